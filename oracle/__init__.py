"""Float64 CPU oracle (test infrastructure only; see muon_oracle.py)."""

from .muon_oracle import (  # noqa: F401
    AGGRESSIVE_ABC,
    DEFAULT_EPS,
    HYBRID_SCHEDULE,
    STANDARD_ABC,
    decay_and_update,
    frobenius_normalise,
    hybrid_newton_schulz,
    momentum,
    muon_step,
    nesterov,
    ns_orthogonalize,
    ns_step,
    orient,
    rescale,
    rescale_none,
    rescale_unit_rms,
    SCALE_MODES,
)

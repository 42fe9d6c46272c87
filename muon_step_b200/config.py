"""Optimizer settings, including the Megatron-Bridge recipe keys.

[V4-breakdown] "Muon 优化器完全拆解…", section "另一条路：开源生态干脆不分片", prints the
Megatron-Bridge DeepSeek-V4-Flash Muon recipe: muon_momentum,
muon_use_nesterov, muon_scale_mode ("unit_rms_norm"), muon_fp32_matmul_prec,
muon_num_ns_steps, muon_extra_scale_factor, muon_coefficient_type
("quintic"; the table also registers "deepseekv4", the hybrid 8 + 2 schedule),
weight_decay and the learning-rate schedule. ``from_megatron`` maps those
keys onto this library's arguments so that such a recipe runs unchanged.

Readings where the recipe's keys are not explained on the pages:

* "quintic" is the (3.4445, -4.7750, 2.0315) step repeated
  muon_num_ns_steps times (the recipe's 5-step quintic loop);
  "deepseekv4" is the hybrid 8 + 2 schedule and fixes 10 steps.
* muon_scale_mode "unit_rms_norm" is the unit-RMS rule (O = O' gamma /
  RMS(O'), gamma = muon_extra_scale_factor). The pages name no value for the
  shape rule; "shape" selects it here, and "none" the plain gamma O'.
* muon_fp32_matmul_prec "highest" asks for full fp32 Newton-Schulz products:
  the fp32 precision of this library. Any other value selects the bf16
  tensor-core path.
* max_lr is the learning rate handed to the step; the warm-up and decay
  schedule, gradient clipping and the data-parallel settings belong to the
  training loop and are returned untouched in ``unused``.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

AGGRESSIVE = (3.4445, -4.7750, 2.0315)
STANDARD = (2.0, -1.5, 0.5)
HYBRID = (AGGRESSIVE,) * 8 + (STANDARD,) * 2

_SCALE_MODES = {"unit_rms_norm": "unit_rms", "unit_rms": "unit_rms", "shape": "shape",
                "none": "none"}


@dataclass
class MuonConfig:
    """Everything a Muon step needs besides the tensors."""

    lr: float = 0.02
    momentum: float = 0.95
    weight_decay: float = 0.1
    gamma: float = 0.2
    nesterov: bool = True
    schedule: Tuple[Tuple[float, float, float], ...] = HYBRID
    scale_mode: str = "shape"
    precision: str = "bf16"
    unused: dict = field(default_factory=dict)

    def plan_kwargs(self) -> dict:
        """Arguments of MuonPlan(...) besides the matrices."""
        return {"precision": self.precision, "schedule": self.schedule,
                "scale_mode": self.scale_mode}

    def execute_kwargs(self) -> dict:
        """Arguments of MuonPlan.execute(...) besides the workspace."""
        return {"lr": self.lr, "momentum": self.momentum, "weight_decay": self.weight_decay,
                "gamma": self.gamma, "nesterov": self.nesterov}


def coefficient_schedule(kind: str, steps: Optional[int]):
    """The Newton-Schulz schedule of a Megatron-Bridge coefficient type."""
    if kind == "quintic":
        n = 5 if steps is None else int(steps)
        if not 1 <= n <= 64:
            raise ValueError(f"muon_num_ns_steps must be in 1 .. 64, got {steps}")
        return (AGGRESSIVE,) * n
    if kind == "deepseekv4":
        if steps not in (None, 10):
            raise ValueError("the deepseekv4 coefficient set is 10 steps (8 + 2)")
        return HYBRID
    raise ValueError(f"unknown muon_coefficient_type {kind!r}")


def from_megatron(**keys) -> MuonConfig:
    """A MuonConfig from Megatron-Bridge recipe keys (unknown keys go to
    ``unused``)."""
    keys = dict(keys)
    cfg = MuonConfig()
    if "muon_momentum" in keys:
        cfg.momentum = float(keys.pop("muon_momentum"))
    if "muon_use_nesterov" in keys:
        cfg.nesterov = bool(keys.pop("muon_use_nesterov"))
    if "muon_scale_mode" in keys:
        mode = keys.pop("muon_scale_mode")
        if mode not in _SCALE_MODES:
            raise ValueError(f"unknown muon_scale_mode {mode!r}")
        cfg.scale_mode = _SCALE_MODES[mode]
    if "muon_extra_scale_factor" in keys:
        cfg.gamma = float(keys.pop("muon_extra_scale_factor"))
    if "muon_fp32_matmul_prec" in keys:
        cfg.precision = "fp32" if keys.pop("muon_fp32_matmul_prec") == "highest" else "bf16"
    kind = keys.pop("muon_coefficient_type", None)
    steps = keys.pop("muon_num_ns_steps", None)
    if kind is not None or steps is not None:
        cfg.schedule = coefficient_schedule(kind or "quintic", steps)
    if "weight_decay" in keys:
        cfg.weight_decay = float(keys.pop("weight_decay"))
    if "max_lr" in keys:
        cfg.lr = float(keys.pop("max_lr"))
    keys.pop("optimizer", None)
    cfg.unused = keys
    return cfg

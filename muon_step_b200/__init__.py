"""Python binding of the B200 Muon step library (argument marshalling only).

Every step of the computation runs in the CUDA kernels of libmuon_step.so,
called through its C ABI (include/muon_step.h). PyTorch supplies device
memory, the workspace and the current stream. There is no fallback: if the
library is missing or the device is not an sm_100 GPU, calls raise.

    plan = MuonPlan([(W, G, M), ...])          # fp32 CUDA tensors, n x m each
    ws = plan.alloc_workspace()
    plan.execute(ws, lr=0.02, momentum=0.95, weight_decay=0.1, gamma=0.2)

    muon_step([(W, G, M)], lr=0.02)            # one-shot
    O = ns_orthogonalize([X])                   # O' per matrix
"""

from __future__ import annotations

import ctypes
from typing import Iterable, Optional, Sequence

import torch

from . import _lib
from ._lib import (MUON_ERR_TIMEOUT, MUON_NS_BF16, MUON_NS_FP32, MUON_OK, AdamwHyper, AdamwParam,
                   MuonHyper, MuonNsMatrix, MuonNsSchedule, MuonParam)

__all__ = ["MuonError", "MuonPlan", "NsPlan", "AdamWPlan", "muon_step", "ns_orthogonalize",
           "adamw_step", "sync_status", "library", "HYBRID_SCHEDULE", "wait_probe",
           "set_wait_limit_ns"]

# the pages' hybrid schedule: 8 aggressive steps, then 2 standard ones
HYBRID_SCHEDULE = ((3.4445, -4.7750, 2.0315),) * 8 + ((2.0, -1.5, 0.5),) * 2


class MuonError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        msg = _lib.load().muon_status_string(status).decode()
        super().__init__(f"{what}: {msg} (status {status})" if what else msg)
        self.status = status


def library() -> ctypes.CDLL:
    return _lib.load()


def _check(status: int, what: str):
    if status != MUON_OK:
        raise MuonError(status, what)


def _precision(p) -> int:
    if p in ("bf16", MUON_NS_BF16, torch.bfloat16):
        return MUON_NS_BF16
    if p in ("fp32", MUON_NS_FP32, torch.float32):
        return MUON_NS_FP32
    raise ValueError(f"precision must be 'bf16' or 'fp32', got {p!r}")


def _matrix(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.float32 or t.dim() != 2 or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous 2-D float32 tensor")
    return t


def _one_device(tensors, what="matrices"):
    """The common device of the tensors (None entries skipped); raise if they differ."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"all {what} must be on one CUDA device, got {sorted(map(str, devs))}")
    return devs.pop()


def _workspace(ws, device):
    """(pointer, size in bytes) of a caller's workspace: a contiguous CUDA
    tensor of any dtype on `device`."""
    if not isinstance(ws, torch.Tensor) or ws.device.type != "cuda":
        raise TypeError("workspace must be a CUDA tensor")
    if not ws.is_contiguous():
        raise TypeError("workspace must be contiguous")
    if ws.device != device:
        raise ValueError(f"workspace is on {ws.device}, the matrices on {device}")
    return ws.data_ptr(), ws.numel() * ws.element_size()


def _schedule(schedule, eps):
    """(struct or None, keep-alive array)."""
    if schedule is None and eps is None:
        return None, None
    sched = HYBRID_SCHEDULE if schedule is None else tuple(tuple(s) for s in schedule)
    flat = (ctypes.c_float * (3 * len(sched)))(*[float(v) for s in sched for v in s])
    st = MuonNsSchedule(len(sched), ctypes.cast(flat, ctypes.POINTER(ctypes.c_float)),
                        1e-7 if eps is None else float(eps))
    return st, flat


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


class _PlanBase:
    _plan = None
    _destroy = None

    def __del__(self):
        # the destroy function is bound at creation: module globals may be gone at exit
        if self._plan and self._destroy is not None:
            self._destroy(self._plan)
            self._plan = None

    @property
    def workspace_bytes(self) -> int:
        n = ctypes.c_size_t()
        _check(_lib.load().muon_plan_workspace_size(self._plan, ctypes.byref(n)), "workspace_size")
        return n.value

    def alloc_workspace(self, device=None) -> torch.Tensor:
        device = self.device if device is None else device
        return torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8, device=device)

    def set_chaining(self, on: bool = True, window: int = 0):
        """Run every Newton-Schulz stage in one chained launch (on, the
        default) or one launch per stage and step (off); `window` is the number
        of matrices the chained launch keeps in flight (0: from the tile
        counts). Results are bit-identical; timing events must be set again."""
        _check(_lib.load().muon_plan_set_chaining(self._plan, 1 if on else 0, int(window)),
               "muon_plan_set_chaining")

    def launches(self):
        """Kinds of the kernels one execute launches (0 elementwise, 1 Gram,
        2 polynomial, 3 apply, 4 apply + update, 5 small-matrix kernel,
        6 RMS reduction, 7 update pass, 8 mid-size kernel, 9 tiny fp32 kernel,
        10 chained Newton-Schulz stages)."""
        lib = _lib.load()
        n = ctypes.c_int()
        _check(lib.muon_plan_launches(self._plan, ctypes.byref(n), None, 0), "launches")
        kinds = (ctypes.c_int * n.value)()
        _check(lib.muon_plan_launches(self._plan, ctypes.byref(n), kinds, n.value), "launches")
        return list(kinds)

    def set_events(self, events: Optional[Sequence[torch.cuda.Event]], materialize=True):
        """Record events[2k] / events[2k+1] around launch k of every execute.

        torch creates an event's cudaEvent_t on its first record; pass
        materialize=False only for events that have been recorded before (for
        instance while capturing a CUDA graph)."""
        lib = _lib.load()
        if not events:
            _check(lib.muon_plan_set_events(self._plan, None, 0), "set_events")
            self._events = None
            return
        if materialize:
            for e in events:
                e.record()
        handles = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        _check(lib.muon_plan_set_events(self._plan, handles, len(events)), "set_events")
        self._events = list(events)

    def flops(self):
        """Useful FLOPs of one execute per stage kind (Gram, poly, apply)."""
        g, p, a = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
        _check(_lib.load().muon_plan_flops(self._plan, ctypes.byref(g), ctypes.byref(p),
                                           ctypes.byref(a)), "flops")
        return g.value, p.value, a.value

    def _ws(self, workspace):
        if workspace is None:
            if getattr(self, "_own_ws", None) is None:
                self._own_ws = self.alloc_workspace()
            workspace = self._own_ws
        return workspace


class MuonPlan(_PlanBase):
    """A planned Muon step over a fixed list of (W, G, M[, O]) fp32 CUDA matrices."""

    def __init__(self, params: Iterable, precision="bf16", schedule=None, eps=None,
                 scale_mode="shape"):
        items = []
        self._tensors = []
        for k, p in enumerate(params):
            W, G, M = (_matrix(t, f"params[{k}].{nm}") for t, nm in zip(p[:3], "WGM"))
            O = p[3] if len(p) > 3 else None
            if O is not None:
                _matrix(O, f"params[{k}].O")
            if not (W.shape == G.shape == M.shape and (O is None or O.shape == W.shape)):
                raise ValueError(f"params[{k}]: W, G, M (and O) must have one shape")
            n, m = W.shape
            items.append(MuonParam(W.data_ptr(), G.data_ptr(), M.data_ptr(),
                                   O.data_ptr() if O is not None else None, n, m))
            self._tensors.append((W, G, M, O))
        if not items:
            raise ValueError("no matrices")
        self.device = _one_device([t for q in self._tensors for t in q])
        arr = (MuonParam * len(items))(*items)
        sched, self._sched_keep = _schedule(schedule, eps)
        plan = ctypes.c_void_p()
        _check(_lib.load().muon_plan_create(arr, len(items), _precision(precision),
                                            ctypes.byref(sched) if sched else None,
                                            ctypes.byref(plan)), "muon_plan_create")
        self._plan = plan
        self._destroy = _lib.load().muon_plan_destroy
        if scale_mode != "shape":
            self.set_scale_mode(scale_mode)

    SCALE_MODES = {"shape": 0, "unit_rms": 1, "none": 2}

    def set_scale_mode(self, mode):
        """Update scale: "shape" (O' sqrt(max(n, m)) gamma, default), "unit_rms"
        (O' gamma / RMS(O')) or "none" (O' gamma). Timing events must be set
        again afterwards (the launch list may change)."""
        _check(_lib.load().muon_plan_set_scale_mode(self._plan, self.SCALE_MODES[mode]),
               "muon_plan_set_scale_mode")

    def set_l2_batching(self, nbytes: int):
        """Run the Newton-Schulz stages batch by batch, each batch's buffers
        at most `nbytes` (0: one pass over every matrix). Results and the
        workspace are unchanged; timing events must be set again."""
        _check(_lib.load().muon_plan_set_l2_batching(self._plan, int(nbytes)),
               "muon_plan_set_l2_batching")

    def set_diagnostics(self, out: Optional[torch.Tensor]):
        """Write per-matrix diagnostics on every later execute into `out`, a
        float32 CUDA tensor of shape (count, 2): column 0 = ||N||_F (the
        orthogonaliser's input), column 1 = RMS of the scaled update O. None
        turns them off. Timing events must be set again afterwards."""
        if out is None:
            ptr = None
        else:
            count = len(self._tensors)
            if (out.dtype != torch.float32 or not out.is_cuda or not out.is_contiguous()
                    or out.numel() != 2 * count or out.device != self.device):
                raise ValueError(f"diagnostics need a contiguous float32 tensor of {2 * count} "
                                 f"elements on {self.device}")
            ptr = out.data_ptr()
        _check(_lib.load().muon_plan_set_diagnostics(self._plan, ptr), "muon_plan_set_diagnostics")
        self._diag = out

    def execute(self, workspace=None, lr=0.02, momentum=0.95, weight_decay=0.1, gamma=0.2,
                nesterov=True, stream=None):
        ptr, nbytes = _workspace(self._ws(workspace), self.device)
        h = MuonHyper(lr, momentum, weight_decay, gamma, 1 if nesterov else 0)
        _check(_lib.load().muon_plan_execute(self._plan, ctypes.byref(h), ptr, nbytes,
                                             _stream_ptr(stream)),
               "muon_plan_execute")


class NsPlan(_PlanBase):
    """A planned ns_orthogonalize over a fixed list of (X, O) fp32 CUDA matrices."""

    def __init__(self, pairs: Iterable, precision="bf16", schedule=None, eps=None):
        items = []
        self._tensors = []
        for k, (X, O) in enumerate(pairs):
            _matrix(X, f"X[{k}]")
            _matrix(O, f"O[{k}]")
            if X.shape != O.shape:
                raise ValueError(f"X[{k}] and O[{k}] differ in shape")
            items.append(MuonNsMatrix(X.data_ptr(), O.data_ptr(), X.shape[0], X.shape[1]))
            self._tensors.append((X, O))
        if not items:
            raise ValueError("no matrices")
        self.device = _one_device([t for q in self._tensors for t in q])
        arr = (MuonNsMatrix * len(items))(*items)
        sched, self._sched_keep = _schedule(schedule, eps)
        plan = ctypes.c_void_p()
        _check(_lib.load().muon_plan_create_ns(arr, len(items), _precision(precision),
                                               ctypes.byref(sched) if sched else None,
                                               ctypes.byref(plan)), "muon_plan_create_ns")
        self._plan = plan
        self._destroy = _lib.load().muon_plan_destroy

    def execute(self, workspace=None, stream=None):
        ptr, nbytes = _workspace(self._ws(workspace), self.device)
        _check(_lib.load().muon_plan_execute(self._plan, None, ptr, nbytes, _stream_ptr(stream)),
               "muon_plan_execute")


def muon_step(params, lr=0.02, momentum=0.95, weight_decay=0.1, gamma=0.2, nesterov=True,
              precision="bf16", schedule=None, eps=None, workspace=None, stream=None):
    """One-shot Muon step (C ABI muon_step) over a list of (W, G, M[, O])."""
    items = []
    keep = []
    for k, p in enumerate(params):
        W, G, M = (_matrix(t, f"params[{k}].{nm}") for t, nm in zip(p[:3], "WGM"))
        O = p[3] if len(p) > 3 else None
        if O is not None:
            _matrix(O, f"params[{k}].O")
        if not (W.shape == G.shape == M.shape and (O is None or O.shape == W.shape)):
            raise ValueError(f"params[{k}]: W, G, M (and O) must have one shape")
        keep.append((W, G, M, O))
        items.append(MuonParam(W.data_ptr(), G.data_ptr(), M.data_ptr(),
                               O.data_ptr() if O is not None else None, *W.shape))
    if not items:
        raise ValueError("no matrices")
    device = _one_device([t for q in keep for t in q])
    arr = (MuonParam * len(items))(*items)
    lib = _lib.load()
    prec = _precision(precision)
    if workspace is None:
        n = ctypes.c_size_t()
        _check(lib.muon_workspace_size(arr, len(items), prec, ctypes.byref(n)), "muon_workspace_size")
        workspace = torch.empty(max(n.value, 256), dtype=torch.uint8, device=device)
    ptr, nbytes = _workspace(workspace, device)
    sched, _keep = _schedule(schedule, eps)
    _check(lib.muon_step(arr, len(items), lr, momentum, weight_decay, gamma, 1 if nesterov else 0,
                         ctypes.byref(sched) if sched else None, prec, ptr, nbytes,
                         _stream_ptr(stream)), "muon_step")
    return workspace


def ns_orthogonalize(xs, out=None, precision="bf16", schedule=None, eps=None, workspace=None,
                     stream=None):
    """O' = NewtonSchulz(X / (||X||_F + eps)) per matrix (C ABI ns_orthogonalize)."""
    xs = [_matrix(x, f"X[{k}]") for k, x in enumerate(xs)]
    if not xs:
        raise ValueError("no matrices")
    if out is None:
        out = [torch.empty_like(x) for x in xs]
    else:
        out = [_matrix(o, f"out[{k}]") for k, o in enumerate(out)]
        if len(out) != len(xs) or any(o.shape != x.shape for x, o in zip(xs, out)):
            raise ValueError("out must hold one matrix of X's shape per input")
    device = _one_device(xs + out)
    items = (MuonNsMatrix * len(xs))(*[MuonNsMatrix(x.data_ptr(), o.data_ptr(), *x.shape)
                                       for x, o in zip(xs, out)])
    lib = _lib.load()
    prec = _precision(precision)
    if workspace is None:
        n = ctypes.c_size_t()
        _check(lib.ns_workspace_size(items, len(xs), prec, ctypes.byref(n)), "ns_workspace_size")
        workspace = torch.empty(max(n.value, 256), dtype=torch.uint8, device=device)
    ptr, nbytes = _workspace(workspace, device)
    sched, _keep = _schedule(schedule, eps)
    _check(lib.ns_orthogonalize(items, len(xs), ctypes.byref(sched) if sched else None, prec,
                                ptr, nbytes, _stream_ptr(stream)),
           "ns_orthogonalize")
    return out


def _flat(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.float32 or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous float32 tensor")
    return t


def _adamw_items(params):
    items, keep = [], []
    for k, q in enumerate(params):
        p, g, m, v = (_flat(t, f"params[{k}].{nm}") for t, nm in zip(q, "pgmv"))
        if not (p.numel() == g.numel() == m.numel() == v.numel()):
            raise ValueError(f"params[{k}]: p, g, m, v must have one size")
        items.append(AdamwParam(p.data_ptr(), g.data_ptr(), m.data_ptr(), v.data_ptr(), p.numel()))
        keep.append((p, g, m, v))
    if not items:
        raise ValueError("no tensors")
    _one_device([t for q in keep for t in q], "tensors")
    return (AdamwParam * len(items))(*items), keep


def _adamw_hyper(lr, betas, eps, weight_decay, step, step_tensor):
    if step_tensor is not None:
        if (step_tensor.dtype != torch.int32 or not step_tensor.is_cuda
                or step_tensor.numel() != 1):
            raise TypeError("step_tensor must be a one-element int32 CUDA tensor")
        return AdamwHyper(lr=lr, eps=eps, weight_decay=weight_decay, step=0, beta1=betas[0],
                          beta2=betas[1], step_dev=step_tensor.data_ptr())
    return AdamwHyper(lr=lr, eps=eps, weight_decay=weight_decay, step=int(step), beta1=betas[0],
                      beta2=betas[1], step_dev=None)


class AdamWPlan:
    """A planned AdamW step over a fixed list of (p, g, m, v) float32 CUDA
    tensors (any shape, contiguous; m and v are the moment buffers, zero at
    the start). One kernel launch per execute (C ABI muon_adamw_plan_*)."""

    _plan = None
    _destroy = None

    def __init__(self, params: Iterable):
        arr, self._tensors = _adamw_items(params)
        self.device = self._tensors[0][0].device
        lib = _lib.load()
        plan = ctypes.c_void_p()
        _check(lib.muon_adamw_plan_create(arr, len(arr), ctypes.byref(plan)), "muon_adamw_plan_create")
        self._plan = plan
        self._destroy = lib.muon_adamw_plan_destroy
        self._ws_cache = None

    def __del__(self):
        if self._plan and self._destroy is not None:
            self._destroy(self._plan)
            self._plan = None

    @property
    def workspace_bytes(self) -> int:
        n = ctypes.c_size_t()
        _check(_lib.load().muon_adamw_plan_workspace_size(self._plan, ctypes.byref(n)),
               "muon_adamw_plan_workspace_size")
        return n.value

    @property
    def numel(self) -> int:
        n = ctypes.c_int64()
        _check(_lib.load().muon_adamw_plan_numel(self._plan, ctypes.byref(n)), "muon_adamw_plan_numel")
        return n.value

    def alloc_workspace(self, device=None) -> torch.Tensor:
        device = self.device if device is None else device
        return torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8, device=device)

    def execute(self, workspace=None, lr=0.02, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.1,
                step=1, step_tensor=None, stream=None):
        """One AdamW step at step number `step` (from 1), or at the number held
        on the device in `step_tensor` (int32, read by the kernel)."""
        if workspace is None:
            if self._ws_cache is None:
                self._ws_cache = self.alloc_workspace()
            workspace = self._ws_cache
        ptr, nbytes = _workspace(workspace, self.device)
        if step_tensor is not None and step_tensor.device != self.device:
            raise ValueError(f"step_tensor is on {step_tensor.device}, the tensors on {self.device}")
        h = _adamw_hyper(lr, betas, eps, weight_decay, step, step_tensor)
        _check(_lib.load().muon_adamw_plan_execute(self._plan, ctypes.byref(h), ptr, nbytes,
                                                   _stream_ptr(stream)),
               "muon_adamw_plan_execute")


def adamw_step(params, step, lr=0.02, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.1,
               workspace=None, stream=None):
    """One-shot AdamW step (C ABI muon_adamw_step) over a list of (p, g, m, v)."""
    arr, keep = _adamw_items(params)
    lib = _lib.load()
    if workspace is None:
        n = ctypes.c_size_t()
        _check(lib.muon_adamw_workspace_size(arr, len(arr), ctypes.byref(n)),
               "muon_adamw_workspace_size")
        workspace = torch.empty(max(n.value, 256), dtype=torch.uint8, device=keep[0][0].device)
    ptr, nbytes = _workspace(workspace, keep[0][0].device)
    h = _adamw_hyper(lr, betas, eps, weight_decay, step, None)
    _check(lib.muon_adamw_step(arr, len(arr), ctypes.byref(h), ptr, nbytes, _stream_ptr(stream)),
           "muon_adamw_step")
    return workspace


def sync_status(stream=None) -> int:
    """Synchronise and return the device error status (MUON_OK or MUON_ERR_TIMEOUT)."""
    return _lib.load().muon_sync_status(_stream_ptr(stream))


def set_tracing(on: bool = True):
    """NVTX ranges around every kernel launch of later executes (off by default)."""
    _lib.load().muon_set_tracing(1 if on else 0)


def set_wait_limit_ns(ns: int):
    _lib.load().muon_set_wait_limit_ns(int(ns))


def wait_probe(flag: torch.Tensor, limit_ns: int, stream=None):
    """Launch one bounded device wait on ``flag`` (int32 CUDA tensor)."""
    if flag.dtype != torch.int32 or flag.device.type != "cuda":
        raise TypeError("flag must be an int32 CUDA tensor")
    _check(_lib.load().muon_wait_probe(flag.data_ptr(), int(limit_ns), _stream_ptr(stream)),
           "muon_wait_probe")


def dep_wait_probe(counter: torch.Tensor, target: int, limit_ns: int, stream=None):
    """Launch the chained launch's dependency wait on ``counter`` (int32 CUDA
    tensor, read as unsigned) until it reaches ``target``, bounded by
    ``limit_ns``."""
    if counter.dtype != torch.int32 or counter.device.type != "cuda":
        raise TypeError("counter must be an int32 CUDA tensor")
    _check(_lib.load().muon_dep_wait_probe(counter.data_ptr(), int(target), int(limit_ns),
                                           _stream_ptr(stream)), "muon_dep_wait_probe")

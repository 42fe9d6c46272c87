"""ctypes declarations of the C ABI in include/muon_step.h."""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmuon_step.so")

MUON_OK = 0
MUON_ERR_INVALID_ARG = 1
MUON_ERR_WORKSPACE = 2
MUON_ERR_CUDA = 3
MUON_ERR_UNSUPPORTED = 4
MUON_ERR_TIMEOUT = 5

MUON_NS_BF16 = 0
MUON_NS_FP32 = 1

MUON_STATIC_SCRATCH_BYTES = 64 << 20

MUON_SCALE_SHAPE = 0
MUON_SCALE_UNIT_RMS = 1
MUON_SCALE_NONE = 2

# every symbol include/muon_step.h declares
EXPORTS = (
    "muon_plan_create", "muon_plan_create_ns", "muon_plan_workspace_size", "muon_plan_execute",
    "muon_plan_launches", "muon_plan_set_events", "muon_plan_flops", "muon_plan_destroy",
    "muon_workspace_size", "muon_step", "ns_workspace_size", "ns_orthogonalize",
    "muon_sync_status", "muon_status_string", "muon_abi_version", "muon_set_wait_limit_ns",
    "muon_wait_probe", "muon_step_static_scratch", "muon_plan_set_scale_mode",
    "muon_plan_set_diagnostics",
    "muon_adamw_plan_create", "muon_adamw_plan_workspace_size", "muon_adamw_plan_execute",
    "muon_adamw_plan_numel", "muon_adamw_plan_destroy", "muon_adamw_workspace_size",
    "muon_adamw_step",
    "muon_shard_workspace_size", "muon_shard_momentum", "muon_shard_update", "muon_copy_segments",
    "muon_plan_set_l2_batching", "muon_set_tracing", "muon_plan_set_chaining",
    "muon_dep_wait_probe",
)


class MuonParam(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("G", ctypes.c_void_p), ("M", ctypes.c_void_p),
                ("O", ctypes.c_void_p), ("n", ctypes.c_int64), ("m", ctypes.c_int64)]


class MuonNsSchedule(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_int), ("abc", ctypes.POINTER(ctypes.c_float)),
                ("eps", ctypes.c_float)]


class MuonNsMatrix(ctypes.Structure):
    _fields_ = [("X", ctypes.c_void_p), ("O", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("m", ctypes.c_int64)]


class AdamwParam(ctypes.Structure):
    _fields_ = [("p", ctypes.c_void_p), ("g", ctypes.c_void_p), ("m", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("numel", ctypes.c_int64)]


class AdamwHyper(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("step", ctypes.c_int32), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("step_dev", ctypes.c_void_p)]


class ShardMomentum(ctypes.Structure):
    _fields_ = [("M", ctypes.c_void_p), ("G", ctypes.c_void_p), ("N", ctypes.c_void_p),
                ("numel", ctypes.c_int64)]


class ShardUpdate(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("O", ctypes.c_void_p), ("numel", ctypes.c_int64),
                ("n", ctypes.c_int64), ("m", ctypes.c_int64)]


class Segment(ctypes.Structure):
    _fields_ = [("dst", ctypes.c_void_p), ("src", ctypes.c_void_p), ("numel", ctypes.c_int64)]


class MuonHyper(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("momentum", ctypes.c_float),
                ("weight_decay", ctypes.c_float), ("gamma", ctypes.c_float),
                ("nesterov", ctypes.c_int)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library; raise if it has not been built (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libmuon_step.so not found at {path}; build it with `python -m muon_step_b200.build`")
    lib = ctypes.CDLL(path)
    st = ctypes.c_int
    vp = ctypes.c_void_p
    P = ctypes.POINTER
    sig = {
        "muon_plan_create": (st, [P(MuonParam), ctypes.c_int, ctypes.c_int, P(MuonNsSchedule), P(vp)]),
        "muon_plan_create_ns": (st, [P(MuonNsMatrix), ctypes.c_int, ctypes.c_int, P(MuonNsSchedule), P(vp)]),
        "muon_plan_workspace_size": (st, [vp, P(ctypes.c_size_t)]),
        "muon_plan_execute": (st, [vp, P(MuonHyper), vp, ctypes.c_size_t, vp]),
        "muon_plan_launches": (st, [vp, P(ctypes.c_int), P(ctypes.c_int), ctypes.c_int]),
        "muon_plan_set_events": (st, [vp, P(vp), ctypes.c_int]),
        "muon_plan_flops": (st, [vp, P(ctypes.c_double), P(ctypes.c_double), P(ctypes.c_double)]),
        "muon_plan_destroy": (None, [vp]),
        "muon_plan_set_scale_mode": (st, [vp, ctypes.c_int]),
        "muon_plan_set_diagnostics": (st, [vp, vp]),
        "muon_plan_set_l2_batching": (st, [vp, ctypes.c_size_t]),
        "muon_plan_set_chaining": (st, [vp, ctypes.c_int, ctypes.c_int]),
        "muon_set_tracing": (None, [ctypes.c_int]),
        "muon_adamw_plan_create": (st, [P(AdamwParam), ctypes.c_int, P(vp)]),
        "muon_adamw_plan_workspace_size": (st, [vp, P(ctypes.c_size_t)]),
        "muon_adamw_plan_execute": (st, [vp, P(AdamwHyper), vp, ctypes.c_size_t, vp]),
        "muon_adamw_plan_numel": (st, [vp, P(ctypes.c_int64)]),
        "muon_adamw_plan_destroy": (None, [vp]),
        "muon_adamw_workspace_size": (st, [P(AdamwParam), ctypes.c_int, P(ctypes.c_size_t)]),
        "muon_adamw_step": (st, [P(AdamwParam), ctypes.c_int, P(AdamwHyper), vp, ctypes.c_size_t,
                                 vp]),
        "muon_shard_workspace_size": (st, [ctypes.c_int, P(ctypes.c_size_t)]),
        "muon_shard_momentum": (st, [P(ShardMomentum), ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                     vp, ctypes.c_size_t, vp]),
        "muon_shard_update": (st, [P(ShardUpdate), ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                   ctypes.c_float, vp, ctypes.c_size_t, vp]),
        "muon_copy_segments": (st, [P(Segment), ctypes.c_int, vp, ctypes.c_size_t, vp]),
        "muon_workspace_size": (st, [P(MuonParam), ctypes.c_int, ctypes.c_int, P(ctypes.c_size_t)]),
        "muon_step": (st, [P(MuonParam), ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                           ctypes.c_float, ctypes.c_int, P(MuonNsSchedule), ctypes.c_int, vp,
                           ctypes.c_size_t, vp]),
        "ns_workspace_size": (st, [P(MuonNsMatrix), ctypes.c_int, ctypes.c_int, P(ctypes.c_size_t)]),
        "ns_orthogonalize": (st, [P(MuonNsMatrix), ctypes.c_int, P(MuonNsSchedule), ctypes.c_int, vp,
                                  ctypes.c_size_t, vp]),
        "muon_sync_status": (st, [vp]),
        "muon_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "muon_abi_version": (ctypes.c_int, []),
        "muon_set_wait_limit_ns": (None, [ctypes.c_uint64]),
        "muon_wait_probe": (st, [vp, ctypes.c_uint64, vp]),
        "muon_dep_wait_probe": (st, [vp, ctypes.c_uint32, ctypes.c_uint64, vp]),
        "muon_step_static_scratch": (st, [P(MuonParam), ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                          ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                          P(MuonNsSchedule), ctypes.c_int, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib

"""Python binding of libmoonep.so — MoonEP-style balanced expert-parallel hot path on B200.

Argument marshalling only: every step runs in the CUDA kernels of
``libmoonep.so`` (C ABI declared in ``include/moonep.h``).  PyTorch provides the
device memory and the stream; nothing here computes.  If the library is not
built this import fails; there is no fallback.

The functions keep the C names::

    moonep_nvs(cfg) / moonep_plan_bytes(cfg) / moonep_workspace_bytes(cfg)
    moonep_plan(cfg, topk_idx, plan_arena, workspace, dev_status, stream=None)
    moonep_plan_static(cfg, topk_idx, plan_arena, dev_status, stream=None)
    moonep_plan_view(cfg, plan_arena) -> dict of int32 tensor views
    moonep_debug_set_wait(limit_ns, phantom_arrivals=0)
    moonep_dispatch(cfg, plan_arena, x, recv, dev_status, stream=None)
    moonep_combine(cfg, plan_arena, y, gates, out, dev_status, stream=None)
    moonep_combine_backward(cfg, plan_arena, dout, y, gates, dy, dgates, dev_status, stream=None)
    moonep_reduce_grad(cfg, plan_arena, rep_grads, home_grads, P, dev_status, stream=None)
    moonep_reduce_grad_f32(cfg, plan_arena, rep_grads, home_grads, P, dev_status, stream=None)
    moonep_dispatch_backward(cfg, plan_arena, d_recv, dx, dev_status, stream=None)
    moonep_prefetch_weight(cfg, plan_arena, weights, rep_weights, W, dev_status, stream=None)
    moonep_dispatch_via_buffer(cfg, plan_arena, x, comm, comm_index, recv, dev_status, stream=None)
    moonep_combine_via_buffer(cfg, plan_arena, y, gates, comm_index, comm, out, dev_status, stream=None)
    moonep_fused_forward(cfg, topk_idx, gates, x, plan_arena, workspace, recv, out, dev_status, stream=None)

Tensor arguments are device tensors (bf16 tensors may be ``torch.bfloat16``
or ``int16``/``uint16`` views); raw integer device addresses are accepted too.
A non-OK return raises :class:`MoonepError`.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Dict, Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoonep.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moonep.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libmoonep.so is not built ({LIB_PATH}); run `python token_dispatch_moonep_b200/build.py` "
        "(nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

MODE_TRAIN = 0
MODE_INFER = 1
MAX_EXPERTS = 1024
MAX_TOPK = 32
STATIC_WORKSPACE_BYTES = 4 << 20

OK = 0
ERR_INVALID_ARG = 1
ERR_CUDA = 2
ERR_UNSUPPORTED = 3

DEV_BAD_EXPERT_ID = 0x1
DEV_CAPACITY = 0x2
DEV_BUDGET = 0x4
DEV_TIMEOUT = 0x8
DEV_BAD_PLAN = 0x10

SEG_NATIVE = 0
SEG_REPLICA = 1
SEG_REMOTE = 2


class MoonepError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {moonep_status_string(status)} (status {status})")


class Config(ctypes.Structure):
    """moonep_config_t."""

    _fields_ = [(n, ctypes.c_int32) for n in ("R", "E", "K", "S", "H", "budget", "mode", "align")]

    def __init__(self, R, E, K, S, H=1, budget=0, mode=MODE_TRAIN, align=1):
        super().__init__(R, E, K, S, H, budget, mode, align)

    @classmethod
    def of(cls, w, **over) -> "Config":
        d = dict(R=w.R, E=w.E, K=w.K, S=w.S, H=w.H, budget=w.budget, mode=w.mode,
                 align=getattr(w, "align", 1))
        d.update(over)
        return cls(**d)

    def __repr__(self):
        return "Config(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


_I32P = ctypes.POINTER(ctypes.c_int32)
_VIEW_FIELDS = ["slot_of", "slot_src", "expert_count", "rank_load", "overflow", "deficit", "n_seg",
                "seg_expert", "seg_start", "seg_len", "seg_kind", "seg_wslot", "piece_expert",
                "piece_rank", "piece_start", "piece_len", "piece_wslot", "piece_ostart",
                "expert_piece_begin", "expert_piece_end", "rep_expert", "replicated_experts",
                "scalars"]


class PlanView(ctypes.Structure):
    """moonep_plan_view_t."""

    _fields_ = [(n, ctypes.c_void_p) for n in _VIEW_FIELDS] + [
        ("nvs", ctypes.c_int64), ("max_pieces", ctypes.c_int32)]


_CP = ctypes.POINTER(Config)
_VP = ctypes.c_void_p
_ST = ctypes.c_int

_lib.moonep_nvs.argtypes = [_CP]
_lib.moonep_nvs.restype = ctypes.c_int64
_lib.moonep_plan_bytes.argtypes = [_CP]
_lib.moonep_plan_bytes.restype = ctypes.c_size_t
_lib.moonep_workspace_bytes.argtypes = [_CP]
_lib.moonep_workspace_bytes.restype = ctypes.c_size_t
_lib.moonep_plan.argtypes = [_CP, _VP, _VP, _VP, _VP, _VP]
_lib.moonep_plan.restype = _ST
_lib.moonep_plan_static.argtypes = [_CP, _VP, _VP, _VP, _VP]
_lib.moonep_plan_static.restype = _ST
_lib.moonep_debug_set_wait.argtypes = [ctypes.c_int64, ctypes.c_int32]
_lib.moonep_debug_set_wait.restype = _ST
_lib.moonep_plan_view.argtypes = [_CP, _VP, ctypes.POINTER(PlanView)]
_lib.moonep_plan_view.restype = _ST
_lib.moonep_dispatch.argtypes = [_CP, _VP, _VP, _VP, _VP, _VP]
_lib.moonep_dispatch.restype = _ST
_lib.moonep_combine.argtypes = [_CP, _VP, _VP, _VP, _VP, _VP, _VP]
_lib.moonep_combine.restype = _ST
_lib.moonep_combine_backward.argtypes = [_CP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]
_lib.moonep_combine_backward.restype = _ST
_lib.moonep_reduce_grad.argtypes = [_CP, _VP, _VP, _VP, ctypes.c_int64, _VP, _VP]
_lib.moonep_reduce_grad.restype = _ST
_lib.moonep_reduce_grad_f32.argtypes = [_CP, _VP, _VP, _VP, ctypes.c_int64, _VP, _VP]
_lib.moonep_reduce_grad_f32.restype = _ST
_lib.moonep_dispatch_backward.argtypes = [_CP, _VP, _VP, _VP, _VP, _VP]
_lib.moonep_dispatch_backward.restype = _ST
_lib.moonep_prefetch_weight.argtypes = [_CP, _VP, _VP, _VP, ctypes.c_int64, _VP, _VP]
_lib.moonep_prefetch_weight.restype = _ST
_lib.moonep_segment_weights.argtypes = [_CP, _VP, _VP, _VP, ctypes.c_int64, _VP, _VP, _VP]
_lib.moonep_segment_weights.restype = _ST
_lib.moonep_dispatch_via_buffer.argtypes = [_CP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]
_lib.moonep_dispatch_via_buffer.restype = _ST
_lib.moonep_combine_via_buffer.argtypes = [_CP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]
_lib.moonep_combine_via_buffer.restype = _ST
_lib.moonep_fused_forward.argtypes = [_CP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]
_lib.moonep_fused_forward.restype = _ST
_lib.moonep_status_string.argtypes = [_ST]
_lib.moonep_status_string.restype = ctypes.c_char_p


def header_functions() -> list:
    """Names of the functions declared in include/moonep.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moonep_[a-z_0-9]+)\s*\(", text)))


# ------------------------------------------------------------- marshalling ---
def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, st: int) -> None:
    if st != OK:
        raise MoonepError(fn, st)


def moonep_status_string(status: int) -> str:
    return _lib.moonep_status_string(int(status)).decode()


def moonep_nvs(cfg: Config) -> int:
    return int(_lib.moonep_nvs(ctypes.byref(cfg)))


def moonep_plan_bytes(cfg: Config) -> int:
    return int(_lib.moonep_plan_bytes(ctypes.byref(cfg)))


def moonep_workspace_bytes(cfg: Config) -> int:
    return int(_lib.moonep_workspace_bytes(ctypes.byref(cfg)))


def moonep_plan(cfg: Config, topk_idx, plan_arena, workspace, dev_status, stream=None) -> None:
    _check("moonep_plan", _lib.moonep_plan(ctypes.byref(cfg), _ptr(topk_idx), _ptr(plan_arena),
                                           _ptr(workspace), _ptr(dev_status), _stream(stream)))


def moonep_plan_static(cfg: Config, topk_idx, plan_arena, dev_status, stream=None) -> None:
    """moonep_plan without a caller workspace: the library's fixed scratch array is used
    (for callers that cannot allocate; see include/moonep.h).  Calls that overlap on the
    GPU share that array and race."""
    _check("moonep_plan_static", _lib.moonep_plan_static(
        ctypes.byref(cfg), _ptr(topk_idx), _ptr(plan_arena), _ptr(dev_status), _stream(stream)))


def moonep_debug_set_wait(limit_ns: int, phantom_arrivals: int = 0) -> None:
    """Time limit of the plan kernel's in-kernel waits; phantom arrivals force a timeout (tests)."""
    _check("moonep_debug_set_wait", _lib.moonep_debug_set_wait(int(limit_ns), int(phantom_arrivals)))


DEFAULT_WAIT_NS = 200 * 1000 * 1000


def moonep_plan_view_ptrs(cfg: Config, plan_arena) -> PlanView:
    v = PlanView()
    _check("moonep_plan_view", _lib.moonep_plan_view(ctypes.byref(cfg), _ptr(plan_arena),
                                                     ctypes.byref(v)))
    return v


def moonep_plan_view(cfg: Config, plan_arena) -> Dict[str, "object"]:
    """int32 tensor views into the plan arena, keyed like moonep_plan_view_t's fields."""
    import torch
    v = moonep_plan_view_ptrs(cfg, plan_arena)
    R, E, K, S, B = cfg.R, cfg.E, cfg.K, cfg.S, cfg.budget
    pm = v.max_pieces
    n = dict(slot_of=R * S * K, slot_src=R * v.nvs, expert_count=E, rank_load=R, overflow=R,
             deficit=R, n_seg=R, seg_expert=R * E, seg_start=R * E, seg_len=R * E, seg_kind=R * E,
             seg_wslot=R * E, piece_expert=pm, piece_rank=pm, piece_start=pm, piece_len=pm,
             piece_wslot=pm, piece_ostart=pm, expert_piece_begin=E, expert_piece_end=E,
             rep_expert=R * B, replicated_experts=E, scalars=8)
    base = _ptr(plan_arena)
    flat = plan_arena.view(torch.uint8).reshape(-1)
    out = {}
    for name in _VIEW_FIELDS:
        off = getattr(v, name) - base
        out[name] = flat[off: off + 4 * n[name]].view(torch.int32)
    out["nvs"] = v.nvs
    return out


def moonep_dispatch(cfg: Config, plan_arena, x, recv, dev_status, stream=None) -> None:
    _check("moonep_dispatch", _lib.moonep_dispatch(ctypes.byref(cfg), _ptr(plan_arena), _ptr(x),
                                                   _ptr(recv), _ptr(dev_status), _stream(stream)))


def moonep_combine(cfg: Config, plan_arena, y, gates, out, dev_status, stream=None) -> None:
    _check("moonep_combine", _lib.moonep_combine(ctypes.byref(cfg), _ptr(plan_arena), _ptr(y),
                                                 _ptr(gates), _ptr(out), _ptr(dev_status),
                                                 _stream(stream)))


def moonep_combine_backward(cfg: Config, plan_arena, dout, y, gates, dy, dgates, dev_status,
                            stream=None) -> None:
    _check("moonep_combine_backward", _lib.moonep_combine_backward(
        ctypes.byref(cfg), _ptr(plan_arena), _ptr(dout), _ptr(y), _ptr(gates), _ptr(dy),
        _ptr(dgates), _ptr(dev_status), _stream(stream)))


def moonep_reduce_grad(cfg: Config, plan_arena, rep_grads, home_grads, P: int, dev_status,
                       stream=None) -> None:
    _check("moonep_reduce_grad", _lib.moonep_reduce_grad(
        ctypes.byref(cfg), _ptr(plan_arena), _ptr(rep_grads), _ptr(home_grads), int(P),
        _ptr(dev_status), _stream(stream)))


def moonep_reduce_grad_f32(cfg: Config, plan_arena, rep_grads, home_grads, P: int, dev_status,
                           stream=None) -> None:
    """reduce_grad over fp32 gradient buffers (float32 tensors [R, budget, P] and [E, P])."""
    _check("moonep_reduce_grad_f32", _lib.moonep_reduce_grad_f32(
        ctypes.byref(cfg), _ptr(plan_arena), _ptr(rep_grads), _ptr(home_grads), int(P),
        _ptr(dev_status), _stream(stream)))


def moonep_dispatch_backward(cfg: Config, plan_arena, d_recv, dx, dev_status, stream=None) -> None:
    _check("moonep_dispatch_backward", _lib.moonep_dispatch_backward(
        ctypes.byref(cfg), _ptr(plan_arena), _ptr(d_recv), _ptr(dx), _ptr(dev_status),
        _stream(stream)))


def moonep_prefetch_weight(cfg: Config, plan_arena, weights, rep_weights, W: int, dev_status,
                           stream=None) -> None:
    _check("moonep_prefetch_weight", _lib.moonep_prefetch_weight(
        ctypes.byref(cfg), _ptr(plan_arena), _ptr(weights), _ptr(rep_weights), int(W),
        _ptr(dev_status), _stream(stream)))


def moonep_segment_weights(cfg: Config, plan_arena, weights, rep_weights, W: int, seg_weights,
                           dev_status, stream=None) -> None:
    """Device pointers [R*E] (an int64 tensor) to the weight matrix of every segment-table
    entry: replica pieces their local slot, native segments and remote pieces the home
    expert's row, unused entries 0 (see include/moonep.h)."""
    _check("moonep_segment_weights", _lib.moonep_segment_weights(
        ctypes.byref(cfg), _ptr(plan_arena), _ptr(weights), _ptr(rep_weights), int(W),
        _ptr(seg_weights), _ptr(dev_status), _stream(stream)))


def moonep_dispatch_via_buffer(cfg: Config, plan_arena, x, comm, comm_index, recv, dev_status,
                               stream=None) -> None:
    _check("moonep_dispatch_via_buffer", _lib.moonep_dispatch_via_buffer(
        ctypes.byref(cfg), _ptr(plan_arena), _ptr(x), _ptr(comm), _ptr(comm_index), _ptr(recv),
        _ptr(dev_status), _stream(stream)))


def moonep_combine_via_buffer(cfg: Config, plan_arena, y, gates, comm_index, comm, out, dev_status,
                              stream=None) -> None:
    _check("moonep_combine_via_buffer", _lib.moonep_combine_via_buffer(
        ctypes.byref(cfg), _ptr(plan_arena), _ptr(y), _ptr(gates), _ptr(comm_index), _ptr(comm),
        _ptr(out), _ptr(dev_status), _stream(stream)))


def moonep_fused_forward(cfg: Config, topk_idx, gates, x, plan_arena, workspace, recv, out,
                         dev_status, stream=None) -> None:
    _check("moonep_fused_forward", _lib.moonep_fused_forward(
        ctypes.byref(cfg), _ptr(topk_idx), _ptr(gates), _ptr(x), _ptr(plan_arena), _ptr(workspace),
        _ptr(recv), _ptr(out), _ptr(dev_status), _stream(stream)))


# ---------------------------------------------------------- allocation help ---
def alloc_plan(cfg: Config, device="cuda"):
    """(plan_arena, workspace, dev_status) device tensors sized for ``cfg`` (torch allocations)."""
    import torch
    pb, wb = moonep_plan_bytes(cfg), moonep_workspace_bytes(cfg)
    if pb == 0 or wb == 0:
        raise MoonepError("alloc_plan", ERR_INVALID_ARG)
    arena = torch.empty(pb, dtype=torch.uint8, device=device)
    ws = torch.empty(wb, dtype=torch.uint8, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    return arena, ws, status


__all__ = [n for n in dir() if n.startswith("moonep_")] + [
    "Config", "PlanView", "MoonepError", "alloc_plan", "LIB_PATH", "header_functions"]

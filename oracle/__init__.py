"""CPU oracle for the MoonEP balanced expert-parallel hot path — TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's ``cpu_baseline``
leg may import this package.  It wraps the plain C implementation in
``moonep_oracle.c`` (built with gcc, strict IEEE arithmetic, no fast-math) and
shares nothing with the CUDA library: no code, header, table or constant.

What each function follows, and what pins it (the ``-m "not gpu"`` tests).
Besides the pins below, property tests draw small plans (1-8 ranks, budgets
0..L, both modes, padding, repeated experts in a token, REMOTE pieces) and
check on each the plan's invariants, the data path, the two gradient folds
and the replica-weight tables:

* ``plan`` — the pages fix the outcome: every rank receives exactly S*K
  token-slots ("Moonshot AI Open-Sources MoonEP", S x K paragraph), overloaded
  experts are duplicated onto other ranks within a per-rank replica-slot budget
  (same page, replica-slot paragraph), buffers have a fixed NvS = S*K +
  alignment padding rows ("MoonshotAI/MoonEP 딥다이브" §4 pattern 2).  The
  tie-breaks are a fixed reading stated in the C file header.  Pinned by:
  a hand-derived worked example; closed-form degenerate routings (all tokens on
  one expert, already-balanced routing); invariants on random routings (S*K
  rows per rank, bijection pairs -> rows, row expert = routed expert, replica
  budget, overflow/deficit accounting, piece-count bound, independence of H);
  and an independent lexsort formulation of the keep/overflow/receiver order.
* ``dispatch`` — the bit-copy definition (§2② zero copy); pinned by the
  round trip and the "every row written exactly once" poison check.
* ``combine`` — fp32 gate-weighted sum (§3③ combine); pinned against the fp64
  closed form sum_k w_k x within the bf16 + fp32 rounding bound (§8 exercise C),
  and its order (ascending k) by three terms whose fp32 sum depends on it.
* ``combine_backward`` — per-element closed forms: dY = w*dOut within half a bf16
  ulp of the fp64 product; dgate = <dOut, x> for the identity expert, in fp64.
* ``reduce_grad`` — with integer-valued bf16 gradients all fp32 sums are
  exact, so home + replicas must equal, bit for bit, the no-replication
  gradient (§4 pattern 3, §8 exercise E); its order (home first, then the
  pieces by ascending receiving rank) by three terms whose sum depends on it.
* ``reduce_grad_f32`` — the same fold over fp32 gradient buffers.  Pinned by the
  no-replication identity with integers past bf16's exact range (so a rounding
  through bf16 fails), and by the order of the fp32 additions: home first, then
  the pieces in ascending receiver, fixed by sums whose result depends on it.
* ``dispatch_backward`` — the adjoint of dispatch: with integer-valued data
  <dispatch(x), dR> = <x, dispatch_backward(dR)> exactly, and
  dispatch_backward(dispatch(x)) = K*x; its order (ascending k) as combine's.
* ``prefetch_weight`` — every local replica slot holds its expert's weights
  bit for bit, every other slot is untouched; closed form for all tokens on
  one expert.
* ``segment_weights`` — the weights each segment computes with: replica pieces
  their local slot, native segments and remote pieces the home expert ("Moonshot
  AI Open-Sources MoonEP", replica-slot paragraph: reads past the budget go to
  the home rank).  Pinned by the worked example by hand, and against the piece
  and replica-slot tables (a route that does not read the segment tables).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

import numpy as np

from .build import LIB_PATH, build

OK = 0
INVALID_ARG = 1
BAD_EXPERT_ID = 2
BUDGET = 4
CAPACITY = 8

KIND_NATIVE = 0
KIND_REPLICA = 1
KIND_REMOTE = 2


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("R", "E", "K", "S", "H", "budget", "mode", "align")]

    def __init__(self, R, E, K, S, H=1, budget=0, mode=0, align=1):
        super().__init__(R, E, K, S, H, budget, mode, align)

    @classmethod
    def of(cls, w, **over) -> "Config":
        d = dict(R=w.R, E=w.E, K=w.K, S=w.S, H=w.H, budget=w.budget, mode=w.mode,
                 align=getattr(w, "align", 1))
        d.update(over)
        return cls(**d)


_I32P = ctypes.POINTER(ctypes.c_int32)
_PLAN_FIELDS = ["expert_count", "rank_load", "overflow", "deficit", "n_seg", "seg_expert",
                "seg_start", "seg_len", "seg_kind", "seg_wslot", "n_piece", "piece_expert",
                "piece_rank", "piece_start", "piece_len", "piece_wslot", "piece_ostart",
                "rep_expert", "n_remote", "slot_of", "slot_src"]


class _PlanOut(ctypes.Structure):
    _fields_ = [(n, _I32P) for n in _PLAN_FIELDS]


_lib = None


def _L():
    global _lib
    if _lib is None:
        # MOONEP_ORACLE_LIB: a deliberately broken oracle build, used only by the test that
        # checks the pins fail against planted mistakes
        lib = ctypes.CDLL(os.environ.get("MOONEP_ORACLE_LIB") or build())
        vp = ctypes.c_void_p
        cp = ctypes.POINTER(Config)
        lib.orc_nvs.argtypes = [cp]
        lib.orc_nvs.restype = ctypes.c_int64
        lib.orc_plan.argtypes = [cp, vp, ctypes.POINTER(_PlanOut)]
        lib.orc_plan.restype = ctypes.c_int
        lib.orc_dispatch.argtypes = [cp, vp, vp, vp]
        lib.orc_dispatch.restype = None
        lib.orc_combine_tokens.argtypes = [cp, vp, vp, vp, vp, ctypes.c_int64, vp]
        lib.orc_combine_tokens.restype = None
        lib.orc_combine_backward_tokens.argtypes = [cp, vp, vp, vp, vp, vp, ctypes.c_int64, vp, vp]
        lib.orc_combine_backward_tokens.restype = None
        lib.orc_reduce_grad.argtypes = [cp, vp, vp, vp, ctypes.c_int32, vp, vp, ctypes.c_int64]
        lib.orc_reduce_grad.restype = None
        lib.orc_reduce_grad_f32.argtypes = [cp, vp, vp, vp, ctypes.c_int32, vp, vp, ctypes.c_int64]
        lib.orc_reduce_grad_f32.restype = None
        lib.orc_dispatch_backward_tokens.argtypes = [cp, vp, vp, vp, ctypes.c_int64, vp]
        lib.orc_dispatch_backward_tokens.restype = None
        lib.orc_prefetch_weight.argtypes = [cp, vp, vp, vp, ctypes.c_int32, vp, vp, ctypes.c_int64]
        lib.orc_prefetch_weight.restype = None
        lib.orc_segment_weights.argtypes = [cp, vp, vp, vp, ctypes.c_int64, vp, vp]
        lib.orc_segment_weights.restype = None
        lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.orc_f32_to_bf16.restype = ctypes.c_uint16
        lib.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_f32.restype = ctypes.c_float
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def nvs(cfg: Config) -> int:
    return int(_L().orc_nvs(ctypes.byref(cfg)))


def plan(cfg: Config, topk_idx: np.ndarray) -> Tuple[int, Dict[str, np.ndarray]]:
    """Run the plan.  Returns (status, tables); tables hold the valid prefix of each."""
    R, E, K, S, B = cfg.R, cfg.E, cfg.K, cfg.S, cfg.budget
    n_pairs = R * S * K
    NvS = nvs(cfg) if R > 0 and cfg.align >= 1 else 0
    sizes = dict(expert_count=E, rank_load=R, overflow=R, deficit=R, n_seg=R, seg_expert=R * E,
                 seg_start=R * E, seg_len=R * E, seg_kind=R * E, seg_wslot=R * E, n_piece=1,
                 piece_expert=E + R, piece_rank=E + R, piece_start=E + R, piece_len=E + R,
                 piece_wslot=E + R, piece_ostart=E + R, rep_expert=max(R * B, 1), n_remote=1,
                 slot_of=max(n_pairs, 1), slot_src=max(R * NvS, 1))
    arrs = {k: np.full(max(v, 1), -7, dtype=np.int32) for k, v in sizes.items()}
    out = _PlanOut(**{k: a.ctypes.data_as(_I32P) for k, a in arrs.items()})
    idx = _c(topk_idx, np.int32).ravel()
    st = int(_L().orc_plan(ctypes.byref(cfg), _p(idx), ctypes.byref(out)))
    arrs["slot_of"] = arrs["slot_of"][:n_pairs]
    arrs["slot_src"] = arrs["slot_src"][:R * NvS]
    arrs["rep_expert"] = arrs["rep_expert"][:R * B]
    np_ = int(arrs["n_piece"][0]) if st in (OK, BUDGET) else 0
    for k in ("piece_expert", "piece_rank", "piece_start", "piece_len", "piece_wslot",
              "piece_ostart"):
        arrs[k] = arrs[k][:np_]
    for k in ("seg_expert", "seg_start", "seg_len", "seg_kind", "seg_wslot"):
        arrs[k] = arrs[k].reshape(R, E)
    arrs["nvs"] = np.array([NvS], np.int64)
    return st, arrs


def dispatch(cfg: Config, slot_of: np.ndarray, x: np.ndarray, recv: Optional[np.ndarray] = None
             ) -> np.ndarray:
    """recv[slot_of[p]] = x[p // K]; ``recv`` (uint16 [R*NvS, H]) is updated in place."""
    NvS = nvs(cfg)
    if recv is None:
        recv = np.zeros((cfg.R * NvS, cfg.H), np.uint16)
    s = _c(slot_of, np.int32)
    xx = _c(x, np.uint16)
    _L().orc_dispatch(ctypes.byref(cfg), _p(s), _p(xx), _p(recv))
    return recv


def combine(cfg: Config, slot_of: np.ndarray, y: np.ndarray, gates: np.ndarray,
            tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """bf16 bits [n_tokens, H] of sum_k w_k y[slot_k] for the listed tokens (all if None)."""
    s = _c(slot_of, np.int32)
    g = _c(gates, np.float32)
    yy = _c(y, np.uint16)
    n = cfg.R * cfg.S if tokens is None else len(tokens)
    tk = None if tokens is None else _c(tokens, np.int64)
    out = np.zeros((n, cfg.H), np.uint16)
    _L().orc_combine_tokens(ctypes.byref(cfg), _p(s), _p(yy), _p(g), _p(tk), n, _p(out))
    return out


def combine_backward(cfg: Config, slot_of: np.ndarray, dout: np.ndarray, y: np.ndarray,
                     gates: np.ndarray, tokens: Optional[np.ndarray] = None
                     ) -> Tuple[np.ndarray, np.ndarray]:
    """(dY rows bf16 [n_tokens, K, H], dgates fp32 [n_tokens, K]) for the listed tokens."""
    s = _c(slot_of, np.int32)
    g = _c(gates, np.float32)
    d = _c(dout, np.uint16)
    yy = _c(y, np.uint16)
    n = cfg.R * cfg.S if tokens is None else len(tokens)
    tk = None if tokens is None else _c(tokens, np.int64)
    dy = np.zeros((n, cfg.K, cfg.H), np.uint16)
    dg = np.zeros((n, cfg.K), np.float32)
    _L().orc_combine_backward_tokens(ctypes.byref(cfg), _p(s), _p(d), _p(yy), _p(g), _p(tk), n,
                                     _p(dy), _p(dg))
    return dy, dg


def reduce_grad(cfg: Config, tables: Dict[str, np.ndarray], rep: np.ndarray, home: np.ndarray,
                inplace: bool = False) -> np.ndarray:
    """New home gradients (bf16 bits [E, P]); ``rep`` is [R, budget, P].  With
    ``inplace`` the result is written into ``home`` itself (a C-contiguous uint16
    array) instead of a copy."""
    if not (inplace and isinstance(home, np.ndarray) and home.dtype == np.uint16
            and home.flags["C_CONTIGUOUS"] and home.flags["WRITEABLE"]):
        home = np.array(home, dtype=np.uint16, copy=True, order="C")
    rep = _c(rep, np.uint16)
    P = home.shape[-1]
    pe = _c(tables["piece_expert"], np.int32)
    pr = _c(tables["piece_rank"], np.int32)
    pw = _c(tables["piece_wslot"], np.int32)
    _L().orc_reduce_grad(ctypes.byref(cfg), _p(pe), _p(pr), _p(pw), len(pe), _p(rep), _p(home), P)
    return home


def reduce_grad_f32(cfg: Config, tables: Dict[str, np.ndarray], rep: np.ndarray,
                    home: np.ndarray) -> np.ndarray:
    """New fp32 home gradients [E, P] (a copy); ``rep`` is fp32 [R, budget, P]: the
    replica pieces added into their home expert in fp32, in plan order."""
    home = np.array(home, dtype=np.float32, copy=True, order="C")
    rep = _c(rep, np.float32)
    P = home.shape[-1]
    pe = _c(tables["piece_expert"], np.int32)
    pr = _c(tables["piece_rank"], np.int32)
    pw = _c(tables["piece_wslot"], np.int32)
    _L().orc_reduce_grad_f32(ctypes.byref(cfg), _p(pe), _p(pr), _p(pw), len(pe), _p(rep), _p(home), P)
    return home


def dispatch_backward(cfg: Config, slot_of: np.ndarray, drecv: np.ndarray,
                      tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """bf16 bits [n_tokens, H] of sum_k dRecv[slot_k] (fp32, k order) for the listed tokens."""
    s = _c(slot_of, np.int32)
    d = _c(drecv, np.uint16)
    n = cfg.R * cfg.S if tokens is None else len(tokens)
    tk = None if tokens is None else _c(tokens, np.int64)
    out = np.zeros((n, cfg.H), np.uint16)
    _L().orc_dispatch_backward_tokens(ctypes.byref(cfg), _p(s), _p(d), _p(tk), n, _p(out))
    return out


def prefetch_weight(cfg: Config, tables: Dict[str, np.ndarray], w: np.ndarray,
                    rep_w: np.ndarray, inplace: bool = False) -> np.ndarray:
    """Replica weight slots after the prefetch (bf16 bits [R, budget, W]); ``w`` is [E, W].
    With ``inplace`` the slots are written into ``rep_w`` itself (C-contiguous uint16)."""
    if not (inplace and isinstance(rep_w, np.ndarray) and rep_w.dtype == np.uint16
            and rep_w.flags["C_CONTIGUOUS"] and rep_w.flags["WRITEABLE"]):
        rep_w = np.array(rep_w, dtype=np.uint16, copy=True, order="C")
    ww = _c(w, np.uint16)
    pe = _c(tables["piece_expert"], np.int32)
    pr = _c(tables["piece_rank"], np.int32)
    pw = _c(tables["piece_wslot"], np.int32)
    _L().orc_prefetch_weight(ctypes.byref(cfg), _p(pe), _p(pr), _p(pw), len(pe), _p(ww), _p(rep_w),
                             ww.shape[-1])
    return rep_w


def segment_weights(cfg: Config, tables: Dict[str, np.ndarray], W: int
                    ) -> Tuple[np.ndarray, np.ndarray]:
    """The weight matrix of every segment-table entry: (buf, off), both [R, E]; buf 0 is
    the home weights [E, W], 1 the replica slots [R, budget, W], -1 none; off the first
    element of the matrix in that buffer, -1 for none."""
    R, E = cfg.R, cfg.E
    se = _c(tables["seg_expert"], np.int32)
    sk = _c(tables["seg_kind"], np.int32)
    sw = _c(tables["seg_wslot"], np.int32)
    buf = np.empty((R, E), np.int32)
    off = np.empty((R, E), np.int64)
    _L().orc_segment_weights(ctypes.byref(cfg), _p(se), _p(sk), _p(sw), int(W), _p(buf), _p(off))
    return buf, off


def f32_to_bf16(v: float) -> int:
    return int(_L().orc_f32_to_bf16(float(v)))


def bf16_to_f32(b: int) -> float:
    return float(_L().orc_bf16_to_f32(int(b)))

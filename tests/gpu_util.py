"""Helpers for the GPU parity tests: move numpy inputs to the device, run the
C-ABI calls through the binding, read results back, compare with the oracle."""
from __future__ import annotations

import numpy as np

import oracle

POISON = 0xFFC1  # a bf16 NaN pattern no kernel writes


def dev():
    import torch
    return torch.device("cuda:0")


def to_dev(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(dev())


def to_np(t, dtype=None) -> np.ndarray:
    a = t.detach().cpu().numpy()
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    return a if dtype is None else a.astype(dtype)


def configs(R, E, K, S, H=8, budget=None, mode=0, align=1):
    import token_dispatch_moonep_b200 as me
    if budget is None:
        budget = E // R
    kw = dict(R=R, E=E, K=K, S=S, H=H, budget=budget, mode=mode, align=align)
    return me.Config(**kw), oracle.Config(**kw)


def gpu_plan(cfg, idx_np):
    """Run moonep_plan twice on one workspace; returns the second call's (dev_status int,
    arena tensor, views dict of numpy, idx tensor).

    The first launch on a workspace finds no expert totals zeroed for it and sums every
    chunk's histogram row; every later launch reads the totals the chunks added by atomics
    (the steady state of a caller).  Both must give the same plan bit for bit, and the
    second is the one the caller compares with the oracle."""
    import torch
    import token_dispatch_moonep_b200 as me
    arena, ws, status = me.alloc_plan(cfg)
    # poison the arena and workspace so nothing depends on stale contents
    arena.fill_(0xA5)
    ws.fill_(0x5A)
    idx = to_dev(np.ascontiguousarray(idx_np, np.int32).ravel())

    def run(st):
        me.moonep_plan(cfg, idx if idx.numel() else None, arena, ws, st)
        torch.cuda.synchronize()
        return int(st.item()), {k: (to_np(v) if not isinstance(v, int) else v)
                                for k, v in me.moonep_plan_view(cfg, arena).items()}

    st1, first = run(status)
    st2, views = run(torch.zeros_like(status))
    assert st1 == st2, (st1, st2)
    for k, v in views.items():
        assert np.array_equal(first[k], v), k
    return st2, arena, views, idx


def compare_plans(cfg, ostatus, ot, gstatus, gv):
    """Bit-exact comparison of every plan table the oracle defines."""
    import token_dispatch_moonep_b200 as me
    R, E, B = cfg.R, cfg.E, cfg.budget
    exp_bits = me.DEV_BUDGET if ostatus == oracle.BUDGET else 0
    assert gstatus == exp_bits, (gstatus, ostatus)
    for k in ("expert_count", "rank_load", "overflow", "deficit", "n_seg", "slot_of", "slot_src",
              "rep_expert"):
        assert np.array_equal(gv[k], ot[k]), k
    for k in ("seg_expert", "seg_start", "seg_len", "seg_kind", "seg_wslot"):
        assert np.array_equal(gv[k].reshape(R, E), ot[k]), k
    n_piece = int(ot["n_piece"][0])
    sc = gv["scalars"]
    assert sc[0] == n_piece and sc[1] == int(ot["n_remote"][0])
    assert sc[2] == n_piece - int(ot["n_remote"][0])
    for k in ("piece_expert", "piece_rank", "piece_start", "piece_len", "piece_wslot",
              "piece_ostart"):
        assert np.array_equal(gv[k][:n_piece], ot[k]), k
    # tables the oracle does not spell out, derived from its piece table
    pe = ot["piece_expert"]
    for e in range(E):
        mine = np.nonzero(pe == e)[0]
        b, en = gv["expert_piece_begin"][e], gv["expert_piece_end"][e]
        if mine.size:
            assert b == mine[0] and en == mine[-1] + 1
        else:
            assert b == en
    local = np.unique(pe[ot["piece_wslot"] >= 0]) if n_piece else np.zeros(0, np.int32)
    assert sc[3] == local.size
    assert np.array_equal(gv["replicated_experts"][:local.size], local)


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / max |ref| (norm-relative, fp64)."""
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    if r.size == 0:
        return 0.0
    den = np.abs(r).max()
    return float(np.abs(g - r).max() / (den if den > 0 else 1.0))

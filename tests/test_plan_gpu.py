"""GPU plan vs the CPU oracle: every table bit-exact.

Covers the small parity workload, tiny random shapes (R in {1,2,3,8}, E/R in
{1,2,4}, alignment in {1,16,128}, budgets down to 0, TRAIN and INFER, skew from
uniform to every token on one expert), ragged histogram chunks, the maximum
expert count, empty batches, bad expert ids, and the full-size workloads.
"""
import numpy as np
import pytest

import oracle
from moonep_inputs import WORKLOADS, make_routing, uniform_routing
from tests.gpu_util import compare_plans, configs, gpu_plan

pytestmark = pytest.mark.gpu


def _run(R, E, K, S, idx, budget=None, mode=0, align=1):
    cfg, ocfg = configs(R, E, K, S, budget=budget, mode=mode, align=align)
    ost, ot = oracle.plan(ocfg, idx)
    gst, arena, gv, _ = gpu_plan(cfg, idx)
    compare_plans(cfg, ost, ot, gst, gv)
    return ot, gv


def test_worked_example():
    idx = np.array([[[0, 1], [0, 1], [1, 2]], [[0, 1], [0, 3], [1, 2]]], np.int32)
    _run(2, 4, 2, 3, idx, budget=2)
    _run(2, 4, 2, 3, idx, budget=2, align=4)
    _run(2, 4, 2, 3, idx, budget=0, mode=1)


def test_small_workload():
    w = WORKLOADS["ep8_e32_k4_s256_h512"]
    for mv in (0.2, 1.0, 5.0, 20.0):
        idx, _, _ = make_routing(w.R, w.E, w.K, w.S, mv, seed=0)
        _run(w.R, w.E, w.K, w.S, idx, budget=w.budget, mode=w.mode)


def _random_cases():
    rng = np.random.default_rng(1234)
    cases = []
    for R in (1, 2, 3, 8):
        for L in (1, 2, 4):
            E = R * L
            for align in (1, 16, 128):
                K = int(rng.integers(1, min(E, 8) + 1))
                S = int(rng.integers(0, 65))
                B = int(rng.integers(0, L + 1))
                mode = int(rng.integers(0, 2))
                skew = ["uniform", "zipf", "first", "last"][int(rng.integers(0, 4))]
                cases.append((R, E, K, S, B, mode, align, skew))
    return cases


@pytest.mark.parametrize("case", _random_cases())
def test_random_tiny(case):
    R, E, K, S, B, mode, align, skew = case
    if skew == "uniform" or S == 0:
        idx = uniform_routing(R, E, K, S, seed=S + E)
    elif skew == "zipf":
        idx, _, _ = make_routing(R, E, K, S, min(3.0, E / K - 1.01) if E > K else 0.1, seed=S)
    elif skew == "first":
        idx = np.tile(np.arange(K, dtype=np.int32), (R, S, 1))
    else:
        idx = np.tile(np.arange(E - K, E, dtype=np.int32), (R, S, 1))
    _run(R, E, K, S, idx.astype(np.int32), budget=B, mode=mode, align=align)


@pytest.mark.parametrize("S", [300, 1025, 4097])
def test_ragged_chunks(S):
    # 8 ranks x S tokens x 8 picks: several 8192-pair chunks and a ragged tail
    idx, _, _ = make_routing(8, 64, 8, S, 6.0, seed=S)
    _run(8, 64, 8, S, idx, budget=8)


def test_repeated_experts_within_a_token():
    idx = uniform_routing(4, 8, 3, 50, seed=5, distinct=False)
    _run(4, 8, 3, 50, idx, budget=1, mode=1, align=2)


def test_maximum_sizes():
    # 1024 experts on 8 ranks, top-32 (MAX_TOPK)
    idx, _, _ = make_routing(8, 1024, 32, 64, 5.0, seed=3)
    _run(8, 1024, 32, 64, idx, budget=128)
    # 1024 ranks with one expert each
    idx = np.zeros((1024, 3, 1), np.int32)
    idx[:, 1, 0] = np.arange(1024)
    _run(1024, 1024, 1, 3, idx, budget=1, mode=1)
    # everything on one expert at scale, alignment 128
    idx = np.zeros((8, 2048, 1), np.int32)
    _run(8, 64, 1, 2048, idx, budget=8, align=128)


def test_empty_batch():
    _run(4, 16, 2, 0, np.zeros((4, 0, 2), np.int32), budget=4)


def test_bad_expert_id_sets_status_and_invalidates_plan():
    import token_dispatch_moonep_b200 as me
    cfg, _ = configs(4, 16, 2, 40)
    idx = uniform_routing(4, 16, 2, 40, seed=1)
    idx[2, 7, 1] = 16
    st, arena, gv, _ = gpu_plan(cfg, idx)
    assert st & me.DEV_BAD_EXPERT_ID
    assert (gv["slot_of"] == -1).all() and (gv["slot_src"] == -1).all()
    idx[2, 7, 1] = -3
    st, arena, gv, _ = gpu_plan(cfg, idx)
    assert st & me.DEV_BAD_EXPERT_ID


def test_bad_expert_id_in_the_first_chunk_of_a_large_plan():
    """A bad id in chunk 0 of 128: every CTA still arrives before the solver moves
    on, so the status is exactly BAD_EXPERT_ID (no timeout) and the plan is invalid."""
    import token_dispatch_moonep_b200 as me
    R, E, K, S = 8, 64, 8, 2048
    cfg, _ = configs(R, E, K, S)
    idx, _, _ = make_routing(R, E, K, S, 3.0, seed=12)
    idx[0, 0, 0] = E + 5
    st, arena, gv, _ = gpu_plan(cfg, idx)
    assert st == me.DEV_BAD_EXPERT_ID
    assert (gv["slot_of"] == -1).all() and (gv["slot_src"] == -1).all()


def test_budget_flag_only_in_training_mode():
    import token_dispatch_moonep_b200 as me
    idx = np.zeros((4, 10, 1), np.int32)  # expert 0 overflows onto 3 ranks
    cfg, _ = configs(4, 8, 1, 10, budget=0, mode=0)
    st, _, gv, _ = gpu_plan(cfg, idx)
    assert st == me.DEV_BUDGET and gv["scalars"][1] == 3
    cfg, _ = configs(4, 8, 1, 10, budget=0, mode=1)
    st, _, gv, _ = gpu_plan(cfg, idx)
    assert st == 0 and gv["scalars"][1] == 3


def test_plan_is_deterministic_across_runs():
    idx, _, _ = make_routing(8, 256, 8, 512, 10.0, seed=7)
    cfg, _ = configs(8, 256, 8, 512)
    _, _, a, _ = gpu_plan(cfg, idx)
    _, _, b, _ = gpu_plan(cfg, idx)
    for k in a:
        if not isinstance(a[k], int):
            assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("name,mv,seed", [
    ("ep8_e256_k8_s4096_h7168", 0.2, 0),
    ("ep8_e256_k8_s4096_h7168_sweep", 20.0, 4),
    ("ep8_e384_k8_s8192_h7168_bwd", 20.0, 0),
    ("ep64_e256_k8_s128_h7168_decode", 1.0, 0),
    ("ep64_e256_k8_s128_h7168_decode", 20.0, 0),
])
def test_full_size_plans(name, mv, seed):
    w = WORKLOADS[name]
    idx, _, _ = make_routing(w.R, w.E, w.K, w.S, mv, seed=seed)
    ot, gv = _run(w.R, w.E, w.K, w.S, idx, budget=w.budget, mode=w.mode)
    if w.mode == 1 and mv >= 20:
        assert int(ot["n_remote"][0]) > 0  # the remote-read path is exercised


def test_several_chunks_per_cta():
    # 1.28M pairs = 157 chunks of 8192: more chunks than co-resident CTAs
    idx, _, _ = make_routing(8, 64, 8, 20000, 4.0, seed=9)
    _run(8, 64, 8, 20000, idx, budget=8)


def test_workspace_reuse_with_arbitrary_contents():
    import torch
    import token_dispatch_moonep_b200 as me
    cfg, ocfg = configs(8, 256, 8, 512)
    arena, ws, _ = me.alloc_plan(cfg)
    for fill, (mv, seed) in [(0x00, (0.2, 0)), (0xFF, (5.0, 1)), (0xA5, (20.0, 2)), (None, (1.0, 3)),
                             (None, (1.0, 3))]:
        if fill is not None:
            ws.fill_(fill)
        idx, _, _ = make_routing(8, 256, 8, 512, mv, seed=seed)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        me.moonep_plan(cfg, torch.from_numpy(idx.ravel().copy()).cuda(), arena, ws, st)
        torch.cuda.synchronize()
        ost, ot = oracle.plan(ocfg, idx)
        gv = {k: (v.cpu().numpy() if not isinstance(v, int) else v)
              for k, v in me.moonep_plan_view(cfg, arena).items()}
        compare_plans(cfg, ost, ot, int(st.item()), gv)


def test_forced_timeout_reports_status_and_context_stays_usable():
    """A wait that runs out (an arrival nothing makes) ends the kernel with TIMEOUT."""
    import torch
    import token_dispatch_moonep_b200 as me
    cfg, ocfg = configs(8, 64, 8, 3000)
    idx, _, _ = make_routing(8, 64, 8, 3000, 3.0, seed=4)
    try:
        me.moonep_debug_set_wait(2_000_000, 1)  # 2 ms, one phantom arrival
        st, _, gv, _ = gpu_plan(cfg, idx)
        assert st & me.DEV_TIMEOUT
        assert (gv["slot_of"] == -1).all() and (gv["slot_src"] == -1).all()
    finally:
        me.moonep_debug_set_wait(me.DEFAULT_WAIT_NS, 0)
    # the context is intact and the next plan is correct
    ost, ot = oracle.plan(ocfg, idx)
    st, _, gv, _ = gpu_plan(cfg, idx)
    compare_plans(cfg, ost, ot, st, gv)


def test_plan_replayed_from_a_cuda_graph():
    """Graph replays reuse the kernel's arguments; the launch epoch must still advance."""
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S = 8, 256, 8, 1024
    cfg, ocfg = configs(R, E, K, S)
    arena, ws, st = me.alloc_plan(cfg)
    idx_dev = torch.zeros(R * S * K, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        me.moonep_plan(cfg, idx_dev, arena, ws, st, stream=s)  # warm up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        me.moonep_plan(cfg, idx_dev, arena, ws, st, stream=s)
    for mv, seed in [(0.2, 0), (20.0, 1), (5.0, 2), (5.0, 2)]:
        idx, _, _ = make_routing(R, E, K, S, mv, seed=seed)
        idx_dev.copy_(torch.from_numpy(idx.ravel().copy()))
        st.zero_()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        ost, ot = oracle.plan(ocfg, idx)
        gv = {k: (v.cpu().numpy() if not isinstance(v, int) else v)
              for k, v in me.moonep_plan_view(cfg, arena).items()}
        compare_plans(cfg, ost, ot, int(st.item()), gv)
    del g

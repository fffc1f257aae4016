"""The allocation-free plan entry point, moonep_plan_static.

Some callers cannot allocate device memory themselves — a plugin inside another
engine that is only handed the tensors of one call, or a serving loop that
reserved all device memory up front and must not call cudaMalloc (which can
synchronise the device) while it runs.  For them the plan's scratch lives in a
fixed array inside the library.  These tests check that this entry point gives
exactly the plan the ordinary entry point gives with a caller workspace, call
after call, while the config changes between calls (so the scratch areas the
previous call left behind sit at other offsets), after a call whose bounded
wait ran out, and that configs too large for the array are refused.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

from moonep_inputs import make_routing


def test_too_large_for_the_static_scratch_is_refused():
    import token_dispatch_moonep_b200 as me
    # 8 ranks x 262144 tokens x 8 picks: 2M pairs need more scratch than the array holds
    cfg = me.Config(R=8, E=256, K=8, S=262144, H=8, budget=32)
    assert me.moonep_workspace_bytes(cfg) > me.STATIC_WORKSPACE_BYTES
    fake = 1 << 30  # refused on the host before any device work
    st = me._lib.moonep_plan_static(ctypes.byref(cfg), fake, fake, fake, None)
    assert st == me.ERR_UNSUPPORTED
    bad = me.Config(R=3, E=8, K=2, S=4, H=8, budget=1)
    assert me._lib.moonep_plan_static(ctypes.byref(bad), fake, fake, fake, None) == \
        me.ERR_INVALID_ARG


def _same_plan(me, cfg, arena_ref, arena_got, what):
    ref = me.moonep_plan_view(cfg, arena_ref)
    got = me.moonep_plan_view(cfg, arena_got)
    n_piece = int(ref["scalars"][0].item())
    for k, v in ref.items():
        if isinstance(v, int):
            assert got[k] == v, (what, k)
            continue
        a, b = v.cpu().numpy(), got[k].cpu().numpy()
        if k.startswith("piece_"):
            a, b = a[:n_piece], b[:n_piece]
        if k == "replicated_experts":
            m = int(ref["scalars"][3].item())
            a, b = a[:m], b[:m]
        assert np.array_equal(a, b), (what, k)


# (R, E, K, S, budget, mode, align, maxvio, seed): the small parity workload, the
# headline forward shape, the training-backward shape, the decode shape (64 ranks,
# inference, 4 slots, remote pieces), an aligned layout, then the first again
CALLS = [
    (8, 32, 4, 256, 4, 0, 1, 5.0, 0),
    (8, 256, 8, 4096, 32, 0, 1, 0.2, 0),
    (8, 384, 8, 8192, 48, 0, 1, 20.0, 1),
    (64, 256, 8, 128, 4, 1, 1, 20.0, 2),
    (8, 64, 8, 512, 8, 0, 16, 6.0, 3),
    (8, 32, 4, 256, 4, 0, 1, 5.0, 0),
]


@pytest.mark.gpu
def test_static_scratch_plan_equals_workspace_plan_call_after_call():
    import torch
    import token_dispatch_moonep_b200 as me
    for call, (R, E, K, S, B, mode, A, mv, seed) in enumerate(CALLS):
        cfg = me.Config(R=R, E=E, K=K, S=S, H=7168, budget=B, mode=mode, align=A)
        assert me.moonep_workspace_bytes(cfg) <= me.STATIC_WORKSPACE_BYTES
        idx_np, _, _ = make_routing(R, E, K, S, mv, seed=seed)
        idx = torch.from_numpy(idx_np.ravel().copy()).cuda()
        # the existing entry point with a caller-allocated workspace
        arena_ref, ws, st_ref = me.alloc_plan(cfg)
        me.moonep_plan(cfg, idx, arena_ref, ws, st_ref)
        # the allocation-free entry point, twice in a row on the same inputs
        for rep in range(2):
            arena = torch.full((me.moonep_plan_bytes(cfg),), 0xA5 - 256, dtype=torch.int8,
                               device="cuda").view(torch.uint8)
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            me.moonep_plan_static(cfg, idx, arena, st)
            torch.cuda.synchronize()
            assert int(st.item()) == int(st_ref.item()) == 0, (call, rep)
            _same_plan(me, cfg, arena_ref, arena, (call, rep))


@pytest.mark.gpu
def test_static_scratch_after_a_timed_out_call():
    """A call whose bounded wait runs out (an arrival nothing makes) leaves the shared
    array as it was at that moment; the next call must still give the exact plan."""
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, B = 8, 64, 8, 3000, 8
    cfg = me.Config(R=R, E=E, K=K, S=S, H=8, budget=B)
    idx_np, _, _ = make_routing(R, E, K, S, 3.0, seed=4)
    idx = torch.from_numpy(idx_np.ravel().copy()).cuda()
    arena = torch.empty(me.moonep_plan_bytes(cfg), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        me.moonep_debug_set_wait(2_000_000, 1)  # 2 ms, one phantom arrival
        me.moonep_plan_static(cfg, idx, arena, st)
        torch.cuda.synchronize()
        assert int(st.item()) & me.DEV_TIMEOUT
    finally:
        me.moonep_debug_set_wait(me.DEFAULT_WAIT_NS, 0)
    arena_ref, ws, st_ref = me.alloc_plan(cfg)
    me.moonep_plan(cfg, idx, arena_ref, ws, st_ref)
    st.zero_()
    me.moonep_plan_static(cfg, idx, arena, st)
    torch.cuda.synchronize()
    assert int(st.item()) == int(st_ref.item()) == 0
    _same_plan(me, cfg, arena_ref, arena, "after timeout")

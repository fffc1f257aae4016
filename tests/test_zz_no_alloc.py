"""The allocation-free plan entry point, moonep_plan_static.

Some callers cannot allocate device memory themselves — a plugin inside another
engine that is only handed the tensors of one call, or a serving loop that
reserved all device memory up front and must not call cudaMalloc (which can
synchronise the device) while it runs.  For them the plan's scratch lives in a
fixed array inside the library.  These tests check that this entry point gives
exactly the plan the ordinary entry point gives with a caller workspace, on two
calls in a row (so stale scratch contents from the first call would show in the
second), and that configs too large for the array are refused.

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


@pytest.mark.gpu
def test_static_scratch_plan_equals_workspace_plan_twice():
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, B = 8, 256, 8, 4096, 32
    cfg = me.Config(R=R, E=E, K=K, S=S, H=7168, budget=B)
    assert me.moonep_workspace_bytes(cfg) <= me.STATIC_WORKSPACE_BYTES
    arena_static = torch.empty(me.moonep_plan_bytes(cfg), dtype=torch.uint8, device="cuda")
    for call, (mv, seed) in enumerate([(0.2, 0), (20.0, 1)]):
        idx_np, _, _ = make_routing(R, E, K, S, mv, seed=seed)
        idx = torch.from_numpy(idx_np.ravel().copy()).cuda()
        # the existing entry point with a caller-allocated workspace
        arena_ref, ws, st_ref = me.alloc_plan(cfg)
        me.moonep_plan(cfg, idx, arena_ref, ws, st_ref)
        # the allocation-free entry point, same arena reused on both calls
        arena_static.fill_(0xA5)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        me.moonep_plan_static(cfg, idx, arena_static, st)
        torch.cuda.synchronize()
        assert int(st.item()) == int(st_ref.item()) == 0, call
        ref = me.moonep_plan_view(cfg, arena_ref)
        got = me.moonep_plan_view(cfg, arena_static)
        n_piece = int(ref["scalars"][0].item())
        for k, v in ref.items():
            if isinstance(v, int):
                assert got[k] == v
                continue
            a, b = v.cpu().numpy(), got[k].cpu().numpy()
            if k.startswith("piece_"):
                a, b = a[:n_piece], b[:n_piece]
            if k == "replicated_experts":
                m = int(ref["scalars"][3].item())
                a, b = a[:m], b[:m]
            assert np.array_equal(a, b), (call, k)

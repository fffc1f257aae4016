"""The fused forward layer (plan + dispatch + combine of the identity expert in one
launch) against the oracle and against the three separate calls.

Bar: every plan table bit-exact; dispatched rows bit-exact with padding untouched;
combine output bit-identical (the same fused multiply-adds in ascending k as the
oracle) and within the contract's 1e-3 norm-relative error.
"""
import numpy as np
import pytest

import oracle
from moonep_inputs import (WORKLOADS, bf16_bits_to_f32, make_gates, make_routing, make_x,
                           uniform_routing)
from tests.gpu_util import POISON, compare_plans, configs, rel_err, to_dev, to_np

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _fused(cfg, idx, gates, x, NvS, poison_recv=True):
    import torch
    import token_dispatch_moonep_b200 as me
    R, S, K, H = cfg.R, cfg.S, cfg.K, cfg.H
    arena, ws, st = me.alloc_plan(cfg)
    arena.fill_(0xA5)
    ws.fill_(0x5A)
    recv = torch.full((R * NvS, H), POISON - 65536, dtype=torch.int16, device="cuda")
    out = torch.full((R * S, H), 7, dtype=torch.int16, device="cuda")
    idx_d = to_dev(np.ascontiguousarray(idx, np.int32).ravel())
    me.moonep_fused_forward(cfg, idx_d if idx_d.numel() else None, to_dev(gates.ravel()),
                            to_dev(x), arena, ws, recv, out, st)
    torch.cuda.synchronize()
    views = {k: (to_np(v) if not isinstance(v, int) else v)
             for k, v in me.moonep_plan_view(cfg, arena).items()}
    return int(st.item()), views, to_np(recv), to_np(out)


SHAPES = [
    # R, E, K, S, H, budget, mode, align, skew
    (8, 32, 4, 256, 512, 4, 0, 1, 5.0),      # the small parity workload
    (2, 4, 2, 9, 24, 2, 0, 1, 1.0),
    (4, 16, 8, 33, 136, 4, 1, 16, 3.0),      # alignment 16, inference budget
    (8, 64, 8, 1200, 1032, 8, 0, 1, 6.0),    # several chunks, ragged vector tail
    (3, 9, 1, 700, 64, 1, 1, 4, 0.0),        # K = 1, uniform routing
    (64, 256, 8, 16, 7168, 4, 1, 1, 20.0),   # decode shape, remote pieces
    (4, 16, 2, 0, 64, 4, 0, 1, 1.0),         # empty batch
]


@pytest.mark.parametrize("shape", SHAPES)
def test_fused_forward_matches_oracle(shape):
    R, E, K, S, H, B, mode, A, mv = shape
    cfg, ocfg = configs(R, E, K, S, H=H, budget=B, mode=mode, align=A)
    if S == 0:
        idx = np.zeros((R, 0, K), np.int32)
    elif mv == 0.0:
        idx = uniform_routing(R, E, K, S, seed=S)
    else:
        idx, _, _ = make_routing(R, E, K, S, mv, seed=S)
    gates = make_gates(R, S, K, seed=7)
    x = make_x(R, S, H, seed=7).reshape(R * S, H)
    ost, ot = oracle.plan(ocfg, idx)
    NvS = int(ot["nvs"][0])
    st, gv, recv, out = _fused(cfg, idx, gates, x, NvS)
    compare_plans(cfg, ost, ot, st, gv)
    ref_recv = oracle.dispatch(ocfg, ot["slot_of"], x, np.full((R * NvS, H), POISON, np.uint16))
    assert np.array_equal(recv, ref_recv)
    if R * S == 0:
        return
    ref_out = oracle.combine(ocfg, ot["slot_of"], ref_recv, gates)
    assert rel_err(bf16_bits_to_f32(out), bf16_bits_to_f32(ref_out)) <= TOL
    assert np.array_equal(out, ref_out)


@pytest.mark.parametrize("mv", [1.0, 20.0])
def test_fused_forward_full_decode_size(mv):
    """64 ranks x 128 tokens x top-8 over 256 experts, H = 7168: the layer the fused call
    is for.  The plan is compared table by table; the dispatch buffer as a whole on the
    device; the combine output on a sample of 2048 tokens (every rank's first and last)."""
    import torch
    w = WORKLOADS["ep64_e256_k8_s128_h7168_decode"]
    R, E, K, S, H, B = w.R, w.E, w.K, w.S, w.H, w.budget
    T = R * S
    cfg, ocfg = configs(R, E, K, S, H=H, budget=B, mode=w.mode)
    idx, _, _ = make_routing(R, E, K, S, mv, seed=0)
    gates = make_gates(R, S, K, seed=0).reshape(T, K)
    x = make_x(R, S, H, seed=0).reshape(T, H)
    ost, ot = oracle.plan(ocfg, idx)
    NvS = int(ot["nvs"][0])
    st, gv, recv, out = _fused(cfg, idx, gates, x, NvS)
    compare_plans(cfg, ost, ot, st, gv)
    assert int(ot["n_remote"][0]) > 0
    src = ot["slot_src"]
    valid = src >= 0
    assert np.array_equal(recv[valid], x[src[valid] // K])
    assert (recv[~valid] == POISON).all()
    rng = np.random.default_rng(2)
    ends = np.unique(np.concatenate([np.arange(R) * S, np.arange(R) * S + S - 1]))
    toks = np.unique(np.concatenate([ends, rng.choice(T, 2048 - ends.size, replace=False)]))
    n = len(toks)
    c1 = oracle.Config(R=1, E=E, K=K, S=n, H=H, budget=B, mode=w.mode)
    ref = oracle.combine(c1, np.arange(n * K, dtype=np.int32), np.repeat(x[toks], K, axis=0),
                         gates[toks])
    assert rel_err(bf16_bits_to_f32(out[toks]), bf16_bits_to_f32(ref)) <= TOL
    assert np.array_equal(out[toks], ref)


def test_fused_forward_equals_separate_calls():
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, H, B = 8, 64, 8, 512, 1024, 8
    cfg, ocfg = configs(R, E, K, S, H=H, budget=B, mode=1)
    idx, _, _ = make_routing(R, E, K, S, 10.0, seed=3)
    gates = make_gates(R, S, K, seed=3)
    x = make_x(R, S, H, seed=3).reshape(R * S, H)
    NvS = me.moonep_nvs(cfg)
    st, gv, recv, out = _fused(cfg, idx, gates, x, NvS)
    arena, ws, st2 = me.alloc_plan(cfg)
    recv2 = torch.full((R * NvS, H), POISON - 65536, dtype=torch.int16, device="cuda")
    out2 = torch.empty((R * S, H), dtype=torch.int16, device="cuda")
    g_d, x_d = to_dev(gates.ravel()), to_dev(x)
    me.moonep_plan(cfg, to_dev(idx.ravel()), arena, ws, st2)
    me.moonep_dispatch(cfg, arena, x_d, recv2, st2)
    me.moonep_combine(cfg, arena, recv2, g_d, out2, st2)
    torch.cuda.synchronize()
    assert st == int(st2.item()) == 0
    assert np.array_equal(recv, to_np(recv2))
    assert np.array_equal(out, to_np(out2))
    sep = {k: (to_np(v) if not isinstance(v, int) else v)
           for k, v in me.moonep_plan_view(cfg, arena).items()}
    n_piece = int(sep["scalars"][0])
    for k, v in sep.items():
        if isinstance(v, int):
            continue
        a, b = v, gv[k]
        if k.startswith("piece_"):
            a, b = a[:n_piece], b[:n_piece]
        if k == "replicated_experts":
            a, b = a[:int(sep["scalars"][3])], b[:int(sep["scalars"][3])]
        assert np.array_equal(a, b), k


def test_fused_forward_bad_expert_id_dispatches_nothing():
    import token_dispatch_moonep_b200 as me
    R, E, K, S, H = 4, 16, 2, 40, 64
    cfg, ocfg = configs(R, E, K, S, H=H, budget=4)
    idx = uniform_routing(R, E, K, S, seed=1)
    idx[1, 3, 0] = E + 2
    gates = make_gates(R, S, K, seed=1)
    x = make_x(R, S, H, seed=1).reshape(R * S, H)
    st, gv, recv, out = _fused(cfg, idx, gates, x, me.moonep_nvs(cfg))
    assert st & me.DEV_BAD_EXPERT_ID
    assert (gv["slot_of"] == -1).all() and (gv["slot_src"] == -1).all()
    assert (recv == POISON).all()
    assert (out == 0).all()

"""GPU dispatch / combine / combine-backward / reduce_grad vs the CPU oracle.

Bar: dispatched rows bit-exact (and padding rows untouched); combine,
combine-backward and reduce_grad within 1e-3 norm-relative error
(max |gpu - ref| / max |ref|) with fp32 accumulation.  Where both sides round
the same fp32 value, computed with the same operations in the same order
(combine: fused multiply-adds in ascending k; dY: one product;
dispatch-backward: additions in ascending k; reduce_grad: additions in piece
order), the results must also be bit-identical.  dgate (an fp32 dot product
on the GPU, fp64 in the oracle) is held to 1e-3 only.
"""
import numpy as np
import pytest

import oracle
from moonep_inputs import (WORKLOADS, bf16_bits_to_f32, integer_bf16, make_gates, make_routing,
                           make_x, normal_bf16, uniform_routing)
from tests.gpu_util import POISON, configs, gpu_plan, rel_err, to_dev, to_np

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _exact(got, ref):
    """The contract's 1e-3 norm-relative bar, and bit-identity (same fp32 steps)."""
    assert rel_err(bf16_bits_to_f32(got), bf16_bits_to_f32(ref)) <= TOL
    assert np.array_equal(got, ref), int((got != ref).sum())


def _setup(R, E, K, S, H, mv=3.0, seed=0, budget=None, mode=0, align=1):
    cfg, ocfg = configs(R, E, K, S, H=H, budget=budget, mode=mode, align=align)
    if S == 0:
        idx = np.zeros((R, 0, K), np.int32)
    elif E > K:
        idx, _, _ = make_routing(R, E, K, S, mv, seed=seed)
    else:
        idx = uniform_routing(R, E, K, S, seed=seed)
    ost, ot = oracle.plan(ocfg, idx)
    gst, arena, gv, _ = gpu_plan(cfg, idx)
    assert np.array_equal(gv["slot_of"], ot["slot_of"])
    return cfg, ocfg, ot, arena


def _dispatch(cfg, arena, x_np, NvS, offset_elems=0):
    """Run dispatch into a poisoned buffer; offset_elems shifts the buffers (alignment tests)."""
    import torch
    import token_dispatch_moonep_b200 as me
    H = cfg.H
    nrows = cfg.R * NvS
    xs = to_dev(np.concatenate([np.zeros(offset_elems, np.uint16), x_np.ravel()]))
    x = xs[offset_elems:]
    rb = torch.full((nrows * H + offset_elems,), POISON - 65536,
                    dtype=torch.int16, device=x.device)
    recv = rb[offset_elems:]
    status = torch.zeros(1, dtype=torch.int32, device=x.device)
    me.moonep_dispatch(cfg, arena, x, recv, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return to_np(recv).reshape(nrows, H)


SHAPES = [
    # R, E, K, S, H, align
    (8, 32, 4, 256, 512, 1),     # the small parity workload
    (2, 4, 2, 9, 24, 1),
    (4, 16, 8, 33, 136, 16),
    (3, 9, 3, 17, 13, 4),        # H not a multiple of 8: scalar path
    (1, 4, 2, 5, 8, 1),
    (8, 64, 6, 40, 1, 1),        # H = 1
    (4, 16, 2, 0, 64, 1),        # empty batch
    (8, 64, 8, 1200, 1032, 1),   # several blocks, ragged vector tail (129 vectors per row)
    (4, 32, 12, 20, 64, 1),      # K > 8: the k-at-a-time kernels
    (2, 64, 32, 9, 40, 1),       # K = MAX_TOPK
]


@pytest.mark.parametrize("shape", SHAPES)
def test_dispatch_bitwise(shape):
    R, E, K, S, H, A = shape
    cfg, ocfg, ot, arena = _setup(R, E, K, S, H, align=A)
    NvS = int(ot["nvs"][0])
    x = make_x(R, S, H, seed=1).reshape(R * S, H)
    got = _dispatch(cfg, arena, x, NvS)
    ref = oracle.dispatch(ocfg, ot["slot_of"], x,
                          np.full((R * NvS, H), POISON, np.uint16))
    assert np.array_equal(got, ref)
    # every valid row written exactly once with its source row, padding untouched
    valid = ot["slot_src"] >= 0
    assert (got[~valid] == POISON).all()


def test_dispatch_misaligned_buffers_take_the_scalar_path():
    cfg, ocfg, ot, arena = _setup(4, 16, 4, 20, 64)
    NvS = int(ot["nvs"][0])
    x = make_x(4, 20, 64, seed=2).reshape(80, 64)
    got = _dispatch(cfg, arena, x, NvS, offset_elems=1)
    ref = oracle.dispatch(ocfg, ot["slot_of"], x, np.full((4 * NvS, 64), POISON, np.uint16))
    assert np.array_equal(got, ref)


def _combine(cfg, arena, y_np, w_np):
    import torch
    import token_dispatch_moonep_b200 as me
    y = to_dev(y_np)
    w = to_dev(w_np.astype(np.float32).ravel())
    out = torch.empty((cfg.R * cfg.S, cfg.H), dtype=torch.int16, device=y.device)
    status = torch.zeros(1, dtype=torch.int32, device=y.device)
    me.moonep_combine(cfg, arena, y, w, out, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return to_np(out)


@pytest.mark.parametrize("shape", SHAPES)
def test_combine_matches_oracle(shape):
    R, E, K, S, H, A = shape
    cfg, ocfg, ot, arena = _setup(R, E, K, S, H, align=A, seed=3)
    NvS = int(ot["nvs"][0])
    y = normal_bf16((R * NvS, H), seed=3, stream=9)
    w = make_gates(R, S, K, seed=3)
    got = _combine(cfg, arena, y, w)
    ref = oracle.combine(ocfg, ot["slot_of"], y, w)
    if ref.size == 0:
        assert got.size == 0
        return
    _exact(got, ref)


@pytest.mark.parametrize("shape", SHAPES[:3])
def test_round_trip_identity_expert(shape):
    """dispatch -> identity expert -> combine == sum_k w_k x (§8 exercise C)."""
    R, E, K, S, H, A = shape
    cfg, ocfg, ot, arena = _setup(R, E, K, S, H, align=A, seed=4)
    NvS = int(ot["nvs"][0])
    x = make_x(R, S, H, seed=4).reshape(R * S, H)
    recv = _dispatch(cfg, arena, x, NvS)
    w = make_gates(R, S, K, seed=4)
    got = _combine(cfg, arena, recv, w)
    ref = oracle.combine(ocfg, ot["slot_of"], oracle.dispatch(ocfg, ot["slot_of"], x), w)
    _exact(got, ref)
    exact = w.reshape(R * S, K).astype(np.float64).sum(1, keepdims=True) * bf16_bits_to_f32(x)
    assert rel_err(bf16_bits_to_f32(got), exact) <= 2 ** -7


def _combine_bwd(cfg, arena, dout_np, y_np, w_np, NvS):
    import torch
    import token_dispatch_moonep_b200 as me
    dout = to_dev(dout_np)
    y = to_dev(y_np)
    w = to_dev(w_np.astype(np.float32).ravel())
    dy = torch.full((cfg.R * NvS, cfg.H), POISON - 65536,
                    dtype=torch.int16, device=y.device)
    dg = torch.full((cfg.R * cfg.S * cfg.K,), float("nan"), dtype=torch.float32, device=y.device)
    status = torch.zeros(1, dtype=torch.int32, device=y.device)
    me.moonep_combine_backward(cfg, arena, dout, y, w, dy, dg, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return to_np(dy), to_np(dg)


@pytest.mark.parametrize("shape", SHAPES)
def test_combine_backward_matches_oracle(shape):
    R, E, K, S, H, A = shape
    cfg, ocfg, ot, arena = _setup(R, E, K, S, H, align=A, seed=5)
    NvS = int(ot["nvs"][0])
    y = normal_bf16((R * NvS, H), seed=5, stream=9)
    dout = normal_bf16((R * S, H), seed=5, stream=3)
    w = make_gates(R, S, K, seed=5)
    dy, dg = _combine_bwd(cfg, arena, dout, y, w, NvS)
    ref_dy, ref_dg = oracle.combine_backward(ocfg, ot["slot_of"], dout, y, w)
    if R * S == 0:
        return
    so = ot["slot_of"]
    got_rows = dy[so].reshape(R * S, K, H)
    _exact(got_rows, ref_dy)
    assert (dy[ot["slot_src"] < 0] == POISON).all()
    assert rel_err(dg.reshape(R * S, K), ref_dg) <= TOL


def _reduce(cfg, arena, rep_np, home_np, P):
    import torch
    import token_dispatch_moonep_b200 as me
    rep = to_dev(rep_np)
    home = to_dev(home_np)
    status = torch.zeros(1, dtype=torch.int32, device=home.device)
    me.moonep_reduce_grad(cfg, arena, rep, home, P, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return to_np(home)


@pytest.mark.parametrize("shape", [(8, 32, 4, 256, 4, 2048), (4, 16, 2, 40, 3, 13),
                                   (8, 64, 8, 64, 8, 1000), (2, 8, 2, 30, 1, 8)])
def test_reduce_grad_matches_oracle(shape):
    R, E, K, S, B, P = shape
    cfg, ocfg, ot, arena = _setup(R, E, K, S, 8, mv=6.0, seed=6, budget=B)
    assert int(ot["n_piece"][0]) > 0
    rep = normal_bf16((R, B, P), seed=6, stream=11)
    home = normal_bf16((E, P), seed=6, stream=12)
    got = _reduce(cfg, arena, rep, home, P)
    ref = oracle.reduce_grad(ocfg, ot, rep, home)
    _exact(got, ref)


def test_reduce_grad_gradient_equivalence_exact():
    """Integer-valued gradients: home + replicas == the no-replication gradient, bit for bit."""
    R, E, K, S, B = 8, 32, 4, 64, 4
    cfg, ocfg, ot, arena = _setup(R, E, K, S, 8, mv=6.0, seed=8, budget=B)
    P = 24
    NvS = int(ot["nvs"][0])
    g = np.random.default_rng(8).integers(-1, 2, size=(R * NvS, P))
    flat = make_routing(R, E, K, S, 6.0, seed=8)[0].ravel()
    ref = np.zeros((E, P), np.int64)
    np.add.at(ref, flat, g[ot["slot_of"]])
    home = np.zeros((E, P), np.int64)
    rep = np.zeros((R, B, P), np.int64)
    L = E // R
    for d in range(R):
        for i in range(int(ot["n_seg"][d])):
            e, s0, ln = ot["seg_expert"][d, i], ot["seg_start"][d, i], ot["seg_len"][d, i]
            part = g[d * NvS + s0: d * NvS + s0 + ln].sum(0)
            if i < L:
                home[e] += part
            else:
                rep[d, ot["seg_wslot"][d, i]] += part
    from moonep_inputs import f32_to_bf16_bits
    got = _reduce(cfg, arena, f32_to_bf16_bits(rep.astype(np.float32)),
                  f32_to_bf16_bits(home.astype(np.float32)), P)
    assert np.array_equal(bf16_bits_to_f32(got).astype(np.int64), ref)


def test_reduce_grad_overlapping_calls_share_one_plan():
    """Two gradient matrices of one plan folded on two streams at once (the data calls
    only read the plan arena): both results exact."""
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, B, P = 8, 256, 8, 256, 32, 16384
    cfg, ocfg, ot, arena = _setup(R, E, K, S, 8, mv=20.0, seed=44, budget=B, mode=1)
    assert int(ot["n_piece"][0]) > 0
    mats = [(normal_bf16((R, B, P), seed=44 + j, stream=11), normal_bf16((E, P), seed=44 + j, stream=12))
            for j in range(2)]
    dev = [(to_dev(r), to_dev(h)) for r, h in mats]
    statuses = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(2)]
    streams = [torch.cuda.Stream() for _ in range(2)]
    torch.cuda.synchronize()
    for _ in range(3):  # three rounds: the replicas are added three times
        for j in range(2):
            with torch.cuda.stream(streams[j]):
                me.moonep_reduce_grad(cfg, arena, dev[j][0], dev[j][1], P, statuses[j],
                                      streams[j].cuda_stream)
    torch.cuda.synchronize()
    for j in range(2):
        assert int(statuses[j].item()) == 0
        rep, ref = mats[j]
        for _ in range(3):
            ref = oracle.reduce_grad(ocfg, ot, rep, ref)
        _exact(to_np(dev[j][1]), ref)


def test_reduce_grad_without_budget_is_a_no_op():
    cfg, ocfg, ot, arena = _setup(4, 16, 2, 40, 8, mv=4.0, seed=9, budget=0, mode=1)
    home = integer_bf16((16, 16), seed=9)
    got = _reduce(cfg, arena, np.zeros((4, 0, 16), np.uint16), home, 16)
    assert np.array_equal(got, home)


def test_reduce_grad_expert_with_many_pieces():
    """All tokens on expert 0: its overflow becomes one piece on each of the 7 other ranks."""
    R, E, K, S, B, P = 8, 16, 1, 64, 2, 520
    cfg, ocfg = configs(R, E, K, S, H=8, budget=B)
    idx = np.zeros((R, S, K), np.int32)
    ost, ot = oracle.plan(ocfg, idx)
    gst, arena, gv, _ = gpu_plan(cfg, idx)
    assert int(ot["n_piece"][0]) == R - 1
    rep = normal_bf16((R, B, P), seed=7, stream=11)
    home = normal_bf16((E, P), seed=7, stream=12)
    got = _reduce(cfg, arena, rep, home, P)
    ref = oracle.reduce_grad(ocfg, ot, rep, home)
    _exact(got, ref)


@pytest.mark.parametrize("R,P", [(80, 10000), (80, 8), (80, 13)])
def test_reduce_grad_more_local_pieces_than_the_cache(R, P):
    """All tokens on expert 0 across 80 ranks: 79 local pieces of one expert.

    More pieces than the reduce kernel keeps in shared memory (64), so its
    producer walks the piece tables again for the rest; P = 10000 makes rows
    of three chunks with a ragged last one, P = 8 a single 16-byte chunk, and
    P = 13 takes the unaligned path."""
    E, K, S, B = R, 1, 8, 1
    cfg, ocfg = configs(R, E, K, S, H=8, budget=B)
    idx = np.zeros((R, S, K), np.int32)
    ost, ot = oracle.plan(ocfg, idx)
    gst, arena, gv, _ = gpu_plan(cfg, idx)
    assert int(ot["n_piece"][0]) == R - 1 and int(ot["n_remote"][0]) == 0
    rep = normal_bf16((R, B, P), seed=17, stream=11)
    home = normal_bf16((E, P), seed=17, stream=12)
    got = _reduce(cfg, arena, rep, home, P)
    ref = oracle.reduce_grad(ocfg, ot, rep, home)
    _exact(got, ref)
    assert np.array_equal(got[1:], home[1:])  # experts without replicas untouched


def _dispatch_bwd(cfg, arena, drecv_np):
    import torch
    import token_dispatch_moonep_b200 as me
    d = to_dev(drecv_np)
    dx = torch.empty((cfg.R * cfg.S, cfg.H), dtype=torch.int16, device=d.device)
    status = torch.zeros(1, dtype=torch.int32, device=d.device)
    me.moonep_dispatch_backward(cfg, arena, d, dx, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return to_np(dx)


@pytest.mark.parametrize("shape", SHAPES)
def test_dispatch_backward_matches_oracle(shape):
    R, E, K, S, H, A = shape
    cfg, ocfg, ot, arena = _setup(R, E, K, S, H, align=A, seed=10)
    NvS = int(ot["nvs"][0])
    drecv = normal_bf16((R * NvS, H), seed=10, stream=13)
    got = _dispatch_bwd(cfg, arena, drecv)
    ref = oracle.dispatch_backward(ocfg, ot["slot_of"], drecv)
    if ref.size == 0:
        assert got.size == 0
        return
    _exact(got, ref)


def test_dispatch_backward_is_adjoint_on_gpu():
    """Integer data: <dispatch(x), dR> == <x, dispatch_backward(dR)> exactly, on the GPU path."""
    R, E, K, S, H = 8, 32, 4, 64, 64
    cfg, ocfg, ot, arena = _setup(R, E, K, S, H, seed=11)
    NvS = int(ot["nvs"][0])
    x = integer_bf16((R * S, H), seed=11, bound=4)
    dR = integer_bf16((R * NvS, H), seed=12, bound=4)
    recv = _dispatch(cfg, arena, x, NvS)
    dx = _dispatch_bwd(cfg, arena, dR)
    valid = ot["slot_src"] >= 0
    lhs = (bf16_bits_to_f32(recv[valid]).astype(np.int64) *
           bf16_bits_to_f32(dR[valid]).astype(np.int64)).sum()
    rhs = (bf16_bits_to_f32(x).astype(np.int64) * bf16_bits_to_f32(dx).astype(np.int64)).sum()
    assert lhs == rhs


@pytest.mark.parametrize("shape", [(8, 32, 4, 256, 4, 4096, 0.2), (8, 64, 8, 64, 8, 1000, 6.0),
                                   (4, 16, 2, 40, 3, 13, 3.0), (64, 256, 8, 16, 4, 512, 20.0)])
def test_prefetch_weight_matches_oracle(shape):
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, B, W, mv = shape
    cfg, ocfg, ot, arena = _setup(R, E, K, S, 8, mv=mv, seed=13, budget=B, mode=1)
    w = normal_bf16((E, W), seed=13, stream=14)
    before = normal_bf16((R, B, W), seed=14, stream=15)
    rep = to_dev(before)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    me.moonep_prefetch_weight(cfg, arena, to_dev(w), rep, W, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = oracle.prefetch_weight(ocfg, ot, w, before)
    assert np.array_equal(to_np(rep), ref)


@pytest.mark.parametrize("shape", [(8, 32, 4, 256, 512, 1), (4, 16, 8, 33, 136, 16),
                                   (8, 64, 8, 1200, 1032, 1), (64, 256, 8, 8, 64, 1)])
def test_copy_through_buffer_path_equals_zero_copy(shape):
    """zero_copy=False: land in a comm buffer in arrival order, permute, and back."""
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, H, A = shape
    cfg, ocfg, ot, arena = _setup(R, E, K, S, H, align=A, seed=16)
    NvS = int(ot["nvs"][0])
    N = R * S * K
    x = make_x(R, S, H, seed=16).reshape(R * S, H)
    ref_recv = oracle.dispatch(ocfg, ot["slot_of"], x, np.full((R * NvS, H), POISON, np.uint16))
    comm = torch.zeros((R * NvS, H), dtype=torch.int16, device="cuda")
    cidx = torch.full((N + R,), -5, dtype=torch.int32, device="cuda")
    recv = torch.full((R * NvS, H), POISON - 65536, dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    me.moonep_dispatch_via_buffer(cfg, arena, to_dev(x), comm, cidx, recv, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert np.array_equal(to_np(recv), ref_recv)
    ci = to_np(cidx)[:N]
    # every rank's S*K comm rows are used exactly once, by pairs sent to that rank
    assert np.array_equal(np.sort(ci), np.sort(
        (np.arange(R)[:, None] * NvS + np.arange(S * K)[None, :]).ravel()))
    assert ((ci // NvS) == (ot["slot_of"] // NvS)).all()
    y = normal_bf16((R * NvS, H), seed=17, stream=9)
    w = make_gates(R, S, K, seed=17)
    out = torch.empty((R * S, H), dtype=torch.int16, device="cuda")
    me.moonep_combine_via_buffer(cfg, arena, to_dev(y), to_dev(w.ravel()), cidx, comm, out, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert np.array_equal(to_np(out), oracle.combine(ocfg, ot["slot_of"], y, w))


def test_chained_calls_without_host_syncs():
    """The whole training chain enqueued back to back, one sync at the end.

    Every data kernel is launched with programmatic dependent launch: it may be
    scheduled while the previous kernel drains and waits on the device for it.
    Here each call consumes what the call just before it wrote (plan ->
    prefetch -> dispatch -> combine -> combine-backward -> dispatch-backward ->
    reduce_grad, and a second plan on new routing), so any read that moved
    ahead of that wait shows up as a mismatch with the oracle."""
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, H, P = 8, 64, 6, 96, 264, 1000
    cfg, ocfg = configs(R, E, K, S, H=H)
    dev = torch.device("cuda")
    NvS = me.moonep_nvs(cfg)
    idx1, _, _ = make_routing(R, E, K, S, 10.0, seed=21)
    idx2, _, _ = make_routing(R, E, K, S, 0.5, seed=22)
    x = make_x(R, S, H, seed=21).reshape(R * S, H)
    g = make_gates(R, S, K, seed=21)
    dout = normal_bf16((R * S, H), seed=21, stream=3)
    w = normal_bf16((E, P), seed=21, stream=4)
    home0 = normal_bf16((E, P), seed=21, stream=5)
    arena, ws, st = me.alloc_plan(cfg)
    arena2, _, _ = me.alloc_plan(cfg)
    idx1_d, idx2_d = to_dev(idx1.ravel().astype(np.int32)), to_dev(idx2.ravel().astype(np.int32))
    x_d, g_d, dout_d, w_d = to_dev(x), to_dev(g.ravel()), to_dev(dout), to_dev(w)
    home = to_dev(home0)
    rep_w = torch.zeros((R * cfg.budget, P), dtype=torch.int16, device=dev)
    recv = torch.zeros((R * NvS, H), dtype=torch.int16, device=dev)
    out = torch.zeros((R * S, H), dtype=torch.int16, device=dev)
    dy = torch.zeros_like(recv)
    dg = torch.zeros(R * S * K, dtype=torch.float32, device=dev)
    dx = torch.zeros_like(out)
    torch.cuda.synchronize()
    me.moonep_plan(cfg, idx1_d, arena, ws, st)
    me.moonep_prefetch_weight(cfg, arena, w_d, rep_w, P, st)
    me.moonep_dispatch(cfg, arena, x_d, recv, st)
    me.moonep_combine(cfg, arena, recv, g_d, out, st)
    me.moonep_combine_backward(cfg, arena, dout_d, recv, g_d, dy, dg, st)
    me.moonep_dispatch_backward(cfg, arena, dy, dx, st)
    me.moonep_reduce_grad(cfg, arena, rep_w, home, P, st)  # replica "grads" = the prefetched weights
    me.moonep_plan(cfg, idx2_d, arena2, ws, st)             # same workspace: the steady-state path
    me.moonep_dispatch(cfg, arena2, out, recv, st)          # second layer reads the first's output
    torch.cuda.synchronize()
    assert int(st.item()) & ~me.DEV_BUDGET == 0

    _, ot = oracle.plan(ocfg, idx1)
    _, ot2 = oracle.plan(ocfg, idx2)
    ref_rep = oracle.prefetch_weight(ocfg, ot, w, np.zeros((R, cfg.budget, P), np.uint16))
    ref_recv1 = oracle.dispatch(ocfg, ot["slot_of"], x)
    ref_out = oracle.combine(ocfg, ot["slot_of"], ref_recv1, g)
    ref_dy_pairs, ref_dg = oracle.combine_backward(ocfg, ot["slot_of"], dout, ref_recv1, g)
    ref_dy = np.zeros((R * NvS, H), np.uint16)  # the oracle gives dY per pair: put it in slot order
    ref_dy[ot["slot_of"]] = ref_dy_pairs.reshape(R * S * K, H)
    ref_dx = oracle.dispatch_backward(ocfg, ot["slot_of"], ref_dy)
    ref_home = oracle.reduce_grad(ocfg, ot, ref_rep, home0)
    ref_recv2 = oracle.dispatch(ocfg, ot2["slot_of"], ref_out)

    close = _exact  # fp32-accumulated results: the bar of the other data tests

    assert np.array_equal(to_np(rep_w).reshape(R, cfg.budget, P), ref_rep)  # copies: bit-exact
    close(to_np(out), ref_out)
    close(to_np(dy)[ot["slot_of"]], ref_dy[ot["slot_of"]])
    assert rel_err(to_np(dg).reshape(R * S, K), ref_dg.reshape(R * S, K)) <= TOL
    close(to_np(dx), ref_dx)
    close(to_np(home), ref_home)
    valid = ot2["slot_src"] >= 0
    close(to_np(recv)[valid], ref_recv2[valid])


def test_reduce_grad_forced_timeout_reports_status_and_context_stays_usable():
    """reduce_grad's pipeline waits are bounded: a stage that expects bytes no copy
    delivers (the debug hook) ends the kernel with TIMEOUT instead of hanging, and
    the next call on the same context is correct."""
    import token_dispatch_moonep_b200 as me
    R, E, K, S, B, P = 8, 32, 4, 256, 4, 2048
    cfg, ocfg, ot, arena = _setup(R, E, K, S, 8, mv=6.0, seed=6, budget=B)
    assert int(ot["n_piece"][0]) > 0
    rep = normal_bf16((R, B, P), seed=6, stream=11)
    home = normal_bf16((E, P), seed=6, stream=12)
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    h = to_dev(home)
    try:
        me.moonep_debug_set_wait(2_000_000, 1)  # 2 ms, 16 bytes that never arrive
        me.moonep_reduce_grad(cfg, arena, to_dev(rep), h, P, status)
        torch.cuda.synchronize()
        assert int(status.item()) & me.DEV_TIMEOUT
    finally:
        me.moonep_debug_set_wait(me.DEFAULT_WAIT_NS, 0)
    got = _reduce(cfg, arena, rep, home, P)
    ref = oracle.reduce_grad(ocfg, ot, rep, home)
    _exact(got, ref)


@pytest.mark.parametrize("R,E,K,S,B,P,mv", [(8, 384, 8, 512, 48, 4096 + 8, 20.0),
                                             (8, 256, 8, 256, 32, 24, 0.2),
                                             (64, 256, 8, 64, 4, 8192, 20.0)])
def test_replica_rows_of_ragged_lengths(R, E, K, S, B, P, mv):
    """reduce_grad and prefetch_weight move expert rows in 8 KB units: rows of one short
    unit, of one full unit plus 16 bytes, and many experts with few units each must all
    come out exact."""
    import torch
    import token_dispatch_moonep_b200 as me
    cfg, ocfg, ot, arena = _setup(R, E, K, S, 8, mv=mv, seed=31, budget=B, mode=1)
    assert int(ot["n_piece"][0]) > 0
    rep = normal_bf16((R, B, P), seed=31, stream=11)
    home = normal_bf16((E, P), seed=31, stream=12)
    _exact(_reduce(cfg, arena, rep, home, P), oracle.reduce_grad(ocfg, ot, rep, home))
    w = normal_bf16((E, P), seed=32, stream=14)
    before = normal_bf16((R, B, P), seed=33, stream=15)
    out = to_dev(before)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    me.moonep_prefetch_weight(cfg, arena, to_dev(w), out, P, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert np.array_equal(to_np(out), oracle.prefetch_weight(ocfg, ot, w, before))

"""GPU parity of moonep_reduce_grad_f32 (replica gradients folded into the home
expert over fp32 gradient buffers) against the oracle's orc_reduce_grad_f32.

Both sides add in fp32 in the same order (home first, then the local pieces in
ascending receiving rank), so results are compared bit for bit; the contract's
1e-3 norm-relative bar is asserted beside it."""
import numpy as np
import pytest

import oracle
from gpu_util import configs, gpu_plan, to_dev, to_np
from moonep_inputs import make_routing

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _plan(R, E, K, S, B, mv=6.0, seed=6, mode=0, idx=None):
    cfg, ocfg = configs(R, E, K, S, H=8, budget=B, mode=mode)
    if idx is None:
        idx, _, _ = make_routing(R, E, K, S, mv, seed=seed)
    _, ot = oracle.plan(ocfg, idx)
    _, arena, gv, _ = gpu_plan(cfg, idx)
    assert np.array_equal(gv["slot_of"], ot["slot_of"])
    return cfg, ocfg, ot, arena


def _fold(cfg, arena, rep, home, P, offset=0):
    """reduce_grad_f32 on device copies; ``offset`` floats shift both buffers off their
    16-byte alignment (the scalar path)."""
    import torch
    import token_dispatch_moonep_b200 as me
    rb = to_dev(np.concatenate([np.zeros(offset, np.float32), rep.ravel()]))
    hb = to_dev(np.concatenate([np.zeros(offset, np.float32), home.ravel()]))
    status = torch.zeros(1, dtype=torch.int32, device=hb.device)
    me.moonep_reduce_grad_f32(cfg, arena, rb[offset:], hb[offset:], P, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return to_np(hb[offset:]).reshape(home.shape)


def _check(got, ref):
    scale = float(np.abs(ref).max()) or 1.0
    assert float(np.abs(got.astype(np.float64) - ref).max()) / scale <= TOL
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), int((got != ref).sum())


@pytest.mark.parametrize("shape", [(8, 32, 4, 256, 4, 2048), (8, 64, 8, 64, 8, 1000),
                                   (4, 16, 2, 40, 3, 13), (8, 256, 8, 256, 32, 2052),
                                   (2, 8, 2, 30, 1, 4), (8, 384, 8, 512, 48, 4096 + 4)])
def test_reduce_grad_f32_matches_oracle(shape):
    """Rows of whole and ragged 8 KB units (2048 floats), a row of one vector, and P = 13
    (the scalar path); the last case has tens of replicated experts."""
    R, E, K, S, B, P = shape
    cfg, ocfg, ot, arena = _plan(R, E, K, S, B, mv=20.0 if E >= 256 else 6.0, mode=1)
    assert int(ot["n_piece"][0]) > 0
    rng = np.random.default_rng(P)
    rep = rng.standard_normal((R, B, P)).astype(np.float32)
    home = rng.standard_normal((E, P)).astype(np.float32)
    _check(_fold(cfg, arena, rep, home, P), oracle.reduce_grad_f32(ocfg, ot, rep, home))


def test_reduce_grad_f32_unaligned_buffers_take_the_scalar_path():
    R, E, K, S, B, P = 8, 32, 4, 256, 4, 2048
    cfg, ocfg, ot, arena = _plan(R, E, K, S, B)
    rng = np.random.default_rng(3)
    rep = rng.standard_normal((R, B, P)).astype(np.float32)
    home = rng.standard_normal((E, P)).astype(np.float32)
    _check(_fold(cfg, arena, rep, home, P, offset=1), oracle.reduce_grad_f32(ocfg, ot, rep, home))


def test_reduce_grad_f32_equals_no_replication():
    """Integer gradients past bf16's exact range: home + replicas equal the gradient
    without replication exactly (nothing is rounded through bf16)."""
    R, E, K, S, B, P = 8, 32, 4, 64, 4, 48
    cfg, ocfg, ot, arena = _plan(R, E, K, S, B, seed=18)
    NvS = int(ot["nvs"][0])
    idx, _, _ = make_routing(R, E, K, S, 6.0, seed=18)
    g = np.random.default_rng(18).integers(-300, 301, size=(R * NvS, P)).astype(np.int64)
    ref = np.zeros((E, P), np.int64)
    np.add.at(ref, idx.ravel(), g[ot["slot_of"]])
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
    assert np.abs(ref).max() > 256
    got = _fold(cfg, arena, rep.astype(np.float32), home.astype(np.float32), P)
    assert np.array_equal(got.astype(np.int64), ref)


@pytest.mark.parametrize("P", [4, 13])
def test_reduce_grad_f32_adds_home_first_then_pieces_by_rank(P):
    """home 1, rank 1's piece 1, rank 2's piece 2**24: only home-first, ascending-rank
    order gives 2**24 + 2 (bulk and scalar paths)."""
    R, E, K, S, B = 3, 3, 1, 4, 1
    idx = np.zeros((R, S, K), np.int32)
    cfg, ocfg, ot, arena = _plan(R, E, K, S, B, idx=idx)
    home = np.zeros((E, P), np.float32)
    home[0] = 1.0
    rep = np.zeros((R, B, P), np.float32)
    rep[1, 0] = 1.0
    rep[2, 0] = 2.0 ** 24
    got = _fold(cfg, arena, rep, home, P)
    assert (got[0] == np.float32(2.0 ** 24 + 2)).all() and (got[1:] == 0).all()


@pytest.mark.parametrize("P", [10000, 8, 13])
def test_reduce_grad_f32_more_local_pieces_than_the_cache(P):
    """All tokens on expert 0 across 80 ranks: 79 local pieces (more than the 64 the
    producer keeps in shared memory)."""
    R = 80
    E, K, S, B = R, 1, 8, 1
    idx = np.zeros((R, S, K), np.int32)
    cfg, ocfg, ot, arena = _plan(R, E, K, S, B, idx=idx)
    assert int(ot["n_piece"][0]) == R - 1
    rng = np.random.default_rng(17)
    rep = rng.standard_normal((R, B, P)).astype(np.float32)
    home = rng.standard_normal((E, P)).astype(np.float32)
    got = _fold(cfg, arena, rep, home, P)
    _check(got, oracle.reduce_grad_f32(ocfg, ot, rep, home))
    assert np.array_equal(got[1:], home[1:])


def test_reduce_grad_f32_without_budget_is_a_no_op():
    R, E, K, S = 4, 16, 2, 40
    cfg, ocfg, ot, arena = _plan(R, E, K, S, 0, mv=4.0, seed=9, mode=1)
    home = np.random.default_rng(9).standard_normal((E, 16)).astype(np.float32)
    got = _fold(cfg, arena, np.zeros((R, 0, 16), np.float32), home, 16)
    assert np.array_equal(got, home)


def test_reduce_grad_f32_forced_timeout_reports_status_and_next_call_is_exact():
    """The fp32 pipeline's waits are bounded like the bf16 one's: a stage that expects
    bytes no copy delivers ends the launch with TIMEOUT, and the next call is exact."""
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, B, P = 8, 32, 4, 256, 4, 2048
    cfg, ocfg, ot, arena = _plan(R, E, K, S, B)
    rng = np.random.default_rng(5)
    rep = rng.standard_normal((R, B, P)).astype(np.float32)
    home = rng.standard_normal((E, P)).astype(np.float32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        me.moonep_debug_set_wait(2_000_000, 1)  # 2 ms, 16 bytes that never arrive
        me.moonep_reduce_grad_f32(cfg, arena, to_dev(rep), to_dev(home), P, status)
        torch.cuda.synchronize()
        assert int(status.item()) & me.DEV_TIMEOUT
    finally:
        me.moonep_debug_set_wait(me.DEFAULT_WAIT_NS, 0)
    _check(_fold(cfg, arena, rep, home, P), oracle.reduce_grad_f32(ocfg, ot, rep, home))

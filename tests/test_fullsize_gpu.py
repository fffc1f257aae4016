"""Parity at the full workload sizes, in the launch configuration bench.py times.

The oracle computes sampled outputs one by one from host inputs (it never reads
a buffer the GPU produced): for the identity expert the K rows a token gathers
are its own row of x.  Whole-buffer properties are checked on the device with
the oracle's plan (every valid row of the dispatch buffer equals its source
token's row; padding rows untouched).

Bar: bit-exact for the plan and dispatched rows.  combine, combine-backward's
dY, dispatch-backward and reduce_grad round one fp32 value per element that
both sides compute with the same operations in the same order (fused
multiply-adds in ascending k, one product, fp32 additions in ascending k or in
piece order), so they must be bit-identical too; the 1e-3 norm-relative bar of
the contract is asserted beside it.  dgate is an fp32 dot product on the GPU
and an fp64 one in the oracle: 1e-3 norm-relative.  reduce_grad over fp32
gradient buffers is the same fp32 additions with no rounding: bit-identical.
"""
import numpy as np
import pytest

import oracle
from moonep_inputs import (WORKLOADS, bf16_bits_to_f32, make_dout, make_gates, make_routing,
                           make_x, row_pool)
from tests.gpu_util import compare_plans, rel_err, to_dev, to_np

pytestmark = pytest.mark.gpu
TOL = 1e-3
N_SAMPLE_TOKENS = 4096
N_SAMPLE_COLS = 16384


def _exact(got, ref, what):
    assert rel_err(bf16_bits_to_f32(got), bf16_bits_to_f32(ref)) <= TOL, what
    assert np.array_equal(got, ref), (what, int((got != ref).sum()))


def _sample_tokens(rng, R, S):
    """About N_SAMPLE_TOKENS tokens over every rank, always the first and last of each."""
    T = R * S
    ends = np.unique(np.concatenate([np.arange(R) * S, np.arange(R) * S + S - 1]))
    if T <= N_SAMPLE_TOKENS:
        return np.arange(T)
    rest = np.setdiff1d(np.arange(T), ends)
    extra = rng.choice(rest, size=N_SAMPLE_TOKENS - ends.size, replace=False)
    return np.sort(np.concatenate([ends, extra]))


def _sample_cols(rng, P):
    """Columns of an expert gradient: every 8 KB chunk boundary of the first rows, the
    last (possibly ragged) columns and a random spread."""
    fixed = np.array([0, 1, 4095, 4096, 4097, 8191, 8192, P - 2, P - 1])
    fixed = fixed[(fixed >= 0) & (fixed < P)]
    rest = rng.choice(P, size=min(P, N_SAMPLE_COLS), replace=False)
    return np.unique(np.concatenate([fixed, rest]))


@pytest.mark.parametrize("name,mv,seed", [("ep8_e256_k8_s4096_h7168", 0.2, 0),
                                          ("ep8_e256_k8_s4096_h7168_sweep", 20.0, 4),
                                          ("ep8_e384_k8_s8192_h7168_bwd", 20.0, 0),
                                          ("ep64_e256_k8_s128_h7168_decode", 1.0, 0),
                                          ("ep64_e256_k8_s128_h7168_decode", 20.0, 0)])
def test_full_size_layer(name, mv, seed):
    import torch
    import token_dispatch_moonep_b200 as me
    w = WORKLOADS[name]
    R, E, K, S, H, B = w.R, w.E, w.K, w.S, w.H, w.budget
    T = R * S
    train = w.mode == 0
    cfg = me.Config.of(w)
    ocfg = oracle.Config.of(w)
    idx, _, _ = make_routing(R, E, K, S, mv, seed=seed)
    gates = make_gates(R, S, K, seed=seed).reshape(T, K)
    x = make_x(R, S, H, seed=seed).reshape(T, H)
    NvS = me.moonep_nvs(cfg)
    dev = torch.device("cuda")
    POISON = -63  # 0xFFC1 as int16

    # ---- plan (bit-exact, every table)
    ost, ot = oracle.plan(ocfg, idx)
    arena, ws, status = me.alloc_plan(cfg)
    idx_d = to_dev(idx.ravel().astype(np.int32))
    # the first launch on a workspace sums every chunk's histogram row; the second (a
    # caller's steady state) reads the totals the chunks added by atomics: both compared
    for _ in range(2):
        status.zero_()
        me.moonep_plan(cfg, idx_d, arena, ws, status)
        torch.cuda.synchronize()
        gv = {k: (to_np(v) if not isinstance(v, int) else v)
              for k, v in me.moonep_plan_view(cfg, arena).items()}
        compare_plans(cfg, ost, ot, int(status.item()), gv)
    if w.mode == 1 and mv >= 20:
        assert int(ot["n_remote"][0]) > 0  # the remote-read path is exercised

    # ---- dispatch
    x_d = to_dev(x)
    recv = torch.full((R * NvS, H), POISON, dtype=torch.int16, device=dev)
    me.moonep_dispatch(cfg, arena, x_d, recv, status)
    torch.cuda.synchronize()
    src = torch.from_numpy(ot["slot_src"].astype(np.int64)).to(dev)
    valid = src >= 0
    # property over the whole buffer: valid rows are their source token's row, padding untouched
    assert torch.equal(recv[valid], x_d[src[valid] // K])
    assert bool((recv[~valid] == POISON).all())
    rng = np.random.default_rng(1)
    rows = rng.choice(np.nonzero(ot["slot_src"] >= 0)[0], size=min(2048, T * K), replace=False)
    got_rows = to_np(recv[torch.from_numpy(rows).to(dev)])
    assert np.array_equal(got_rows, x[ot["slot_src"][rows] // K])

    # ---- combine (identity expert: y = the dispatch buffer)
    g_d = to_dev(gates.ravel())
    out = torch.empty((T, H), dtype=torch.int16, device=dev)
    me.moonep_combine(cfg, arena, recv, g_d, out, status)
    torch.cuda.synchronize()
    toks = _sample_tokens(rng, R, S)
    n = len(toks)
    c1 = oracle.Config(R=1, E=E, K=K, S=n, H=H, budget=B, mode=w.mode)
    y_rows = np.repeat(x[toks], K, axis=0)                 # row k of token t is x[t]
    compact = np.arange(n * K, dtype=np.int32)
    ref_out = oracle.combine(c1, compact, y_rows, gates[toks])
    toks_d = torch.from_numpy(toks).to(dev)
    _exact(to_np(out[toks_d]), ref_out, "combine")
    del out
    torch.cuda.synchronize()

    if not train:
        assert int(status.item()) == 0
        return

    # ---- combine-backward
    dout = make_dout(R, S, H, seed=seed).reshape(T, H)
    dout_d = to_dev(dout)
    dy = torch.full((R * NvS, H), POISON, dtype=torch.int16, device=dev)
    dg = torch.empty(T * K, dtype=torch.float32, device=dev)
    me.moonep_combine_backward(cfg, arena, dout_d, recv, g_d, dy, dg, status)
    torch.cuda.synchronize()
    ref_dy, ref_dg = oracle.combine_backward(c1, compact, dout[toks], y_rows, gates[toks])
    so = torch.from_numpy(ot["slot_of"].reshape(T, K)[toks].ravel().astype(np.int64)).to(dev)
    _exact(to_np(dy[so]).reshape(n, K, H), ref_dy, "combine_backward dY")
    got_dg = to_np(dg).reshape(T, K)[toks]
    assert rel_err(got_dg, ref_dg) <= TOL
    assert bool((dy[~valid] == POISON).all())
    del recv, dout_d, x_d, dg
    torch.cuda.empty_cache()

    # ---- dispatch-backward of the combine-backward's dY (the oracle sums its own dY rows)
    dx = torch.empty((T, H), dtype=torch.int16, device=dev)
    me.moonep_dispatch_backward(cfg, arena, dy, dx, status)
    torch.cuda.synchronize()
    ref_dx = oracle.dispatch_backward(c1, compact, ref_dy.reshape(n * K, H))
    _exact(to_np(dx[toks_d]), ref_dx, "dispatch_backward")
    del dy, dx
    torch.cuda.empty_cache()

    # ---- reduce_grad on [2048 x H] expert gradients built from a pool of rows
    P = w.P or 2048 * H
    pool = row_pool(12, P, seed=3)                          # 12 bf16 rows of P elements
    rep_map = (np.arange(R * B) * 7 + 3) % 12               # replica slot -> pool row
    home_map = (np.arange(E) * 5 + 1) % 12                  # expert -> pool row
    pool_d = to_dev(pool)
    rep = pool_d[torch.from_numpy(rep_map).to(dev)]         # [R*B, P] on the device
    home = pool_d[torch.from_numpy(home_map).to(dev)]       # [E, P]
    me.moonep_reduce_grad(cfg, arena, rep, home, P, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    cols = _sample_cols(rng, P)
    rep_cols = pool[rep_map][:, cols].reshape(R, B, len(cols))
    home_cols = pool[home_map][:, cols]
    ref_home = oracle.reduce_grad(ocfg, ot, rep_cols, home_cols)
    got_home = to_np(home[:, torch.from_numpy(cols).to(dev)])
    _exact(got_home, ref_home, "reduce_grad")
    touched = np.zeros(E, bool)
    touched[ot["piece_expert"][ot["piece_wslot"] >= 0]] = True
    assert touched.any()
    assert np.array_equal(got_home[~touched], home_cols[~touched])  # untouched experts unchanged

    # ---- the same fold over fp32 gradient buffers (the pool's rows as fp32)
    del rep, home
    torch.cuda.empty_cache()
    pool32 = bf16_bits_to_f32(pool)
    pool32_d = torch.from_numpy(pool32).to(dev)
    rep32 = pool32_d[torch.from_numpy(rep_map).to(dev)]     # [R*B, P] fp32
    home32 = pool32_d[torch.from_numpy(home_map).to(dev)]   # [E, P] fp32
    me.moonep_reduce_grad_f32(cfg, arena, rep32, home32, P, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref32 = oracle.reduce_grad_f32(ocfg, ot, pool32[rep_map][:, cols].reshape(R, B, len(cols)),
                                   pool32[home_map][:, cols])
    got32 = home32[:, torch.from_numpy(cols).to(dev)].cpu().numpy()
    assert float(np.abs(got32.astype(np.float64) - ref32).max()) <= TOL * float(np.abs(ref32).max())
    assert np.array_equal(got32.view(np.uint32), ref32.view(np.uint32)), int((got32 != ref32).sum())
    assert np.array_equal(got32[~touched], pool32[home_map][:, cols][~touched])
    del rep32, home32, pool32_d
    torch.cuda.empty_cache()

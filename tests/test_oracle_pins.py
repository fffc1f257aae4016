"""Pins for the CPU oracle: facts fixed by the MoonEP pages and by mathematics.

None of these re-types the oracle's own loops.  They check it against
* a worked example derived by hand from the planning rule,
* closed forms of degenerate routings,
* invariants every balanced plan must satisfy ("every rank receives exactly
  S x K token-slots", "Moonshot AI Open-Sources MoonEP"; replica budget, same
  page; fixed NvS, "MoonshotAI/MoonEP 딥다이브" §4 pattern 2),
* brute force over all pair -> rank assignments on tiny inputs,
* an independent sort-based formulation of the keep / overflow / receiver order,
* fp64 closed forms of combine and combine-backward (§8 exercise C),
* exact integer arithmetic for reduce_grad (§4 pattern 3, §8 exercise E).
"""
import itertools

import numpy as np
import pytest

import oracle
from moonep_inputs import (bf16_bits_to_f32, f32_to_bf16_bits, integer_bf16, make_gates,
                           make_routing, make_x, normal_bf16, uniform_routing)

# ----------------------------------------------------------------- helpers ---


def cfg(R, E, K, S, H=8, budget=None, mode=0, align=1):
    if budget is None:
        budget = E // R
    return oracle.Config(R=R, E=E, K=K, S=S, H=H, budget=budget, mode=mode, align=align)


def check_invariants(c, idx, st, t):
    """Properties any plan obeying the pages' contract must have."""
    R, E, K, S, A, B = c.R, c.E, c.K, c.S, c.align, c.budget
    L = E // R
    SK = S * K
    NvS = int(t["nvs"][0])
    assert NvS >= SK
    if A == 1:
        assert NvS == SK
    idx = np.asarray(idx).ravel()
    n = idx.size
    # counts and loads
    cnt = np.bincount(idx, minlength=E)
    assert (t["expert_count"] == cnt).all()
    load = cnt.reshape(R, L).sum(1)
    assert (t["rank_load"] == load).all()
    assert (t["overflow"] == np.maximum(load - SK, 0)).all()
    assert (t["deficit"] == np.maximum(SK - load, 0)).all()
    # slot_of: a bijection from pairs onto the valid rows
    so = t["slot_of"]
    src = t["slot_src"]
    assert so.shape == (n,) and src.shape == (R * NvS,)
    assert (so >= 0).all() and (so < R * NvS).all()
    assert np.unique(so).size == n
    assert (src[so] == np.arange(n)).all()
    assert (src >= -1).all()
    assert ((src >= 0).sum()) == n
    # every rank holds exactly S*K valid rows
    per_rank = np.bincount(so // max(NvS, 1), minlength=R) if n else np.zeros(R, int)
    assert (per_rank == SK).all()
    # each row belongs to a segment whose expert is the routed expert
    row_expert = np.full(R * NvS, -1, np.int64)
    row_kind = np.full(R * NvS, -1, np.int64)
    n_rep_per_rank = np.zeros(R, np.int64)
    for d in range(R):
        ns = int(t["n_seg"][d])
        assert L <= ns <= E
        prev_end = 0
        for i in range(ns):
            e, st0, ln = t["seg_expert"][d, i], t["seg_start"][d, i], t["seg_len"][d, i]
            kind, ws = t["seg_kind"][d, i], t["seg_wslot"][d, i]
            assert st0 % A == 0 and st0 >= prev_end
            prev_end = st0 + ln
            assert prev_end <= NvS
            if i < L:
                assert e == d * L + i and kind == oracle.KIND_NATIVE and ws == -1
            else:
                assert e // L != d, "a rank never receives a replica of its own expert"
                assert ln > 0
                assert kind in (oracle.KIND_REPLICA, oracle.KIND_REMOTE)
                j = i - L
                if j < B:
                    assert kind == oracle.KIND_REPLICA and ws == j
                    assert t["rep_expert"][d * B + j] == e
                else:
                    assert kind == oracle.KIND_REMOTE and ws == -1
                n_rep_per_rank[d] += 1
            row_expert[d * NvS + st0: d * NvS + st0 + ln] = e
            row_kind[d * NvS + st0: d * NvS + st0 + ln] = kind
        # replicas only on ranks that had a deficit, and each expert at most once
        reps = t["seg_expert"][d, L:ns]
        assert np.unique(reps).size == reps.size
        if t["deficit"][d] == 0:
            assert ns == L
        for i in range(ns, E):
            assert t["seg_expert"][d, i] == -1
    assert (row_expert[so] == idx).all()
    # padding rows carry no source
    assert (src[row_expert < 0] == -1).all()
    # pairs that stay home are exactly S*K per overloaded rank and all of an underloaded one
    home_rank = idx // L
    on_home = (so // max(NvS, 1)) == home_rank
    kept_per_rank = np.bincount(home_rank[on_home], minlength=R)
    assert (kept_per_rank == np.minimum(load, SK)).all()
    moved_in = np.bincount((so // max(NvS, 1))[~on_home], minlength=R)
    assert (moved_in == t["deficit"]).all()
    moved_out = np.bincount(home_rank[~on_home], minlength=R)
    assert (moved_out == t["overflow"]).all()
    # piece accounting
    n_piece = int(t["n_piece"][0])
    n_over_items = sum(1 for e in range(E) if ((~on_home) & (idx == e)).any())
    n_recv = int((t["deficit"] > 0).sum())
    if n_piece:
        assert n_piece <= n_over_items + n_recv - 1
    assert n_piece == int(n_rep_per_rank.sum())
    remote = int((t["piece_wslot"] < 0).sum())
    assert remote == int(t["n_remote"][0])
    assert remote == int(np.maximum(n_rep_per_rank - B, 0).sum())
    expect_st = oracle.BUDGET if (c.mode == 0 and remote > 0) else oracle.OK
    assert st == expect_st


# ------------------------------------------------------ worked example pin ---


def test_worked_example_by_hand():
    """R=2 ranks, E=4 experts (L=2), S=3 tokens per rank, K=2, alignment 1.

    rank 0 tokens pick {0,1}, {0,1}, {1,2}; rank 1 tokens pick {0,1}, {0,3}, {1,2}.
    By hand: counts [4,5,2,1]; loads [9,3]; S*K = 6 so rank 0 sheds 3, rank 1
    takes 3.  Rank 0's stream is e0 = [r0t0, r0t1, r1t0, r1t1] then
    e1 = [r0t0, r0t1, r0t2, r1t0, r1t2]; the first 6 stay, so e1's r0t2, r1t0,
    r1t2 move to rank 1 as one replica piece of e1 in weight slot 0, after rank
    1's native rows (e2: r0t2, r1t2; e3: r1t1).
    """
    c = cfg(2, 4, 2, 3, budget=2)
    idx = np.array([[[0, 1], [0, 1], [1, 2]], [[0, 1], [0, 3], [1, 2]]], np.int32)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK
    assert t["expert_count"].tolist() == [4, 5, 2, 1]
    assert t["rank_load"].tolist() == [9, 3]
    assert t["overflow"].tolist() == [3, 0]
    assert t["deficit"].tolist() == [0, 3]
    NvS = 6
    # (rank,row) per (r, t, k) in flat order
    expect = [(0, 0), (0, 4),  # r0t0
              (0, 1), (0, 5),  # r0t1
              (1, 3), (1, 0),  # r0t2
              (0, 2), (1, 4),  # r1t0
              (0, 3), (1, 2),  # r1t1
              (1, 5), (1, 1)]  # r1t2
    assert t["slot_of"].tolist() == [d * NvS + r for d, r in expect]
    assert t["slot_src"].tolist() == [0, 2, 6, 8, 1, 3, 5, 11, 9, 4, 7, 10]
    assert int(t["n_piece"][0]) == 1
    assert t["piece_expert"].tolist() == [1] and t["piece_rank"].tolist() == [1]
    assert t["piece_start"].tolist() == [3] and t["piece_len"].tolist() == [3]
    assert t["piece_wslot"].tolist() == [0] and t["piece_ostart"].tolist() == [0]
    assert t["rep_expert"].tolist() == [-1, -1, 1, -1]
    assert t["n_seg"].tolist() == [2, 3]
    assert t["seg_expert"][1, :3].tolist() == [2, 3, 1]
    assert t["seg_start"][1, :3].tolist() == [0, 2, 3]
    assert t["seg_kind"][1, :3].tolist() == [0, 0, 1]
    check_invariants(c, idx, st, t)


def test_worked_example_with_alignment_by_hand():
    """Same routing with alignment A=4: NvS = 6 + 3*min(4, 6) = 18.

    Rank 0 segments: e0 len 4 at 0, e1 len 2 at 4.  Rank 1: e2 len 2 at 0,
    e3 len 1 at 4, the e1 piece len 3 at 8; rows 2,3,5,6,7,11.. are padding.
    """
    c = cfg(2, 4, 2, 3, budget=2, align=4)
    idx = np.array([[[0, 1], [0, 1], [1, 2]], [[0, 1], [0, 3], [1, 2]]], np.int32)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK
    NvS = 18
    assert int(t["nvs"][0]) == NvS
    expect = [(0, 0), (0, 4), (0, 1), (0, 5), (1, 8), (1, 0),
              (0, 2), (1, 9), (0, 3), (1, 4), (1, 10), (1, 1)]
    assert t["slot_of"].tolist() == [d * NvS + r for d, r in expect]
    src = t["slot_src"]
    valid_rows = sorted(d * NvS + r for d, r in expect)
    assert sorted(np.nonzero(src >= 0)[0].tolist()) == valid_rows
    check_invariants(c, idx, st, t)


# ------------------------------------------------------ closed-form routings ---


@pytest.mark.parametrize("R,S,B", [(4, 5, 1), (8, 3, 1), (3, 7, 0)])
def test_all_tokens_on_first_expert(R, S, B):
    """K=1, E=R (one expert per rank), every token picks expert 0.

    Rank 0 keeps the first S pairs in (rank, token) order, i.e. its own
    tokens; the overflow stream is ranks 1..R-1's tokens in order and the
    receivers 1..R-1 (ascending) take S each, so token (r, s) lands on rank r,
    row s, as a replica of expert 0 (weight slot 0 if the budget allows).
    """
    c = cfg(R, R, 1, S, budget=B, mode=1)
    idx = np.zeros((R, S, 1), np.int32)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK
    r, s = np.meshgrid(np.arange(R), np.arange(S), indexing="ij")
    assert (t["slot_of"] == (r * S + s).ravel()).all()
    assert int(t["n_piece"][0]) == R - 1
    assert t["piece_rank"].tolist() == list(range(1, R))
    assert t["piece_wslot"].tolist() == ([0] * (R - 1) if B >= 1 else [-1] * (R - 1))
    assert int(t["n_remote"][0]) == (0 if B >= 1 else R - 1)
    check_invariants(c, idx, st, t)


@pytest.mark.parametrize("R,S", [(4, 5), (2, 9)])
def test_all_tokens_on_last_expert(R, S):
    """K=1, E=R, every token picks expert R-1 (home rank R-1).

    Rank R-1 keeps the first S pairs, which are rank 0's tokens; the overflow
    (ranks 1..R-1's tokens) goes to receivers 0..R-2 in order, so rank r's
    tokens land on rank r-1 for r >= 1.
    """
    c = cfg(R, R, 1, S, budget=1)
    idx = np.full((R, S, 1), R - 1, np.int32)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK
    dest = np.array([R - 1] + list(range(R - 1)))
    expect = (dest[:, None] * S + np.arange(S)[None, :]).ravel()
    assert (t["slot_of"] == expect).all()
    check_invariants(c, idx, st, t)


@pytest.mark.parametrize("R,K,S", [(2, 2, 3), (4, 3, 5), (8, 8, 4)])
def test_already_balanced_routing(R, K, S):
    """L=K and token (r,s) picks its own rank's experts rK..rK+K-1 in order.

    Every load is exactly S*K: nothing moves, and expert rK+k holds tokens
    (r, 0..S-1) in order in rows k*S..k*S+S-1 of rank r.
    """
    E = R * K
    c = cfg(R, E, K, S)
    idx = (np.arange(R)[:, None, None] * K + np.arange(K)[None, None, :]).repeat(S, axis=1)
    idx = idx.astype(np.int32)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK
    r, s, k = np.meshgrid(np.arange(R), np.arange(S), np.arange(K), indexing="ij")
    assert (t["slot_of"] == (r * S * K + k * S + s).ravel()).all()
    assert int(t["n_piece"][0]) == 0
    check_invariants(c, idx, st, t)


def test_empty_and_single_rank():
    st, t = oracle.plan(cfg(4, 8, 2, 0), np.zeros((4, 0, 2), np.int32))
    assert st == oracle.OK and t["slot_of"].size == 0 and t["slot_src"].size == 0
    assert (t["expert_count"] == 0).all() and int(t["n_piece"][0]) == 0
    idx = uniform_routing(1, 6, 3, 10, seed=3)
    c = cfg(1, 6, 3, 10)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK and int(t["n_piece"][0]) == 0
    check_invariants(c, idx, st, t)


def test_rejects_bad_input():
    assert oracle.plan(cfg(2, 4, 2, 3), np.full((2, 3, 2), 4, np.int32))[0] == oracle.BAD_EXPERT_ID
    assert oracle.plan(cfg(2, 4, 2, 3), np.full((2, 3, 2), -1, np.int32))[0] == oracle.BAD_EXPERT_ID
    assert oracle.plan(cfg(3, 4, 2, 3), np.zeros((3, 3, 2), np.int32))[0] == oracle.INVALID_ARG
    assert oracle.plan(cfg(2, 4, 5, 3), np.zeros((2, 3, 5), np.int32))[0] == oracle.INVALID_ARG


# ------------------------------------------------------- invariants, random ---


RANDOM_CASES = [
    # R, E, K, S, budget, mode, align, maxvio
    (8, 32, 4, 256, 4, 0, 1, 0.2),
    (8, 32, 4, 256, 4, 0, 1, 5.0),
    (8, 64, 8, 64, 8, 0, 16, 3.0),
    (4, 16, 2, 33, 1, 1, 1, 3.0),
    (3, 9, 3, 17, 2, 1, 8, 1.0),
    (2, 2, 1, 50, 1, 0, 1, 0.5),
    (16, 64, 6, 40, 2, 1, 4, 8.0),
    (64, 256, 8, 16, 4, 1, 1, 20.0),
]


@pytest.mark.parametrize("case", RANDOM_CASES)
def test_invariants_random(case):
    R, E, K, S, B, mode, A, mv = case
    idx, _, _ = make_routing(R, E, K, S, mv, seed=11)
    c = cfg(R, E, K, S, budget=B, mode=mode, align=A)
    st, t = oracle.plan(c, idx)
    check_invariants(c, idx, st, t)


from hypothesis import given, settings, strategies as hs  # noqa: E402


@settings(max_examples=150, deadline=None, derandomize=True)
@given(R=hs.integers(1, 8), L=hs.integers(1, 4), K=hs.integers(1, 8), S=hs.integers(0, 40),
       budget_frac=hs.floats(0, 1), mode=hs.integers(0, 1), align=hs.sampled_from([1, 2, 3, 4, 16]),
       alpha=hs.floats(0, 3), seed=hs.integers(0, 2**31 - 1))
def test_invariants_property(R, L, K, S, budget_frac, mode, align, alpha, seed):
    """The contract's invariants over drawn configs: ranks 1-8, 1-4 experts per
    rank, top-1..8 with ids that may repeat inside a token, budgets 0..L, both
    modes, alignments 1-16, popularity from uniform to steep Zipf."""
    E = R * L
    K = min(K, E)
    B = int(round(budget_frac * L))
    p = (np.arange(E) + 1.0) ** -alpha
    rng = np.random.default_rng(seed)
    idx = rng.choice(E, size=(R, S, K), p=p / p.sum()).astype(np.int32)
    c = cfg(R, E, K, S, budget=B, mode=mode, align=align)
    st, t = oracle.plan(c, idx)
    check_invariants(c, idx, st, t)


def test_invariants_with_repeated_experts_in_a_token():
    idx = uniform_routing(4, 8, 3, 20, seed=5, distinct=False)
    c = cfg(4, 8, 3, 20, budget=1, mode=1, align=2)
    st, t = oracle.plan(c, idx)
    check_invariants(c, idx, st, t)


def test_plan_independent_of_hidden_size_and_repeatable():
    idx, _, _ = make_routing(8, 32, 4, 64, 2.0, seed=1)
    st1, t1 = oracle.plan(cfg(8, 32, 4, 64, H=8), idx)
    st2, t2 = oracle.plan(cfg(8, 32, 4, 64, H=7168), idx)
    st3, t3 = oracle.plan(cfg(8, 32, 4, 64, H=8), idx)
    assert st1 == st2 == st3
    for k in t1:
        assert np.array_equal(t1[k], t2[k]) and np.array_equal(t1[k], t3[k])


# ----------------------------------------- independent sort-based ordering ---


@pytest.mark.parametrize("case", RANDOM_CASES[:6])
def test_order_against_sort_formulation(case):
    """Keep/overflow/receiver order re-derived with a stable lexsort.

    Sorting pairs by (home rank, expert, flat pair id) gives each home stream;
    its first S*K entries stay; the rest, concatenated over ranks, is the
    overflow stream, cut into consecutive runs of deficit_d for ascending d.
    """
    R, E, K, S, B, mode, A, mv = case
    idx, _, _ = make_routing(R, E, K, S, mv, seed=23)
    c = cfg(R, E, K, S, budget=B, mode=mode, align=A)
    st, t = oracle.plan(c, idx)
    flat = idx.ravel().astype(np.int64)
    L, SK, NvS = E // R, S * K, int(t["nvs"][0])
    pid = np.arange(flat.size)
    order = np.lexsort((pid, flat, flat // L))       # primary: home, then expert, then pair
    home_sorted = (flat // L)[order]
    first_of_home = np.searchsorted(home_sorted, np.arange(R))
    pos_in_stream = np.arange(flat.size) - first_of_home[home_sorted]
    stays = pos_in_stream < SK
    dest_rank = np.empty(flat.size, np.int64)
    dest_rank[order[stays]] = home_sorted[stays]
    leaving = order[~stays]                          # overflow stream O, in order
    deficit = np.maximum(SK - np.bincount(flat // L, minlength=R), 0)
    recv_of_o = np.repeat(np.arange(R), deficit)
    assert recv_of_o.size == leaving.size
    dest_rank[leaving] = recv_of_o
    assert ((t["slot_of"] // NvS) == dest_rank).all()
    # inside each (rank, expert) segment rows follow the stream order
    so = t["slot_of"]
    for d in range(R):
        for e in np.unique(flat[dest_rank == d]):
            mine = np.nonzero((dest_rank == d) & (flat == e))[0]  # ascending pair id
            rows = so[mine]
            assert (np.diff(rows) == 1).all()


# ------------------------------------------------------------ brute force ---


def _brute_min_moves(idx, R, L, SK):
    """Fewest pairs away from their home rank over all assignments with loads = S*K."""
    flat = np.asarray(idx).ravel()
    best = None
    for assign in itertools.product(range(R), repeat=flat.size):
        a = np.array(assign)
        if (np.bincount(a, minlength=R) != SK).any():
            continue
        moves = int((a != flat // L).sum())
        best = moves if best is None else min(best, moves)
    return best


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_balance_is_minimal(seed):
    """On tiny inputs: S*K per rank is attainable and the plan moves the fewest pairs."""
    rng = np.random.default_rng(seed)
    R = [2, 3][seed % 2]
    L = 1 + seed % 2
    E, K = R * L, 1 + (seed % 2)
    S = max(1, 8 // (R * K))
    idx = np.stack([np.stack([rng.choice(E, size=K, replace=False) for _ in range(S)])
                    for _ in range(R)]).astype(np.int32)
    idx[0, :, 0] = 0  # skew towards rank 0
    c = cfg(R, E, K, S, budget=E)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK
    NvS = int(t["nvs"][0])
    moved = int(((t["slot_of"] // NvS) != idx.ravel() // L).sum())
    assert moved == _brute_min_moves(idx, R, L, S * K)
    assert moved == int(t["overflow"].sum())


# -------------------------------------------------------------- bf16 helper ---


def test_bf16_rounding_matches_library():
    import torch
    specials = np.array([0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9,
                         -1.0 - 2 ** -8, 65504.0, 3.3895313892515355e38, 1e-40, -1e-42,
                         np.inf, -np.inf, 2 ** -126, 0.1, -7.3e-3], np.float32)
    rnd = np.random.default_rng(0).standard_normal(2000).astype(np.float32) * 1e3
    vals = np.concatenate([specials, rnd])
    ours = np.array([oracle.f32_to_bf16(v) for v in vals], np.uint16)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # ties go to even
    assert oracle.f32_to_bf16(1.0 + 2 ** -8) == 0x3F80
    assert oracle.f32_to_bf16(1.0 + 3 * 2 ** -8) == 0x3F82
    for b in [0x3F80, 0xC2F7, 0x0001, 0x7F7F]:
        assert f32_to_bf16_bits(np.array([oracle.bf16_to_f32(b)], np.float32))[0] == b


# ------------------------------------------------------ dispatch / combine ---


def _bf16_half_ulp(v):
    """Half a bf16 ulp at |v| (2**-8 relative to the binade), 2**-134 floor."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 8)


@pytest.mark.parametrize("case", [(8, 32, 4, 64, 40, 2.0), (2, 4, 2, 9, 24, 0.5),
                                  (4, 16, 8, 16, 16, 5.0)])
def test_round_trip_identity_expert(case):
    """dispatch -> identity expert -> combine equals sum_k w_k x (§8 exercise C)."""
    R, E, K, S, H, mv = case
    idx, _, _ = make_routing(R, E, K, S, mv, seed=2)
    c = cfg(R, E, K, S, H=H)
    st, t = oracle.plan(c, idx)
    x = make_x(R, S, H, seed=2).reshape(R * S, H)
    w = make_gates(R, S, K, seed=2).reshape(R * S, K)
    recv = oracle.dispatch(c, t["slot_of"], x)
    # every valid row is an exact copy of its source token's row
    valid = t["slot_src"] >= 0
    assert np.array_equal(recv[valid], x[t["slot_src"][valid] // K])
    out = oracle.combine(c, t["slot_of"], recv, w)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    exact = w.astype(np.float64).sum(1, keepdims=True) * xf
    got = bf16_bits_to_f32(out).astype(np.float64)
    bound = _bf16_half_ulp(exact) * (1 + 2 ** -7) + K * 2.0 ** -24 * np.abs(exact) * 2
    assert (np.abs(got - exact) <= bound).all()


def test_combine_general_rows_closed_form():
    """combine over arbitrary expert outputs y against the fp64 gate-weighted sum."""
    R, E, K, S, H = 4, 16, 4, 24, 32
    idx, _, _ = make_routing(R, E, K, S, 3.0, seed=4)
    c = cfg(R, E, K, S, H=H)
    st, t = oracle.plan(c, idx)
    NvS = int(t["nvs"][0])
    y = normal_bf16((R * NvS, H), seed=4, stream=9)
    w = make_gates(R, S, K, seed=4).reshape(R * S, K)
    out = oracle.combine(c, t["slot_of"], y, w)
    yf = bf16_bits_to_f32(y).astype(np.float64)
    rows = t["slot_of"].reshape(R * S, K)
    terms = w.astype(np.float64)[:, :, None] * yf[rows]
    exact = terms.sum(1)
    got = bf16_bits_to_f32(out).astype(np.float64)
    bound = _bf16_half_ulp(exact) * (1 + 2 ** -7) + K * 2.0 ** -23 * np.abs(terms).sum(1)
    assert (np.abs(got - exact) <= bound).all()
    # dropping any single k would break the bound somewhere
    partial = terms[:, 1:, :].sum(1)
    assert (np.abs(partial - exact) > bound).any()
    # a subset of tokens gives the same rows as the full call
    tok = np.array([0, 5, R * S - 1])
    assert np.array_equal(oracle.combine(c, t["slot_of"], y, w, tokens=tok), out[tok])


def test_combine_backward_closed_form():
    R, E, K, S, H = 4, 16, 4, 24, 48
    idx, _, _ = make_routing(R, E, K, S, 2.0, seed=6)
    c = cfg(R, E, K, S, H=H)
    st, t = oracle.plan(c, idx)
    x = make_x(R, S, H, seed=6).reshape(R * S, H)
    dout = normal_bf16((R * S, H), seed=6, stream=3)
    w = make_gates(R, S, K, seed=6).reshape(R * S, K)
    y = oracle.dispatch(c, t["slot_of"], x)      # identity expert: y[slot_k] = x[t]
    dy, dg = oracle.combine_backward(c, t["slot_of"], dout, y, w)
    d64 = bf16_bits_to_f32(dout).astype(np.float64)
    prod = w.astype(np.float64)[:, :, None] * d64[:, None, :]
    got = bf16_bits_to_f32(dy).astype(np.float64)
    assert (np.abs(got - prod) <= _bf16_half_ulp(prod) * (1 + 2 ** -7) + 1e-45).all()
    ref = (d64 * bf16_bits_to_f32(x).astype(np.float64)).sum(1)  # <dOut[t], x[t]>, all k
    absum = np.abs(d64 * bf16_bits_to_f32(x)).sum(1)
    tol = 2.0 ** -24 * np.abs(ref) + H * 2.0 ** -52 * absum
    assert (np.abs(dg.astype(np.float64) - ref[:, None]) <= tol[:, None]).all()


# ------------------------------------------------------------- reduce_grad ---


@pytest.mark.parametrize("case", [(8, 32, 4, 64, 4, 6.0), (4, 16, 2, 40, 3, 3.0),
                                  (8, 64, 8, 32, 8, 15.0)])
def test_reduce_grad_equals_no_replication(case):
    """Replica gradients summed home equal the gradient without replication.

    Each row of the dispatch buffer contributes an integer-valued gradient g[row]
    (exact in bf16 and fp32).  Without replication expert e's gradient is the
    sum of g over all rows that hold e's pairs.  With the plan, the home rank
    accumulates its native rows and each replica piece its own rows;
    reduce_grad must then reproduce the no-replication sum bit for bit.
    """
    R, E, K, S, B, mv = case
    idx, _, _ = make_routing(R, E, K, S, mv, seed=8)
    c = cfg(R, E, K, S, budget=B)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK
    assert int(t["n_piece"][0]) > 0
    P = 24
    NvS = int(t["nvs"][0])
    g = np.random.default_rng(8).integers(-1, 2, size=(R * NvS, P)).astype(np.int64)
    so = t["slot_of"]
    flat = idx.ravel()
    # no-replication gradient: per expert, the sum over all its rows
    ref = np.zeros((E, P), np.int64)
    np.add.at(ref, flat, g[so])
    # the planned split: home accumulates native rows, replica slots their piece rows
    home = np.zeros((E, P), np.int64)
    rep = np.zeros((R, B, P), np.int64)
    L = E // R
    for d in range(R):
        for i in range(int(t["n_seg"][d])):
            e, s0, ln = t["seg_expert"][d, i], t["seg_start"][d, i], t["seg_len"][d, i]
            part = g[d * NvS + s0: d * NvS + s0 + ln].sum(0)
            if i < L:
                home[e] += part
            else:
                rep[d, t["seg_wslot"][d, i]] += part
    assert np.abs(ref).max() <= 256 and np.abs(home).max() <= 256 and np.abs(rep).max() <= 256
    to_bf16 = lambda a: f32_to_bf16_bits(a.astype(np.float32))
    new = oracle.reduce_grad(c, t, to_bf16(rep), to_bf16(home))
    assert np.array_equal(bf16_bits_to_f32(new).astype(np.int64), ref)


def test_reduce_grad_leaves_unreplicated_experts_alone():
    R, E, K, S, B = 4, 16, 2, 30, 2
    idx, _, _ = make_routing(R, E, K, S, 4.0, seed=9)
    c = cfg(R, E, K, S, budget=B)
    st, t = oracle.plan(c, idx)
    P = 10
    home = integer_bf16((E, P), seed=9, bound=64)
    rep = integer_bf16((R, B, P), seed=10, bound=16)
    new = oracle.reduce_grad(c, t, rep, home)
    touched = np.zeros(E, bool)
    touched[t["piece_expert"][t["piece_wslot"] >= 0]] = True
    assert np.array_equal(new[~touched], home[~touched])
    # touched experts: home + the replicas of that expert (integers, exact)
    hf = bf16_bits_to_f32(home).astype(np.int64)
    rf = bf16_bits_to_f32(rep).astype(np.int64)
    for e in np.nonzero(touched)[0]:
        want = hf[e].copy()
        for i in np.nonzero((t["piece_expert"] == e) & (t["piece_wslot"] >= 0))[0]:
            want += rf[t["piece_rank"][i], t["piece_wslot"][i]]
        assert np.array_equal(bf16_bits_to_f32(new[e]).astype(np.int64), want)


# ------------------------------------------------------- dispatch-backward ---


@pytest.mark.parametrize("case", [(8, 32, 4, 48, 24, 3.0), (3, 9, 3, 17, 8, 1.0),
                                  (4, 16, 8, 10, 16, 5.0)])
def test_dispatch_backward_is_the_adjoint_of_dispatch(case):
    """<dispatch(x), dR> = <x, dispatch_backward(dR)> with integers (all sums exact)."""
    R, E, K, S, H, mv = case
    idx, _, _ = make_routing(R, E, K, S, mv, seed=12)
    c = cfg(R, E, K, S, H=H)
    st, t = oracle.plan(c, idx)
    NvS = int(t["nvs"][0])
    x = integer_bf16((R * S, H), seed=12, bound=4)
    dR = integer_bf16((R * NvS, H), seed=13, bound=4)
    recv = oracle.dispatch(c, t["slot_of"], x)
    dx = oracle.dispatch_backward(c, t["slot_of"], dR)
    valid = t["slot_src"] >= 0
    lhs = (bf16_bits_to_f32(recv[valid]).astype(np.int64) *
           bf16_bits_to_f32(dR[valid]).astype(np.int64)).sum()
    rhs = (bf16_bits_to_f32(x).astype(np.int64) * bf16_bits_to_f32(dx).astype(np.int64)).sum()
    assert lhs == rhs
    # per element: dx[t] is the sum of the K rows that token t was sent to
    ref = bf16_bits_to_f32(dR).astype(np.int64)[t["slot_of"]].reshape(R * S, K, H).sum(1)
    assert np.array_equal(bf16_bits_to_f32(dx).astype(np.int64), ref)


def test_dispatch_backward_of_dispatch_is_k_times_x():
    R, E, K, S, H = 4, 16, 4, 20, 32
    idx, _, _ = make_routing(R, E, K, S, 2.0, seed=14)
    c = cfg(R, E, K, S, H=H)
    st, t = oracle.plan(c, idx)
    x = integer_bf16((R * S, H), seed=14, bound=32)
    dx = oracle.dispatch_backward(c, t["slot_of"], oracle.dispatch(c, t["slot_of"], x))
    assert np.array_equal(bf16_bits_to_f32(dx), K * bf16_bits_to_f32(x))


def test_dispatch_backward_rounding_bound():
    R, E, K, S, H = 4, 16, 8, 12, 40
    idx, _, _ = make_routing(R, E, K, S, 3.0, seed=15)
    c = cfg(R, E, K, S, H=H)
    st, t = oracle.plan(c, idx)
    NvS = int(t["nvs"][0])
    dR = normal_bf16((R * NvS, H), seed=15, stream=21)
    dx = oracle.dispatch_backward(c, t["slot_of"], dR)
    terms = bf16_bits_to_f32(dR).astype(np.float64)[t["slot_of"]].reshape(R * S, K, H)
    exact = terms.sum(1)
    bound = _bf16_half_ulp(exact) * (1 + 2 ** -7) + K * 2.0 ** -23 * np.abs(terms).sum(1)
    assert (np.abs(bf16_bits_to_f32(dx) - exact) <= bound).all()


# --------------------------------------------------------- prefetch_weight ---


@pytest.mark.parametrize("case", [(8, 32, 4, 64, 4, 6.0), (4, 16, 2, 40, 1, 4.0)])
def test_prefetch_copies_home_weights_into_local_slots(case):
    R, E, K, S, B, mv = case
    idx, _, _ = make_routing(R, E, K, S, mv, seed=16)
    c = cfg(R, E, K, S, budget=B, mode=1)
    st, t = oracle.plan(c, idx)
    W = 20
    w = normal_bf16((E, W), seed=16, stream=22)
    before = normal_bf16((R, B, W), seed=17, stream=23)
    after = oracle.prefetch_weight(c, t, w, before)
    filled = np.zeros((R, B), bool)
    for d in range(R):
        for j in range(B):
            e = t["rep_expert"][d * B + j]
            if e >= 0:
                assert np.array_equal(after[d, j], w[e])
                filled[d, j] = True
    assert np.array_equal(after[~filled], before[~filled])
    assert filled.sum() == int((t["piece_wslot"] >= 0).sum())


def test_prefetch_all_tokens_on_one_expert():
    """Expert 0's overflow lands on every other rank, each holding its weights in slot 0."""
    R, S = 4, 6
    c = cfg(R, R, 1, S, budget=2, mode=1)
    st, t = oracle.plan(c, np.zeros((R, S, 1), np.int32))
    w = normal_bf16((R, 8), seed=18, stream=24)
    after = oracle.prefetch_weight(c, t, w, np.zeros((R, 2, 8), np.uint16))
    assert np.array_equal(after[1:, 0], np.broadcast_to(w[0], (R - 1, 8)))
    assert not after[0].any() and not after[1:, 1].any()


# ------------------------------------------------------- segment weights ---


def test_segment_weights_worked_example():
    """The worked example by hand (R=2, E=4, S=3, K=2): rank 0 holds experts 0 and 1
    natively; rank 1 holds 2 and 3 and the overflow of expert 1 as a replica piece in
    weight slot 0.  With W = 5: native segments read home rows e * 5, the piece reads
    replica slot (rank 1 * budget 2 + slot 0) * 5; the remaining entries read nothing."""
    c = cfg(2, 4, 2, 3, budget=2)
    idx = np.array([[[0, 1], [0, 1], [1, 2]], [[0, 1], [0, 3], [1, 2]]], np.int32)
    _, t = oracle.plan(c, idx)
    buf, off = oracle.segment_weights(c, t, 5)
    assert buf.tolist() == [[0, 0, -1, -1], [0, 0, 1, -1]]
    assert off.tolist() == [[0, 5, -1, -1], [10, 15, 10, -1]]
    # past the budget (budget 0) the piece is remote: it reads the home expert's row
    c0 = cfg(2, 4, 2, 3, budget=0, mode=1)
    _, t0 = oracle.plan(c0, idx)
    buf0, off0 = oracle.segment_weights(c0, t0, 5)
    assert buf0[1, 2] == 0 and off0[1, 2] == 1 * 5


@pytest.mark.parametrize("case", [(8, 64, 8, 96, 8, 20.0, 0), (8, 64, 8, 96, 2, 20.0, 1),
                                  (4, 32, 4, 50, 0, 5.0, 1), (3, 9, 3, 40, 3, 3.0, 0)])
def test_segment_weights_against_piece_tables(case):
    """Derived from the piece list and the replica-slot table instead of the segment
    table: each local piece reads slot (rank * budget + slot) and that slot holds the
    piece's expert; each remote piece and each native expert reads the home row; every
    rank has exactly n_seg entries that read something."""
    R, E, K, S, B, mv, mode = case
    c = cfg(R, E, K, S, budget=B, mode=mode)
    idx, _, _ = make_routing(R, E, K, S, mv, seed=31)
    st, t = oracle.plan(c, idx)
    W = 7
    buf, off = oracle.segment_weights(c, t, W)
    L = E // R
    expect = {}  # (rank, expert) -> (buf, off)
    for d in range(R):
        for i in range(L):
            expect[(d, d * L + i)] = (0, (d * L + i) * W)
    n_piece = int(t["n_piece"][0])
    for p in range(n_piece):
        d, e, j = int(t["piece_rank"][p]), int(t["piece_expert"][p]), int(t["piece_wslot"][p])
        if j >= 0:
            assert t["rep_expert"][d * B + j] == e
            expect[(d, e)] = (1, (d * B + j) * W)
        else:
            expect[(d, e)] = (0, e * W)
    got = {}
    for d in range(R):
        for i in range(E):
            if buf[d, i] >= 0:
                got[(d, int(t["seg_expert"][d, i]))] = (int(buf[d, i]), int(off[d, i]))
            else:
                assert off[d, i] == -1
        assert (buf[d] >= 0).sum() == t["n_seg"][d]
    assert got == expect


# ------------------------------------------------------- reduce_grad, fp32 ---


@pytest.mark.parametrize("case", [(8, 32, 4, 64, 4, 6.0), (8, 64, 8, 32, 8, 15.0)])
def test_reduce_grad_f32_equals_no_replication(case):
    """The fp32 fold reproduces the no-replication gradient exactly with integer
    gradients up to a few thousand: exact in fp32 but not in bf16 (integers past 256
    round there), so a fold that rounds through bf16 anywhere fails."""
    R, E, K, S, B, mv = case
    idx, _, _ = make_routing(R, E, K, S, mv, seed=18)
    c = cfg(R, E, K, S, budget=B)
    st, t = oracle.plan(c, idx)
    assert st == oracle.OK and int(t["n_piece"][0]) > 0
    P = 16
    NvS = int(t["nvs"][0])
    g = np.random.default_rng(18).integers(-300, 301, size=(R * NvS, P)).astype(np.int64)
    ref = np.zeros((E, P), np.int64)
    np.add.at(ref, idx.ravel(), g[t["slot_of"]])
    home = np.zeros((E, P), np.int64)
    rep = np.zeros((R, B, P), np.int64)
    L = E // R
    for d in range(R):
        for i in range(int(t["n_seg"][d])):
            e, s0, ln = t["seg_expert"][d, i], t["seg_start"][d, i], t["seg_len"][d, i]
            part = g[d * NvS + s0: d * NvS + s0 + ln].sum(0)
            if i < L:
                home[e] += part
            else:
                rep[d, t["seg_wslot"][d, i]] += part
    assert np.abs(ref).max() > 256 and np.abs(ref).max() < 2 ** 24  # beyond bf16, exact in fp32
    new = oracle.reduce_grad_f32(c, t, rep.astype(np.float32), home.astype(np.float32))
    assert new.dtype == np.float32
    assert np.array_equal(new.astype(np.int64), ref)


def test_reduce_grad_f32_adds_home_first_then_pieces_by_rank():
    """All tokens on expert 0 of 3 ranks: its overflow is one piece on rank 1 and one on
    rank 2.  home = 1, rank 1's piece = 1, rank 2's = 2**24: ((1 + 1) + 2**24) = 2**24 + 2
    exactly, while the other orders lose a 1 to rounding (2**24 + 1 is not an fp32)."""
    R, E, K, S, B = 3, 3, 1, 4, 1
    c = cfg(R, E, K, S, budget=B)
    idx = np.zeros((R, S, K), np.int32)
    st, t = oracle.plan(c, idx)
    n = int(t["n_piece"][0])
    pe, pr, pw = t["piece_expert"][:n], t["piece_rank"][:n], t["piece_wslot"][:n]
    assert list(pe) == [0, 0] and list(pr) == [1, 2] and list(pw) == [0, 0]
    P = 2
    home = np.zeros((E, P), np.float32)
    home[0] = 1.0
    rep = np.zeros((R, B, P), np.float32)
    rep[1, 0] = 1.0
    rep[2, 0] = 2.0 ** 24
    new = oracle.reduce_grad_f32(c, t, rep, home)
    assert (new[0] == np.float32(2.0 ** 24 + 2)).all()
    assert np.float32(np.float32(1.0 + 2.0 ** 24) + 1.0) == np.float32(2.0 ** 24)  # the other orders
    assert (new[1:] == 0).all()


def test_reduce_grad_f32_leaves_unreplicated_experts_alone():
    R, E, K, S, B = 4, 16, 2, 30, 2
    idx, _, _ = make_routing(R, E, K, S, 4.0, seed=9)
    c = cfg(R, E, K, S, budget=B)
    st, t = oracle.plan(c, idx)
    P = 10
    rng = np.random.default_rng(19)
    home = rng.standard_normal((E, P)).astype(np.float32)
    rep = rng.standard_normal((R, B, P)).astype(np.float32)
    new = oracle.reduce_grad_f32(c, t, rep, home)
    touched = np.zeros(E, bool)
    touched[t["piece_expert"][t["piece_wslot"] >= 0]] = True
    assert touched.any() and not touched.all()
    assert np.array_equal(new[~touched], home[~touched])


# ------------------------------------------ the order of the fp32 additions ---
# Three terms 2**24, 1, -2**24 (each exact in bf16): added in that order they give 0,
# because 2**24 + 1 rounds back to 2**24 in fp32; in any other order the 1 survives.
# So these pin the order each fold takes (the reading: ascending k for a token's
# slots, the home gradient first and then the pieces by ascending receiving rank),
# which the rounding bounds and the integer identities above do not see.
_ORDERED = np.array([2.0 ** 24, 1.0, -(2.0 ** 24)], np.float32)


def test_combine_accumulates_in_ascending_k():
    c = cfg(1, 3, 3, 1, H=2, budget=0)
    slot_of = np.array([0, 1, 2], np.int32)
    y = f32_to_bf16_bits(np.repeat(_ORDERED[:, None], 2, axis=1))
    out = oracle.combine(c, slot_of, y, np.ones(3, np.float32))
    assert (bf16_bits_to_f32(out) == 0.0).all()
    rev = oracle.combine(c, slot_of[::-1].copy(), y, np.ones(3, np.float32))
    assert (bf16_bits_to_f32(rev) == 1.0).all()  # the same three rows in the other order


def test_dispatch_backward_adds_in_ascending_k():
    c = cfg(1, 3, 3, 1, H=2, budget=0)
    slot_of = np.array([0, 1, 2], np.int32)
    drecv = f32_to_bf16_bits(np.repeat(_ORDERED[:, None], 2, axis=1))
    assert (bf16_bits_to_f32(oracle.dispatch_backward(c, slot_of, drecv)) == 0.0).all()
    rev = oracle.dispatch_backward(c, slot_of[::-1].copy(), drecv)
    assert (bf16_bits_to_f32(rev) == 1.0).all()


def test_reduce_grad_adds_home_first_then_pieces_by_rank():
    """All tokens on expert 0 of 3 ranks: its overflow is one piece on rank 1 and one on
    rank 2.  home = 2**24, rank 1's piece 1, rank 2's piece -2**24 fold to 0."""
    R, E, K, S, B = 3, 3, 1, 4, 1
    c = cfg(R, E, K, S, budget=B)
    st, t = oracle.plan(c, np.zeros((R, S, K), np.int32))
    n = int(t["n_piece"][0])
    assert list(t["piece_expert"][:n]) == [0, 0] and list(t["piece_rank"][:n]) == [1, 2]
    P = 2
    home = np.zeros((E, P), np.float32)
    home[0] = _ORDERED[0]
    rep = np.zeros((R, B, P), np.float32)
    rep[1, 0] = _ORDERED[1]
    rep[2, 0] = _ORDERED[2]
    new = oracle.reduce_grad(c, t, f32_to_bf16_bits(rep), f32_to_bf16_bits(home))
    assert (bf16_bits_to_f32(new) == 0.0).all()
    new32 = oracle.reduce_grad_f32(c, t, rep, home)
    assert (new32 == 0.0).all()


@settings(max_examples=120, deadline=None, derandomize=True)
@given(R=hs.integers(1, 8), L=hs.integers(1, 4), K=hs.integers(1, 8), S=hs.integers(1, 40),
       budget_frac=hs.floats(0, 1), mode=hs.integers(0, 1), align=hs.sampled_from([1, 2, 4]),
       alpha=hs.floats(0, 3), seed=hs.integers(0, 2**31 - 1))
def test_reduce_grad_folds_property(R, L, K, S, budget_frac, mode, align, alpha, seed):
    """Both folds over drawn plans, REMOTE pieces included.  Each buffer row carries an
    integer gradient; home rows sum a rank's native segments, replica slots their local
    pieces.  After the fold every expert holds the gradient of all its pairs except the
    rows of its REMOTE pieces (they have no replica slot and add nothing)."""
    E = R * L
    K = min(K, E)
    B = int(round(budget_frac * L))
    p = (np.arange(E) + 1.0) ** -alpha
    rng = np.random.default_rng(seed)
    idx = rng.choice(E, size=(R, S, K), p=p / p.sum()).astype(np.int32)
    c = cfg(R, E, K, S, budget=B, mode=mode, align=align)
    st, t = oracle.plan(c, idx)
    assert st in (oracle.OK, oracle.BUDGET)
    NvS, P = int(t["nvs"][0]), 3
    g = rng.integers(-2, 3, size=(R * NvS, P)).astype(np.int64)
    want = np.zeros((E, P), np.int64)
    np.add.at(want, idx.ravel(), g[t["slot_of"]])  # no replication: all of e's pairs
    home = np.zeros((E, P), np.int64)
    rep = np.zeros((R, max(B, 1), P), np.int64)
    for d in range(R):
        for i in range(int(t["n_seg"][d])):
            e, s0, ln = t["seg_expert"][d, i], t["seg_start"][d, i], t["seg_len"][d, i]
            part = g[d * NvS + s0: d * NvS + s0 + ln].sum(0)
            if i < L:
                home[e] += part
            elif t["seg_wslot"][d, i] >= 0:
                rep[d, t["seg_wslot"][d, i]] += part
            else:
                want[e] -= part  # a REMOTE piece: its rows are not folded
    got32 = oracle.reduce_grad_f32(c, t, rep[:, :B].astype(np.float32), home.astype(np.float32))
    assert np.array_equal(got32.astype(np.int64), want)
    if max(np.abs(want).max(), np.abs(home).max(), np.abs(rep).max()) <= 256:  # exact in bf16
        to_bf16 = lambda a: f32_to_bf16_bits(a.astype(np.float32))
        got = oracle.reduce_grad(c, t, to_bf16(rep[:, :B]), to_bf16(home))
        assert np.array_equal(bf16_bits_to_f32(got).astype(np.int64), want)


@settings(max_examples=100, deadline=None, derandomize=True)
@given(R=hs.integers(1, 8), L=hs.integers(1, 4), K=hs.integers(1, 8), S=hs.integers(1, 40),
       budget_frac=hs.floats(0, 1), mode=hs.integers(0, 1), alpha=hs.floats(0, 3),
       seed=hs.integers(0, 2**31 - 1))
def test_replica_weights_property(R, L, K, S, budget_frac, mode, alpha, seed):
    """prefetch_weight and segment_weights over drawn plans, REMOTE pieces included:
    every local piece's slot holds its expert's row and every other slot is untouched;
    every segment reads its replica slot (local piece) or the home row (native segment,
    REMOTE piece), derived here from the piece list rather than the segment table."""
    E = R * L
    K = min(K, E)
    B = int(round(budget_frac * L))
    p = (np.arange(E) + 1.0) ** -alpha
    rng = np.random.default_rng(seed)
    idx = rng.choice(E, size=(R, S, K), p=p / p.sum()).astype(np.int32)
    c = cfg(R, E, K, S, budget=B, mode=mode)
    st, t = oracle.plan(c, idx)
    W = 5
    w = rng.integers(0, 1 << 16, size=(E, W)).astype(np.uint16)
    before = rng.integers(0, 1 << 16, size=(R, B, W)).astype(np.uint16)
    after = oracle.prefetch_weight(c, t, w, before)
    n = int(t["n_piece"][0])
    pe, pr, pw = t["piece_expert"][:n], t["piece_rank"][:n], t["piece_wslot"][:n]
    filled = np.zeros((R, B), bool)
    expect = {(d, d * L + i): (0, (d * L + i) * W) for d in range(R) for i in range(L)}
    for e, d, j in zip(pe, pr, pw):
        if j >= 0:
            assert np.array_equal(after[d, j], w[e])
            filled[d, j] = True
            expect[(int(d), int(e))] = (1, (int(d) * B + int(j)) * W)
        else:
            expect[(int(d), int(e))] = (0, int(e) * W)
    assert np.array_equal(after[~filled], before[~filled])
    buf, off = oracle.segment_weights(c, t, W)
    got = {(d, int(t["seg_expert"][d, i])): (int(buf[d, i]), int(off[d, i]))
           for d in range(R) for i in range(E) if buf[d, i] >= 0}
    assert got == expect


@settings(max_examples=100, deadline=None, derandomize=True)
@given(R=hs.integers(1, 8), L=hs.integers(1, 4), K=hs.integers(1, 8), S=hs.integers(1, 40),
       budget_frac=hs.floats(0, 1), mode=hs.integers(0, 1), align=hs.sampled_from([1, 2, 4, 16]),
       alpha=hs.floats(0, 3), seed=hs.integers(0, 2**31 - 1))
def test_data_path_property(R, L, K, S, budget_frac, mode, align, alpha, seed):
    """dispatch, the identity expert's combine and dispatch-backward over drawn plans
    (repeated experts in a token, padding rows, REMOTE pieces): every valid row is its
    source token's row and padding rows keep what was there; combine equals sum_k w_k x
    within the bf16 + fp32 rounding bound; dispatch-backward of dispatch is K x exactly
    on small integers (§8 exercise C; the adjoint of dispatch)."""
    E = R * L
    K = min(K, E)
    B = int(round(budget_frac * L))
    p = (np.arange(E) + 1.0) ** -alpha
    rng = np.random.default_rng(seed)
    idx = rng.choice(E, size=(R, S, K), p=p / p.sum()).astype(np.int32)
    c = cfg(R, E, K, S, H=4, budget=B, mode=mode, align=align)
    st, t = oracle.plan(c, idx)
    T, H, NvS = R * S, 4, int(t["nvs"][0])
    x = f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    poison = np.full((R * NvS, H), 0xFFC1, np.uint16)
    recv = oracle.dispatch(c, t["slot_of"], x, poison.copy())
    valid = t["slot_src"] >= 0
    assert np.array_equal(recv[valid], x[t["slot_src"][valid] // K])
    assert (recv[~valid] == 0xFFC1).all()
    z = rng.standard_normal((T, K))
    w = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    out = oracle.combine(c, t["slot_of"], recv, w)
    exact = w.astype(np.float64).sum(1, keepdims=True) * bf16_bits_to_f32(x).astype(np.float64)
    bound = _bf16_half_ulp(exact) * (1 + 2 ** -7) + K * 2.0 ** -24 * np.abs(exact) * 2
    assert (np.abs(bf16_bits_to_f32(out).astype(np.float64) - exact) <= bound).all()
    xi = f32_to_bf16_bits(rng.integers(-16, 17, size=(T, H)).astype(np.float32))
    dx = oracle.dispatch_backward(c, t["slot_of"], oracle.dispatch(c, t["slot_of"], xi))
    assert np.array_equal(bf16_bits_to_f32(dx), K * bf16_bits_to_f32(xi))

"""The C-ABI library loads and exports what include/moonep.h declares (no GPU needed).

Only host-side calls run here: size queries, plan-view pointer arithmetic and
argument checks that return before any CUDA call.
"""
import ctypes

import numpy as np
import pytest

import oracle
import token_dispatch_moonep_b200 as me


def test_exports_every_declared_function():
    names = me.header_functions()
    assert {"moonep_plan", "moonep_dispatch", "moonep_combine", "moonep_combine_backward",
            "moonep_reduce_grad", "moonep_nvs", "moonep_plan_bytes", "moonep_workspace_bytes",
            "moonep_plan_view", "moonep_status_string"} <= set(names)
    lib = ctypes.CDLL(me.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    for n in names:  # and the binding exposes each under the same name
        assert callable(getattr(me, n)), n


def test_library_keeps_internal_symbols_hidden():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", me.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert {n for n in exported if n.startswith("moonep_")} == set(me.header_functions())


@pytest.mark.parametrize("shape", [(8, 32, 4, 256, 1), (8, 256, 8, 4096, 1), (2, 4, 2, 3, 4),
                                   (64, 256, 8, 128, 1), (3, 9, 3, 17, 8), (4, 8, 2, 0, 16),
                                   (8, 64, 8, 64, 128)])
def test_nvs_matches_oracle(shape):
    R, E, K, S, A = shape
    c = me.Config(R=R, E=E, K=K, S=S, H=8, budget=E // R, align=A)
    oc = oracle.Config(R=R, E=E, K=K, S=S, H=8, budget=E // R, align=A)
    assert me.moonep_nvs(c) == oracle.nvs(oc)
    if A == 1:
        assert me.moonep_nvs(c) == S * K


@pytest.mark.parametrize("bad", [dict(R=3, E=8), dict(E=0), dict(K=0), dict(K=33, E=64),
                                 dict(K=9, E=8), dict(S=-1), dict(budget=-1), dict(budget=9),
                                 dict(mode=2), dict(align=0), dict(align=5000), dict(E=2048, R=8),
                                 dict(R=0)])
def test_invalid_configs_rejected_on_host(bad):
    kw = dict(R=2, E=8, K=2, S=4, H=8, budget=4, mode=0, align=1)
    kw.update(bad)
    c = me.Config(**kw)
    assert me.moonep_nvs(c) == -1
    assert me.moonep_plan_bytes(c) == 0
    assert me.moonep_workspace_bytes(c) == 0
    # the check happens before any CUDA call, so it is safe without a device
    fake = 1 << 20
    st = me._lib.moonep_plan(ctypes.byref(c), fake, fake, fake, fake, 0)
    assert st == me.ERR_INVALID_ARG
    st = me._lib.moonep_dispatch(ctypes.byref(c), fake, fake, fake, fake, 0)
    assert st == me.ERR_INVALID_ARG


def test_too_many_pairs_rejected():
    c = me.Config(R=8, E=256, K=8, S=1 << 25, H=8, budget=32)
    assert me.moonep_plan_bytes(c) == 0


def test_null_and_misaligned_pointers_rejected_on_host():
    c = me.Config(R=2, E=4, K=2, S=3, H=8, budget=2)
    base = 1 << 30
    L = me._lib
    cp = ctypes.byref(c)
    assert L.moonep_plan(cp, None, base, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan(cp, base, None, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan(cp, base, base, None, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan(cp, base, base, base, None, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan(cp, base, base + 16, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan(cp, base, base, base + 8, base, 0) == me.ERR_INVALID_ARG
    # the allocation-free plan checks the same arguments before any CUDA call
    assert L.moonep_plan_static(cp, None, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan_static(cp, base, None, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan_static(cp, base, base, None, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan_static(cp, base, base + 16, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_dispatch(cp, base, None, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_combine(cp, base, base, None, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_combine_backward(cp, base, base, base, base, None, base, base, 0) == \
        me.ERR_INVALID_ARG
    assert L.moonep_reduce_grad(cp, base, base, base, 0, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_reduce_grad(cp, base, None, base, 16, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_reduce_grad_f32(cp, base, base, base, 0, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_reduce_grad_f32(cp, base, None, base, 16, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_reduce_grad_f32(cp, base, base, None, 16, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_reduce_grad_f32(cp, base, base, base, 16, None, 0) == me.ERR_INVALID_ARG
    assert L.moonep_reduce_grad_f32(cp, base + 16, base, base, 16, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_plan_view(cp, None, ctypes.byref(me.PlanView())) == me.ERR_INVALID_ARG
    assert L.moonep_dispatch_backward(cp, base, None, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_dispatch_backward(cp, base, base, None, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_prefetch_weight(cp, base, None, base, 16, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_prefetch_weight(cp, base, base, None, 16, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_prefetch_weight(cp, base, base, base, 0, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_dispatch_via_buffer(cp, base, base, None, base, base, base, 0) == \
        me.ERR_INVALID_ARG
    assert L.moonep_segment_weights(cp, base, None, base, 16, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_segment_weights(cp, base, base, None, 16, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_segment_weights(cp, base, base, base, 0, base, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_segment_weights(cp, base, base, base, 16, None, base, 0) == me.ERR_INVALID_ARG
    assert L.moonep_segment_weights(cp, base, base, base, 16, base + 4, base, 0) == \
        me.ERR_INVALID_ARG
    assert L.moonep_segment_weights(cp, base + 16, base, base, 16, base, base, 0) == \
        me.ERR_INVALID_ARG
    assert L.moonep_combine_via_buffer(cp, base, base, base, None, base, base, base, 0) == \
        me.ERR_INVALID_ARG
    c13 = me.Config(R=2, E=4, K=2, S=3, H=13, budget=2)  # rows not 16-byte multiples
    assert L.moonep_dispatch_via_buffer(ctypes.byref(c13), base, base, base, base, base, base, 0) == \
        me.ERR_UNSUPPORTED


def test_empty_batch_enqueues_nothing():
    # S = 0: data calls return OK without touching any pointer or the device
    c = me.Config(R=2, E=4, K=2, S=0, H=8, budget=2)
    base = 1 << 30
    L = me._lib
    cp = ctypes.byref(c)
    assert L.moonep_dispatch(cp, base, None, None, base, 0) == me.OK
    assert L.moonep_combine(cp, base, None, None, None, base, 0) == me.OK
    assert L.moonep_combine_backward(cp, base, None, None, None, None, None, base, 0) == me.OK


@pytest.mark.parametrize("shape", [(8, 256, 8, 4096, 32), (2, 4, 2, 3, 0), (64, 256, 8, 128, 4)])
def test_plan_view_layout(shape):
    R, E, K, S, B = shape
    c = me.Config(R=R, E=E, K=K, S=S, H=8, budget=B)
    base = 1 << 32
    v = me.moonep_plan_view_ptrs(c, base)
    total = me.moonep_plan_bytes(c)
    NvS = me.moonep_nvs(c)
    assert v.nvs == NvS and v.max_pieces == E + R
    sizes = dict(slot_of=R * S * K, slot_src=R * NvS, expert_count=E, rank_load=R, overflow=R,
                 deficit=R, n_seg=R, seg_expert=R * E, seg_start=R * E, seg_len=R * E,
                 seg_kind=R * E, seg_wslot=R * E, piece_expert=E + R, piece_rank=E + R,
                 piece_start=E + R, piece_len=E + R, piece_wslot=E + R, piece_ostart=E + R,
                 expert_piece_begin=E, expert_piece_end=E, rep_expert=R * B,
                 replicated_experts=E, scalars=8)
    spans = []
    for name, n in sizes.items():
        p = getattr(v, name)
        assert p % 256 == 0
        spans.append((p - base, p - base + 4 * n))
    spans.sort()
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0
    assert spans[-1][1] <= total
    assert me.moonep_workspace_bytes(c) > 0


def test_status_strings():
    for s in (me.OK, me.ERR_INVALID_ARG, me.ERR_CUDA, me.ERR_UNSUPPORTED):
        assert me.moonep_status_string(s)
    assert me.moonep_status_string(99) == "unknown status"


def test_debug_wait_knob_validates_arguments():
    assert me._lib.moonep_debug_set_wait(-1, 0) == me.ERR_INVALID_ARG
    assert me._lib.moonep_debug_set_wait(1000, 33) == me.ERR_INVALID_ARG
    assert me._lib.moonep_debug_set_wait(1000, -1) == me.ERR_INVALID_ARG
    assert me._lib.moonep_debug_set_wait(me.DEFAULT_WAIT_NS, 0) == me.OK


def test_fused_forward_checks_arguments_on_host():
    """The fused layer refuses, before any CUDA call, what its one-launch design cannot
    do: K not dividing 512 or above 8, rows that are not 16-byte multiples, misaligned
    rows; and null pointers."""
    L = me._lib
    base = 1 << 30
    ok = me.Config(R=2, E=8, K=2, S=4, H=16, budget=2)
    cp = ctypes.byref(ok)
    assert L.moonep_fused_forward(cp, None, base, base, base, base, base, base, base, 0) == \
        me.ERR_INVALID_ARG
    assert L.moonep_fused_forward(cp, base, base, base, base, base, base, base, None, 0) == \
        me.ERR_INVALID_ARG
    assert L.moonep_fused_forward(cp, base, base, base, base + 16, base, base, base, base, 0) == \
        me.ERR_INVALID_ARG
    assert L.moonep_fused_forward(cp, base, base, base + 2, base, base, base, base, base, 0) == \
        me.ERR_UNSUPPORTED
    for bad in (me.Config(R=2, E=8, K=3, S=4, H=16, budget=2),
                me.Config(R=2, E=32, K=16, S=4, H=16, budget=2),
                me.Config(R=2, E=8, K=2, S=4, H=12, budget=2)):
        assert L.moonep_fused_forward(ctypes.byref(bad), base, base, base, base, base, base, base,
                                      base, 0) == me.ERR_UNSUPPORTED

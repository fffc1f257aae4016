"""The GPU path adds in the order the oracle's pins fix.

Three terms 2**24, 1, -2**24 (each exact in bf16) sum to 0 only in that order
(2**24 + 1 rounds back to 2**24 in fp32) and to 1 in any other.  Placing them in a
token's slots k = 0, 1, 2 (combine, dispatch-backward) or in the home gradient and
the pieces of ranks 1 and 2 (reduce_grad) checks the kernels' order directly, on the
vector paths and on the scalar ones (rows that are not whole 16-byte vectors)."""
import numpy as np
import pytest

from gpu_util import configs, gpu_plan, to_dev, to_np
from moonep_inputs import bf16_bits_to_f32, f32_to_bf16_bits, make_routing

pytestmark = pytest.mark.gpu

_ORDERED = np.array([2.0 ** 24, 1.0, -(2.0 ** 24)], np.float32)


def _slot_rows(H):
    """A plan with K = 3 and rows y[slot_of[t, k]] = _ORDERED[k] for every token."""
    import token_dispatch_moonep_b200 as me
    R, E, K, S = 2, 4, 3, 16
    cfg, _ = configs(R, E, K, S, H=H, budget=2)
    idx, _, _ = make_routing(R, E, K, S, 0.2, seed=2)
    _, arena, gv, _ = gpu_plan(cfg, idx)
    so = gv["slot_of"].reshape(R * S, K)
    y = np.zeros((R * me.moonep_nvs(cfg), H), np.float32)
    for k in range(K):
        y[so[:, k]] = _ORDERED[k]
    return cfg, arena, f32_to_bf16_bits(y), R * S


@pytest.mark.parametrize("H", [8, 2048, 5])
def test_combine_accumulates_in_ascending_k(H):
    import torch
    import token_dispatch_moonep_b200 as me
    cfg, arena, y, T = _slot_rows(H)
    out = torch.full((T, H), 0x3F80, dtype=torch.int16, device="cuda")  # 1.0: must be overwritten
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    me.moonep_combine(cfg, arena, to_dev(y), to_dev(np.ones(T * cfg.K, np.float32)), out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert (bf16_bits_to_f32(to_np(out)) == 0.0).all()


@pytest.mark.parametrize("H", [8, 2048, 5])
def test_dispatch_backward_adds_in_ascending_k(H):
    import torch
    import token_dispatch_moonep_b200 as me
    cfg, arena, drecv, T = _slot_rows(H)
    dx = torch.full((T, H), 0x3F80, dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    me.moonep_dispatch_backward(cfg, arena, to_dev(drecv), dx, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert (bf16_bits_to_f32(to_np(dx)) == 0.0).all()


@pytest.mark.parametrize("P", [8, 4096 + 8, 13])
def test_reduce_grad_adds_home_first_then_pieces_by_rank(P):
    """All tokens on expert 0 of 3 ranks: pieces on ranks 1 and 2 (bulk and scalar paths)."""
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, B = 3, 3, 1, 4, 1
    cfg, _ = configs(R, E, K, S, H=8, budget=B)
    _, arena, gv, _ = gpu_plan(cfg, np.zeros((R, S, K), np.int32))
    home = np.zeros((E, P), np.float32)
    home[0] = _ORDERED[0]
    rep = np.zeros((R, B, P), np.float32)
    rep[1, 0] = _ORDERED[1]
    rep[2, 0] = _ORDERED[2]
    h = to_dev(f32_to_bf16_bits(home))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    me.moonep_reduce_grad(cfg, arena, to_dev(f32_to_bf16_bits(rep)), h, P, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert (bf16_bits_to_f32(to_np(h)) == 0.0).all()

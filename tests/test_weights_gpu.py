"""moonep_segment_weights against the oracle: the weight matrix of every entry of the
plan's segment tables, as device pointers into the home and replica weight buffers."""
import numpy as np
import pytest

import oracle
from moonep_inputs import make_routing
from tests.gpu_util import configs, gpu_plan

pytestmark = pytest.mark.gpu


def _decode(ptrs, w_base, w_bytes, r_base, r_bytes):
    """(buffer, element offset) of each pointer: 0 home, 1 replica, -1 null."""
    buf = np.full(ptrs.shape, -2, np.int32)
    off = np.full(ptrs.shape, -2, np.int64)
    null = ptrs == 0
    buf[null], off[null] = -1, -1
    home = (ptrs >= w_base) & (ptrs < w_base + w_bytes)
    buf[home], off[home] = 0, (ptrs[home] - w_base) // 2
    rep = (ptrs >= r_base) & (ptrs < r_base + r_bytes)
    buf[rep], off[rep] = 1, (ptrs[rep] - r_base) // 2
    return buf, off


@pytest.mark.parametrize("case", [(8, 64, 8, 96, 8, 0, 20.0, 1), (8, 64, 8, 96, 2, 1, 20.0, 1),
                                  (4, 32, 4, 50, 0, 1, 5.0, 1), (3, 9, 3, 40, 3, 0, 3.0, 16),
                                  (64, 256, 8, 128, 4, 1, 20.0, 1)])
def test_segment_weights_match_oracle(case):
    import torch
    import token_dispatch_moonep_b200 as me
    R, E, K, S, B, mode, mv, A = case
    W = 24
    cfg, ocfg = configs(R, E, K, S, budget=B, mode=mode, align=A)
    idx, _, _ = make_routing(R, E, K, S, mv, seed=33)
    st, arena, gv, _ = gpu_plan(cfg, idx)
    _, ot = oracle.plan(ocfg, idx)
    ref_buf, ref_off = oracle.segment_weights(ocfg, ot, W)
    w = torch.zeros((E, W), dtype=torch.int16, device="cuda")
    rep = torch.zeros((max(R * B, 1), W), dtype=torch.int16, device="cuda")
    ptrs = torch.full((R * E,), -7, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    me.moonep_segment_weights(cfg, arena, w, rep if B > 0 else None, W, ptrs, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    buf, off = _decode(ptrs.cpu().numpy().reshape(R, E), w.data_ptr(), E * W * 2,
                       rep.data_ptr(), R * B * W * 2)
    assert np.array_equal(buf, ref_buf)
    assert np.array_equal(off, ref_off)
    if mode == 1 and mv >= 20:
        assert (ot["seg_kind"] == 2).any()  # remote pieces are among the entries checked

"""The oracle and the GPU path against the stored fixtures in tests/golden/."""
import glob
import json
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
FIXTURES = sorted(glob.glob(os.path.join(HERE, "golden", "*.json")))


def _load(path):
    with open(path) as f:
        r = json.load(f)
    c = r["config"]
    idx = np.array(r["topk_idx"], np.int32).reshape(c["R"], c["S"], c["K"])
    gates = np.array([float.fromhex(h) for h in r["gates_f32_hex"]], np.float32)
    x = np.array(r["x_bf16_bits"], np.uint16).reshape(c["R"] * c["S"], c["H"])
    return r, c, idx, gates.reshape(-1, c["K"]), x


@pytest.mark.parametrize("path", FIXTURES, ids=[os.path.basename(p) for p in FIXTURES])
def test_oracle_reproduces_fixture(path):
    r, c, idx, gates, x = _load(path)
    cfg = oracle.Config(**c)
    st, t = oracle.plan(cfg, idx)
    assert st == r["status"]
    for k, v in r["plan"].items():
        assert np.asarray(t[k]).ravel().tolist() == v, k
    recv = oracle.dispatch(cfg, t["slot_of"], x)
    out = oracle.combine(cfg, t["slot_of"], recv, gates)
    assert out.ravel().tolist() == r["combine_identity_bf16_bits"]


@pytest.mark.gpu
@pytest.mark.parametrize("path", FIXTURES, ids=[os.path.basename(p) for p in FIXTURES])
def test_gpu_reproduces_fixture(path):
    import torch
    import token_dispatch_moonep_b200 as me
    from tests.gpu_util import gpu_plan, to_dev, to_np
    r, c, idx, gates, x = _load(path)
    cfg = me.Config(**c)
    st, arena, gv, _ = gpu_plan(cfg, idx)
    exp_st = me.DEV_BUDGET if r["status"] == oracle.BUDGET else 0
    assert st == exp_st
    n_piece = r["plan"]["n_piece"][0]
    for k in ("slot_of", "slot_src", "expert_count", "rank_load", "overflow", "deficit", "n_seg",
              "seg_expert", "seg_start", "seg_len", "seg_kind", "seg_wslot", "rep_expert"):
        assert gv[k].ravel().tolist() == r["plan"][k], k
    for k in ("piece_expert", "piece_rank", "piece_start", "piece_len", "piece_wslot",
              "piece_ostart"):
        assert gv[k][:n_piece].tolist() == r["plan"][k], k
    NvS = me.moonep_nvs(cfg)
    recv = torch.zeros((c["R"] * NvS, c["H"]), dtype=torch.int16, device="cuda")
    out = torch.empty((c["R"] * c["S"], c["H"]), dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    me.moonep_dispatch(cfg, arena, to_dev(x), recv, status)
    me.moonep_combine(cfg, arena, recv, to_dev(gates.ravel()), out, status)
    torch.cuda.synchronize()
    assert to_np(out).ravel().tolist() == r["combine_identity_bf16_bits"]

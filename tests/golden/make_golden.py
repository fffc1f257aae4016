"""Write the golden fixtures in this directory from the CPU oracle (and nothing else).

Each fixture stores its inputs and the oracle's outputs, so later changes to the
oracle or the kernels can be checked against a fixed record.  Run:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from moonep_inputs import make_gates, make_routing, make_x  # noqa: E402

CASES = [
    # name, R, E, K, S, H, budget, mode, align, maxvio, seed
    ("plan_r4_e16_k2_s24_a1_train", 4, 16, 2, 24, 8, 4, 0, 1, 3.0, 0),
    ("plan_r4_e16_k2_s24_a4_infer_b1", 4, 16, 2, 24, 8, 1, 1, 4, 3.0, 0),
    ("plan_r8_e32_k4_s16_a1_train", 8, 32, 4, 16, 16, 4, 0, 1, 6.0, 1),
]


def main():
    for name, R, E, K, S, H, B, mode, A, mv, seed in CASES:
        cfg = oracle.Config(R=R, E=E, K=K, S=S, H=H, budget=B, mode=mode, align=A)
        idx, _, _ = make_routing(R, E, K, S, mv, seed)
        gates = make_gates(R, S, K, seed).reshape(R * S, K)
        x = make_x(R, S, H, seed).reshape(R * S, H)
        st, t = oracle.plan(cfg, idx)
        recv = oracle.dispatch(cfg, t["slot_of"], x)
        out = oracle.combine(cfg, t["slot_of"], recv, gates)
        rec = {
            "what": "inputs and CPU-oracle outputs (written by tests/golden/make_golden.py)",
            "config": dict(R=R, E=E, K=K, S=S, H=H, budget=B, mode=mode, align=A),
            "topk_idx": idx.ravel().tolist(),
            "gates_f32_hex": [float(g).hex() for g in gates.ravel()],
            "x_bf16_bits": x.ravel().tolist(),
            "status": st,
            "plan": {k: np.asarray(v).ravel().tolist() for k, v in t.items()},
            "combine_identity_bf16_bits": out.ravel().tolist(),
        }
        with open(os.path.join(HERE, name + ".json"), "w") as f:
            json.dump(rec, f, separators=(",", ":"))
        print(name, "status", st, "pieces", int(t["n_piece"][0]))


if __name__ == "__main__":
    main()

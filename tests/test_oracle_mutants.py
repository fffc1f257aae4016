"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a scratch copy of oracle/moonep_oracle.c
(wrong keep/overflow cut, wrong receiver order, wrong layout, wrong weight
slot, a dropped term, a missing gate, a skipped replica, ignored alignment,
truncating instead of rounding, reversed per-expert order, a half dot
product, a remote piece or a replica slot mapped to the wrong weights, an fp32
fold that rounds through bf16, adds its pieces in the wrong order or adds the
home gradient last, a combine, dispatch-backward or bf16 fold that adds its
terms in the wrong order),
builds it with gcc, and runs the pin tests against it: at least one
pin must fail.  Everything runs on the CPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moonep_oracle.c")

MUTANTS = {
    "keep_tail_not_head": ("if (t < SK) {", "if (t >= out->rank_load[h] - SK) {"),
    "receivers_descending": ("for (d = 0; d < R; d++) {\n    int64_t need",
                             "for (d = R - 1; d >= 0; d--) {\n    int64_t need"),
    "native_segments_missing": ("for (e = d * L; e < (d + 1) * L; e++) {\n      int64_t idx = d * E + nseg;",
                                "for (e = d * L; e < (d + 1) * L && 0; e++) {\n      int64_t idx = d * E + nseg;"),
    "weight_slot_off_by_one": ("out->piece_wslot[n_piece] = (int32_t)j;",
                               "out->piece_wslot[n_piece] = (int32_t)(j + 1 < B ? j + 1 : j);"),
    "combine_drops_last_k": ("for (int64_t k = 0; k < K; k++) {\n        int64_t row = slot_of[t * K + k];\n        acc = fmaf",
                             "for (int64_t k = 0; k < K - 1; k++) {\n        int64_t row = slot_of[t * K + k];\n        acc = fmaf"),
    "backward_without_gate": ("float prod = w * g;", "float prod = g;"),
    "reduce_skips_first_piece": ("acc = acc + orc_bf16_to_f32(rep[slot * P + q]);",
                                 "if (i > 0) acc = acc + orc_bf16_to_f32(rep[slot * P + q]);"),
    "alignment_ignored": ("cursor += roundup64(kept[e], A);", "cursor += kept[e];"),
    "truncate_not_round": ("u += 0x7FFFu + lsb;", "u += 0;"),
    "expert_list_reversed": ("list[list_begin[e] + fill[e]] = p;",
                             "list[list_begin[e + 1] - 1 - fill[e]] = p;"),
    "dispatch_backward_drops_first_k": ("acc = acc + orc_bf16_to_f32(drecv[row * H + h]);",
                                        "if (k > 0) acc = acc + orc_bf16_to_f32(drecv[row * H + h]);"),
    "prefetch_wrong_expert": ("rep_w[slot * W + q] = w[(int64_t)piece_expert[i] * W + q];",
                              "rep_w[slot * W + q] = w[(int64_t)((piece_expert[i] + 1) % c->E) * W + q];"),
    "half_dot_product": ("dot += (double)g * (double)orc_bf16_to_f32(y[row * H + h]);",
                         "if (h % 2 == 0) dot += (double)g * (double)orc_bf16_to_f32(y[row * H + h]);"),
    "remote_piece_reads_replica_slot": ("} else if (seg_kind[q] == KIND_NATIVE || seg_kind[q] == KIND_REMOTE) {",
                                        "} else if (seg_kind[q] == KIND_NATIVE) {"),
    "replica_slot_of_rank_zero": ("off[q] = (d * B + seg_wslot[q]) * W;", "off[q] = seg_wslot[q] * W;"),
    "combine_k_descending": ("      for (int64_t k = 0; k < K; k++) {\n        int64_t row = slot_of[t * K + k];\n"
                             "        acc = fmaf(",
                             "      for (int64_t k = K - 1; k >= 0; k--) {\n        int64_t row = slot_of[t * K + k];\n"
                             "        acc = fmaf("),
    "dispatch_backward_k_descending": ("      for (int64_t k = 0; k < K; k++) {\n        int64_t row = slot_of[t * K + k];\n"
                                       "        acc = acc + orc_bf16_to_f32(drecv",
                                       "      for (int64_t k = K - 1; k >= 0; k--) {\n        int64_t row = slot_of[t * K + k];\n"
                                       "        acc = acc + orc_bf16_to_f32(drecv"),
    "reduce_pieces_descending": ("for (int32_t i = 0; i < n_piece; i++) {\n        if (piece_expert[i] != e"
                                 " || piece_wslot[i] < 0) continue;\n        int64_t slot = (int64_t)"
                                 "piece_rank[i] * B + piece_wslot[i];\n        acc = acc + orc_bf16_to_f32(rep[",
                                 "for (int32_t i = n_piece - 1; i >= 0; i--) {\n        if (piece_expert[i] != e"
                                 " || piece_wslot[i] < 0) continue;\n        int64_t slot = (int64_t)"
                                 "piece_rank[i] * B + piece_wslot[i];\n        acc = acc + orc_bf16_to_f32(rep["),
    "reduce_f32_rounds_through_bf16": ("      home[e * P + q] = acc;",
                                       "      home[e * P + q] = orc_bf16_to_f32(orc_f32_to_bf16(acc));"),
    "reduce_f32_pieces_descending": ("for (int32_t i = 0; i < n_piece; i++) {\n        if (piece_expert[i] != e"
                                     " || piece_wslot[i] < 0) continue;\n        int64_t slot = (int64_t)"
                                     "piece_rank[i] * B + piece_wslot[i];\n        acc = acc + rep[",
                                     "for (int32_t i = n_piece - 1; i >= 0; i--) {\n        if (piece_expert[i] != e"
                                     " || piece_wslot[i] < 0) continue;\n        int64_t slot = (int64_t)"
                                     "piece_rank[i] * B + piece_wslot[i];\n        acc = acc + rep["),
    "reduce_f32_home_added_last": ("      float acc = home[e * P + q];\n      for (int32_t i = 0; i < n_piece; i++) {\n"
                                   "        if (piece_expert[i] != e || piece_wslot[i] < 0) continue;\n"
                                   "        int64_t slot = (int64_t)piece_rank[i] * B + piece_wslot[i];\n"
                                   "        acc = acc + rep[slot * P + q];\n      }\n      home[e * P + q] = acc;",
                                   "      float acc = 0.0f;\n      for (int32_t i = 0; i < n_piece; i++) {\n"
                                   "        if (piece_expert[i] != e || piece_wslot[i] < 0) continue;\n"
                                   "        int64_t slot = (int64_t)piece_rank[i] * B + piece_wslot[i];\n"
                                   "        acc = acc + rep[slot * P + q];\n      }\n"
                                   "      home[e * P + q] = acc + home[e * P + q];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {name}"
    mut_c = tmp_path / "mutant.c"
    mut_c.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-w", "-o", str(lib), str(mut_c), "-lm"])
    env = dict(os.environ, MOONEP_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin caught the mutant '{name}':\n{r.stdout[-1500:]}"

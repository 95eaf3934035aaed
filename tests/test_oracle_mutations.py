"""Plants plausible mistakes in a temporary copy of the oracle (on the CPU)
and checks that the pins (tests/_pins.py) catch each one.

The mistakes cover the scoring definition (a dropped ReLU, a transposed
operand, a wrong sign, a dropped head), the visibility rule, the order and
padding of a row, and every helper the GPU parity tests and the smoke check
call: the max |score| that scales the tolerance rule (no absolute value, an
invisible key included, the wrong row's weights), the score of a given key
(a dropped batch offset, no visibility check) and the FP8 scales."""

import os
import subprocess

import pytest

import oracle
from tests import _pins

_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                    "oracle.c")

MUTATIONS = {
    # the score and the row
    "drop_relu": ("double r = dot > 0.0 ? dot : 0.0;", "double r = dot;"),
    "visibility_off_by_one": ("(v + 1) * m - 1 <= t", "(v + 1) * m - 1 < t"),
    "tie_rule_reversed": ("return (x->j < y->j) ? -1 : (x->j > y->j);\n}\n\nstatic int cmp_pairf",
                          "return (x->j > y->j) ? -1 : (x->j < y->j);\n}\n\nstatic int cmp_pairf"),
    "transposed_q": ("bf16_to_f64(qr[h * D + d]) * bf16_to_f64(kr[d])",
                     "bf16_to_f64(qr[d * H + h]) * bf16_to_f64(kr[d])"),
    "wrong_sign": ("        s += (double)wr[h] * r;", "        s -= (double)wr[h] * r;"),
    "dropped_head": ("    double s = 0.0;\n    for (int h = 0; h < H; h++) {\n        double dot = 0.0;\n"
                     "        for (int d = 0; d < D; d++) dot += bf16",
                     "    double s = 0.0;\n    for (int h = 1; h < H; h++) {\n        double dot = 0.0;\n"
                     "        for (int d = 0; d < D; d++) dot += bf16"),
    "pad_zero": ("out_score[r] = r < V ? p[r].s : -INFINITY;", "out_score[r] = r < V ? p[r].s : 0.0;"),
    "ascending": ("    if (x->s > y->s) return -1;\n    if (x->s < y->s) return 1;\n"
                  "    return (x->j < y->j) ? -1 : (x->j > y->j);\n}\n\nstatic int cmp_pairf",
                  "    if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;\n"
                  "    return (x->j < y->j) ? -1 : (x->j > y->j);\n}\n\nstatic int cmp_pairf"),
    # indexer_topk_rows_absmax: the rows and the tolerance scale
    "absmax_no_abs": ("            if (fabs(p[j].s) > mx) mx = fabs(p[j].s);",
                      "            if (p[j].s > mx) mx = p[j].s;"),
    "absmax_over_all_T": (
        "        for (int j = 0; j < V; j++)\n            if (fabs(p[j].s) > mx) mx = fabs(p[j].s);",
        "        for (int j = 0; j < T; j++)\n"
        "            if (fabs(oracle_score_row(qr, wr, kcb, H, D, j)) > mx)\n"
        "                mx = fabs(oracle_score_row(qr, wr, kcb, H, D, j));"),
    "absmax_row_weights_of_row_0": ("        const float* wr = w_rows + (int64_t)i * H;\n"
                                    "        const uint16_t* kcb = kc + b * T * (int64_t)D;",
                                    "        const float* wr = w_rows;\n"
                                    "        const uint16_t* kcb = kc + b * T * (int64_t)D;"),
    "absmax_rows_pad_zero": ("            out_score[(int64_t)i * k + r] = r < V ? p[r].s : -INFINITY;\n"
                             "        }\n        out_absmax[i] = mx;",
                             "            out_score[(int64_t)i * k + r] = r < V ? p[r].s : 0.0;\n"
                             "        }\n        out_absmax[i] = mx;"),
    "absmax_rows_no_batch_offset": ("        const uint16_t* kcb = kc + b * T * (int64_t)D;\n"
                                    "        pair_t* p",
                                    "        const uint16_t* kcb = kc;\n        pair_t* p"),
    # score_keys_rows: the score of a given key
    "score_keys_no_batch_offset": ("                                                        "
                                   "kc + b * T * (int64_t)D, H, D, j);",
                                   "                                                        "
                                   "kc, H, D, j);"),
    "score_keys_no_visibility": ("            if (j < 0 || j >= V) continue;\n"
                                 "            out[(int64_t)i * kk + r] = oracle_score_row(",
                                 "            if (j < 0) continue;\n"
                                 "            out[(int64_t)i * kk + r] = oracle_score_row("),
    "score_keys_weights_of_row_0": ("                                                        "
                                    "w_rows + (int64_t)i * H,\n",
                                    "                                                        "
                                    "w_rows,\n"),
    # row_absmax_rows
    "row_absmax_over_all_T": ("        for (int j = 0; j < V; j++) {\n            double s = fabs(",
                              "        for (int j = 0; j < T; j++) {\n            double s = fabs("),
    # FP8
    "fp8_key_scale_dropped": ("double skj = (double)skb[j];", "double skj = 1.0;"),
    "fp8_query_scale_dropped": ("double x = (double)sqr[h] * skj * dot;", "double x = skj * dot;"),
    "fp8_score_keys_no_batch_offset": ("                k8 + b * T * (int64_t)D, sk + b * T, H, D, j);",
                                       "                k8, sk, H, D, j);"),
    "fp8_score_keys_no_visibility": ("            if (j < 0 || j >= V) continue;\n"
                                     "            out[(int64_t)i * kk + r] = oracle_score_row_fp8(",
                                     "            if (j < 0) continue;\n"
                                     "            out[(int64_t)i * kk + r] = oracle_score_row_fp8("),
    # sparse attention over the listed entries
    "attn_scale_dropped": ("                l[r] = scale * s;", "                l[r] = s;"),
    "attn_query_of_head_0": ("            const uint16_t* qh = qa_rows + ((int64_t)i * H + h) * D;",
                             "            const uint16_t* qh = qa_rows + ((int64_t)i * H) * D;"),
    "attn_no_batch_offset": ("        const uint16_t* vb = va + batch[i] * (int64_t)T * D;",
                             "        const uint16_t* vb = va;"),
    "attn_value_of_first_entry": ("                    const double v = bf16_to_f64(vb[(int64_t)j * D + d]);",
                                  "                    const double v = bf16_to_f64(vb[(int64_t)ir[0] * D + d]);"),
    "attn_normaliser_skips_first": ("            double Z = 0.0;\n            for (int r = 0; r < k; r++) {",
                                    "            double Z = 0.0;\n            for (int r = 1; r < k; r++) {"),
    "attn_absw_without_abs": ("                    ah[d] += p * fabs(v);", "                    ah[d] += p * v;"),
    # MX block FP8: the scale rule, the quantiser and the score
    "mx_exponent_off_by_one": ("    int e = (E - 1) - 8;", "    int e = (E - 1) - 7;"),
    "mx_round_instead_of_floor": ("    int e = (E - 1) - 8;", "    int e = E - 8;"),
    "mx_no_low_clamp": ("    if (e < -127) e = -127;\n", ""),
    "mx_zero_block_scale_one": ("if (!(amax > 0.0)) return 0;", "if (!(amax > 0.0)) return 127;"),
    "mx_signed_block_max": ("double v = fabs(bf16_to_f64(xb[i]));", "double v = bf16_to_f64(xb[i]);"),
    "mx_key_scale_of_block_0": ("(int)ks[d / MX_BLOCK] - 127", "(int)ks[0] - 127"),
    "mx_query_scales_of_head_0": ("(int)qsr[h * nb + d / MX_BLOCK] - 127",
                                  "(int)qsr[d / MX_BLOCK] - 127"),
    "mx_no_relu": ("        s += (double)wr[h] * (dot > 0.0 ? dot : 0.0);",
                   "        s += (double)wr[h] * dot;"),
    "mx_no_batch_offset": ("k8 + b * T * (int64_t)D, ks + b * T * (int64_t)nb", "k8, ks"),
    # topk_scores: the selection on given fp32 values
    "topk_scores_tie_reversed": (
        "    const pairf_t* y = (const pairf_t*)b;\n    if (x->s > y->s) return -1;\n"
        "    if (x->s < y->s) return 1;\n    return (x->j < y->j) ? -1 : (x->j > y->j);",
        "    const pairf_t* y = (const pairf_t*)b;\n    if (x->s > y->s) return -1;\n"
        "    if (x->s < y->s) return 1;\n    return (x->j > y->j) ? -1 : (x->j < y->j);"),
    "topk_scores_pad_zero": ("                out_score[(int64_t)i * k + r] = -INFINITY;",
                             "                out_score[(int64_t)i * k + r] = 0.0f;"),
    "topk_scores_visibility_all_T": ("        const float* xr = X + row * (int64_t)T;\n"
                                     "        pairf_t* p = (pairf_t*)malloc(sizeof(pairf_t) * (size_t)(V > 0 ? V : 1));",
                                     "        const float* xr = X + row * (int64_t)T;\n        V = T;\n"
                                     "        pairf_t* p = (pairf_t*)malloc(sizeof(pairf_t) * (size_t)(V > 0 ? V : 1));"),
    # the per-row E4M3 quantiser
    "e4m3_ties_away": ("    return fmod(f, 2.0) == 0.0 ? f : f + 1.0;", "    return f + 1.0;"),
    "e4m3_saturate_to_nan": ("    if (a >= 448.0) return sign | 0x7E;", "    if (a >= 448.0) return sign | 0x7F;"),
    "e4m3_drop_sign": ("    uint8_t sign = signbit(y) ? 0x80 : 0x00;", "    uint8_t sign = 0x00;"),
    "e4m3_row_scale_240": ("        volatile float s = amax / 448.0f;", "        volatile float s = amax / 240.0f;"),
    "e4m3_row_amax_signed": ("            float v = fabsf((float)bf16_to_f64(xr[c]));",
                             "            float v = (float)bf16_to_f64(xr[c]);"),
}


def _build(tmp_path, name, src):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
                           "-o", str(so), str(c), "-lm"])
    return oracle.load_copy(str(so))


def _pins_pass(o) -> bool:
    try:
        _pins.run_all(o)
    except (AssertionError, ValueError):
        return False
    return True


def test_unmutated_copy_passes(tmp_path):
    assert _pins_pass(_build(tmp_path, "orig", open(_SRC).read()))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    src = open(_SRC).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} found {src.count(old)} times"
    o = _build(tmp_path, name, src.replace(old, new, 1))
    assert not _pins_pass(o), f"pins did not catch mutation {name}"

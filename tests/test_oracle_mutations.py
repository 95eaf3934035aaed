"""Plants plausible mistakes in a temporary copy of the oracle (on the CPU)
and checks that the pins catch each one: a dropped ReLU, an off-by-one
visibility rule, a reversed tie rule, a transposed operand, a wrong sign, a
dropped head, a wrong padding value and an ascending sort."""

import ctypes
import os
import subprocess

import numpy as np
import pytest

import synth
from oracle import brute
from tests import _golden

_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                    "oracle.c")

MUTATIONS = {
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
}


def _build(tmp_path, name, src):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
                           "-o", str(so), str(c), "-lm"])
    lib = ctypes.CDLL(str(so))
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.oracle_indexer_topk.argtypes = [P, P, P, I, I, I, I, I, I, P, I, P, P]
    lib.oracle_indexer_topk.restype = I
    return lib


def _run(lib, q, w, kc, m, k):
    q = np.ascontiguousarray(q, np.uint16)
    w = np.ascontiguousarray(w, np.float32)
    kc = np.ascontiguousarray(kc, np.uint16)
    B, S, H, D = q.shape
    rows = np.arange(B * S, dtype=np.int64)
    idx = np.empty((B * S, k), np.int32)
    sc = np.empty((B * S, k), np.float64)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    lib.oracle_indexer_topk(p(q), p(w), p(kc), B, S, H, D, m, k, p(rows), B * S, p(idx), p(sc))
    return idx, sc


def _pins_pass(lib) -> bool:
    """The hand-worked cases and an exact-rational brute-force comparison."""
    for c in _golden.cases():
        idx, sc = _run(lib, c["q"], c["w"], c["kc"], c["m"], c["k"])
        if not np.array_equal(idx, c["idx"]):
            return False
        same = (sc == c["score"]) | (np.isinf(sc) & np.isinf(c["score"]) & (sc == c["score"]))
        if not np.all(same):
            return False
    g = np.random.default_rng(11)
    B, S, m, H, D, k = 1, 12, 2, 3, 4, 4
    q = synth.f32_to_bf16_bits(g.integers(-8, 9, size=(B, S, H, D)).astype(np.float32) / 8)
    kc = synth.f32_to_bf16_bits(g.integers(-8, 9, size=(B, S // m, D)).astype(np.float32) / 8)
    w = (g.integers(-8, 9, size=(B, S, H)).astype(np.float32) / 8)
    bi, _ = brute.topk(q, w, kc, m, k)
    idx, _ = _run(lib, q, w, kc, m, k)
    return np.array_equal(idx, np.array(bi))


def test_unmutated_copy_passes(tmp_path):
    assert _pins_pass(_build(tmp_path, "orig", open(_SRC).read()))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    src = open(_SRC).read()
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    lib = _build(tmp_path, name, src.replace(old, new, 1))
    assert not _pins_pass(lib), f"pins did not catch mutation {name}"

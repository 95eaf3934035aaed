"""The FP8 accuracy rule of the GPU tests (tests/_fp8.py), checked on the CPU
with the oracle alone: the error bound E(j) covers the exact difference
between the FP8 and the bf16-input scores of every key, and needs both of
its terms; the FP8 oracle's own rows meet the rule; a row whose extra key
scores far below the bound is rejected."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from tests import _fp8


def _case():
    sh = synth.small(1, 256, 4, 8, 64, 16, seed=13, kc_kind="ar1")
    q, w, kc = synth.gen_q(sh, 13), synth.gen_w(sh, 13), synth.gen_kc(sh, 13)
    rows = np.arange(sh.S // 2, sh.S, 3)
    q8r, sqr, k8, sk = _fp8.oracle_quantized(sh, q, kc, rows)
    return sh, q, w, kc, rows, q8r, sqr, k8, sk


def _all_keys(sh, rows):
    V = np.minimum(sh.T, (rows % sh.S + 1) // sh.m)
    js = np.full((len(rows), sh.T), -1, dtype=np.int32)
    for i, v in enumerate(V):
        js[i, :v] = np.arange(v)
    return js


def _exact_rows(g, shape):
    """bf16 bit patterns of rows that per-row E4M3 holds exactly: E4M3 values
    times 2^-6 with each row's first element 448 * 2^-6, so the row scale is
    2^-6 and every element is a code times the scale."""
    tab = _fp8.e4m3_table()
    fin = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
    v = tab[g.choice(fin, size=shape)] * 2.0 ** -6
    v[..., 0] = 448 * 2.0 ** -6
    b = v.astype(np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0)
    return (b >> 16).astype(np.uint16)


@pytest.mark.parametrize("exact", [None, "q", "kc"])
def test_bound_covers_every_key(exact):
    """|s8 - s| <= E(j) for every visible key.  With exactly representable
    queries (dq = 0) or keys (dk = 0) the bound reduces to its other term,
    and the difference is still nonzero: a bound without that term fails."""
    sh, q, w, kc, rows, q8r, sqr, k8, sk = _case()
    g = np.random.default_rng(3)
    if exact == "q":
        q = _exact_rows(g, q.shape)
    elif exact == "kc":
        kc = _exact_rows(g, kc.shape)
    q8r, sqr, k8, sk = _fp8.oracle_quantized(sh, q, kc, rows)
    js = _all_keys(sh, rows)
    qr, wr = q.reshape(-1, sh.H, sh.D)[rows], w.reshape(-1, sh.H)[rows]
    s = oracle.score_keys_rows(qr, wr, kc, sh.S, sh.m, rows, js)
    s8 = oracle.score_keys_fp8_rows(q8r, sqr, wr, k8, sk, sh.S, sh.m, rows, js)
    E = _fp8.quant_error_bound(sh, q, w, kc, q8r, sqr, k8, sk, rows, js)
    ok = js >= 0
    diff = np.abs(s8 - s)[ok]
    assert np.all(diff <= E[ok] * (1 + 1e-12) + 1e-300)
    assert np.any(diff > 0)
    if exact is not None:
        # the side that is exact contributes nothing to the bound
        tab = _fp8.e4m3_table()
        side = (tab[q8r] * sqr.astype(np.float64)[..., None] if exact == "q"
                else tab[k8] * sk.astype(np.float64)[..., None])
        src = qr if exact == "q" else kc
        assert np.array_equal(side, synth.bf16_bits_to_f32(src).astype(np.float64))


def test_fp8_oracle_rows_meet_the_rule():
    sh, q, w, kc, rows, q8r, sqr, k8, sk = _case()
    qr, wr = q.reshape(-1, sh.H, sh.D)[rows], w.reshape(-1, sh.H)[rows]
    oi, os_, amax = oracle.indexer_topk_rows_absmax(qr, wr, kc, sh.S, sh.m, sh.topk, rows)
    ref = {"rows": rows, "k": sh.topk, "idx": oi, "score": os_, "absmax": amax}
    fi, _ = oracle.indexer_topk_fp8_rows(q8r, sqr, wr, k8, sk, sh.S, sh.m, sh.topk, rows)
    mean, mn = _fp8.accuracy_vs_bf16(sh, q, w, kc, q8r, sqr, k8, sk, rows, fi, ref)
    assert 0.8 < mn <= mean <= 1.0
    # a row whose FP8 selection swaps a kept key for the visible key that
    # sits furthest below the rule's floor (lowest s + E): rejected
    js = _all_keys(sh, rows)
    s = oracle.score_keys_rows(qr, wr, kc, sh.S, sh.m, rows, js)
    E = _fp8.quant_error_bound(sh, q, w, kc, q8r, sqr, k8, sk, rows, js)
    i = len(rows) - 1
    v = int((js[i] >= 0).sum())
    low = int(np.argmin(s[i, :v] + E[i, :v]))
    assert low not in fi[i]
    bad = fi.copy()
    bad[i, sh.topk - 1] = low
    with pytest.raises(AssertionError):
        _fp8.accuracy_vs_bf16(sh, q, w, kc, q8r, sqr, k8, sk, rows, bad, ref)

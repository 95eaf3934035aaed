"""Pins for the fp64 CPU oracle: each check ties it to something other than
itself (hand-worked values, exact rational arithmetic, a numpy special case,
library sorting, closed forms and invariants)."""

import numpy as np
import pytest

import oracle
import synth
from oracle import brute
from tests import _golden


def _close_scores(got, want):
    both_inf = np.isinf(got) & np.isinf(want)
    assert np.all(both_inf | (got == want)), (got, want)


@pytest.mark.parametrize("case", _golden.cases(), ids=lambda c: c["name"])
def test_hand_worked(case):
    idx, sc = oracle.indexer_topk(case["q"], case["w"], case["kc"], case["m"], case["k"])
    np.testing.assert_array_equal(idx, case["idx"])
    _close_scores(sc, case["score"])


@pytest.mark.parametrize("case", _golden.cases(), ids=lambda c: c["name"])
def test_hand_worked_rows_interface(case):
    q, w = case["q"], case["w"]
    B, S = q.shape[:2]
    rows = np.arange(B * S)
    idx, sc = oracle.indexer_topk_rows(q.reshape(B * S, *q.shape[2:]), w.reshape(B * S, -1),
                                       case["kc"], S, case["m"], case["k"], rows)
    np.testing.assert_array_equal(idx, case["idx"])
    _close_scores(sc, case["score"])


@pytest.mark.parametrize("case", _golden.cases(), ids=lambda c: c["name"])
def test_brute_force_agrees_with_hand_worked(case):
    idx, sc = brute.topk(case["q"], case["w"], case["kc"], case["m"], case["k"])
    np.testing.assert_array_equal(np.array(idx), case["idx"])
    got = np.array([[-np.inf if s is None else float(s) for s in r] for r in sc])
    _close_scores(got, case["score"])


def _dyadic_inputs(seed, B, S, m, H, D):
    """Values on the grid k/8, |k| <= 8: every product and sum is exact in
    fp64, and exact ties are frequent."""
    g = np.random.default_rng(seed)
    T = S // m
    q = g.integers(-8, 9, size=(B, S, H, D)).astype(np.float32) / 8
    kc = g.integers(-8, 9, size=(B, T, D)).astype(np.float32) / 8
    w = g.integers(-8, 9, size=(B, S, H)).astype(np.float32) / 8
    return synth.f32_to_bf16_bits(q), w, synth.f32_to_bf16_bits(kc)


@pytest.mark.parametrize("seed,B,S,m,H,D,k", [
    (0, 1, 12, 1, 1, 2, 3), (1, 2, 12, 2, 3, 4, 4), (2, 1, 16, 4, 2, 3, 2),
    (3, 1, 9, 3, 4, 8, 5), (4, 2, 8, 2, 2, 2, 8)])
def test_brute_force_exact_dyadic(seed, B, S, m, H, D, k):
    q, w, kc = _dyadic_inputs(seed, B, S, m, H, D)
    bi, bs = brute.topk(q, w, kc, m, k)
    oi, os_ = oracle.indexer_topk(q, w, kc, m, k)
    np.testing.assert_array_equal(oi, np.array(bi))
    ref = np.array([[-np.inf if s is None else float(s) for s in r] for r in bs])
    _close_scores(os_, ref)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_random_bf16(seed):
    sh = synth.small(1, 16, 2, 3, 8, 4, seed=seed)
    q, w, kc = synth.gen_q(sh, seed), synth.gen_w(sh, seed), synth.gen_kc(sh, seed)
    bi, bs = brute.topk(q, w, kc, sh.m, sh.topk)
    oi, os_ = oracle.indexer_topk(q, w, kc, sh.m, sh.topk)
    np.testing.assert_array_equal(oi, np.array(bi))
    for r in range(oi.shape[0]):
        for c in range(oi.shape[1]):
            if bs[r][c] is None:
                assert os_[r, c] == -np.inf
            else:
                assert abs(os_[r, c] - float(bs[r][c])) <= 1e-15 * max(1.0, abs(float(bs[r][c])))


def _numpy_scores(q, w, kc):
    """Independent fp64 computation of all scores with numpy matmul:
    [B,S,T] = sum_h w * relu(q @ kc^T)."""
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    kf = synth.bf16_bits_to_f32(kc).astype(np.float64)
    dots = np.einsum("bshd,btd->bsht", qf, kf)
    return np.einsum("bsh,bsht->bst", w.astype(np.float64), np.maximum(dots, 0.0))


def test_single_head_unit_weight_matches_numpy_lexsort():
    """H=1, w=1: the ranking is that of max(0, q.k), computed by numpy matmul
    and ordered by np.lexsort (score desc, index asc)."""
    sh = synth.small(1, 256, 4, 1, 32, 16, seed=5)
    q, kc = synth.gen_q(sh, 5), synth.gen_kc(sh, 5)
    w = np.ones((1, 256, 1), dtype=np.float32)
    oi, os_ = oracle.indexer_topk(q, w, kc, sh.m, sh.topk)
    s = _numpy_scores(q, w, kc)[0]
    for t in range(sh.S):
        V = min(sh.T, (t + 1) // sh.m)
        order = np.lexsort((np.arange(V), -s[t, :V]))[: sh.topk]
        n = order.size
        np.testing.assert_array_equal(oi[t, :n], order)
        np.testing.assert_allclose(os_[t, :n], s[t, order], rtol=1e-12, atol=1e-15)
        assert np.all(oi[t, n:] == -1)


def test_invariants_tiny_shape():
    sh = synth.shape("tiny")
    q, w, kc = synth.gen_q(sh), synth.gen_w(sh), synth.gen_kc(sh)
    oi, os_ = oracle.indexer_topk(q, w, kc, sh.m, sh.topk)
    s = _numpy_scores(q, w, kc)[0]
    total_visible = 0
    for t in range(sh.S):
        V = min(sh.T, (t + 1) // sh.m)
        assert V == oracle.visible(t, sh.T, sh.m)
        total_visible += V
        n = min(sh.topk, V)
        sel = oi[t, :n]
        # visibility, count and padding
        assert np.all((sel >= 0) & (sel < V))
        assert np.all(oi[t, n:] == -1) and np.all(np.isneginf(os_[t, n:]))
        assert np.unique(sel).size == n
        # sorted: scores non-increasing, equal scores in increasing index
        d = np.diff(os_[t, :n])
        assert np.all(d <= 0)
        eq = d == 0
        assert np.all(np.diff(sel)[eq] > 0)
        # scores agree with the independent numpy computation
        np.testing.assert_allclose(os_[t, :n], s[t, sel], rtol=1e-12, atol=1e-15)
        # every selected score >= every unselected visible score
        if n < V:
            rest = np.setdiff1d(np.arange(V), sel)
            assert os_[t, n - 1] >= s[t, rest].max() - 1e-12
        if t < sh.m - 1:
            assert np.all(oi[t] == -1)
    # closed form of the causal pair count when S = m*T
    T, m = sh.T, sh.m
    assert total_visible == m * T * (T - 1) // 2 + T


def test_topk_scores_matches_lexsort():
    """Selection on given fp32 values: np.lexsort on the values with -0
    folded into +0 (both compare equal), truncated to k, is the same order."""
    for kind in ["normal", "ties", "const", "inf"]:
        X = synth.gen_scores(2, 40, 13, seed=3, kind=kind)
        for m, k in [(3, 4), (1, 13), (2, 20)]:
            oi, os_ = oracle.topk_scores(X, m, k)
            for r in range(2 * 40):
                b, t = divmod(r, 40)
                V = min(13, (t + 1) // m)
                x = X[b, t, :V].copy()
                key = np.where(x == 0, np.float32(0), x)  # -0 -> +0
                order = np.lexsort((np.arange(V), -key.astype(np.float64)))[:k]
                n = order.size
                np.testing.assert_array_equal(oi[r, :n], order)
                # bit patterns of the input values
                np.testing.assert_array_equal(os_[r, :n].view(np.uint32),
                                              x[order].view(np.uint32))
                assert np.all(oi[r, n:] == -1) and np.all(np.isneginf(os_[r, n:]))


def test_rejects_bad_arguments():
    q = np.zeros((1, 6, 1, 1), np.uint16)
    with pytest.raises(ValueError):
        oracle.indexer_topk(q, np.zeros((1, 6, 1), np.float32), np.zeros((1, 1, 1), np.uint16), 4, 1)


# ---------------------------------------------------------------------------
# the helpers the GPU parity tests and the smoke check call, pinned one by one
# (tests/_pins.py; the mutation tests run the same checks on planted mistakes)

from tests import _pins  # noqa: E402


def test_pins_hand_cases_all_row_entries():
    _pins.check_hand_cases(oracle)


def test_pins_dyadic_brute_force_all_row_entries():
    _pins.check_dyadic_brute_force(oracle)


def test_pins_fp8_rows_and_key_scores_brute_force():
    _pins.check_fp8_brute_force(oracle)


def test_pins_decode_rows_brute_force():
    _pins.check_decode_brute_force(oracle)


def test_pins_sparse_attention_library_and_closed_forms():
    _pins.check_sparse_attention(oracle)


def test_pins_pivot_brute_force_and_special_cases():
    _pins.check_pivot(oracle)


def test_row_helpers_match_numpy_two_batches():
    """Random bf16 inputs, two batches, rows t < m - 1 included: the max
    |score| over visible keys and the scores of given keys (visible, -1 and
    beyond the visible range) against an independent numpy fp64 computation."""
    sh = synth.small(2, 256, 4, 8, 64, 16, seed=8, kc_kind="ar1")
    q, w, kc = synth.gen_q(sh, 8), synth.gen_w(sh, 8), synth.gen_kc(sh, 8)
    s = _numpy_scores(q, w, kc).reshape(2 * sh.S, sh.T)
    g = np.random.default_rng(0)
    rows = np.union1d(g.choice(2 * sh.S, 60, replace=False), [0, 1, 2, sh.S, sh.S + 2, 2 * sh.S - 1])
    t = rows % sh.S
    V = np.minimum(sh.T, (t + 1) // sh.m)
    qr, wr = q.reshape(-1, sh.H, sh.D)[rows], w.reshape(-1, sh.H)[rows]
    want_amax = np.array([np.abs(s[r, :v]).max() if v else 0.0 for r, v in zip(rows, V)])
    oi, os_, amax = oracle.indexer_topk_rows_absmax(qr, wr, kc, sh.S, sh.m, sh.topk, rows)
    np.testing.assert_allclose(amax, want_amax, rtol=1e-12, atol=0)
    np.testing.assert_allclose(oracle.row_absmax_rows(qr, wr, kc, sh.S, sh.m, rows), want_amax,
                               rtol=1e-12, atol=0)
    for i, (r, v) in enumerate(zip(rows, V)):
        n = min(sh.topk, v)
        np.testing.assert_allclose(os_[i, :n], np.sort(s[r, :v])[::-1][:n], rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(os_[i, :n], s[r, oi[i, :n]], rtol=1e-12, atol=1e-15)
    js = g.integers(-1, sh.T, size=(rows.size, 40)).astype(np.int32)
    got = oracle.score_keys_rows(qr, wr, kc, sh.S, sh.m, rows, js)
    vis = (js >= 0) & (js < V[:, None])
    assert np.all(np.isnan(got[~vis]))
    np.testing.assert_allclose(got[vis], s[np.repeat(rows, 40).reshape(-1, 40)[vis], js[vis]],
                               rtol=1e-12, atol=1e-15)


def test_pins_mxfp8():
    _pins.check_mxfp8(oracle)

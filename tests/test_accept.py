"""The acceptance rule every GPU parity test applies (oracle/accept.py),
checked on the CPU: the oracle's own rows pass, and each kind of wrong
result (a key below the tolerance, a duplicate, an invisible key, padding
out of place, a wrong count, a differing row that sees at most k keys, a
recall below the bar) is flagged."""

from __future__ import annotations

import numpy as np

import oracle
import synth
from oracle import accept


def _case(seed=7):
    sh = synth.small(1, 96, 4, 4, 32, 8, seed=seed, kc_kind="ar1")
    q, w, kc = synth.gen_q(sh, seed), synth.gen_w(sh, seed), synth.gen_kc(sh, seed)
    rows = np.arange(sh.S)
    qr, wr = q.reshape(-1, sh.H, sh.D), w.reshape(-1, sh.H)
    oi, os_, amax = oracle.indexer_topk_rows_absmax(qr, wr, kc, sh.S, sh.m, sh.topk, rows)
    V = np.array([oracle.visible(int(t), sh.T, sh.m) for t in rows])

    def score(cand):
        return oracle.score_keys_rows(qr, wr, kc, sh.S, sh.m, rows, cand)

    return sh, rows, V, oi, os_, amax, score


def _run(sh, rows, V, oi, os_, amax, score, cand, **kw):
    return accept.check(rows, V, sh.topk, oi, os_, cand, score(cand), amax, **kw)


def test_oracle_rows_pass():
    sh, rows, V, oi, os_, amax, score = _case()
    res = _run(sh, rows, V, oi, os_, amax, score, oi.copy())
    assert accept.passed(res) and res["mean_recall"] == 1.0 and res["min_recall"] == 1.0


def _full_row(V, k):
    return int(np.nonzero(V > k + 4)[0][-1])


def test_near_tie_swap_within_tolerance_passes_and_far_key_fails():
    sh, rows, V, oi, os_, amax, score = _case()
    r = _full_row(V, sh.topk)
    # the best unselected key, scored by the oracle: within 1e-3 of the k-th
    # score (ranked just below it), so swapping it in keeps the rule
    s_all = oracle.score_keys_rows(*_score_args(sh, r), rows[r:r + 1],
                                   np.arange(V[r], dtype=np.int32)[None, :])[0]
    order = np.lexsort((np.arange(V[r]), -s_all))
    nxt, worst = int(order[sh.topk]), int(order[-1])
    cand = oi.copy()
    cand[r, -1] = nxt
    gap = os_[r, sh.topk - 1] - s_all[nxt]
    res = _run(sh, rows, V, oi, os_, amax, score, cand, tol_rel=gap / amax[r] + 1e-9)
    assert not res["violations"] and res["min_recall"] < 1.0
    res = _run(sh, rows, V, oi, os_, amax, score, cand, tol_rel=0.5 * gap / amax[r])
    assert res["violations"] and res["violations"][0][:2] == (r, nxt)
    cand[r, -1] = worst
    res = _run(sh, rows, V, oi, os_, amax, score, cand, tol_rel=1e-9)
    assert res["violations"] and not accept.passed(res)


def _score_args(sh, r):
    seed = 7
    q, w, kc = synth.gen_q(sh, seed), synth.gen_w(sh, seed), synth.gen_kc(sh, seed)
    return (q.reshape(-1, sh.H, sh.D)[r:r + 1], w.reshape(-1, sh.H)[r:r + 1], kc, sh.S, sh.m)


def test_structural_errors_are_flagged():
    sh, rows, V, oi, os_, amax, score = _case()
    r = _full_row(V, sh.topk)
    for name, mutate in [
        ("duplicate", lambda c: c.__setitem__((r, 1), c[r, 0])),
        ("not visible", lambda c: c.__setitem__((r, 0), V[r])),
        ("count/padding", lambda c: c.__setitem__((r, sh.topk - 1), -1)),
    ]:
        cand = oi.copy()
        mutate(cand)
        res = _run(sh, rows, V, oi, os_, amax, score, cand)
        assert any(e[0] == r and e[1] == name for e in res["struct_errors"]), name
        assert not accept.passed(res), name
    # padding ahead of a real entry in a row that sees fewer than k keys
    rs = int(np.nonzero((V > 1) & (V < sh.topk))[0][0])
    cand = oi.copy()
    cand[rs, 0], cand[rs, V[rs]] = -1, oi[rs, 0]
    res = _run(sh, rows, V, oi, os_, amax, score, cand)
    assert any(e == (rs, "count/padding") for e in res["struct_errors"])


def test_rows_seeing_at_most_k_keys_must_match_exactly():
    sh, rows, V, oi, os_, amax, score = _case()
    rs = int(np.nonzero((V > 2) & (V <= sh.topk))[0][-1])
    cand = oi.copy()
    # every visible key is selected, so any change drops one: here the first
    # entry repeats the second
    cand[rs, 0] = cand[rs, 1]
    res = _run(sh, rows, V, oi, os_, amax, score, cand)
    assert rs in res["exact_errors"] and not accept.passed(res)


def test_recall_bar():
    sh, rows, V, oi, os_, amax, score = _case()
    full = np.nonzero(V > sh.topk + 4)[0]
    cand = oi.copy()
    # every full row loses its k-th key to the next-best one: recall (k-1)/k
    for r in full:
        s_all = oracle.score_keys_rows(*_score_args(sh, r), rows[r:r + 1],
                                       np.arange(V[r], dtype=np.int32)[None, :])[0]
        order = np.lexsort((np.arange(V[r]), -s_all))
        cand[r, -1] = int(order[sh.topk])
    res = _run(sh, rows, V, oi, os_, amax, score, cand, tol_rel=1.0)
    want = 1.0 - full.size / len(rows) / sh.topk
    assert abs(res["mean_recall"] - want) < 1e-12 and not res["violations"]
    assert res["mean_recall"] < 0.999 and not accept.passed(res)
    assert accept.passed(res, mean_recall_min=want - 1e-12)


def test_rows_that_see_no_key():
    sh, rows, V, oi, os_, amax, score = _case()
    r0 = np.nonzero(V == 0)[0]
    assert r0.size and np.all(oi[r0] == -1)
    res = _run(sh, rows, V, oi, os_, amax, score, oi.copy())
    assert res["min_recall"] == 1.0
    cand = oi.copy()
    cand[r0[0], 0] = 0  # a key where none is visible
    res = _run(sh, rows, V, oi, os_, amax, score, cand)
    assert not accept.passed(res)

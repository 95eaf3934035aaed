"""The query-group candidate scan on the GPU (si_indexer_pivot): its exact
special cases bit for bit against the exact step, the general case against
the oracle's reading of the scan, and its recall against the exact oracle
(what the approximation gives up)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import streaming_top_lightning_b200 as stl
from tests import _gpu

pytestmark = pytest.mark.gpu


def _recall(g, o):
    """|G & O| / |O| of two index rows (-1 padding), 1 when O is empty."""
    o = o[o >= 0]
    return 1.0 if o.size == 0 else np.intersect1d(g[g >= 0], o).size / o.size


def run_pivot(sh, q, w, kc, G, C):
    idx, sc = stl.indexer_pivot(_gpu.to_dev_bf16(q), torch.from_numpy(w).cuda(),
                                _gpu.to_dev_bf16(kc), sh.m, sh.topk, G, C)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    return idx, sc


@pytest.mark.parametrize("G,C,H", [(1, None, 64), (16, "T", 64), (8, "T", 16)])
def test_pivot_exact_special_cases(G, C, H):
    """Groups of one query (each query its own representative, C = k) and
    C >= T (every visible key is a candidate) reduce the scan to the exact
    step: every row keeps the exact step's keys.  The candidate pass may run
    on a narrower tile, whose epilogue sums the heads in another order, so
    scores agree to fp32 rounding (and keys a rounding apart may swap places)
    rather than bit for bit."""
    sh = synth.small(1, 4096, 4, H, 128, 256, seed=G + H, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=G + H)
    C = sh.topk if C is None else sh.T
    pi, ps = run_pivot(sh, q, w, kc, G, C)
    ei, es = _gpu.run_bf16(sh, q, w, kc)
    pi, ps = pi.reshape(-1, sh.topk).cpu().numpy(), ps.reshape(-1, sh.topk).cpu().numpy()
    ei, es = ei.reshape(-1, sh.topk).cpu().numpy(), es.reshape(-1, sh.topk).cpu().numpy()
    for r in range(pi.shape[0]):
        assert np.array_equal(np.sort(pi[r]), np.sort(ei[r])), r
    # the same key's score from both paths, and the same order up to rounding
    for r in range(0, pi.shape[0], 7):
        real = ei[r] >= 0
        if not real.any():
            continue
        pos = {int(j): n for n, j in enumerate(pi[r])}
        sp = np.array([ps[r, pos[int(j)]] for j in ei[r][real]])
        scale = np.abs(es[r][real]).max()
        assert np.abs(sp - es[r][real]).max() <= 1e-5 * scale, r
        assert np.all(np.diff(ps[r][pi[r] >= 0]) <= 0), r


@pytest.mark.parametrize("S,G,C,k", [(4096, 16, 512, 256), (8192, 64, 1024, 512),
                                     (4096, 32, 128, 128)])
def test_pivot_against_oracle(S, G, C, k):
    sh = synth.small(1, S, 4, 64, 128, k, seed=S + G, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=S + G)
    gi, gs = run_pivot(sh, q, w, kc, G, C)
    rows = np.union1d(np.arange(0, S, 53), np.arange(S - 2 * G, S))
    oi, os_, amax = oracle.pivot_rows(q, w, kc, sh.m, k, G, C, rows)
    gi_r = gi.reshape(-1, k)[rows].cpu().numpy()
    gs_r = gs.reshape(-1, k)[rows].cpu().numpy()
    # the oracle's scores of the keys the GPU kept (nan for keys a row cannot see)
    qr, wr = q.reshape(-1, sh.H, sh.D)[rows], w.reshape(-1, sh.H)[rows]
    extra = oracle.score_keys_rows(qr, wr, kc, sh.S, sh.m, rows, gi_r)
    # structure: distinct visible keys, padding after them, scores descending
    # (ties by index), and as many keys as the oracle's row (the candidates a
    # query sees, at most k)
    V = _gpu.visible(rows % S, sh.T, sh.m)
    for r in range(rows.size):
        g = gi_r[r][gi_r[r] >= 0]
        n = g.size
        assert np.all(gi_r[r][n:] == -1) and np.all(np.isneginf(gs_r[r][n:])), rows[r]
        assert np.unique(g).size == n and (n == 0 or g.max() < V[r]), rows[r]
        d = np.diff(gs_r[r][:n].astype(np.float64))
        assert np.all(d <= 0) and np.all(np.diff(g)[d == 0] > 0), rows[r]
    # a representative's near-tie can swap one candidate between the fp32 and
    # fp64 rankings, so rows are compared by recall, not exactly
    rec_scan = [_recall(g, o) for g, o in zip(gi_r, oi)]
    assert np.mean(rec_scan) >= 0.995, np.mean(rec_scan)
    real = gi_r >= 0
    err = np.abs(gs_r.astype(np.float64) - extra)[real]
    assert (err / np.maximum(np.repeat(amax[:, None], k, axis=1)[real], 1e-30)).max() <= 1e-3
    # what the scan gives up against the exact step
    ref = _gpu.oracle_ref(sh, q, w, kc, rows)
    rec = [_recall(g, o) for g, o in zip(gi_r, ref["idx"])]
    _gpu.record("pivot_recall", {"S": S, "G": G, "C": C, "k": k,
                                 "recall_vs_scan_oracle": float(np.mean(rec_scan)),
                                 "recall_vs_exact_mean": float(np.mean(rec)),
                                 "recall_vs_exact_min": float(np.min(rec))})


def test_pivot_rejects_bad_groups():
    sh = synth.small(1, 512, 4, 64, 128, 64, seed=1)
    q, w, kc = _gpu.inputs(sh, seed=1)
    for G, C in [(3, 128), (16, 32), (16, 4096)]:  # S % G, C < k, C > 2048
        with pytest.raises(stl.StreamIndexError) as e:
            run_pivot(sh, q, w, kc, G, C)
        assert e.value.status == -8, (G, C)

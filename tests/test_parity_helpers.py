"""The GPU parity tests' own checks (tests/_gpu.py) run on the CPU with the
oracle's rows standing in for the device's, as CPU tensors: the oracle's
rows pass check_rows and structural on a batch of two with ragged rows, and
rows from a wrong batch, a shifted row, unsorted or badly padded rows, or
scores off by more than the tolerance fail."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _gpu


def _case():
    sh = synth.small(2, 300, 3, 8, 64, 12, seed=17, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=17)
    rows = np.arange(sh.B * sh.S)
    qr, wr = q.reshape(-1, sh.H, sh.D), w.reshape(-1, sh.H)
    oi, os_ = oracle.indexer_topk_rows(qr, wr, kc, sh.S, sh.m, sh.topk, rows)
    idx = torch.from_numpy(oi.astype(np.int32))
    sc = torch.from_numpy(os_.astype(np.float32))
    return sh, q, w, kc, rows, idx, sc


def test_oracle_rows_pass_the_helpers():
    sh, q, w, kc, rows, idx, sc = _case()
    res = _gpu.check_rows(sh, q, w, kc, idx, sc, rows)
    assert res["mean_recall"] == 1.0 and res["max_score_err_rel"] < 1e-6
    _gpu.structural(sh, idx, sc, rows)


def test_wrong_rows_fail_check_rows():
    sh, q, w, kc, rows, idx, sc = _case()
    S, k = sh.S, sh.topk
    # batch 1's rows replaced by batch 0's: same positions, other keys
    bad = idx.clone()
    bad[S:] = idx[:S]
    bads = sc.clone()
    bads[S:] = sc[:S]
    with pytest.raises(AssertionError):
        _gpu.check_rows(sh, q, w, kc, bad, bads, rows)
    # every row shifted by one position
    bad = torch.roll(idx, 1, dims=0)
    with pytest.raises(AssertionError):
        _gpu.check_rows(sh, q, w, kc, bad, torch.roll(sc, 1, dims=0), rows)
    # scores off by 1 % of the row's scale on one row
    r = S + S - 1
    qr, wr = q.reshape(-1, sh.H, sh.D), w.reshape(-1, sh.H)
    amax = oracle.indexer_topk_rows_absmax(qr, wr, kc, S, sh.m, k, rows)[2][r]
    bads = sc.clone()
    bads[r, 0] += float(0.01 * amax)
    with pytest.raises(AssertionError):
        _gpu.check_rows(sh, q, w, kc, idx, bads, rows)
    # padding scored 0 instead of -inf on a row that sees fewer than k keys
    rs = int(np.nonzero(np.minimum(sh.T, (rows % S + 1) // sh.m) < k)[0][-1])
    bads = sc.clone()
    bads[rs, -1] = 0.0
    with pytest.raises(AssertionError):
        _gpu.check_rows(sh, q, w, kc, idx, bads, rows)


def test_structural_catches_order_and_padding():
    sh, q, w, kc, rows, idx, sc = _case()
    r = sh.B * sh.S - 1
    bad, bads = idx.clone(), sc.clone()
    bad[r, 0], bad[r, 1] = idx[r, 1], idx[r, 0]
    bads[r, 0], bads[r, 1] = sc[r, 1], sc[r, 0]
    with pytest.raises(AssertionError):
        _gpu.structural(sh, bad, bads, rows)
    rs = 2  # sees one key ((2 + 1) // 3): one real entry, then padding
    bad = idx.clone()
    bad[rs, 1] = 0
    with pytest.raises(AssertionError):
        _gpu.structural(sh, bad, sc, rows)


def test_decode_check_on_oracle_rows():
    """The decode tests' check (check_decode) with the decode oracle's rows as
    the device's: they pass; the rows of the sequences in the wrong order,
    or one query's row given to its neighbour, fail."""
    from tests.test_gpu_decode import _decode_shape, check_decode

    ds = _decode_shape(3, 4, 700, 300, 8, 64, 3, 16, seed=5)
    q, w, kc = synth.gen_decode(ds, seed=5)
    oi, os_, _ = oracle.indexer_decode(q, w, kc, ds.t0, ds.seq.m, ds.seq.topk)
    gi, gs = oi.astype(np.int32), os_.astype(np.float32)
    check_decode(ds, q, w, kc, gi, gs)
    check_decode(ds, q, w, kc, gi, gs, batches=[2, 0])
    S_q = ds.S_q
    swapped = np.concatenate([gi[S_q:2 * S_q], gi[:S_q], gi[2 * S_q:]])
    sws = np.concatenate([gs[S_q:2 * S_q], gs[:S_q], gs[2 * S_q:]])
    with pytest.raises(AssertionError):
        check_decode(ds, q, w, kc, swapped, sws)
    shifted, shs = gi.copy(), gs.copy()
    shifted[1], shs[1] = gi[0], gs[0]
    with pytest.raises(AssertionError):
        check_decode(ds, q, w, kc, shifted, shs)

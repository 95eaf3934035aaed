"""Sparse attention over the selected entries on the GPU (si_sparse_attention),
checked element by element against the fp64 attention oracle.

Tolerance, from the arithmetic: the logits are fp32 sums of exact bf16
products (relative error ~1e-6), the softmax is fp32, and the probabilities
are rounded to bf16 (relative error <= 2^-9) before they weight the value
rows, while the normaliser sums the unrounded ones (another <= 2^-9 of the
output).  So |o_gpu - o| <= 2^-8 * a + 2^-9 * |o| + fp32 terms, with
a = sum_j p_j |v_j| (the oracle's weighted magnitude, >= |o|); the test
allows 2^-7 * a + 1e-6."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import streaming_top_lightning_b200 as stl
from tests import _gpu

pytestmark = pytest.mark.gpu

TOL_REL = 2.0 ** -7


def _dev(bits):
    return _gpu.to_dev_bf16(bits)


def run(qa, ka, va, idx, scale=None):
    out = stl.sparse_attention(_dev(qa), _dev(ka), _dev(va), torch.from_numpy(idx).cuda(), scale)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    return out.cpu().numpy()


def check(qa, ka, va, idx, out, scale, rows=None):
    B, S, H, D = qa.shape
    rows = np.arange(B * S) if rows is None else np.asarray(rows)
    ref, absw = oracle.sparse_attention_rows(qa.reshape(B * S, H, D)[rows], ka, va,
                                             idx.reshape(B * S, -1)[rows], rows // S, scale)
    got = out.reshape(B * S, H, D)[rows].astype(np.float64)
    err = np.abs(got - ref)
    bad = err > TOL_REL * absw + 1e-6
    assert not bad.any(), (int(bad.sum()), float((err / (absw + 1e-30)).max()))
    return float((err / np.maximum(absw, 1e-30)).max())


def _idx_rows(g, B, S, T, k):
    """Index rows with the structures the kernel must handle: a full row,
    -1 padding from a random point on, an out-of-range entry, a row that
    lists nothing, a row with one entry, entries only in the last tile."""
    idx = np.stack([g.permutation(T)[:k] for _ in range(B * S)]).astype(np.int32)
    for r in range(B * S):
        kind = r % 6
        if kind == 1:
            idx[r, g.integers(1, k):] = -1
        elif kind == 2:
            idx[r, g.integers(0, k)] = T + 5
        elif kind == 3:
            idx[r] = -1
        elif kind == 4:
            idx[r, 1:] = -1
        elif kind == 5 and k > 128:
            idx[r, : (k - 1) // 128 * 128] = -1
    return idx.reshape(B, S, k)


@pytest.mark.parametrize("B,S,T,k", [(2, 13, 300, 200), (1, 12, 4096, 2048), (3, 7, 100, 64),
                                     (1, 6, 5000, 1000)])
def test_attention_against_oracle(B, S, T, k):
    g = np.random.default_rng(B * 1000 + k)
    qa, ka, va = synth.gen_attention(B, S, T, seed=k)
    idx = _idx_rows(g, B, S, T, k)
    scale = 1.0 / np.sqrt(128.0)
    out = run(qa, ka, va, idx, scale)
    rel = check(qa, ka, va, idx, out, scale)
    _gpu.record("attention_error", {"case": [B, S, T, k], "max_err_over_weighted_abs": rel})
    # a row that lists nothing is exactly zero
    empty = np.all(idx.reshape(B * S, k) < 0, axis=1) | np.all(idx.reshape(B * S, k) >= T, axis=1)
    assert np.all(out.reshape(B * S, -1)[empty] == 0)


def test_attention_peaked_softmax():
    """A scale of 1 makes the logits spread by ~11: the running maximum moves
    across tiles and the rescaling of the accumulated output is exercised."""
    g = np.random.default_rng(3)
    qa, ka, va = synth.gen_attention(1, 8, 2048, seed=3)
    idx = np.stack([g.permutation(2048) for _ in range(8)]).astype(np.int32)[None]
    out = run(qa, ka, va, idx, 1.0)
    check(qa, ka, va, idx, out, 1.0)


def test_attention_over_indexer_rows():
    """The composition: the indexer's top-k rows (with their -1 padding for
    early queries) select the entries the attention reads."""
    sh = synth.small(1, 2048, 4, 64, 128, 256, seed=8, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=8)
    gi, _ = _gpu.run_bf16(sh, q, w, kc)
    idx = gi.cpu().numpy()
    qa, ka, va = synth.gen_attention(1, sh.S, sh.T, seed=9)
    scale = 1.0 / np.sqrt(128.0)
    out = run(qa, ka, va, idx, scale)
    rows = np.union1d(np.arange(0, sh.S, 97), [0, 1, 2, 3, 4, sh.S - 1])
    check(qa, ka, va, idx, out, scale, rows)
    assert np.all(out[0, :3] == 0)  # queries 0..2 see no key: every entry is -1


def test_attention_rejects_bad_arguments():
    qa, ka, va = synth.gen_attention(1, 2, 16, seed=1)
    idx = torch.zeros((1, 2, 4), dtype=torch.int32, device="cuda")
    lib = stl._lib.load()
    out = torch.empty((1, 2, 128, 128), dtype=torch.float32, device="cuda")
    q, k, v = _dev(qa), _dev(ka), _dev(va)
    P = stl._ptr
    assert lib.si_sparse_attention(P(q), P(k), P(v), P(idx), 1, 2, 16, 64, 128, 4, 1.0, P(out),
                                   None, None) == -2
    assert lib.si_sparse_attention(P(q), P(k), P(v), P(idx), 1, 2, 16, 128, 128, 0, 1.0, P(out),
                                   None, None) == -3
    assert lib.si_sparse_attention(P(q), P(k), P(v), P(idx), 1, 2, 16, 128, 128, 4,
                                   float("inf"), P(out), None, None) == -8
    assert lib.si_sparse_attention(None, P(k), P(v), P(idx), 1, 2, 16, 128, 128, 4, 1.0, P(out),
                                   None, None) == -1

"""Decode steps on the GPU: the newest queries of each sequence against the
keys compressed so far (si_indexer_decode), checked against the decode
oracle, against rows of the prefill path on the same sequence, and across key
chunkings."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import streaming_top_lightning_b200 as stl
from oracle import accept
from tests import _gpu

pytestmark = pytest.mark.gpu


def _decode_shape(B, S_q, t0, T, H, D, m, k, seed):
    seq = synth.small(B, m * T, m, H, D, k, seed=seed, kc_kind="ar1")
    return synth.DecodeShape(f"decode_{B}x{S_q}_t{t0}_T{T}", seq, t0, S_q)


def _run(ds, q, w, kc, opts=None):
    idx, sc = stl.indexer_decode(_gpu.to_dev_bf16(q), torch.from_numpy(w).cuda(),
                                 _gpu.to_dev_bf16(kc), ds.t0, ds.seq.m, ds.seq.topk, opts=opts)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    return idx.cpu().numpy().reshape(-1, ds.seq.topk), sc.cpu().numpy().reshape(-1, ds.seq.topk)


def check_decode(ds, q, w, kc, gi, gs, batches=None):
    """The acceptance rule of the prefill tests, with each query's visible
    count from its own position t0 + i; ``batches`` limits the check to those
    sequences (all by default)."""
    sh, k = ds.seq, ds.seq.topk
    B, S_q = sh.B, ds.S_q
    bsel = np.arange(B) if batches is None else np.asarray(batches)
    qs, ws_, kcs = q[bsel], w[bsel], kc[bsel]
    oi, os_, amax = oracle.indexer_decode(qs, ws_, kcs, ds.t0, sh.m, k)
    flat = (bsel[:, None] * S_q + np.arange(S_q)[None, :]).reshape(-1)
    gi, gs = gi[flat], gs[flat]
    S_eq, rows = oracle.decode_rows(len(bsel), S_q, ds.t0, ds.T, sh.m)
    extra = oracle.score_keys_rows(qs.reshape(-1, sh.H, sh.D), ws_.reshape(-1, sh.H), kcs, S_eq,
                                   sh.m, rows, gi)
    V = np.tile(_gpu.visible(ds.t0 + np.arange(S_q), ds.T, sh.m), len(bsel))
    res = accept.check(flat, V, k, oi, os_, gi, extra, amax)
    assert accept.passed(res), {kk: (v[:5] if isinstance(v, list) else v) for kk, v in res.items()}
    real = gi >= 0
    assert np.all(np.isneginf(gs[~real]))
    err = np.abs(gs.astype(np.float64) - extra)[real]
    scale = np.repeat(amax[:, None], k, axis=1)[real]
    assert (err / np.maximum(scale, 1e-30)).max(initial=0.0) <= 1e-3
    return res


# (B, S_q, t0, T, H, D, m, k): one query that sees every key; keys in kc past
# the queries' reach; top-k above V (padding); positions 0.. that see no key;
# top-2048 with chunked keys; the decode workload's per-sequence size; eight
# heads (16 queries per half-width tile) with m = 3; a query tile wider than
# one tile
CASES = [
    (1, 1, 4095, 1024, 64, 128, 4, 512),
    (3, 5, 100, 64, 32, 64, 4, 16),
    (2, 3, 50, 40, 16, 128, 4, 2048),
    (1, 7, 0, 16, 64, 128, 4, 8),
    (4, 2, 2999, 800, 64, 128, 4, 2048),
    (2, 1, 65535, 16384, 64, 128, 4, 2048),
    (2, 9, 1234, 500, 8, 128, 3, 100),
    (1, 40, 5000, 2000, 64, 128, 4, 256),
]


@pytest.mark.parametrize("B,S_q,t0,T,H,D,m,k", CASES)
def test_decode_against_oracle(B, S_q, t0, T, H, D, m, k):
    ds = _decode_shape(B, S_q, t0, T, H, D, m, k, seed=t0 + T)
    q, w, kc = synth.gen_decode(ds, seed=t0 + T)
    gi, gs = _run(ds, q, w, kc)
    res = check_decode(ds, q, w, kc, gi, gs)
    _gpu.record("decode_recall", {"case": [B, S_q, t0, T, H, D, m, k],
                                  "mean_recall": res["mean_recall"],
                                  "min_recall": res["min_recall"]})


@pytest.mark.parametrize("t0,S_q", [(1000, 8), (4090, 6), (0, 3)])
def test_decode_equals_prefill_rows(t0, S_q):
    """A decode step over positions t0 .. t0+S_q-1 computes the same fp32
    scores and selects from the same keys as those rows of the prefill step on
    the whole sequence, so the two agree bit for bit."""
    seq = synth.small(1, 4096, 4, 64, 128, 512, seed=5, kc_kind="ar1")
    q, w, kc = _gpu.inputs(seq, seed=5)
    pi, ps = _gpu.run_bf16(seq, q, w, kc)
    ds = synth.DecodeShape("decode_eq", seq, t0, S_q)
    dq, dw, dkc = synth.gen_decode(ds, seed=5)
    assert np.array_equal(dq[0], q[0, t0:t0 + S_q]) and np.array_equal(dkc, kc)
    gi, gs = _run(ds, dq, dw, dkc)
    assert np.array_equal(gi, pi[0, t0:t0 + S_q].cpu().numpy())
    assert np.array_equal(gs.view(np.uint32), ps[0, t0:t0 + S_q].cpu().numpy().view(np.uint32))


@pytest.mark.parametrize("chunk", [128, 512, 4096])
def test_decode_chunkings_agree(chunk):
    """Key chunking changes where candidates are merged, not the scores: any
    chunk length gives the default plan's result bit for bit."""
    ds = _decode_shape(3, 2, 16383, 4096, 64, 128, 4, 1024, seed=9)
    q, w, kc = synth.gen_decode(ds, seed=9)
    gi, gs = _run(ds, q, w, kc)
    ci, cs = _run(ds, q, w, kc, opts=stl.options(key_chunk=chunk))
    assert np.array_equal(gi, ci) and np.array_equal(gs.view(np.uint32), cs.view(np.uint32))


def test_decode_workload_sampled_batches():
    """The decode workload (64 sequences of 16,384 keys, top-2048, the launch
    configuration the benchmark times) on the oracle for four sequences."""
    ds = synth.DECODE_SHAPES["decode_b64_t16k"]
    q, w, kc = synth.gen_decode(ds)
    plan = stl.decode_plan(ds.seq.B, ds.S_q, ds.t0, ds.T, ds.seq.H, ds.seq.D, ds.seq.m,
                           ds.seq.topk)
    assert plan["mma_n"] == 128 and plan["key_chunks"] > 1, plan
    gi, gs = _run(ds, q, w, kc)
    res = check_decode(ds, q, w, kc, gi, gs, batches=[0, 21, 42, 63])
    _gpu.record("decode_recall", {"case": "decode_b64_t16k", "mean_recall": res["mean_recall"],
                                  "min_recall": res["min_recall"]})


def test_decode_rejects_bad_sizes():
    ds = _decode_shape(1, 2, 10, 8, 64, 128, 4, 4, seed=1)
    q, w, kc = synth.gen_decode(ds, seed=1)
    qd, wd, kd = _gpu.to_dev_bf16(q), torch.from_numpy(w).cuda(), _gpu.to_dev_bf16(kc)
    for t0, m, k, status in [(-1, 4, 4, -2), (10, 0, 4, -2), (10, 4, 0, -3), (10, 4, 2049, -3)]:
        with pytest.raises(stl.StreamIndexError) as e:
            stl.indexer_decode(qd, wd, kd, t0, m, k)
        assert e.value.status == status, (t0, m, k)

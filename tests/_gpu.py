"""Helpers for the GPU parity tests: inputs to the device, the library call,
and the oracle's acceptance rule on the same seeded inputs."""

from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
import synth
import streaming_top_lightning_b200 as stl
from oracle import accept


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def inputs(sh: synth.Shape, seed: int = 0):
    q = synth.gen_q(sh, seed)
    w = synth.gen_w(sh, seed)
    kc = synth.gen_kc(sh, seed)
    return q, w, kc


def visible(t, T, m):
    return np.minimum(T, (np.asarray(t) + 1) // m)


def run_bf16(sh, q, w, kc, opts=None):
    idx, sc = stl.indexer_topk(to_dev_bf16(q), torch.from_numpy(w).cuda(), to_dev_bf16(kc), sh.m,
                               sh.topk, opts=opts)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    return idx, sc


def oracle_ref(sh, q, w, kc, rows, k=None):
    """The oracle's rows (top-k with k >= the topk to check; a shorter top-k is
    its prefix, since rows are sorted), scores and max |score| on the listed
    flat rows, for reuse across runs of the same inputs."""
    k = k or sh.topk
    qr = q.reshape(-1, sh.H, sh.D)[rows]
    wr = w.reshape(-1, sh.H)[rows]
    oi, os_, amax = oracle.indexer_topk_rows_absmax(qr, wr, kc, sh.S, sh.m, k, rows)
    return {"rows": np.asarray(rows), "k": k, "idx": oi, "score": os_, "absmax": amax}


def check_rows(sh, q, w, kc, gpu_idx, gpu_score, rows, mean_recall_min=0.999, ref=None):
    """Acceptance rule on the listed flat rows; returns the result dict.  ``ref``
    is an ``oracle_ref`` of the same inputs and rows (computed here if None)."""
    k = sh.topk
    gi = gpu_idx.reshape(-1, k)[rows].cpu().numpy()
    gs = gpu_score.reshape(-1, k)[rows].cpu().numpy()
    qr = q.reshape(-1, sh.H, sh.D)[rows]
    wr = w.reshape(-1, sh.H)[rows]
    if ref is None:
        ref = oracle_ref(sh, q, w, kc, rows)
    assert np.array_equal(ref["rows"], rows) and ref["k"] >= k
    oi, os_, amax = ref["idx"][:, :k], ref["score"][:, :k], ref["absmax"]
    extra = oracle.score_keys_rows(qr, wr, kc, sh.S, sh.m, rows, gi)
    V = visible(np.asarray(rows) % sh.S, sh.T, sh.m)
    res = accept.check(rows, V, k, oi, os_, gi, extra, amax)
    # score values: fp32 accumulation against the fp64 oracle at the same keys
    real = gi >= 0
    err = np.abs(gs.astype(np.float64) - extra)[real]
    scale = np.repeat(amax[:, None], k, axis=1)[real]
    res["max_score_err_rel"] = float((err / np.maximum(scale, 1e-30)).max()) if err.size else 0.0
    res["pad_ok"] = bool(np.all(np.isneginf(gs[~real])))
    assert accept.passed(res, mean_recall_min), {kk: (v[:5] if isinstance(v, list) else v)
                                                 for kk, v in res.items()}
    assert res["pad_ok"]
    assert res["max_score_err_rel"] <= 1e-3, res["max_score_err_rel"]
    return res


def structural(sh, gpu_idx, gpu_score, rows):
    """Sortedness, visibility, count and padding on the listed rows (no oracle)."""
    k = sh.topk
    gi = gpu_idx.reshape(-1, k)[rows].cpu().numpy()
    gs = gpu_score.reshape(-1, k)[rows].cpu().numpy()
    for r, row in enumerate(rows):
        V = int(visible(row % sh.S, sh.T, sh.m))
        n = min(k, V)
        sel = gi[r, :n]
        assert np.all((sel >= 0) & (sel < V)), row
        assert np.all(gi[r, n:] == -1) and np.all(np.isneginf(gs[r, n:])), row
        assert np.unique(sel).size == n, row
        d = np.diff(gs[r, :n].astype(np.float64))
        assert np.all(d <= 0), row
        assert np.all(np.diff(sel)[d == 0] > 0), row


def record(name: str, entry: dict) -> None:
    """Append one JSON line to $SI_RECORD_DIR/<name>.jsonl when that variable
    is set (measured recall and peak memory for the committed summaries)."""
    d = os.environ.get("SI_RECORD_DIR")
    if not d:
        return
    os.makedirs(d, exist_ok=True)
    with open(os.path.join(d, f"{name}.jsonl"), "a") as f:
        f.write(json.dumps(entry) + "\n")


def run_bf16_counted(sh, q, w, kc, opts=None):
    """The indexer step with its workspace allocated by torch, so the torch
    allocator's peak after a reset covers inputs, outputs and scratch (the
    inclusive peak of the 20 GB cap).  Returns (idx, score, peak bytes)."""
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats()
    qd, wd, kd = to_dev_bf16(q), torch.from_numpy(w).cuda(), to_dev_bf16(kc)
    idx, sc = stl.indexer_topk(qd, wd, kd, sh.m, sh.topk, opts=opts or stl.options())
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    peak = torch.cuda.max_memory_allocated()
    del qd, wd, kd
    return idx, sc, peak

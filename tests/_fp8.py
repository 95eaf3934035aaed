"""FP8 helpers for the GPU tests: the oracle's side of an FP8 run (codes,
scales, the FP8 oracle's rows) and the accuracy rule of the FP8 path against
the bf16-input oracle.

Accuracy rule.  Write q^ = s_q * e4m3(q8) and k^ = s_k * e4m3(k8) for the
dequantised rows, dq = q^ - q, dk = k^ - k.  Per head the FP8 dot product is
sum_d q^ k^ = sum_d q k + sum_d (dq k^ + q dk), and ReLU is 1-Lipschitz, so
for every key j of a query

    |s8(j) - s(j)| <= E(j) = sum_h |w_h| sum_d (|dq_hd| |k^_jd| + |q_hd| |dk_jd|),

s the bf16-input score and s8 the FP8 one (both exact).  The FP8 path keeps
the K best keys by s8 (up to its fp32 accumulation, bounded by eps =
1e-3 * max|row score| as in the bf16 rule), so every key j it selects that the
bf16 oracle does not beats every key o the oracle selects that it does not:
s8(j) >= s8(o) - 2 eps.  Hence

    s(j) >= max over such o of (s(o) - E(o)) - E(j) - 2 eps,

a property of the exact scores that holds at any size.  The test checks it for
every such j, and reports the set recall against the bf16 oracle.
"""

from __future__ import annotations

import numpy as np

import oracle
import synth
from oracle import accept

_E4M3 = None


def e4m3_table() -> np.ndarray:
    """Exact values of the 256 E4M3 codes, from the oracle's decoder."""
    global _E4M3
    if _E4M3 is None:
        _E4M3 = np.array([oracle.e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return _E4M3


def oracle_quantized(sh, q, kc, rows):
    """The oracle's own quantisation of the listed query rows and of every
    key (per-row scaling: a row's codes depend on that row only)."""
    qr = q.reshape(-1, sh.H, sh.D)[rows]
    q8r, sqr = oracle.quantize_e4m3_rows(qr)
    k8, sk = oracle.quantize_e4m3_rows(kc)
    return q8r, sqr, k8, sk


def fp8_oracle_ref(sh, w, q8r, sqr, k8, sk, rows, k):
    """The FP8 oracle's rows on the listed rows, and each row's max |FP8
    score| over its visible keys (the scale of the tolerance rule)."""
    wr = w.reshape(-1, sh.H)[rows]
    oi, os_ = oracle.indexer_topk_fp8_rows(q8r, sqr, wr, k8, sk, sh.S, sh.m, k, rows)
    V = np.minimum(sh.T, (np.asarray(rows) % sh.S + 1) // sh.m)
    allj = np.full((len(rows), sh.T), -1, dtype=np.int32)
    for i, v in enumerate(V):
        allj[i, :v] = np.arange(v)
    sc = oracle.score_keys_fp8_rows(q8r, sqr, wr, k8, sk, sh.S, sh.m, rows, allj)
    amax = np.nanmax(np.abs(np.where(allj >= 0, sc, 0.0)), axis=1, initial=0.0)
    return {"rows": np.asarray(rows), "k": k, "idx": oi, "score": os_, "absmax": amax}


def quant_error_bound(sh, q, w, kc, q8r, sqr, k8, sk, rows, js):
    """E(j) of the module docstring for keys js[i, :] of the listed rows
    (nan where js < 0); q8r and sqr hold the codes and scales of exactly
    those rows, in the same order."""
    assert len(q8r) == len(rows) == len(sqr) == len(js)
    tab = e4m3_table()
    qf = synth.bf16_bits_to_f32(q.reshape(-1, sh.H, sh.D)[rows]).astype(np.float64)
    qh = tab[q8r] * sqr.astype(np.float64)[..., None]
    wa = np.abs(w.reshape(-1, sh.H)[rows].astype(np.float64))
    kf = synth.bf16_bits_to_f32(kc).astype(np.float64)            # [B,T,D]
    kh = tab[k8] * sk.astype(np.float64)[..., None]
    dq, dk = np.abs(qh - qf), np.abs(kh - kf)
    out = np.full(js.shape, np.nan)
    for i, r in enumerate(rows):
        b = int(r) // sh.S
        j = js[i]
        ok = j >= 0
        if not ok.any():
            continue
        jj = j[ok]
        # sum_h |w_h| (|dq_h| . |k^_j| + |q_h| . |dk_j|)
        t1 = dq[i] @ np.abs(kh[b, jj]).T            # [H, n]
        t2 = np.abs(qf[i]) @ dk[b, jj].T            # [H, n]
        out[i, ok] = wa[i] @ (t1 + t2)
    return out


def accuracy_vs_bf16(sh, q, w, kc, q8r, sqr, k8, sk, rows, gi_rows, bf16_ref, tol_rel=1e-3):
    """Check the accuracy rule of the module docstring on the listed rows and
    return (mean recall, min recall) of the FP8 rows against the bf16 oracle.

    gi_rows [n, k]: the FP8 path's indices on those rows; bf16_ref: an
    oracle_ref of the bf16 inputs on the same rows."""
    k = gi_rows.shape[1]
    oi = bf16_ref["idx"][:, :k]
    os_ = bf16_ref["score"][:, :k]
    amax = bf16_ref["absmax"]
    qr, wr = q.reshape(-1, sh.H, sh.D)[rows], w.reshape(-1, sh.H)[rows]
    recalls = []
    bad = []
    for i in range(len(rows)):
        o = oi[i][oi[i] >= 0]
        g = gi_rows[i][gi_rows[i] >= 0]
        recalls.append(np.intersect1d(g, o).size / o.size if o.size else 1.0)
        extra = np.setdiff1d(g, o)
        if extra.size == 0:
            continue
        missed = np.setdiff1d(o, g)
        assert missed.size >= 1, rows[i]
        js = np.concatenate([extra, missed]).astype(np.int32)[None, :]
        E = quant_error_bound(sh, q, w, kc, q8r[i:i + 1], sqr[i:i + 1], k8, sk, rows[i:i + 1],
                              js)[0]
        s = oracle.score_keys_rows(qr[i:i + 1], wr[i:i + 1], kc, sh.S, sh.m, rows[i:i + 1], js)[0]
        ne = extra.size
        floor = np.max(s[ne:] - E[ne:]) - 2 * tol_rel * amax[i]
        for x in range(ne):
            if not s[x] >= floor - E[x]:
                bad.append((int(rows[i]), int(extra[x]), float(s[x]), float(floor - E[x])))
    assert not bad, bad[:5]
    return float(np.mean(recalls)), float(np.min(recalls))


# --------------------------------------------------------------------------- GPU side


def fp8_run(sh, q, w, kc, opts=None):
    """The FP8 step on the GPU from the bf16 inputs: the library's quantiser,
    then the FP8 indexer.  Returns (idx, score, q8, s_q, k8, s_k) on the device."""
    import torch

    import streaming_top_lightning_b200 as stl
    from tests import _gpu

    q8, sq = stl.quantize_fp8_rows(_gpu.to_dev_bf16(q))
    k8, sk = stl.quantize_fp8_rows(_gpu.to_dev_bf16(kc))
    gi, gs = stl.indexer_topk_fp8(q8, sq, torch.from_numpy(w).cuda(), k8, sk, sh.m, sh.topk,
                                  opts=opts)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    return gi, gs, q8, sq, k8, sk


def check_fp8_rows(sh, q, w, kc, rows, gpu, oq=None, fp8_ref=None, bf16_ref=None,
                   check_codes=True):
    """Kernel parity against the FP8 oracle run on the oracle's own codes
    (which must equal the library's bit for bit), then accuracy against the
    bf16-input oracle.  Returns the recalls: against the FP8 oracle (kernel
    parity) and against the bf16 oracle (accuracy), mean and min."""
    from tests import _gpu

    gi, gs, q8, sq, k8, sk = gpu
    k = sh.topk
    q8r, sqr, k8o, sko = oq if oq is not None else oracle_quantized(sh, q, kc, rows)
    if check_codes:  # the library's codes and scales are the oracle's
        assert np.array_equal(q8.cpu().numpy().reshape(-1, sh.H, sh.D)[rows], q8r)
        assert np.array_equal(sq.cpu().numpy().reshape(-1, sh.H)[rows].view(np.uint32),
                              sqr.view(np.uint32))
        assert np.array_equal(k8.cpu().numpy(), k8o)
        assert np.array_equal(sk.cpu().numpy().view(np.uint32), sko.view(np.uint32))
    ref = fp8_ref if fp8_ref is not None else fp8_oracle_ref(sh, w, q8r, sqr, k8o, sko,
                                                                  rows, k)
    wr = w.reshape(-1, sh.H)[rows]
    gi_r = gi.reshape(-1, k)[rows].cpu().numpy()
    gs_r = gs.reshape(-1, k)[rows].cpu().numpy()
    extra = oracle.score_keys_fp8_rows(q8r, sqr, wr, k8o, sko, sh.S, sh.m, rows, gi_r)
    V = _gpu.visible(np.asarray(rows) % sh.S, sh.T, sh.m)
    res = accept.check(rows, V, k, ref["idx"][:, :k], ref["score"][:, :k], gi_r, extra,
                       ref["absmax"])
    assert accept.passed(res), {kk: (v[:5] if isinstance(v, list) else v) for kk, v in res.items()}
    real = gi_r >= 0
    err = np.abs(gs_r.astype(np.float64) - extra)[real]
    scale = np.repeat(ref["absmax"][:, None], k, axis=1)[real]
    assert (err / np.maximum(scale, 1e-30)).max(initial=0.0) <= 1e-3
    if bf16_ref is None:
        bf16_ref = _gpu.oracle_ref(sh, q, w, kc, rows)
    mean, mn = accuracy_vs_bf16(sh, q, w, kc, q8r, sqr, k8o, sko, rows, gi_r, bf16_ref)
    return {"mean_recall_fp8_oracle": res["mean_recall"], "min_recall_fp8_oracle": res["min_recall"],
            "mean_recall_bf16_oracle": mean, "min_recall_bf16_oracle": mn}

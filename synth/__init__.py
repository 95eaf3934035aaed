"""Seeded synthetic inputs for the CSA lightning-indexer step.

This module only draws random numbers and stores them in the input dtypes
(bf16 as raw uint16 bit patterns, fp32).  It contains none of the indexer's
arithmetic: no scores, no masking, no selection, no FP8 quantisation.  Both the
CPU oracle and the CUDA path take their inputs from here.

The StreamIndex abstract ("StreamIndex: Memory-Bounded Compressed Sparse
Attention via Streaming Top-k", Abstract) measures on "synthetic-but-realistic
V4-shaped inputs" that are not published.  The recipe below stands in for them:

* q  [B,S,H_I,d_I]  iid N(0,1)/sqrt(d_I), rounded to bf16 (round to nearest even)
* w  [B,S,H_I]      iid fp32 N(0,1)*w_scale (1/sqrt(8) for the tiny shape, 1/8 else)
* kc [B,T,d_I]      "iid":   N(0,1)/sqrt(d_I)
                    "ar1":   AR(1) along j with rho=0.9 and N(0,1/d_I) marginals,
                             then round(0.02*T) heavy rows scaled by 4
                    then rounded to bf16 via fp32 (both steps round to nearest even)

Every tensor is drawn in blocks of ``BLOCK`` rows along its sequence axis, each
block from its own PCG64 stream keyed by (seed, tensor id, batch, block).  So
any subset of query rows can be regenerated without drawing the whole tensor.
"""

from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

BLOCK = 1024

# tensor ids used in the SeedSequence spawn keys
_TID_Q, _TID_W, _TID_KC, _TID_HEAVY, _TID_ROWS = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Shape:
    """One indexer-step workload: dimensions plus the input distribution."""

    name: str
    B: int
    S: int
    m: int
    H: int          # H_I, indexer heads
    D: int          # d_I, indexer head dim
    topk: int
    kc_kind: str    # "iid" or "ar1"
    w_scale: float
    sample_rows: int  # 0 = every row is checked against the oracle

    @property
    def T(self) -> int:
        return self.S // self.m


# The five workloads of the indexer step.  Names say what they are.
SHAPES = {
    "tiny": Shape("tiny", 1, 2048, 4, 8, 64, 64, "iid", 1.0 / math.sqrt(8.0), 0),
    "v4flash_s16k": Shape("v4flash_s16k", 1, 16384, 4, 64, 128, 512, "ar1", 1.0 / 8.0, 0),
    "large_s64k": Shape("large_s64k", 1, 65536, 4, 64, 128, 2048, "ar1", 1.0 / 8.0, 256),
    "sweep_s32k": Shape("sweep_s32k", 1, 32768, 4, 64, 128, 512, "ar1", 1.0 / 8.0, 256),
    "long_s256k": Shape("long_s256k", 1, 262144, 4, 64, 128, 2048, "ar1", 1.0 / 8.0, 64),
}


def shape(name: str, **overrides) -> Shape:
    return dataclasses.replace(SHAPES[name], **overrides)


def _rng(seed: int, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=seed, spawn_key=tuple(int(k) for k in key))
    return np.random.Generator(np.random.PCG64(ss))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), round to nearest, ties to even.

    Inputs are finite by construction; no NaN handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------- q, w


def _q_block(sh: Shape, seed: int, b: int, blk: int) -> np.ndarray:
    r0 = blk * BLOCK
    n = min(BLOCK, sh.S - r0)
    z = _rng(seed, _TID_Q, b, blk).standard_normal((n, sh.H, sh.D), dtype=np.float32)
    z *= np.float32(1.0 / math.sqrt(sh.D))
    return f32_to_bf16_bits(z)


def _w_block(sh: Shape, seed: int, b: int, blk: int) -> np.ndarray:
    r0 = blk * BLOCK
    n = min(BLOCK, sh.S - r0)
    z = _rng(seed, _TID_W, b, blk).standard_normal((n, sh.H), dtype=np.float32)
    z *= np.float32(sh.w_scale)
    return z


def _fill_blocks(out: np.ndarray, sh: Shape, seed: int, fn, threads: int) -> None:
    nblk = (sh.S + BLOCK - 1) // BLOCK
    jobs = [(b, k) for b in range(sh.B) for k in range(nblk)]

    def run(job):
        b, k = job
        blk = fn(sh, seed, b, k)
        out[b, k * BLOCK : k * BLOCK + blk.shape[0]] = blk

    if threads <= 1:
        for j in jobs:
            run(j)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, jobs))


def gen_q(sh: Shape, seed: int = 0, out: np.ndarray | None = None, threads: int = 8) -> np.ndarray:
    """q as bf16 bits, shape [B,S,H,D] uint16.  ``out`` may be a preallocated
    (e.g. pinned-memory backed) uint16 array of that shape."""
    if out is None:
        out = np.empty((sh.B, sh.S, sh.H, sh.D), dtype=np.uint16)
    _fill_blocks(out, sh, seed, _q_block, threads)
    return out


def gen_w(sh: Shape, seed: int = 0, out: np.ndarray | None = None, threads: int = 8) -> np.ndarray:
    if out is None:
        out = np.empty((sh.B, sh.S, sh.H), dtype=np.float32)
    _fill_blocks(out, sh, seed, _w_block, threads)
    return out


def gen_rows(sh: Shape, rows: np.ndarray, seed: int = 0):
    """Regenerate only the given flat rows (b*S + t) of q and w.

    Returns (q_rows [n,H,D] uint16, w_rows [n,H] float32), identical to the
    corresponding rows of gen_q / gen_w.
    """
    rows = np.asarray(rows, dtype=np.int64)
    qo = np.empty((rows.size, sh.H, sh.D), dtype=np.uint16)
    wo = np.empty((rows.size, sh.H), dtype=np.float32)
    cache = {}
    for i, r in enumerate(rows):
        b, t = divmod(int(r), sh.S)
        blk = t // BLOCK
        if (b, blk) not in cache:
            cache[(b, blk)] = (_q_block(sh, seed, b, blk), _w_block(sh, seed, b, blk))
        qb, wb = cache[(b, blk)]
        qo[i] = qb[t - blk * BLOCK]
        wo[i] = wb[t - blk * BLOCK]
    return qo, wo


# --------------------------------------------------------------------------- kc


def gen_kc(sh: Shape, seed: int = 0) -> np.ndarray:
    """Compressed keys as bf16 bits, shape [B,T,D] uint16."""
    T, D = sh.T, sh.D
    out = np.empty((sh.B, T, D), dtype=np.uint16)
    nblk = (T + BLOCK - 1) // BLOCK
    for b in range(sh.B):
        z = np.empty((T, D), dtype=np.float64)
        for k in range(nblk):
            n = min(BLOCK, T - k * BLOCK)
            z[k * BLOCK : k * BLOCK + n] = _rng(seed, _TID_KC, b, k).standard_normal((n, D))
        z *= 1.0 / math.sqrt(D)
        if sh.kc_kind == "iid":
            x = z
        elif sh.kc_kind == "ar1":
            rho = 0.9
            c = math.sqrt(1.0 - rho * rho)
            x = np.empty_like(z)
            x[0] = z[0]
            for j in range(1, T):
                x[j] = rho * x[j - 1] + c * z[j]
            nh = int(round(0.02 * T))
            if nh > 0:
                heavy = _rng(seed, _TID_HEAVY, b).choice(T, size=nh, replace=False)
                x[heavy] *= 4.0
        else:
            raise ValueError(sh.kc_kind)
        out[b] = f32_to_bf16_bits(x.astype(np.float32))
    return out


def sample_rows(sh: Shape, seed: int = 0) -> np.ndarray:
    """Flat rows (b*S + t) checked against the oracle: every row when
    ``sample_rows`` is 0, else that many rows per batch drawn uniformly without
    replacement, plus the last row of each batch, sorted."""
    if sh.sample_rows == 0:
        return np.arange(sh.B * sh.S, dtype=np.int64)
    rows = []
    for b in range(sh.B):
        r = _rng(seed, _TID_ROWS, b).choice(sh.S, size=sh.sample_rows, replace=False)
        r = np.union1d(r, [sh.S - 1])
        rows.append(r.astype(np.int64) + b * sh.S)
    return np.concatenate(rows)


def gen_scores(B: int, S: int, T: int, seed: int = 0, kind: str = "normal") -> np.ndarray:
    """A given fp32 score tensor [B,S,T] for the selection-only entry point.

    kinds: "normal" (iid N(0,1)); "ties" (values drawn from a 16-value set that
    includes +0 and -0, so equal scores are frequent); "const" (every score
    equal); "inf" (normal with ~5% +-inf mixed in).
    """
    g = _rng(seed, 7, B, S, T)
    if kind == "normal":
        return g.standard_normal((B, S, T), dtype=np.float32)
    if kind == "ties":
        vals = np.array([-2, -1, -0.5, -0.0, 0.0, 0.25, 0.5, 1, 1.5, 2, 3, 4, -3, 7, 0.0, -0.0],
                        dtype=np.float32)
        return vals[g.integers(0, vals.size, size=(B, S, T))]
    if kind == "const":
        return np.full((B, S, T), 0.5, dtype=np.float32)
    if kind == "inf":
        x = g.standard_normal((B, S, T), dtype=np.float32)
        u = g.random((B, S, T))
        x[u < 0.025] = np.inf
        x[(u >= 0.025) & (u < 0.05)] = -np.inf
        return x
    raise ValueError(kind)


# --------------------------------------------------------------------------- decode


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    """A decode step: the S_q newest queries (positions t0 .. t0+S_q-1) of
    each of the B sequences described by ``seq``, against the seq.T keys
    compressed so far.  Its inputs are rows of the sequence's own q and w
    and the sequence's kc, so a decode step reproduces rows of the prefill
    workload ``seq``."""

    name: str
    seq: Shape
    t0: int
    S_q: int

    @property
    def T(self) -> int:
        return self.seq.T


DECODE_SHAPES = {
    # 64 sequences of 65,536 tokens (16,384 compressed keys each), the next
    # token of each: the memory-bound regime (268 MB of keys per step)
    "decode_b64_t16k": DecodeShape(
        "decode_b64_t16k", Shape("decode_b64_t16k", 64, 65536, 4, 64, 128, 2048, "ar1", 1.0 / 8.0,
                                 0), 65535, 1),
}


def gen_decode(ds: DecodeShape, seed: int = 0):
    """(q [B,S_q,H,D] bf16 bits, w [B,S_q,H] fp32, kc [B,T,D] bf16 bits) of a
    decode step: rows t0 .. t0+S_q-1 of the sequence's q and w, and its kc."""
    sh = ds.seq
    rows = (np.arange(sh.B, dtype=np.int64)[:, None] * sh.S
            + np.minimum(ds.t0 + np.arange(ds.S_q), sh.S - 1)[None, :]).reshape(-1)
    q, w = gen_rows(sh, rows, seed)
    return (q.reshape(sh.B, ds.S_q, sh.H, sh.D), w.reshape(sh.B, ds.S_q, sh.H), gen_kc(sh, seed))


# --------------------------------------------------------------------------- attention


# Query-group candidate scans: (indexer workload, group size G, candidates C).
PIVOT_SCANS = {
    "pivot_s16k": ("v4flash_s16k", 16, 1024),   # top-512
    "pivot_s256k": ("long_s256k", 64, 2048),    # top-2048
}

# A layer: the indexer step of SHAPES[indexer] followed by the attention of
# 128 heads of dim 128 over the entries it selects.
ATTENTION_LAYERS = {
    "layer_s16k": "v4flash_s16k",     # S = 16,384, top-512
    "layer_s64k": "large_s64k",       # S = 65,536, top-2048
}


def gen_attention(B: int, S: int, T: int, H: int = 128, D: int = 128, seed: int = 0):
    """Inputs of the sparse attention over the selected entries: query heads
    qa [B,S,H,D] and the entries' key and value rows ka, va [B,T,D], all iid
    N(0,1) rounded to bf16 bits (the softmax scale 1/sqrt(D) then gives
    logits of unit spread)."""
    g = _rng(seed, 16, B, S, T)
    qa = f32_to_bf16_bits(g.standard_normal((B, S, H, D), dtype=np.float32))
    ka = f32_to_bf16_bits(g.standard_normal((B, T, D), dtype=np.float32))
    va = f32_to_bf16_bits(g.standard_normal((B, T, D), dtype=np.float32))
    return qa, ka, va


def small(B: int, S: int, m: int, H: int, D: int, topk: int, seed: int = 0, kc_kind: str = "iid",
          w_scale: float = 0.125) -> Shape:
    """An ad-hoc small workload (tests use these for ragged and edge shapes)."""
    return Shape(f"small_{B}x{S}_m{m}_h{H}_d{D}_k{topk}", B, S, m, H, D, topk, kc_kind, w_scale, 0)

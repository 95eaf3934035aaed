"""Exact-rational brute force for tiny indexer inputs (test infrastructure).

Every input value (bf16 bits, fp32) is converted to a ``fractions.Fraction``
exactly and the score is formed with exact rational arithmetic:

    score(t, j) = sum_h w[t,h] * max(0, sum_d q[t,h,d] * kc[j,d])

over the keys visible to t ((j+1)*m - 1 <= t).  Ranking is by exact score
descending, then index ascending; missing slots are -1.  No floating point is
involved, so ties are decided exactly.  Pure Python loops: tiny inputs only.
"""

from __future__ import annotations

import struct
from fractions import Fraction


def _f32(x: float) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<f", float(x)))[0])


def _bf16(bits: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0])


def visible_count(t: int, T: int, m: int) -> int:
    return sum(1 for j in range(T) if (j + 1) * m - 1 <= t)


def score(q, w, kc, b: int, t: int, j: int) -> Fraction:
    H, D = q.shape[2], q.shape[3]
    s = Fraction(0)
    for h in range(H):
        dot = Fraction(0)
        for d in range(D):
            dot += _bf16(q[b, t, h, d]) * _bf16(kc[b, j, d])
        s += _f32(w[b, t, h]) * max(Fraction(0), dot)
    return s


def topk(q, w, kc, m: int, k: int):
    """q [B,S,H,D] bf16 bits, w [B,S,H] fp32, kc [B,T,D] bf16 bits.
    Returns (idx, score) as nested lists [B*S][k]; score entries are Fractions
    or None in padded slots."""
    B, S = q.shape[0], q.shape[1]
    T = kc.shape[1]
    out_idx, out_sc = [], []
    for b in range(B):
        for t in range(S):
            V = visible_count(t, T, m)
            pairs = [(score(q, w, kc, b, t, j), j) for j in range(V)]
            pairs.sort(key=lambda p: (-p[0], p[1]))
            sel = pairs[:k]
            out_idx.append([j for _, j in sel] + [-1] * (k - len(sel)))
            out_sc.append([s for s, _ in sel] + [None] * (k - len(sel)))
    return out_idx, out_sc


def topk_decode(q, w, kc, m: int, k: int, t0: int):
    """Decode form: query i of batch b sits at sequence position t0 + i and
    sees the keys j with (j+1)*m - 1 <= t0 + i (all T of them once the
    position is past the last key).  q [B,S_q,H,D], w [B,S_q,H], kc [B,T,D].
    Returns (idx, score) as in topk()."""
    B, S = q.shape[0], q.shape[1]
    T = kc.shape[1]
    out_idx, out_sc = [], []
    for b in range(B):
        for i in range(S):
            V = visible_count(t0 + i, T, m)
            pairs = [(score(q, w, kc, b, i, j), j) for j in range(V)]
            pairs.sort(key=lambda p: (-p[0], p[1]))
            sel = pairs[:k]
            out_idx.append([j for _, j in sel] + [-1] * (k - len(sel)))
            out_sc.append([s for s, _ in sel] + [None] * (k - len(sel)))
    return out_idx, out_sc


def topk_pivot(q, w, kc, m: int, k: int, G: int, C: int):
    """Query-group candidate scan in exact arithmetic: the last position of
    each group of G keeps its C best visible keys; every query of the group
    ranks the candidates it can see by its own score and keeps k."""
    B, S = q.shape[0], q.shape[1]
    T = kc.shape[1]
    out_idx, out_sc = [], []
    for b in range(B):
        cand = {}
        for t in range(S):
            rep = min(t // G * G + G - 1, S - 1)
            if rep not in cand:
                Vr = visible_count(rep, T, m)
                pr = sorted(((score(q, w, kc, b, rep, j), j) for j in range(Vr)),
                            key=lambda p: (-p[0], p[1]))
                cand[rep] = [j for _, j in pr[:C]]
            V = visible_count(t, T, m)
            pairs = [(score(q, w, kc, b, t, j), j) for j in cand[rep] if j < V]
            pairs.sort(key=lambda p: (-p[0], p[1]))
            sel = pairs[:k]
            out_idx.append([j for _, j in sel] + [-1] * (k - len(sel)))
            out_sc.append([s for s, _ in sel] + [None] * (k - len(sel)))
    return out_idx, out_sc


def e4m3_value(code: int) -> Fraction:
    """Exact value of an OCP E4M3 code (bias 7, 3 mantissa bits, exponent
    field 0 subnormal), written out from the format's definition."""
    s = -1 if code & 0x80 else 1
    e = (code >> 3) & 15
    mnt = code & 7
    if e == 0:
        v = Fraction(mnt, 8) * Fraction(1, 2 ** 6)
    else:
        v = (1 + Fraction(mnt, 8)) * (Fraction(2) ** (e - 7))
    return s * v


def score_fp8(q8, s_q, w, k8, s_k, b: int, t: int, j: int) -> Fraction:
    """Exact FP8 score of key j for query (b, t):
    sum_h w * max(0, s_q[t,h] * s_k[j] * sum_d e4m3(q8) * e4m3(k8))."""
    H, D = q8.shape[2], q8.shape[3]
    s = Fraction(0)
    for h in range(H):
        dot = sum((e4m3_value(int(q8[b, t, h, d])) * e4m3_value(int(k8[b, j, d]))
                   for d in range(D)), Fraction(0))
        x = _f32(s_q[b, t, h]) * _f32(s_k[b, j]) * dot
        s += _f32(w[b, t, h]) * max(Fraction(0), x)
    return s


def topk_fp8(q8, s_q, w, k8, s_k, m: int, k: int):
    """Exact-rational FP8 score top-k:
    score = sum_h w * max(0, s_q[t,h] * s_k[j] * sum_d e4m3(q8) * e4m3(k8))."""
    B, S = q8.shape[:2]
    T = k8.shape[1]
    out_idx, out_sc = [], []
    for b in range(B):
        for t in range(S):
            V = visible_count(t, T, m)
            pairs = [(score_fp8(q8, s_q, w, k8, s_k, b, t, j), j) for j in range(V)]
            pairs.sort(key=lambda p: (-p[0], p[1]))
            sel = pairs[:k]
            out_idx.append([j for _, j in sel] + [-1] * (k - len(sel)))
            out_sc.append([s for s, _ in sel] + [None] * (k - len(sel)))
    return out_idx, out_sc

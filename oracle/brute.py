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


def _e4m3_finite_codes():
    """Non-negative finite E4M3 codes and their exact values, ascending."""
    return [(c, e4m3_value(c)) for c in range(0x7F)]


def mx_quantize_block(bits):
    """MX block scaling of one block of bf16 values (given as bit patterns),
    found by search rather than by formula: the scale exponent e is the one
    integer with 256 <= amax / 2^e < 512 (clamped to [-127, 127]; -127 for a
    block of zeros), and each element's code is the non-negative E4M3 code
    whose value is nearest to |x| / 2^e (ties to the even code, 448 for
    anything above), with x's sign bit.  Returns (codes, scale byte)."""
    vals = [_bf16(b) for b in bits]
    amax = max(abs(v) for v in vals)
    if amax == 0:
        e = -127
    else:
        e = 0
        while amax / Fraction(2) ** e >= 512:
            e += 1
        while amax / Fraction(2) ** e < 256:
            e -= 1
        e = max(-127, min(127, e))
    X = Fraction(2) ** e
    table = _e4m3_finite_codes()
    codes = []
    for b, v in zip(bits, vals):
        y = abs(v) / X
        best = None
        for c, cv in table:
            d = abs(cv - y)
            if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
                best = (d, c)
        codes.append(best[1] | (0x80 if int(b) & 0x8000 else 0))
    return codes, e + 127


def mx_value(code: int, scale_byte: int) -> Fraction:
    """Exact value of an MX element: its E4M3 value times 2^(byte - 127)."""
    return e4m3_value(code) * Fraction(2) ** (scale_byte - 127)


def topk_mxfp8(q8, qs, w, k8, ks, m: int, k: int):
    """Exact-rational MXFP8 score top-k; q8 [B,S,H,D], qs [B,S,H,D/32], w
    [B,S,H], k8 [B,T,D], ks [B,T,D/32]:
    score = sum_h w * max(0, sum_d mx(q8, qs) * mx(k8, ks)), the block of
    element d being d // 32."""
    B, S, H, D = q8.shape
    T = k8.shape[1]
    out_idx, out_sc = [], []
    for b in range(B):
        for t in range(S):
            V = visible_count(t, T, m)
            pairs = []
            for j in range(V):
                s = Fraction(0)
                for h in range(H):
                    dot = sum((mx_value(int(q8[b, t, h, d]), int(qs[b, t, h, d // 32])) *
                               mx_value(int(k8[b, j, d]), int(ks[b, j, d // 32]))
                               for d in range(D)), Fraction(0))
                    s += _f32(w[b, t, h]) * max(Fraction(0), dot)
                pairs.append((s, j))
            pairs.sort(key=lambda p: (-p[0], p[1]))
            sel = pairs[:k]
            out_idx.append([j for _, j in sel] + [-1] * (k - len(sel)))
            out_sc.append([s for s, _ in sel] + [None] * (k - len(sel)))
    return out_idx, out_sc

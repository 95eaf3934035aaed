"""The oracle's pins as one suite over an oracle API object.

Each check ties an oracle function to something other than the oracle itself:
the hand-worked values of tests/golden/hand_cases.json, exact rational
arithmetic (oracle/brute.py) and the visibility rule written out.  The same
suite runs on the built oracle (tests/test_oracle.py) and on copies with a
planted mistake (tests/test_oracle_mutations.py), which it must reject.

``o`` is the ``oracle`` module or ``oracle.load_copy(path)``.  Every check
covers the functions the GPU parity tests and the smoke check call:
indexer_topk, indexer_topk_rows, indexer_topk_rows_absmax (the rows, their
scores and the max |score| that scales the tolerance rule), score_keys_rows
(the score of a key outside the oracle's own top-k), row_absmax_rows and the
FP8 pair indexer_topk_fp8_rows / score_keys_fp8_rows, and the MX block
FP8 functions (mx_scale_byte, quantize_mxfp8_rows, indexer_topk_mxfp8_rows).
"""

from __future__ import annotations

import numpy as np

import synth
from oracle import brute
from tests import _golden


def _same_scores(got, want) -> bool:
    """fp64 scores equal, or both the same infinity (padding)."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return bool(np.all((got == want) | (np.isinf(got) & np.isinf(want) & (got == want))))


def _brute_scores(q, w, kc, m):
    """Exact scores of every key for every query, as fp64 (None where the key
    is not visible).  Values are dyadic with few bits, so fp64 holds them
    exactly and fp64 equality is exact equality."""
    B, S = q.shape[:2]
    T = kc.shape[1]
    out = np.full((B * S, T), np.nan)
    for b in range(B):
        for t in range(S):
            for j in range(brute.visible_count(t, T, m)):
                out[b * S + t, j] = float(brute.score(q, w, kc, b, t, j))
    return out


def _dyadic(seed, B, S, m, H, D):
    """Values on the grid i/8, |i| <= 8: every fp64 product and sum of the
    oracle is exact, and exact ties are frequent."""
    g = np.random.default_rng(seed)
    T = S // m
    q = g.integers(-8, 9, size=(B, S, H, D)).astype(np.float32) / 8
    kc = g.integers(-8, 9, size=(B, T, D)).astype(np.float32) / 8
    w = g.integers(-8, 9, size=(B, S, H)).astype(np.float32) / 8
    return synth.f32_to_bf16_bits(q), w, synth.f32_to_bf16_bits(kc)


# (seed, B, S, m, H, D, k): two batches (batch offsets), rows t < m-1 that see
# no key, rows that see fewer keys than k, m = 1
DYADIC = [(11, 1, 12, 2, 3, 4, 4), (12, 2, 12, 3, 2, 3, 3), (13, 2, 8, 1, 2, 2, 5),
          (14, 2, 16, 4, 3, 2, 2)]


def check_hand_cases(o) -> None:
    """The hand-worked rows through every row-producing entry, and the max
    |score| of each row against the exact brute-force scores."""
    for c in _golden.cases():
        q, w, kc, m, k = c["q"], c["w"], c["kc"], c["m"], c["k"]
        B, S = q.shape[:2]
        rows = np.arange(B * S)
        qr, wr = q.reshape(B * S, *q.shape[2:]), w.reshape(B * S, -1)
        idx, sc = o.indexer_topk(q, w, kc, m, k)
        assert np.array_equal(idx, c["idx"]) and _same_scores(sc, c["score"]), c["name"]
        idx, sc = o.indexer_topk_rows(qr, wr, kc, S, m, k, rows)
        assert np.array_equal(idx, c["idx"]) and _same_scores(sc, c["score"]), c["name"]
        idx, sc, amax = o.indexer_topk_rows_absmax(qr, wr, kc, S, m, k, rows)
        assert np.array_equal(idx, c["idx"]) and _same_scores(sc, c["score"]), c["name"]
        exact = _brute_scores(q, w, kc, m)
        want = np.max(np.abs(np.nan_to_num(exact, nan=0.0)), axis=1)
        assert np.array_equal(amax, want), (c["name"], amax, want)


def check_dyadic_brute_force(o) -> None:
    """Every row function against exact rational arithmetic on dyadic inputs:
    rows and scores, the visible-key max |score|, and the score of every key
    j in [-1, T] (nan exactly where the key is not visible)."""
    for seed, B, S, m, H, D, k in DYADIC:
        q, w, kc = _dyadic(seed, B, S, m, H, D)
        T = S // m
        bi, bs = brute.topk(q, w, kc, m, k)
        bi = np.array(bi)
        bsf = np.array([[-np.inf if s is None else float(s) for s in r] for r in bs])
        exact = _brute_scores(q, w, kc, m)
        absmax = np.max(np.abs(np.nan_to_num(exact, nan=0.0)), axis=1)
        rows = np.arange(B * S)
        qr, wr = q.reshape(B * S, H, D), w.reshape(B * S, H)
        oi, os_ = o.indexer_topk(q, w, kc, m, k)
        assert np.array_equal(oi, bi) and _same_scores(os_, bsf), ("indexer_topk", seed)
        oi, os_ = o.indexer_topk_rows(qr, wr, kc, S, m, k, rows)
        assert np.array_equal(oi, bi) and _same_scores(os_, bsf), ("indexer_topk_rows", seed)
        oi, os_, am = o.indexer_topk_rows_absmax(qr, wr, kc, S, m, k, rows)
        assert np.array_equal(oi, bi) and _same_scores(os_, bsf), ("rows_absmax", seed)
        assert np.array_equal(am, absmax), ("rows_absmax: absmax", seed, am, absmax)
        assert np.array_equal(o.row_absmax_rows(qr, wr, kc, S, m, rows), absmax), ("row_absmax",
                                                                                  seed)
        # a reversed row subset: each row still finds its own batch and position
        sub = rows[::-1][: max(1, rows.size // 2)]
        oi, _, am = o.indexer_topk_rows_absmax(qr[sub], wr[sub], kc, S, m, k, sub)
        assert np.array_equal(oi, bi[sub]) and np.array_equal(am, absmax[sub]), ("subset", seed)
        # scores of given keys: every j in [-1, T], visible or not
        js = np.broadcast_to(np.arange(-1, T + 1, dtype=np.int32), (B * S, T + 2))
        js = np.where(js > T - 1, -1, js).astype(np.int32)
        got = o.score_keys_rows(qr, wr, kc, S, m, rows, js)
        want = np.where(js >= 0, exact[rows[:, None], np.maximum(js, 0)], np.nan)
        same = (got == want) | (np.isnan(got) & np.isnan(want))
        assert np.all(same), ("score_keys_rows", seed, got, want)


def check_fp8_brute_force(o) -> None:
    """The FP8 rows and key scores against exact rational arithmetic on the
    decoded codes (codes and scales drawn directly, two batches)."""
    g = np.random.default_rng(21)
    B, S, m, H, D, k = 2, 12, 3, 2, 4, 3
    T = S // m
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    q8 = g.choice(codes, size=(B, S, H, D))
    k8 = g.choice(codes, size=(B, T, D))
    s_q = (g.integers(1, 16, size=(B, S, H)) / 8).astype(np.float32)
    s_k = (g.integers(1, 16, size=(B, T)) / 4).astype(np.float32)
    w = (g.integers(-8, 9, size=(B, S, H)) / 8).astype(np.float32)
    bi, bs = brute.topk_fp8(q8, s_q, w, k8, s_k, m, k)
    rows = np.arange(B * S)
    oi, os_ = o.indexer_topk_fp8_rows(q8.reshape(B * S, H, D), s_q.reshape(B * S, H),
                                      w.reshape(B * S, H), k8, s_k, S, m, k, rows)
    assert np.array_equal(oi, np.array(bi)), ("fp8 rows", oi, bi)
    # a reversed row subset with its own rows' codes: each row finds its batch
    sub = rows[::-1][::2].copy()
    si, ss = o.indexer_topk_fp8_rows(q8.reshape(B * S, H, D)[sub], s_q.reshape(B * S, H)[sub],
                                     w.reshape(B * S, H)[sub], k8, s_k, S, m, k, sub)
    assert np.array_equal(si, oi[sub]) and np.array_equal(ss, os_[sub]), "fp8 row subset"
    for r in range(B * S):
        for c in range(k):
            want = -np.inf if bs[r][c] is None else float(bs[r][c])
            assert os_[r, c] == want or abs(os_[r, c] - want) <= 1e-14 * abs(want), ("fp8 score",
                                                                                   r, c)
    js = np.broadcast_to(np.arange(-1, T, dtype=np.int32), (B * S, T + 1)).copy()
    got = o.score_keys_fp8_rows(q8.reshape(B * S, H, D), s_q.reshape(B * S, H),
                                w.reshape(B * S, H), k8, s_k, S, m, rows, js)
    for r in range(B * S):
        b, t = divmod(r, S)
        V = brute.visible_count(t, T, m)
        for c, j in enumerate(js[r]):
            if j < 0 or j >= V:
                assert np.isnan(got[r, c]), ("fp8 key score of an invisible key", r, j)
            else:
                want = float(brute.score_fp8(q8, s_q, w, k8, s_k, b, t, int(j)))
                assert abs(got[r, c] - want) <= 1e-14 * max(abs(want), 1e-300), ("fp8 key", r, j)


# (seed, B, T, m, H, D, k, t0, S_q): positions that see no key, fewer keys
# than k, exactly the last key (t0 + i = m*T - 1) and past it (all T keys)
DECODE = [(31, 2, 4, 3, 2, 3, 3, 0, 4), (32, 2, 4, 3, 2, 3, 3, 9, 6), (33, 1, 5, 2, 3, 2, 4, 8, 5),
          (34, 3, 3, 1, 2, 2, 2, 1, 4)]


def check_decode_brute_force(o) -> None:
    """The decode oracle (rows, scores, max |score|, key scores through the
    decode rows) against exact rational arithmetic with each query's own
    position, on dyadic inputs."""
    for seed, B, T, m, H, D, k, t0, S_q in DECODE:
        g = np.random.default_rng(seed)
        q = synth.f32_to_bf16_bits(g.integers(-8, 9, size=(B, S_q, H, D)).astype(np.float32) / 8)
        kc = synth.f32_to_bf16_bits(g.integers(-8, 9, size=(B, T, D)).astype(np.float32) / 8)
        w = (g.integers(-8, 9, size=(B, S_q, H)) / 8).astype(np.float32)
        bi, bs = brute.topk_decode(q, w, kc, m, k, t0)
        bsf = np.array([[-np.inf if x is None else float(x) for x in r] for r in bs])
        oi, os_, am = o.indexer_decode(q, w, kc, t0, m, k)
        assert np.array_equal(oi, np.array(bi)) and _same_scores(os_, bsf), ("decode", seed)
        exact = np.full((B * S_q, T), np.nan)
        for b in range(B):
            for i in range(S_q):
                for j in range(brute.visible_count(t0 + i, T, m)):
                    exact[b * S_q + i, j] = float(brute.score(q, w, kc, b, i, j))
        assert np.array_equal(am, np.max(np.abs(np.nan_to_num(exact, nan=0.0)), axis=1)), (
            "decode absmax", seed)
        S, rows = o.decode_rows(B, S_q, t0, T, m)
        js = np.broadcast_to(np.arange(-1, T, dtype=np.int32), (B * S_q, T + 1)).copy()
        got = o.score_keys_rows(q.reshape(B * S_q, H, D), w.reshape(B * S_q, H), kc, S, m, rows,
                                js)
        want = np.where(js >= 0, exact[np.arange(B * S_q)[:, None], np.maximum(js, 0)], np.nan)
        assert np.all((got == want) | (np.isnan(got) & np.isnan(want))), ("decode keys", seed)


def _sdpa_rows(qa, ka, va, idx, batch, scale):
    """The same attention through a library routine: torch's scaled dot-product
    attention in fp64 on the CPU, with a boolean mask over all T entries
    selecting the listed ones (rows with no listed entry give 0)."""
    import torch

    n, H, D = qa.shape
    T = ka.shape[1]
    out = np.zeros((n, H, D))
    for i in range(n):
        sel = idx[i][(idx[i] >= 0) & (idx[i] < T)]
        if sel.size == 0:
            continue
        mask = torch.zeros((1, 1, 1, T), dtype=torch.bool)
        mask[..., torch.from_numpy(sel.astype(np.int64))] = True
        q = torch.from_numpy(synth.bf16_bits_to_f32(qa[i]).astype(np.float64))[None, :, None, :]
        kk = torch.from_numpy(synth.bf16_bits_to_f32(ka[batch[i]]).astype(np.float64))
        vv = torch.from_numpy(synth.bf16_bits_to_f32(va[batch[i]]).astype(np.float64))
        kk = kk[None, None].expand(1, H, T, D)
        vv = vv[None, None].expand(1, H, T, D)
        o = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, attn_mask=mask,
                                                             scale=scale)
        out[i] = o[0, :, 0, :].numpy()
    return out


def check_sparse_attention(o) -> None:
    """The attention oracle against (a) torch's fp64 scaled dot-product
    attention with a mask of the listed entries, on random rows with padding,
    out-of-range entries and two batches; (b) closed forms: one listed entry
    gives its value row exactly, all-equal logits give the mean of the listed
    value rows, two entries whose logits differ by ln 3 get weights 1/4 and
    3/4; (c) the weighted magnitude equals the output when every value is
    non-negative, and is 0 with the output for a row with no entry."""
    g = np.random.default_rng(41)
    B, T, H, D, k, n = 2, 9, 3, 4, 5, 7
    qa = synth.f32_to_bf16_bits(g.standard_normal((n, H, D)).astype(np.float32))
    ka = synth.f32_to_bf16_bits(g.standard_normal((B, T, D)).astype(np.float32))
    va = synth.f32_to_bf16_bits(g.standard_normal((B, T, D)).astype(np.float32))
    idx = np.stack([g.permutation(T)[:k] for _ in range(n)]).astype(np.int32)
    idx[1, 3:] = -1          # padding
    idx[2, 0] = T            # out of range: skipped
    idx[3, :] = -1           # no entry
    batch = np.array([0, 1, 1, 0, 1, 0, 1], dtype=np.int64)
    scale = 0.37
    out, absw = o.sparse_attention_rows(qa, ka, va, idx, batch, scale)
    ref = _sdpa_rows(qa, ka, va, idx, batch, scale)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-13), ("sparse attention vs sdpa", out, ref)
    assert np.all(out[3] == 0) and np.all(absw[3] == 0), "row with no entry"
    # closed forms, on dyadic values
    one = lambda x: synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))  # noqa: E731
    ka1 = one([[[1, 0], [0, 1], [0.5, 0.5], [1, 1]]])                          # [1, 4, 2]
    va1 = one([[[2, -3], [0.25, 4], [-1, 1], [8, 0.5]]])
    qa1 = one([[[1, 0], [0, 0]]])                                             # head 1: q = 0
    out1, _ = o.sparse_attention_rows(qa1, ka1, va1, np.array([[2, -1, -1]], np.int32),
                                      np.array([0]), 1.0)
    assert np.array_equal(out1[0, 0], [-1.0, 1.0]) and np.array_equal(out1[0, 1], [-1.0, 1.0])
    out2, _ = o.sparse_attention_rows(qa1, ka1, va1, np.array([[0, 1, 3]], np.int32),
                                      np.array([0]), 1.0)
    assert np.allclose(out2[0, 1], (np.array([2, -3]) + [0.25, 4] + [8, 0.5]) / 3, rtol=1e-15)
    out3, _ = o.sparse_attention_rows(qa1, ka1, va1, np.array([[1, 0]], np.int32), np.array([0]),
                                      float(np.log(3.0)))
    # head 0: logits 0 (entry 1) and ln 3 (entry 0): weights 1/4 and 3/4
    assert np.allclose(out3[0, 0], 0.25 * np.array([0.25, 4]) + 0.75 * np.array([2, -3]),
                       rtol=1e-14, atol=1e-15)
    vpos = one(np.abs(g.standard_normal((B, T, D))))
    outp, absp = o.sparse_attention_rows(qa, ka, vpos, idx, batch, scale)
    assert np.allclose(outp, absp, rtol=1e-14, atol=0), "weighted magnitude, non-negative values"
    # the weighted magnitude is the attention output of |v| (library route)
    vabs = one(np.abs(synth.bf16_bits_to_f32(va)))
    assert np.allclose(absw, _sdpa_rows(qa, ka, vabs, idx, batch, scale), rtol=1e-12, atol=1e-13)


def check_pivot(o) -> None:
    """The query-group scan against exact arithmetic on dyadic inputs (groups
    of 2 and 3, fewer and more candidates than k), and its two special cases:
    groups of one query with C = k, and C at least T, both equal the exact
    indexer rows."""
    for seed, B, S, m, H, D, k, G, C in [(51, 2, 12, 2, 2, 3, 2, 3, 3), (52, 1, 12, 3, 2, 2, 3, 2, 2),
                                         (53, 2, 8, 1, 2, 2, 2, 4, 5)]:
        q, w, kc = _dyadic(seed, B, S, m, H, D)
        rows = np.arange(B * S)
        bi, bs = brute.topk_pivot(q, w, kc, m, k, G, C)
        bsf = np.array([[-np.inf if x is None else float(x) for x in r] for r in bs])
        oi, os_, _ = o.pivot_rows(q, w, kc, m, k, G, C, rows)
        assert np.array_equal(oi, np.array(bi)) and _same_scores(os_, bsf), ("pivot", seed)
        # a subset of the rows in another order gives those rows' results
        sub = rows[::-1][::2].copy()
        si, ss, _ = o.pivot_rows(q, w, kc, m, k, G, C, sub)
        assert np.array_equal(si, oi[sub]) and _same_scores(ss, os_[sub]), ("pivot rows", seed)
        ei, es = o.indexer_topk(q, w, kc, m, k)
        oi, os_, _ = o.pivot_rows(q, w, kc, m, k, 1, k, rows)
        assert np.array_equal(oi, ei) and _same_scores(os_, es), ("pivot G=1", seed)
        oi, os_, _ = o.pivot_rows(q, w, kc, m, k, G, S // m, rows)
        assert np.array_equal(oi, ei) and _same_scores(os_, es), ("pivot C>=T", seed)


def _bf16_bits(x) -> np.ndarray:
    """fp32 values that bf16 holds exactly -> their bf16 bit patterns."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not exact in bf16"
    return (b >> 16).astype(np.uint16)


def check_mxfp8(o) -> None:
    """MX block scaling and the MXFP8 score.

    The scale byte at worked values of the rule (the largest magnitude
    scaled into [256, 512), clamped to 2^-127 .. 2^127, zeros at 2^-127);
    the quantiser against a search over the E4M3 value table
    (brute.mx_quantize_block) on blocks of five magnitudes, signed zeros,
    a saturating block and round-to-even ties; exact round trips of values
    the format holds; the MXFP8 rows against exact rational arithmetic (two
    batches, blocks with different scales); and, with one scale per row, the
    per-row FP8 oracle on the same codes."""
    # worked values: amax -> e = floor(log2 amax) - 8, byte e + 127
    for amax, byte in [(1.0, 119), (448.0, 127), (500.0, 127), (511.0, 127), (256.0, 127),
                       (255.0, 126), (512.0, 128), (0.0, 0), (3 * 2.0 ** -130, 0),
                       (2.0 ** -118, 1), (2.0 ** 135, 254), (2.0 ** 140, 254), (0.75, 118)]:
        assert o.mx_scale_byte(amax) == byte, ("mx scale byte", amax)
    # the quantiser against the search, block by block
    g = np.random.default_rng(41)
    blocks = []
    for mag in (1e-30, 1e-3, 1.0, 7.0, 1e20):
        blocks.append(g.standard_normal(32) * mag)
    blocks.append(np.zeros(32))
    sat = g.standard_normal(32)
    sat[5] = 500.0  # e = 0: 500 saturates to 448; -3 and 1.0625 (a tie) keep theirs
    sat[6], sat[7], sat[8] = -3.0, 1.0625, -0.0
    blocks.append(sat)
    tiny = g.standard_normal(32) * 1e-39  # bf16 subnormals: the scale clamps at 2^-127
    blocks.append(tiny)
    x = np.stack(blocks).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16).reshape(4, 64)  # truncation: any bf16
    codes, scales = o.quantize_mxfp8_rows(bits)
    assert codes.shape == (4, 64) and scales.shape == (4, 2)
    for r in range(4):
        for blk in range(2):
            bc, bs = brute.mx_quantize_block(bits[r, blk * 32:(blk + 1) * 32].tolist())
            assert scales[r, blk] == bs, ("mx scale", r, blk)
            assert codes[r, blk * 32:(blk + 1) * 32].tolist() == bc, ("mx codes", r, blk)
    # exact round trip: E4M3 values times 2^e whose block maximum fixes e
    vals = np.array([brute.e4m3_value(c) for c in range(0x7F)], dtype=object)
    for e in (-20, 0, 9):
        pick = g.choice(np.arange(0x7F), size=32)
        pick[0] = 0x7E  # 448: the block's maximum, so its exponent is e
        v = np.array([float(vals[c]) * 2.0 ** e for c in pick], dtype=np.float32)
        v[1::2] *= -1
        c2, s2 = o.quantize_mxfp8_rows(_bf16_bits(v).reshape(1, 32))
        assert s2[0, 0] == e + 127
        back = np.array([float(brute.mx_value(int(c), int(s2[0, 0]))) for c in c2[0]])
        assert np.array_equal(back, v.astype(np.float64)), ("mx round trip", e)
    # MXFP8 rows against exact rational arithmetic
    B, S, m, H, D, k = 2, 6, 2, 2, 64, 3
    T = S // m
    fin = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    q8 = g.choice(fin, size=(B, S, H, D))
    k8 = g.choice(fin, size=(B, T, D))
    qs = g.integers(118, 136, size=(B, S, H, D // 32)).astype(np.uint8)
    ks = g.integers(118, 136, size=(B, T, D // 32)).astype(np.uint8)
    w = (g.integers(-8, 9, size=(B, S, H)) / 8).astype(np.float32)
    bi, bsc = brute.topk_mxfp8(q8, qs, w, k8, ks, m, k)
    rows = np.arange(B * S)
    oi, os_ = o.indexer_topk_mxfp8_rows(q8.reshape(B * S, H, D), qs.reshape(B * S, H, D // 32),
                                        w.reshape(B * S, H), k8, ks, S, m, k, rows)
    assert np.array_equal(oi, np.array(bi)), ("mxfp8 rows", oi, bi)
    for r in range(B * S):
        for c in range(k):
            want = -np.inf if bsc[r][c] is None else float(bsc[r][c])
            assert os_[r, c] == want or abs(os_[r, c] - want) <= 1e-14 * abs(want), ("mx score",
                                                                                   r, c)
    # one scale per row: the per-row FP8 oracle with s = 2^(byte - 127)
    qb = g.integers(118, 136, size=(B, S, H)).astype(np.uint8)
    kb = g.integers(118, 136, size=(B, T)).astype(np.uint8)
    qs1 = np.repeat(qb[..., None], D // 32, axis=-1)
    ks1 = np.repeat(kb[..., None], D // 32, axis=-1)
    mi, ms = o.indexer_topk_mxfp8_rows(q8.reshape(B * S, H, D), qs1.reshape(B * S, H, D // 32),
                                       w.reshape(B * S, H), k8, ks1, S, m, k, rows)
    fi, fs = o.indexer_topk_fp8_rows(q8.reshape(B * S, H, D),
                                     np.ldexp(1.0, qb.astype(np.int32) - 127).astype(
                                         np.float32).reshape(B * S, H),
                                     w.reshape(B * S, H), k8,
                                     np.ldexp(1.0, kb.astype(np.int32) - 127).astype(np.float32),
                                     S, m, k, rows)
    assert np.array_equal(mi, fi) and np.allclose(ms, fs, rtol=1e-13, atol=0), "mx vs fp8"


def check_topk_scores(o) -> None:
    """The selection on given fp32 values (the bit-exact tests' reference)
    against numpy's lexsort with -0 folded into +0, on normal, tied,
    constant and infinite scores, with fewer visible keys than k."""
    for kind in ["normal", "ties", "const", "inf"]:
        X = synth.gen_scores(2, 40, 13, seed=3, kind=kind)
        for m, k in [(3, 4), (1, 13), (2, 20)]:
            oi, os_ = o.topk_scores(X, m, k)
            for r in range(2 * 40):
                b, t = divmod(r, 40)
                V = min(13, (t + 1) // m)
                x = X[b, t, :V].copy()
                key = np.where(x == 0, np.float32(0), x)  # -0 -> +0
                order = np.lexsort((np.arange(V), -key.astype(np.float64)))[:k]
                n = order.size
                assert np.array_equal(oi[r, :n], order), ("topk_scores order", kind, r)
                assert np.array_equal(os_[r, :n].view(np.uint32), x[order].view(np.uint32))
                assert np.all(oi[r, n:] == -1) and np.all(np.isneginf(os_[r, n:])), "padding"


def check_fp8_quantiser(o) -> None:
    """The per-row E4M3 quantiser: the encoder against torch's float8_e4m3fn
    conversion (a library route) on values spread over the format's range,
    including the subnormal grid and exact ties, and hand values from the
    format's definition (saturation, signed zero); the row scale is the
    row's largest magnitude over 448, which lands that element on +-448."""
    import torch

    g = np.random.default_rng(5)
    ys = (np.exp2(g.uniform(-11, 8.8, size=4000)) * g.choice([-1, 1], size=4000)).astype(np.float32)
    ties = np.array([1.0625, 1.1875, 3 * 2.0 ** -10, 5 * 2.0 ** -10, 2.0 ** -11, 17.0, 19.0, 464.0],
                    dtype=np.float32)
    ys = np.concatenate([ys[np.abs(ys) <= 448], ties])
    want = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([o.e4m3_encode(float(y)) for y in ys], dtype=np.uint8)
    assert np.array_equal(got, want), "e4m3 encoder vs torch"
    assert o.e4m3_encode(500.0) == 0x7E and o.e4m3_encode(-1000.0) == 0xFE, "saturation"
    assert o.e4m3_encode(-0.0) == 0x80 and o.e4m3_encode(0.0) == 0x00, "signed zero"
    sh = synth.small(1, 16, 4, 4, 64, 8, seed=2)
    q = synth.gen_q(sh, 2)
    codes, scale = o.quantize_e4m3_rows(q)
    x = synth.bf16_bits_to_f32(q)
    amax = np.abs(x).max(axis=-1)
    assert np.array_equal(scale, (amax / np.float32(448)).astype(np.float32)), "row scale"
    am = np.abs(x).argmax(axis=-1)
    top = np.take_along_axis(codes, am[..., None], axis=-1)[..., 0]
    assert np.all((top & 0x7F) == 0x7E), "row maximum on 448"
    y = (x / scale[..., None]).astype(np.float32)
    want = torch.from_numpy(np.clip(y, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, want), "row codes vs torch"


def run_all(o) -> None:
    check_hand_cases(o)
    check_topk_scores(o)
    check_fp8_quantiser(o)
    check_dyadic_brute_force(o)
    check_fp8_brute_force(o)
    check_decode_brute_force(o)
    check_sparse_attention(o)
    check_pivot(o)
    check_mxfp8(o)

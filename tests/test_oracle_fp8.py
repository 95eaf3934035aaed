"""Pins for the oracle's FP8 E4M3 path: the encoder and decoder against
torch's float8_e4m3fn conversion (a library routine) and against hand values
from the format's definition; the FP8 score against exact rational arithmetic
and against the bf16 oracle where both represent the same values exactly."""

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import brute


def test_decode_all_codes_match_torch():
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue  # NaN codes
        want = torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float().item()
        assert oracle.e4m3_decode(c) == want, c
        assert float(brute.e4m3_value(c)) == want, c


def test_encode_hand_values():
    # from the definition: 1.0 = 2^0 * (1 + 0/8) -> field 7, mantissa 0 -> 0x38
    assert oracle.e4m3_encode(1.0) == 0x38
    assert oracle.e4m3_encode(448.0) == 0x7E          # 2^8 * 1.75, largest finite
    assert oracle.e4m3_encode(500.0) == 0x7E          # saturates
    assert oracle.e4m3_encode(-1000.0) == 0xFE
    assert oracle.e4m3_encode(2.0 ** -9) == 0x01       # smallest subnormal
    assert oracle.e4m3_encode(2.0 ** -6) == 0x08       # smallest normal
    assert oracle.e4m3_encode(1.0625) == 0x38          # halfway 1 / 1.125: even mantissa 0
    assert oracle.e4m3_encode(1.1875) == 0x3A          # halfway 1.125 / 1.25: even mantissa 2
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02  # 1.5 subnormal steps: even -> 2 steps
    assert oracle.e4m3_encode(5 * 2.0 ** -10) == 0x02  # 2.5 subnormal steps: even -> 2 steps
    assert oracle.e4m3_encode(2.0 ** -11) == 0x00      # 0.25 of a step rounds to zero
    assert oracle.e4m3_encode(-0.0) == 0x80


def test_encode_matches_torch_random():
    g = np.random.default_rng(0)
    mags = np.exp2(g.uniform(-14, 8.8, size=200000)).astype(np.float32)
    ys = (mags * g.choice([-1, 1], size=mags.size)).astype(np.float32)
    ys = ys[np.abs(ys) <= 448]
    want = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(y)) for y in ys[:20000]], dtype=np.uint8)
    np.testing.assert_array_equal(got, want[:20000])


def test_quantize_rows_properties():
    sh = synth.small(1, 64, 4, 4, 128, 8, seed=1)
    q = synth.gen_q(sh, 1)
    codes, scale = oracle.quantize_e4m3_rows(q)
    x = synth.bf16_bits_to_f32(q)
    amax = np.abs(x).max(axis=-1)
    np.testing.assert_array_equal(scale, (amax / np.float32(448)).astype(np.float32))
    # the largest element of each row lands on +-448
    am = np.abs(x).argmax(axis=-1)
    top = np.take_along_axis(codes, am[..., None], axis=-1)[..., 0]
    assert np.all((top & 0x7F) == 0x7E)
    # codes = torch's E4M3 rounding of x / scale computed in fp32
    y = (x / scale[..., None]).astype(np.float32)
    want = torch.from_numpy(np.clip(y, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, want)
    # all-zero rows get scale 1 and zero codes
    z = np.zeros((2, 16), np.uint16)
    c0, s0 = oracle.quantize_e4m3_rows(z)
    assert np.all(c0 == 0) and np.all(s0 == 1.0)


@pytest.mark.parametrize("seed", [0, 1])
def test_fp8_score_brute_force(seed):
    sh = synth.small(1, 12, 2, 2, 4, 3, seed=seed)
    q, w, kc = synth.gen_q(sh, seed), synth.gen_w(sh, seed), synth.gen_kc(sh, seed)
    q8, sq = oracle.quantize_e4m3_rows(q)
    k8, sk = oracle.quantize_e4m3_rows(kc)
    bi, bs = brute.topk_fp8(q8, sq, w, k8, sk, sh.m, sh.topk)
    rows = np.arange(sh.S)
    oi, os_ = oracle.indexer_topk_fp8_rows(q8[0], sq[0], w[0], k8, sk, sh.S, sh.m, sh.topk, rows)
    np.testing.assert_array_equal(oi, np.array(bi))
    for r in range(sh.S):
        for c in range(sh.topk):
            if bs[r][c] is None:
                assert os_[r, c] == -np.inf
            else:
                assert abs(os_[r, c] - float(bs[r][c])) <= 1e-14 * max(1.0, abs(float(bs[r][c])))


def test_fp8_unit_scales_reduce_to_bf16_oracle():
    """Integer values |v| <= 8 are exact in both E4M3 and bf16: with unit
    scales the FP8 score equals the bf16 score of the same values."""
    g = np.random.default_rng(3)
    B, S, m, H, D, k = 1, 24, 3, 3, 8, 4
    T = S // m
    qv = g.integers(-8, 9, size=(B, S, H, D)).astype(np.float32)
    kv = g.integers(-8, 9, size=(B, T, D)).astype(np.float32)
    w = g.standard_normal((B, S, H)).astype(np.float32)
    enc = np.vectorize(oracle.e4m3_encode, otypes=[np.uint8])
    q8, k8 = enc(qv), enc(kv)
    sq = np.ones((S, H), np.float32)
    sk = np.ones((B, T), np.float32)
    oi8, os8 = oracle.indexer_topk_fp8_rows(q8[0], sq, w[0], k8, sk, S, m, k, np.arange(S))
    oi, os_ = oracle.indexer_topk(synth.f32_to_bf16_bits(qv), w, synth.f32_to_bf16_bits(kv), m, k)
    np.testing.assert_array_equal(oi8, oi)
    np.testing.assert_array_equal(os8, os_)

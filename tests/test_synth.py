"""The seeded generator: deterministic, row-regenerable, and drawing the
distributions the workloads name."""

import numpy as np

import synth


def test_rows_regenerate_exactly():
    sh = synth.small(2, 2500, 4, 8, 64, 16, kc_kind="ar1")
    q, w = synth.gen_q(sh, 3), synth.gen_w(sh, 3)
    rows = np.array([0, 1023, 1024, 2499, 2500, 4999, 3333])
    qr, wr = synth.gen_rows(sh, rows, 3)
    np.testing.assert_array_equal(qr, q.reshape(-1, sh.H, sh.D)[rows])
    np.testing.assert_array_equal(wr, w.reshape(-1, sh.H)[rows])


def test_deterministic_and_threads_agree():
    sh = synth.small(1, 3000, 4, 8, 64, 16)
    a = synth.gen_q(sh, 0, threads=1)
    b = synth.gen_q(sh, 0, threads=4)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, synth.gen_q(sh, 1))


def test_distributions():
    sh = synth.shape("v4flash_s16k")
    kc = synth.bf16_bits_to_f32(synth.gen_kc(sh)).astype(np.float64)[0]
    T = sh.T
    norms = np.linalg.norm(kc, axis=1)
    heavy = norms > 2.5 * np.median(norms)
    assert abs(heavy.sum() - round(0.02 * T)) <= 3
    light = kc[~heavy]
    assert abs(light.std() - 1 / np.sqrt(128)) < 0.01
    # lag-1 correlation along j of the non-heavy rows is about 0.9
    x = kc[:-1][~heavy[:-1] & ~heavy[1:]]
    y = kc[1:][~heavy[:-1] & ~heavy[1:]]
    r = (x * y).sum() / np.sqrt((x * x).sum() * (y * y).sum())
    assert 0.87 < r < 0.93
    qs = synth.bf16_bits_to_f32(synth.gen_q(synth.small(1, 1024, 4, 64, 128, 8)))
    assert abs(qs.std() - 1 / np.sqrt(128)) < 0.002
    ws = synth.gen_w(sh)
    assert abs(ws.std() - 1 / 8) < 0.002


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], np.float32)
    got = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    np.testing.assert_array_equal(got, np.array([1.0, 1.0, 1.0 + 4 * 2 ** -8, 1.0, -2.5], np.float32))


def test_sample_rows():
    sh = synth.shape("large_s64k")
    r = synth.sample_rows(sh)
    assert r.size == 257 and r[-1] == sh.S - 1 and np.all(np.diff(r) > 0)

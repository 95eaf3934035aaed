"""FP8 (E4M3) score path: the quantiser bit-exact against the oracle's, the
FP8 kernel against the oracle run on the same codes and scales (kernel
parity), and its recall against the bf16-input oracle (accuracy)."""

import numpy as np
import pytest
import torch

import oracle
import synth
import streaming_top_lightning_b200 as stl
from oracle import accept
from tests import _gpu

pytestmark = pytest.mark.gpu


def test_quantize_bit_exact():
    sh = synth.small(1, 512, 4, 64, 128, 8, seed=2, kc_kind="ar1")
    q, _, kc = _gpu.inputs(sh, seed=2)
    for x in (q, kc):
        codes, scale = stl.quantize_fp8_rows(_gpu.to_dev_bf16(x))
        oc, os_ = oracle.quantize_e4m3_rows(x)
        np.testing.assert_array_equal(codes.cpu().numpy(), oc)
        np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    z = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    zc, zs = stl.quantize_fp8_rows(z)
    assert torch.all(zc == 0) and torch.all(zs == 1.0)


@pytest.mark.parametrize("rows,cols", [(37, 64), (1001, 128), (5, 256), (7, 136), (3, 4096)])
def test_quantize_shapes_bit_exact(rows, cols):
    # the lane-group kernels (64, 128, 256 values per row, ragged row counts)
    # and the warp-per-row kernel (any other length), against the oracle
    g = np.random.default_rng(rows * 7919 + cols)
    x = g.standard_normal((rows, cols)).astype(np.float32)
    x[0] *= 1e-30  # tiny values: codes underflow to zero / subnormals
    x[-1] = 0.0     # an all-zero row has scale 1
    if rows > 2:
        x[1] *= 1e30  # huge values
    bits = synth.f32_to_bf16_bits(x)
    codes, scale = stl.quantize_fp8_rows(_gpu.to_dev_bf16(bits))
    oc, os_ = oracle.quantize_e4m3_rows(bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)
    np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), os_.view(np.uint32))


def _fp8_case(sh, seed, rows, opts=None):
    q, w, kc = _gpu.inputs(sh, seed=seed)
    q8, sq = stl.quantize_fp8_rows(_gpu.to_dev_bf16(q))
    k8, sk = stl.quantize_fp8_rows(_gpu.to_dev_bf16(kc))
    gi, gs = stl.indexer_topk_fp8(q8, sq, torch.from_numpy(w).cuda(), k8, sk, sh.m, sh.topk,
                                  opts=opts)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    k = sh.topk
    q8n = q8.cpu().numpy().reshape(-1, sh.H, sh.D)[rows]
    sqn = sq.cpu().numpy().reshape(-1, sh.H)[rows]
    wr = w.reshape(-1, sh.H)[rows]
    k8n, skn = k8.cpu().numpy(), sk.cpu().numpy()
    oi, os_ = oracle.indexer_topk_fp8_rows(q8n, sqn, wr, k8n, skn, sh.S, sh.m, k, rows)
    gi_r = gi.reshape(-1, k)[rows].cpu().numpy()
    extra = oracle.score_keys_fp8_rows(q8n, sqn, wr, k8n, skn, sh.S, sh.m, rows, gi_r)
    # row scale: max |score| over visible keys, from every visible key's FP8 score
    V = _gpu.visible(np.asarray(rows) % sh.S, sh.T, sh.m)
    allj = np.array([np.pad(np.arange(v), (0, sh.T - v), constant_values=-1) for v in V],
                    dtype=np.int32)
    amax = np.nanmax(np.abs(oracle.score_keys_fp8_rows(q8n, sqn, wr, k8n, skn, sh.S, sh.m, rows,
                                                       allj)), axis=1, initial=0.0)
    res = accept.check(rows, V, k, oi, os_, gi_r, extra, amax)
    assert accept.passed(res), {kk: (v[:5] if isinstance(v, list) else v) for kk, v in res.items()}
    # accuracy against the bf16-input oracle (reported; FP8 rounding moves keys
    # near the k-th score)
    qr, wr16 = q.reshape(-1, sh.H, sh.D)[rows], w.reshape(-1, sh.H)[rows]
    bi, _ = oracle.indexer_topk_rows(qr, wr16, kc, sh.S, sh.m, k, rows)
    rec = [np.intersect1d(gi_r[i][gi_r[i] >= 0], bi[i][bi[i] >= 0]).size / max(1, (bi[i] >= 0).sum())
           for i in range(len(rows))]
    return float(np.mean(rec))


def test_fp8_tiny_all_rows():
    sh = synth.small(1, 2048, 4, 8, 128, 64, seed=1, w_scale=1 / np.sqrt(8))
    rec = _fp8_case(sh, 1, np.arange(sh.S))
    assert rec > 0.9


def test_fp8_v4flash_sampled():
    sh = synth.shape("v4flash_s16k")
    rows = np.union1d(np.random.default_rng(2).choice(sh.S, 128, replace=False), [sh.S - 1])
    rec = _fp8_case(sh, 0, rows)
    assert rec > 0.9


@pytest.mark.parametrize("chunk", [0, 1024])
def test_fp8_chunked(chunk):
    sh = synth.small(1, 4096, 4, 64, 128, 128, seed=6, kc_kind="ar1")
    rows = np.arange(0, sh.S, 13)
    _fp8_case(sh, 6, rows, opts=stl.options(key_chunk=chunk) if chunk else None)

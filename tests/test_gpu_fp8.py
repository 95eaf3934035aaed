"""FP8 (E4M3) score path: the quantiser bit-exact against the oracle's, the
FP8 kernel against the FP8 oracle run on the oracle's own codes and scales
(kernel parity), and its accuracy against the bf16-input oracle: every key it
selects that the bf16 oracle does not is within the quantisation error bound
of tests/_fp8.py, and the set recall is recorded."""

import numpy as np
import pytest
import torch

import oracle
import synth
import streaming_top_lightning_b200 as stl
from oracle import accept
from tests import _fp8, _gpu

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


def test_fp8_tiny_all_rows():
    sh = synth.small(1, 2048, 4, 8, 128, 64, seed=1, w_scale=1 / np.sqrt(8))
    q, w, kc = _gpu.inputs(sh, seed=1)
    rows = np.arange(sh.S)
    rec = _fp8.check_fp8_rows(sh, q, w, kc, rows, _fp8.fp8_run(sh, q, w, kc))
    _gpu.record("recall", {"workload": "tiny_h8_d128", "path": "fp8-e4m3", "rows": int(rows.size),
                           **rec})


def test_fp8_v4flash_sampled():
    sh = synth.shape("v4flash_s16k")
    q, w, kc = _gpu.inputs(sh)
    rows = np.union1d(np.random.default_rng(2).choice(sh.S, 128, replace=False), [sh.S - 1])
    rec = _fp8.check_fp8_rows(sh, q, w, kc, rows, _fp8.fp8_run(sh, q, w, kc))
    _gpu.record("recall", {"workload": sh.name, "path": "fp8-e4m3", "rows": int(rows.size),
                           **rec})


@pytest.mark.parametrize("chunk", [0, 1024])
def test_fp8_chunked(chunk):
    sh = synth.small(1, 4096, 4, 64, 128, 128, seed=6, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=6)
    rows = np.arange(0, sh.S, 13)
    _fp8.check_fp8_rows(sh, q, w, kc, rows,
                   _fp8.fp8_run(sh, q, w, kc, opts=stl.options(key_chunk=chunk) if chunk else None))

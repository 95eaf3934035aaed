"""The design-space sweep at S = 32,768 (T = 8,192, H_I = 64, d_I = 128):
key chunk, key tile and top-k, each swept with the other two at the library's
defaults, on the bf16 and the FP8-e4m3 score paths.  Every cell is checked on
256 sampled query rows (plus the last row) against the oracle: the acceptance
rule for bf16, kernel parity against the FP8 oracle plus the accuracy rule
against the bf16-input oracle for FP8.  Mean and min recall of every cell are
recorded when SI_RECORD_DIR is set.  ("StreamIndex: Memory-Bounded
Compressed Sparse Attention via Streaming Top-k", Abstract: three 5-point
sweeps of chunk size, key-tile size and top-k, with mean and minimum recall
per cell.)"""

import numpy as np
import pytest
import torch

import synth
import streaming_top_lightning_b200 as stl
from tests import _fp8, _gpu

pytestmark = pytest.mark.gpu

CELLS = ([("key_chunk", c) for c in (1024, 2048, 4096, 8192, 16384)] +
         [("key_tile", t) for t in (32, 64, 128, 256, 512, 1024)] +
         [("topk", k) for k in (128, 256, 512, 1024, 2048)])


@pytest.fixture(scope="module")
def sweep():
    sh = synth.shape("sweep_s32k")
    q, w, kc = _gpu.inputs(sh)
    rows = synth.sample_rows(sh)
    d = {"sh": sh, "q": q, "w": w, "kc": kc, "rows": rows,
         "qd": _gpu.to_dev_bf16(q), "wd": torch.from_numpy(w).cuda(), "kd": _gpu.to_dev_bf16(kc)}
    # the oracle's rows at the largest top-k; smaller ones are their prefixes
    d["bf16_ref"] = _gpu.oracle_ref(sh, q, w, kc, rows, k=2048)
    d["oq"] = _fp8.oracle_quantized(sh, q, kc, rows)
    d["fp8_ref"] = _fp8.fp8_oracle_ref(sh, w, *d["oq"], rows, 2048)
    q8, sq = stl.quantize_fp8_rows(d["qd"])
    k8, sk = stl.quantize_fp8_rows(d["kd"])
    torch.cuda.synchronize()
    q8r, sqr, k8o, sko = d["oq"]
    assert np.array_equal(q8.cpu().numpy().reshape(-1, sh.H, sh.D)[rows], q8r)
    assert np.array_equal(sq.cpu().numpy().reshape(-1, sh.H)[rows].view(np.uint32),
                          sqr.view(np.uint32))
    assert np.array_equal(k8.cpu().numpy(), k8o)
    assert np.array_equal(sk.cpu().numpy().view(np.uint32), sko.view(np.uint32))
    d["fp8"] = (q8, sq, k8, sk)
    return d


@pytest.mark.parametrize("path", ["bf16", "fp8"])
@pytest.mark.parametrize("axis,value", CELLS)
def test_sweep_cell(sweep, path, axis, value):
    base = sweep["sh"]
    sh = synth.shape("sweep_s32k", topk=value if axis == "topk" else base.topk)
    opts = stl.options(key_chunk=value if axis == "key_chunk" else 0,
                       key_tile=value if axis == "key_tile" else 0)
    q, w, kc, rows = sweep["q"], sweep["w"], sweep["kc"], sweep["rows"]
    entry = {"workload": sh.name, "path": "bf16" if path == "bf16" else "fp8-e4m3",
             "topk": sh.topk, "key_chunk": opts.key_chunk or "one", "key_tile": opts.key_tile or
             "auto", "rows": int(rows.size)}
    if path == "bf16":
        gi, gs = stl.indexer_topk(sweep["qd"], sweep["wd"], sweep["kd"], sh.m, sh.topk, opts=opts)
        torch.cuda.synchronize()
        assert stl.device_error() == 0
        res = _gpu.check_rows(sh, q, w, kc, gi, gs, rows, ref=sweep["bf16_ref"])
        entry.update(mean_recall=res["mean_recall"], min_recall=res["min_recall"])
    else:
        q8, sq, k8, sk = sweep["fp8"]
        gi, gs = stl.indexer_topk_fp8(q8, sq, sweep["wd"], k8, sk, sh.m, sh.topk, opts=opts)
        torch.cuda.synchronize()
        assert stl.device_error() == 0
        rec = _fp8.check_fp8_rows(sh, q, w, kc, rows, (gi, gs, q8, sq, k8, sk), oq=sweep["oq"],
                                  fp8_ref=sweep["fp8_ref"], bf16_ref=sweep["bf16_ref"],
                                  check_codes=False)
        entry.update(rec)
    _gpu.structural(sh, gi, gs, np.arange(0, sh.S, 97))
    _gpu.record("sweep_recall", entry)

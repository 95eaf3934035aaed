"""The allocation-free entry point, si_indexer_topk_noalloc.

It serves callers that cannot allocate device memory themselves or let a
library do so: a serving runtime that owns a fixed memory pool, a plugin
inside another framework, or a latency-critical loop where an allocator call
may block or fail under fragmentation.  Its scratch is a fixed device array
inside the library, so it must give exactly what the allocating entry point
gives, call after call, and must not take any device memory.

This file sorts last so that, in a run that stops at the first failure, every
other test has already run.
"""

import ctypes

import numpy as np
import pytest
import torch

import synth
import streaming_top_lightning_b200 as stl
from streaming_top_lightning_b200 import _lib
from tests import _gpu

pytestmark = pytest.mark.gpu


def _noalloc(lib, qd, wd, kd, m, k, idx, score):
    B, S, H, D = qd.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.si_indexer_topk_noalloc(p(qd), p(wd), p(kd), B, S, H, D, m, k, p(idx), p(score),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name", ["small", "v4flash_s16k"])
def test_noalloc_matches_allocating_entry_point(name):
    # two batches of a ragged small shape, and the V4-Flash-shaped step
    sh = (synth.small(2, 2048, 4, 64, 128, 96, seed=12, kc_kind="ar1") if name == "small"
          else synth.shape(name))
    q, w, kc = _gpu.inputs(sh, seed=12 if name == "small" else 0)
    qd, wd, kd = _gpu.to_dev_bf16(q), torch.from_numpy(w).cuda(), _gpu.to_dev_bf16(kc)
    ref_idx, ref_score = stl.indexer_topk(qd, wd, kd, sh.m, sh.topk)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    lib = _lib.load()
    idx = torch.empty_like(ref_idx)
    score = torch.empty_like(ref_score)

    def call_and_check():
        idx.fill_(-7)
        score.fill_(7.0)
        assert _noalloc(lib, qd, wd, kd, sh.m, sh.topk, idx, score) == 0
        torch.cuda.synchronize()
        assert stl.device_error() == 0
        assert torch.equal(idx, ref_idx)
        assert torch.equal(score.view(torch.int32), ref_score.view(torch.int32))

    # the first call on the device looks up the fixed array; with lazy module
    # loading the runtime may materialise the array's memory at that point
    call_and_check()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(2):  # two calls in a row, each identical to the reference
        call_and_check()
    assert torch.cuda.mem_get_info()[0] >= free_before

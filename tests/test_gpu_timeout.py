"""Failure detection without a GPU fault: a debug flag makes the producer skip
its first key-tile load, so the consumer's bounded wait on that stage must run
out.  The kernel then drains its own copies and MMAs, frees TMEM, records the
timeout in the device error word and exits; the context stays usable."""

import numpy as np
import pytest
import torch

import synth
import streaming_top_lightning_b200 as stl
from tests import _gpu

pytestmark = pytest.mark.gpu


def test_wait_expires_and_context_survives():
    sh = synth.small(1, 2048, 4, 64, 128, 64, seed=8)
    q, w, kc = _gpu.inputs(sh, seed=8)
    qd, wd, kd = _gpu.to_dev_bf16(q), torch.from_numpy(w).cuda(), _gpu.to_dev_bf16(kc)
    assert stl.device_error() == 0
    stl.indexer_topk(qd, wd, kd, sh.m, sh.topk, opts=stl.options(timeout_ms=100, debug_flags=1))
    assert stl.device_error() == -7  # SI_ERR_DEVICE_TIMEOUT
    assert stl.device_error() == 0   # the word is cleared by the read
    gi, gs = _gpu.run_bf16(sh, q, w, kc)
    _gpu.check_rows(sh, q, w, kc, gi, gs, np.arange(0, sh.S, 5))

"""End-to-end indexer step through the C ABI against the fp64 oracle: mean
recall >= 0.999, exact sets where a row sees <= k keys, every extra key within
1e-3 * max|row score| of the oracle's k-th score, and the structural
invariants (order, visibility, count, padding)."""

import numpy as np
import pytest
import torch

import synth
import streaming_top_lightning_b200 as stl
from tests import _gpu

pytestmark = pytest.mark.gpu


def test_tiny_all_rows():
    sh = synth.shape("tiny")
    q, w, kc = _gpu.inputs(sh)
    gi, gs = _gpu.run_bf16(sh, q, w, kc)
    rows = np.arange(sh.B * sh.S)
    res = _gpu.check_rows(sh, q, w, kc, gi, gs, rows)
    assert res["mean_recall"] == 1.0
    _gpu.structural(sh, gi, gs, rows)


SMALL = [
    # B, S, m, H, D, k
    (2, 100, 4, 8, 64, 16),     # S not a multiple of the 32-query tile, 2 batches
    (1, 256, 2, 16, 128, 32),
    (1, 520, 4, 32, 64, 40),
    (2, 1024, 4, 64, 128, 100),
    (1, 64, 8, 64, 128, 3),     # m=8: the first query tile sees no key at all
    (1, 1024, 1, 64, 128, 2048),  # k above every row's visible count
    (1, 3000, 4, 64, 64, 333),  # ragged T (750)
    (3, 200, 4, 16, 64, 7),
]


@pytest.mark.parametrize("B,S,m,H,D,k", SMALL)
def test_small_shapes(B, S, m, H, D, k):
    sh = synth.small(B, S, m, H, D, k, seed=S + H, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=S + H)
    gi, gs = _gpu.run_bf16(sh, q, w, kc)
    rows = np.arange(B * S)
    _gpu.check_rows(sh, q, w, kc, gi, gs, rows)
    _gpu.structural(sh, gi, gs, rows)


@pytest.mark.parametrize("S,H,D,k", [(2048, 64, 128, 1200), (4096, 8, 128, 512), (8704, 32, 64, 2048)])
def test_half_width_tiles(S, H, D, k):
    # top-k large enough for the half-width (N = 128) query tile: two (H=64),
    # four (H=32) or sixteen (H=8) queries per tile; sampled rows including
    # the last ones, which see more than k keys
    sh = synth.small(1, S, 4, H, D, k, seed=S + k, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=S + k)
    gi, gs = _gpu.run_bf16(sh, q, w, kc)
    rows = np.union1d(np.arange(0, S, 37), np.arange(S - 96, S))
    _gpu.check_rows(sh, q, w, kc, gi, gs, rows)
    _gpu.structural(sh, gi, gs, np.arange(S))


def test_topk_above_the_shape_limit_is_rejected():
    # with eight heads a 128-column query tile holds 16 queries; their pools
    # hold top-1056 candidates each at d_I = 128, not top-1057
    sh = synth.small(1, 512, 4, 8, 128, 1057, seed=1)
    q, w, kc = _gpu.inputs(sh, seed=1)
    with pytest.raises(stl.StreamIndexError) as e:
        _gpu.run_bf16(sh, q, w, kc)
    assert e.value.status == -3



@pytest.mark.parametrize("chunk", [128, 256, 1024])
def test_chunked_equals_unchunked(chunk):
    """Chunking changes only where the selection happens, not the fp32 scores,
    so the chunked partition-merge path returns exactly the same result, and
    both meet the acceptance rule against the oracle."""
    sh = synth.small(1, 8192, 4, 64, 128, 256, seed=3, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=3)
    gi0, gs0 = _gpu.run_bf16(sh, q, w, kc)
    gi1, gs1 = _gpu.run_bf16(sh, q, w, kc, opts=stl.options(key_chunk=chunk))
    assert torch.equal(gi0, gi1)
    assert torch.equal(gs0.view(torch.int32), gs1.view(torch.int32))
    rows = np.union1d(np.arange(0, sh.S, 29), np.arange(sh.S - 8, sh.S))
    _gpu.check_rows(sh, q, w, kc, gi1, gs1, rows)


@pytest.mark.parametrize("B,S,m,H,D,k", [(1, 2048, 4, 8, 64, 64), (2, 1024, 4, 64, 128, 100),
                                         (1, 4096, 4, 64, 128, 512), (1, 2048, 4, 64, 128, 1200)])
def test_rows_finished_in_fused_kernel_equal_merge(B, S, m, H, D, k):
    """Finishing the rows in the fused kernel's selection warps or in the
    merge kernel selects from the same fp32 scores under the same total
    order, so the two return exactly the same rows (sorted in registers for
    k <= 512, by the row-sort kernel above)."""
    sh = synth.small(B, S, m, H, D, k, seed=S + k, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=S + k)
    gi0, gs0 = _gpu.run_bf16(sh, q, w, kc, opts=stl.options(row_finish=2))
    gi1, gs1 = _gpu.run_bf16(sh, q, w, kc, opts=stl.options(row_finish=1))
    assert torch.equal(gi0, gi1)
    assert torch.equal(gs0.view(torch.int32), gs1.view(torch.int32))
    _gpu.structural(sh, gi1, gs1, np.arange(B * S))
    rows = np.union1d(np.arange(0, B * S, 13), [B * S - 1])
    _gpu.check_rows(sh, q, w, kc, gi1, gs1, rows)


@pytest.mark.parametrize("key_tile,strip_slots", [(128, 2), (256, 3), (512, 4), (1024, 2), (128, 4),
                                                  (32, 4), (64, 2), (64, 4), (32, 0)])
def test_strip_options_do_not_change_rows(key_tile, strip_slots):
    """The strip length and the number of strips in flight change only how the
    scores travel from the epilogue to the selection warps (and so the pool
    room the planner leaves), never which keys are selected: the rows are
    bit-identical to the default plan's."""
    sh = synth.small(1, 6144, 4, 64, 128, 300, seed=11, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=11)
    gi0, gs0 = _gpu.run_bf16(sh, q, w, kc)
    gi1, gs1 = _gpu.run_bf16(sh, q, w, kc,
                             opts=stl.options(key_tile=key_tile, strip_slots=strip_slots))
    assert torch.equal(gi0, gi1)
    assert torch.equal(gs0.view(torch.int32), gs1.view(torch.int32))
    rows = np.union1d(np.arange(0, sh.S, 31), [sh.S - 1])
    _gpu.check_rows(sh, q, w, kc, gi1, gs1, rows)


@pytest.mark.parametrize("key_tile", [32, 64])
@pytest.mark.parametrize("B,S,m,chunk", [(2, 1000, 4, 256), (1, 3003, 3, 0), (3, 712, 8, 128)])
def test_short_strips_ragged(key_tile, B, S, m, chunk):
    """Strips shorter than a key tile (each lane quadrant of a tile handed
    over on its own) on ragged shapes, with key chunks that end inside a
    query tile's reach and units that see no key: the rows equal the default
    plan's bit for bit and pass the oracle rule."""
    sh = synth.small(B, S, m, 64, 128, 100, seed=S + key_tile, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=S + key_tile)
    gi0, gs0 = _gpu.run_bf16(sh, q, w, kc, opts=stl.options(key_chunk=chunk))
    gi1, gs1 = _gpu.run_bf16(sh, q, w, kc, opts=stl.options(key_chunk=chunk, key_tile=key_tile))
    assert torch.equal(gi0, gi1)
    assert torch.equal(gs0.view(torch.int32), gs1.view(torch.int32))
    _gpu.structural(sh, gi1, gs1, np.arange(B * S))
    rows = np.union1d(np.arange(0, B * S, 7), [B * S - 1])
    _gpu.check_rows(sh, q, w, kc, gi1, gs1, rows)


def test_repeatable():
    sh = synth.small(1, 4096, 4, 64, 128, 512, seed=4, kc_kind="ar1")
    q, w, kc = _gpu.inputs(sh, seed=4)
    a = _gpu.run_bf16(sh, q, w, kc)
    b = _gpu.run_bf16(sh, q, w, kc)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1].view(torch.int32), b[1].view(torch.int32))


def test_v4flash_all_rows():
    # every one of the 16,384 rows against the oracle (about 20 s of fp64 on
    # the host cores), the visibility boundary rows among them
    sh = synth.shape("v4flash_s16k")
    q, w, kc = _gpu.inputs(sh)
    gi, gs = _gpu.run_bf16(sh, q, w, kc)
    rows = np.arange(sh.S)
    res = _gpu.check_rows(sh, q, w, kc, gi, gs, rows)
    _gpu.structural(sh, gi, gs, rows)
    _gpu.record("recall", {"workload": sh.name, "path": "bf16", "rows": int(rows.size),
                           "mean_recall": res["mean_recall"], "min_recall": res["min_recall"]})


CAP = 20 * 10 ** 9  # the peak-HBM cap of the large configurations, in bytes


def test_large_s64k_sampled_rows():
    sh = synth.shape("large_s64k")
    q, w, kc = _gpu.inputs(sh)
    gi, gs, peak = _gpu.run_bf16_counted(sh, q, w, kc)
    assert peak < CAP, peak
    rows = synth.sample_rows(sh)
    res = _gpu.check_rows(sh, q, w, kc, gi, gs, rows)
    _gpu.structural(sh, gi, gs, np.arange(0, sh.S, 61))
    _gpu.record("recall", {"workload": sh.name, "path": "bf16", "rows": int(rows.size),
                           "mean_recall": res["mean_recall"], "min_recall": res["min_recall"],
                           "peak_hbm_bytes": int(peak)})


def test_long_s256k_sampled_rows():
    # S = 262,144 (T = 65,536, top-2048): inclusive peak HBM (inputs, outputs
    # and the bounded scratch) under the cap, the sampled rows against the
    # oracle, and the structural invariants on a stride of rows
    sh = synth.shape("long_s256k")
    q = synth.gen_q(sh, 0, threads=16)
    w = synth.gen_w(sh, 0)
    kc = synth.gen_kc(sh, 0)
    gi, gs, peak = _gpu.run_bf16_counted(sh, q, w, kc)
    assert peak < CAP, peak
    rows = synth.sample_rows(sh)
    res = _gpu.check_rows(sh, q, w, kc, gi, gs, rows)
    _gpu.structural(sh, gi, gs, np.arange(0, sh.S, 509))
    _gpu.record("recall", {"workload": sh.name, "path": "bf16", "rows": int(rows.size),
                           "mean_recall": res["mean_recall"], "min_recall": res["min_recall"],
                           "peak_hbm_bytes": int(peak)})

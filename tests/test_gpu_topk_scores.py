"""Selection stage on given fp32 scores: bit-exact (indices and score bits)
against the oracle, including ties, +-0, +-inf, constant rows, rows with fewer
visible keys than k, ragged sizes and the chunked partition-merge path."""

import numpy as np
import pytest
import torch

import oracle
import synth
import streaming_top_lightning_b200 as stl

pytestmark = pytest.mark.gpu

CASES = [
    # B, S, T, m, k, key_chunk
    (1, 64, 16, 4, 8, 0),
    (2, 37, 13, 3, 5, 0),          # ragged: S not a multiple of the query tile
    (1, 1000, 700, 1, 64, 0),      # T not a multiple of 128
    (1, 2048, 512, 4, 64, 128),    # chunked: 4 chunks + merge
    (1, 4096, 1024, 4, 512, 256),
    (1, 2048, 2048, 1, 2048, 0),   # k at its maximum, many candidates per strip
    (1, 300, 5000, 1, 2048, 1024), # chunked with k at its maximum
    (3, 100, 300, 2, 300, 128),    # k > T
    (1, 5, 3, 1, 1, 0),            # k = 1, tiny
]


@pytest.mark.parametrize("kind", ["normal", "ties", "const", "inf"])
@pytest.mark.parametrize("B,S,T,m,k,chunk", CASES)
def test_bit_exact(kind, B, S, T, m, k, chunk):
    X = synth.gen_scores(B, S, T, seed=B * 7 + S, kind=kind)
    opts = stl.options(key_chunk=chunk) if chunk else None
    gi, gs = stl.topk_scores(torch.from_numpy(X).cuda(), m, k, opts=opts)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    oi, os_ = oracle.topk_scores(X, m, k)
    gi = gi.reshape(-1, k).cpu().numpy()
    gs = gs.reshape(-1, k).cpu().numpy()
    np.testing.assert_array_equal(gi, oi)
    np.testing.assert_array_equal(gs.view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("kind", ["normal", "ties", "inf"])
@pytest.mark.parametrize("B,S,T,m,k,chunk", [c for c in CASES if c[5] == 0])
def test_bit_exact_rows_finished_by_selection_warps(kind, B, S, T, m, k, chunk):
    """With one key chunk the selection warps can finish the rows themselves
    (exact select, in-register sort for k <= 512, row sort above): still
    bit-exact against the oracle."""
    X = synth.gen_scores(B, S, T, seed=B * 7 + S, kind=kind)
    gi, gs = stl.topk_scores(torch.from_numpy(X).cuda(), m, k, opts=stl.options(row_finish=1))
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    oi, os_ = oracle.topk_scores(X, m, k)
    np.testing.assert_array_equal(gi.reshape(-1, k).cpu().numpy(), oi)
    np.testing.assert_array_equal(gs.reshape(-1, k).cpu().numpy().view(np.uint32),
                                  os_.view(np.uint32))


def test_increasing_rows_worst_case():
    """Scores rising along j: every key beats the running k-th, so every strip
    overflows the candidate buffer."""
    B, S, T, m, k = 1, 64, 4096, 1, 1024
    X = np.broadcast_to(np.arange(T, dtype=np.float32), (B, S, T)).copy()
    X += np.random.default_rng(0).standard_normal((B, S, T)).astype(np.float32) * 1e-3
    gi, gs = stl.topk_scores(torch.from_numpy(X).cuda(), m, k)
    oi, os_ = oracle.topk_scores(X, m, k)
    np.testing.assert_array_equal(gi.reshape(-1, k).cpu().numpy(), oi)
    np.testing.assert_array_equal(gs.reshape(-1, k).cpu().numpy().view(np.uint32), os_.view(np.uint32))


def test_chunk_sizes_agree():
    X = synth.gen_scores(1, 512, 3000, seed=5, kind="ties")
    ref = None
    for chunk in [0, 128, 384, 1024, 2048]:
        opts = stl.options(key_chunk=chunk) if chunk else None
        gi, gs = stl.topk_scores(torch.from_numpy(X).cuda(), 1, 700, opts=opts)
        cur = (gi.cpu().numpy(), gs.cpu().numpy().view(np.uint32))
        if ref is None:
            ref = cur
        np.testing.assert_array_equal(cur[0], ref[0])
        np.testing.assert_array_equal(cur[1], ref[1])


def test_small_scratch_budget_many_blocks():
    """A 1 MiB scratch budget forces many query blocks; the result is unchanged."""
    X = synth.gen_scores(2, 256, 2048, seed=9, kind="normal")
    opts = stl.options(key_chunk=256, scratch_mb=1)
    gi, gs = stl.topk_scores(torch.from_numpy(X).cuda(), 2, 256, opts=opts)
    oi, os_ = oracle.topk_scores(X, 2, 256)
    np.testing.assert_array_equal(gi.reshape(-1, 256).cpu().numpy(), oi)
    np.testing.assert_array_equal(gs.reshape(-1, 256).cpu().numpy().view(np.uint32), os_.view(np.uint32))


# The fused kernel's own selection plans: the test entry selects with the
# queries per tile, strip length, pool room and partial-list length the
# indexer plans for that shape (si_options.plan_heads / plan_dim / plan_fp8),
# so the pruning and radix-select steps the product runs are checked bit for
# bit, not only through the end-to-end tolerance rule.
PLANS = [
    # H_I, d_I, fp8, k, S, T, m, key_chunk
    (64, 128, 0, 512, 6000, 4096, 1, 0),     # V4-Flash step: 4 queries, 512-key strips
    (64, 128, 0, 2048, 9000, 8192, 1, 0),    # top-2048 steps: half-width tile, 2 queries
    (64, 128, 0, 512, 4000, 8192, 1, 1024),  # the sweep's chunked cells
    (64, 128, 0, 1024, 4000, 8192, 1, 2048),
    (8, 64, 0, 64, 2048, 512, 4, 0),         # tiny step: 32 queries, 128-key strips
    (64, 128, 1, 512, 6000, 4096, 1, 0),     # FP8 plan of the V4-Flash step
    (64, 128, 1, 2048, 9000, 8192, 1, 0),
]


@pytest.mark.parametrize("kind", ["normal", "ties", "inf"])
@pytest.mark.parametrize("H,D,fp8,k,S,T,m,chunk", PLANS)
def test_bit_exact_on_the_indexer_plans(kind, H, D, fp8, k, S, T, m, chunk):
    X = synth.gen_scores(1, S, T, seed=S + k + H, kind=kind)
    opts = stl.options(key_chunk=chunk, plan_heads=H, plan_dim=D, plan_fp8=fp8)
    gi, gs = stl.topk_scores(torch.from_numpy(X).cuda(), m, k, opts=opts)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    oi, os_ = oracle.topk_scores(X, m, k)
    np.testing.assert_array_equal(gi.reshape(-1, k).cpu().numpy(), oi)
    np.testing.assert_array_equal(gs.reshape(-1, k).cpu().numpy().view(np.uint32),
                                  os_.view(np.uint32))


@pytest.mark.parametrize("kind", ["normal", "ties"])
@pytest.mark.parametrize("fp8,k,key_tile", [(0, 512, 32), (0, 512, 64), (1, 2048, 64),
                                            (0, 2048, 32)])
def test_bit_exact_on_short_strip_plans(kind, fp8, k, key_tile):
    """Plans with strips of 32 or 64 keys (a quarter or half of a key tile per
    hand-over): the selection steps on those strips are bit-exact too."""
    S, T = 3000, 4096
    X = synth.gen_scores(1, S, T, seed=k + key_tile, kind=kind)
    opts = stl.options(plan_heads=64, plan_dim=128, plan_fp8=fp8, key_tile=key_tile)
    gi, gs = stl.topk_scores(torch.from_numpy(X).cuda(), 1, k, opts=opts)
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    oi, os_ = oracle.topk_scores(X, 1, k)
    np.testing.assert_array_equal(gi.reshape(-1, k).cpu().numpy(), oi)
    np.testing.assert_array_equal(gs.reshape(-1, k).cpu().numpy().view(np.uint32),
                                  os_.view(np.uint32))


@pytest.mark.parametrize("H,D,fp8,k", [(64, 128, 0, 512), (64, 128, 0, 2048)])
def test_increasing_rows_on_the_indexer_plans(H, D, fp8, k):
    """Scores rising along j on the product's plans: every key beats the
    running k-th, every strip overflows the pools, every prune is exercised."""
    S = T = 8192
    X = np.broadcast_to(np.arange(T, dtype=np.float32), (1, S, T)).copy()
    X += np.random.default_rng(1).standard_normal((1, S, T)).astype(np.float32) * 1e-3
    opts = stl.options(plan_heads=H, plan_dim=D, plan_fp8=fp8)
    gi, gs = stl.topk_scores(torch.from_numpy(X).cuda(), 1, k, opts=opts)
    oi, os_ = oracle.topk_scores(X, 1, k)
    np.testing.assert_array_equal(gi.reshape(-1, k).cpu().numpy(), oi)
    np.testing.assert_array_equal(gs.reshape(-1, k).cpu().numpy().view(np.uint32),
                                  os_.view(np.uint32))

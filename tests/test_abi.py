"""The C-ABI library: builds, loads, exports every symbol include/*.h declares,
and rejects bad arguments on the host before any CUDA work."""

import ctypes
import glob
import os
import re

import pytest

from streaming_top_lightning_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(si_[a-z0-9_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared, "no declarations found"
    assert declared == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    assert lib.si_status_string(0) == b"ok"
    for code in range(-1, -10, -1):
        assert lib.si_status_string(code) != b"unknown status"
    assert lib.si_version() >= 100


def _ws(lib, B, S, H, D, m, k, opts=None):
    n = ctypes.c_size_t(0)
    rc = lib.si_indexer_topk_workspace_size(B, S, H, D, m, k,
                                            ctypes.byref(opts) if opts else None, ctypes.byref(n))
    return rc, n.value


def test_workspace_size_and_validation(lib):
    rc, n = _ws(lib, 1, 16384, 64, 128, 4, 512)
    assert rc == 0 and n >= 4          # single chunk: just the unit counter
    opts = _lib.SiOptions(1024, 64, 0, 0, 0)
    rc, n2 = _ws(lib, 1, 16384, 64, 128, 4, 512, opts)
    assert rc == 0 and 64 << 20 >= n2 - 256 > 0  # bounded by the scratch budget
    big = _lib.SiOptions(1024, 64, 0, 0, 0)
    rc, n3 = _ws(lib, 1, 262144, 64, 128, 4, 2048, big)
    assert rc == 0 and n3 - 256 <= 64 << 20      # independent of S
    assert _ws(lib, 1, 16383, 64, 128, 4, 512)[0] == -2   # S % m
    assert _ws(lib, 1, 16384, 48, 128, 4, 512)[0] == -2   # H_I
    assert _ws(lib, 1, 16384, 64, 96, 4, 512)[0] == -2    # d_I
    assert _ws(lib, 1, 16384, 64, 128, 4, 0)[0] == -3     # topk
    assert _ws(lib, 1, 16384, 64, 128, 4, 2049)[0] == -3
    assert _ws(lib, 1, 16384, 64, 128, 4, 512, _lib.SiOptions(100, 0, 0, 0, 0))[0] == -8


def test_noalloc_size_check_comes_first(lib):
    # one query tile over B=1024 batches with top-2048 needs about 86 MB of
    # partial-list scratch (1024 batches x 4 queries x 2624 candidates x 8
    # bytes), more than the fixed 64 MiB array: refused before any pointer is
    # looked at (the tensors here are NULL, so a problem that fits is then
    # refused for its NULL pointers, and nothing can reach a launch)
    P = ctypes.c_void_p
    assert lib.si_indexer_topk_noalloc(None, None, None, 1024, 8192, 64, 128, 4, 2048,
                                       None, None, None) == -5
    assert lib.si_indexer_topk_noalloc(None, None, None, 1, 8192, 64, 128, 4, 2048,
                                       None, None, None) == -1
    assert lib.si_indexer_topk_noalloc(P(0x1000), P(0x1000), P(0x1000), 1, 8191, 64, 128, 4,
                                       512, P(0x1000), P(0x1000), None) == -2


def test_row_finish_option(lib):
    # rows finished in the fused kernel need no partial lists: the workspace
    # is the unit counter and one query tile's weights (256 columns of fp32,
    # for a last tile that S leaves partial), whatever the problem size
    for B, S, H, D, k in [(1, 262144, 64, 128, 2048), (64, 65536, 8, 64, 64)]:
        o = _lib.SiOptions(0, 0, 0, 0, 0)
        o.row_finish = 1
        rc, n = _ws(lib, B, S, H, D, 4, k, o)
        assert rc == 0 and 0 < n <= 256 + 1024
        o.row_finish = 2
        rc, n2 = _ws(lib, B, S, H, D, 4, k, o)
        assert rc == 0 and n2 > 256 + 1024
    o = _lib.SiOptions(0, 0, 0, 0, 0)
    o.row_finish = 3
    assert _ws(lib, 1, 16384, 64, 128, 4, 512, o)[0] == -8


def test_strip_options_validated(lib):
    # strips of 32 or 64 keys: a tile's 128/key_tile strips take whole slot groups
    for kt, ss, ok in [(0, 0, True), (128, 2, True), (1024, 4, True), (100, 0, False),
                       (2048, 0, False), (0, 1, False), (0, 5, False), (256, -1, False),
                       (32, 0, True), (32, 4, True), (32, 2, False), (32, 3, False),
                       (64, 0, True), (64, 2, True), (64, 4, True), (64, 3, False),
                       (16, 0, False), (96, 0, False)]:
        o = _lib.SiOptions(0, 0, 0, 0, 0)
        o.key_tile = kt
        o.strip_slots = ss
        rc, _ = _ws(lib, 1, 16384, 64, 128, 4, 512, o)
        assert (rc == 0) == ok, (kt, ss, rc)
        if not ok:
            assert rc == -8


def _plan(lib, B, S, H, D, m, k, fp8=0, opts=None):
    info = _lib.SiPlanInfo()
    rc = lib.si_indexer_topk_plan(B, S, H, D, m, k, fp8, ctypes.byref(opts) if opts else None,
                                  ctypes.byref(info))
    return rc, info


def test_plan_query(lib):
    # host-only: on a machine without a GPU the plan is made for the sm_100
    # limits, so these hold on the CPU and on a B200 alike
    rc, p = _plan(lib, 1, 16384, 64, 128, 4, 512)
    assert rc == 0
    assert (p.queries_per_tile, p.mma_n, p.key_chunks, p.query_blocks, p.launches) == (4, 256, 1,
                                                                                        1, 2)
    assert p.pool_keys >= 512 + 64 and p.partial_len == 704
    assert p.smem_bytes <= 227 * 1024
    rc, n = _ws(lib, 1, 16384, 64, 128, 4, 512)
    assert rc == 0 and p.workspace_bytes <= n
    # top-2048 keeps the full-width tile (its pools still hold 1.5K keys);
    # its 2624-key lists at S = 262,144 need eleven query blocks
    rc, p = _plan(lib, 1, 262144, 64, 128, 4, 2048)
    assert rc == 0 and (p.queries_per_tile, p.mma_n, p.query_blocks, p.launches) == (4, 256, 11,
                                                                                      22)
    assert p.pool_keys >= 3 * 2048 // 2
    # chunked: score + merge per block and the row sort above k = 512
    o = _lib.SiOptions(1024, 0, 0, 0, 0)
    rc, p = _plan(lib, 1, 32768, 64, 128, 4, 1024, opts=o)
    assert rc == 0 and (p.key_chunks, p.query_blocks, p.launches) == (8, 6, 13)
    # errors: topk above the shape's limit, a strip above the tile's limit,
    # bad dims and a bad fp8 flag
    assert _plan(lib, 1, 4096, 8, 128, 4, 1056)[0] == 0
    assert _plan(lib, 1, 4096, 8, 128, 4, 1057)[0] == -3
    o = _lib.SiOptions(0, 0, 0, 0, 0)
    o.key_tile = 1024
    assert _plan(lib, 1, 4096, 8, 128, 4, 64, opts=o)[0] == -8   # 32 queries: strips <= 128
    assert _plan(lib, 1, 4096, 64, 128, 4, 64, opts=o)[0] == 0
    assert _plan(lib, 1, 4095, 64, 128, 4, 64)[0] == -2
    assert _plan(lib, 1, 4096, 64, 128, 4, 64, fp8=2)[0] == -8
    assert lib.si_indexer_topk_plan(1, 4096, 64, 128, 4, 64, 0, None, None) == -1


def test_plan_short_strips(lib):
    """Strips of 32 or 64 keys keep the tile and its pools; the strip ring
    holds whole groups of a tile's 128/key_tile strips (4 for 32; 2 or 4 for
    64), and the smaller strips leave the pools no less room."""
    rc, p0 = _plan(lib, 1, 32768, 64, 128, 4, 512)
    assert rc == 0
    for kt, ss, want_slots in [(32, 0, 4), (32, 4, 4), (64, 0, 4), (64, 2, 2)]:
        o = _lib.SiOptions(0, 0, 0, 0, 0)
        o.key_tile, o.strip_slots = kt, ss
        for fp8 in (0, 1):
            rc, p = _plan(lib, 1, 32768, 64, 128, 4, 512, fp8=fp8, opts=o)
            assert rc == 0, (kt, ss, fp8)
            assert (p.key_tile, p.strip_slots, p.mma_n) == (kt, want_slots, 256), (kt, ss, fp8)
            assert p.pool_keys >= p0.pool_keys and p.smem_bytes <= 227 * 1024
            assert p.launches == p0.launches


def test_plan_hint_options_validated(lib):
    for heads, dim, fp8, ok in [(0, 0, 0, True), (64, 128, 0, True), (8, 64, 1, True),
                                (48, 128, 0, False), (64, 96, 0, False), (64, 128, 2, False)]:
        o = _lib.SiOptions(0, 0, 0, 0, 0)
        o.plan_heads, o.plan_dim, o.plan_fp8 = heads, dim, fp8
        rc, _ = _ws(lib, 1, 16384, 64, 128, 4, 512, o)
        assert (rc == 0) == ok, (heads, dim, fp8, rc)


def test_decode_pivot_attention_argument_errors(lib):
    """The host-side checks of the decode, query-group and attention entry
    points (nothing is launched: every case fails before any device access)."""
    Z = ctypes.c_size_t
    n = Z(0)
    # decode: bad position, bad m, bad topk
    assert lib.si_indexer_decode_workspace_size(1, 1, -1, 16, 64, 128, 4, 8, None,
                                                ctypes.byref(n)) == -2
    assert lib.si_indexer_decode_workspace_size(1, 1, 0, 16, 64, 128, 0, 8, None,
                                                ctypes.byref(n)) == -2
    assert lib.si_indexer_decode_workspace_size(1, 1, 0, 16, 64, 128, 4, 0, None,
                                                ctypes.byref(n)) == -3
    assert lib.si_indexer_decode_workspace_size(1, 2, 9, 16, 64, 128, 4, 8, None,
                                                ctypes.byref(n)) == 0 and n.value > 0
    # query-group scan: S not a multiple of G, C below topk, C above 2048
    for G, C, rc in [(3, 128, -8), (16, 32, -8), (16, 4096, -8), (16, 128, 0)]:
        assert lib.si_indexer_pivot_workspace_size(1, 512, 64, 128, 4, 64, G, C, None,
                                                   ctypes.byref(n)) == rc, (G, C)
    # attention: NULL, heads other than 128, topk, a non-finite scale (fake device
    # pointers: each call fails before using them)
    fake = ctypes.c_void_p(256)
    assert lib.si_sparse_attention(None, fake, fake, fake, 1, 2, 16, 128, 128, 4, 1.0, fake,
                                   None, None) == -1
    assert lib.si_sparse_attention(fake, fake, fake, fake, 1, 2, 16, 64, 128, 4, 1.0, fake,
                                   None, None) == -2
    assert lib.si_sparse_attention(fake, fake, fake, fake, 1, 2, 16, 128, 128, 0, 1.0, fake,
                                   None, None) == -3
    for bad in (float("nan"), float("inf"), -0.5):
        assert lib.si_sparse_attention(fake, fake, fake, fake, 1, 2, 16, 128, 128, 4, bad, fake,
                                       None, None) == -8


# The largest top-k per (fp8, H_I, d_I) that the header documents; every other
# shape takes top-2048.
DOCUMENTED_MAX_TOPK = {(0, 8, 128): 1056, (0, 8, 64): 1312, (1, 8, 128): 1280, (1, 8, 64): 1408}


@pytest.mark.parametrize("fp8", [0, 1])
@pytest.mark.parametrize("H", [8, 16, 32, 64])
@pytest.mark.parametrize("D", [64, 128])
def test_plan_limits_and_invariants(lib, fp8, H, D):
    """Host-only planner sweep: the documented largest top-k holds exactly,
    and every plan below it fits the 227 KB of shared memory, gives each
    query a pool of at least K + 64 keys, a tile of QT = N / H_I queries, a
    strip no longer than the tile allows and a strip ring that holds whole
    groups of a tile's strips."""
    kmax = DOCUMENTED_MAX_TOPK.get((fp8, H, D), 2048)
    assert _plan(lib, 1, 16384, H, D, 4, kmax, fp8=fp8)[0] == 0
    if kmax < 2048:
        assert _plan(lib, 1, 16384, H, D, 4, kmax + 1, fp8=fp8)[0] == -3
    for k in sorted({1, 2, 31, 64, 100, 128, 255, 512, 777, 1024, kmax // 2, kmax}):
        if k > kmax:
            continue
        for kt, ss in [(0, 0), (32, 0), (64, 2), (128, 0), (512, 3)]:
            o = _lib.SiOptions(0, 0, 0, 0, 0)
            o.key_tile, o.strip_slots = kt, ss
            rc, p = _plan(lib, 1, 16384, H, D, 4, k, fp8=fp8, opts=o)
            if rc != 0:
                # only a strip longer than this tile allows, or pools that no
                # longer fit beside a requested strip ring, may be refused
                assert rc in (-8, -3) and kt >= 512, (k, kt, ss, rc)
                continue
            assert p.smem_bytes <= 227 * 1024, (k, kt, p.smem_bytes)
            assert p.pool_keys >= ((k + 64 + 31) // 32) * 32, (k, kt, p.pool_keys)
            assert p.mma_n in (128, 256) and p.queries_per_tile * H == p.mma_n
            assert 2 <= p.strip_slots <= 4 and (ss == 0 or p.strip_slots == ss)
            assert kt == 0 or p.key_tile == kt
            if p.key_tile < 128:
                assert p.strip_slots % (128 // p.key_tile) == 0
            assert p.partial_len >= k and p.partial_len % 32 == 0

"""fp64 CPU oracle for the CSA lightning-indexer top-k step (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never does, and the two share no code: the only thing both use is the
seeded input generator in ``synth``.

The arithmetic lives in ``oracle.c`` (plain loops, fp64, qsort); this module
compiles it with gcc on first use and marshals numpy arrays to it.  The C
file's header states the definition it follows ("StreamIndex: Memory-Bounded
Compressed Sparse Attention via Streaming Top-k", Abstract) and the readings it
takes where that text is silent.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2, OpenMP, no fast-math, no
    FMA contraction, so every fp64 operation rounds once as written)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def declare(lib):
    """Declare the argument types of every oracle symbol on a loaded CDLL
    (the built oracle, or a test's modified copy of it)."""
    P = ctypes.c_void_p
    I, L = ctypes.c_int, ctypes.c_int64
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = I
    lib.oracle_visible.argtypes = [I, I, I]
    lib.oracle_visible.restype = I
    lib.oracle_indexer_topk.argtypes = [P, P, P, I, I, I, I, I, I, P, I, P, P]
    lib.oracle_indexer_topk.restype = I
    lib.oracle_indexer_topk_rows.argtypes = [P, P, P, I, I, I, I, I, I, P, I, P, P]
    lib.oracle_indexer_topk_rows.restype = I
    lib.oracle_indexer_topk_rows_absmax.argtypes = [P, P, P, I, I, I, I, I, I, P, I, P, P, P]
    lib.oracle_indexer_topk_rows_absmax.restype = I
    lib.oracle_score_keys_rows.argtypes = [P, P, P, I, I, I, I, P, I, P, I, P]
    lib.oracle_score_keys_rows.restype = None
    lib.oracle_row_absmax_rows.argtypes = [P, P, P, I, I, I, I, P, I, P]
    lib.oracle_row_absmax_rows.restype = None
    lib.oracle_topk_scores.argtypes = [P, I, I, I, I, I, P, I, P, P]
    lib.oracle_topk_scores.restype = I
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_quantize_e4m3_rows.argtypes = [P, L, I, P, P]
    lib.oracle_quantize_e4m3_rows.restype = None
    lib.oracle_indexer_topk_fp8_rows.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, I, P, P]
    lib.oracle_indexer_topk_fp8_rows.restype = I
    lib.oracle_score_keys_fp8_rows.argtypes = [P, P, P, P, P, I, I, I, I, P, I, P, I, P]
    lib.oracle_score_keys_fp8_rows.restype = None
    lib.oracle_mx_scale_byte.argtypes = [ctypes.c_double]
    lib.oracle_mx_scale_byte.restype = ctypes.c_uint8
    lib.oracle_quantize_mxfp8_rows.argtypes = [P, L, I, P, P]
    lib.oracle_quantize_mxfp8_rows.restype = I
    lib.oracle_indexer_topk_mxfp8_rows.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, I, P, P]
    lib.oracle_indexer_topk_mxfp8_rows.restype = I
    lib.oracle_sparse_attention_rows.argtypes = [P, P, P, P, P, I, I, I, I, I, I, ctypes.c_double,
                                                 P, P]
    lib.oracle_sparse_attention_rows.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = declare(ctypes.CDLL(build()))
    return _lib


class _Bound:
    """The module's functions bound to another compiled copy of oracle.c."""

    def __init__(self, path: str):
        self._cdll = declare(ctypes.CDLL(path))

    def __getattr__(self, name):
        fn = _API[name]
        return lambda *a, **kw: fn(*a, lib=self._cdll, **kw)


def load_copy(path: str) -> "_Bound":
    """The oracle API on a separately compiled copy of oracle.c (used by the
    tests that plant mistakes in a copy and check that the pins catch them)."""
    return _Bound(path)


def _use(lib):
    return lib if lib is not None else _load()


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def threads(lib=None) -> int:
    """OpenMP threads the oracle's row loops use."""
    return _use(lib).oracle_threads()


def visible(t: int, T: int, m: int, lib=None) -> int:
    """Number of compressed keys visible to query t (keys j with (j+1)m-1 <= t)."""
    return _use(lib).oracle_visible(int(t), int(T), int(m))


def indexer_topk(q, w, kc, m: int, k: int, rows=None, lib=None):
    """Oracle top-k from full tensors.

    q [B,S,H,D] uint16 (bf16 bits), w [B,S,H] float32, kc [B,T,D] uint16.
    rows: flat positions b*S+t to evaluate (default: all).
    Returns (idx [n,k] int32, score [n,k] float64).
    """
    q, w, kc = _c(q, np.uint16), _c(w, np.float32), _c(kc, np.uint16)
    B, S, H, D = q.shape
    rows = _c(np.arange(B * S) if rows is None else rows, np.int64)
    n = rows.size
    idx = np.empty((n, k), dtype=np.int32)
    sc = np.empty((n, k), dtype=np.float64)
    rc = _use(lib).oracle_indexer_topk(_p(q), _p(w), _p(kc), B, S, H, D, m, k, _p(rows), n,
              _p(idx), _p(sc))
    if rc != 0:
        raise ValueError("oracle_indexer_topk: bad arguments")
    return idx, sc


def indexer_topk_rows(q_rows, w_rows, kc, S: int, m: int, k: int, rows, lib=None):
    """Oracle top-k given only the listed queries' rows of q and w
    (q_rows [n,H,D], w_rows [n,H]); rows are their flat positions b*S+t."""
    q_rows, w_rows, kc = _c(q_rows, np.uint16), _c(w_rows, np.float32), _c(kc, np.uint16)
    rows = _c(rows, np.int64)
    n, H, D = q_rows.shape
    B = kc.shape[0]
    idx = np.empty((n, k), dtype=np.int32)
    sc = np.empty((n, k), dtype=np.float64)
    rc = _use(lib).oracle_indexer_topk_rows(_p(q_rows), _p(w_rows), _p(kc), B, S, H, D, m, k,
              _p(rows), n, _p(idx), _p(sc))
    if rc != 0:
        raise ValueError("oracle_indexer_topk_rows: bad arguments")
    return idx, sc


def indexer_topk_rows_absmax(q_rows, w_rows, kc, S: int, m: int, k: int, rows, lib=None):
    """``indexer_topk_rows`` plus each row's max |score| over its visible keys."""
    q_rows, w_rows, kc = _c(q_rows, np.uint16), _c(w_rows, np.float32), _c(kc, np.uint16)
    rows = _c(rows, np.int64)
    n, H, D = q_rows.shape
    B = kc.shape[0]
    idx = np.empty((n, k), dtype=np.int32)
    sc = np.empty((n, k), dtype=np.float64)
    amax = np.empty(n, dtype=np.float64)
    rc = _use(lib).oracle_indexer_topk_rows_absmax(_p(q_rows), _p(w_rows), _p(kc), B, S, H, D, m,
              k, _p(rows), n, _p(idx), _p(sc), _p(amax))
    if rc != 0:
        raise ValueError("oracle_indexer_topk_rows_absmax: bad arguments")
    return idx, sc, amax


def score_keys_rows(q_rows, w_rows, kc, S: int, m: int, rows, js, lib=None):
    """fp64 scores of keys js[i, :] for the listed queries; keys a query cannot
    see (j < 0 or j >= V_t) give nan."""
    q_rows, w_rows, kc = _c(q_rows, np.uint16), _c(w_rows, np.float32), _c(kc, np.uint16)
    rows, js = _c(rows, np.int64), _c(js, np.int32)
    n, H, D = q_rows.shape
    out = np.full(js.shape, np.nan, dtype=np.float64)
    _use(lib).oracle_score_keys_rows(_p(q_rows), _p(w_rows), _p(kc), S, H, D, m, _p(rows), n,
         _p(js), js.shape[1], _p(out))
    return out


def row_absmax_rows(q_rows, w_rows, kc, S: int, m: int, rows, lib=None):
    """max over visible keys of |score| for each listed query."""
    q_rows, w_rows, kc = _c(q_rows, np.uint16), _c(w_rows, np.float32), _c(kc, np.uint16)
    rows = _c(rows, np.int64)
    n, H, D = q_rows.shape
    out = np.empty(n, dtype=np.float64)
    _use(lib).oracle_row_absmax_rows(_p(q_rows), _p(w_rows), _p(kc), S, H, D, m, _p(rows), n,
         _p(out))
    return out


def decode_rows(B: int, S_q: int, t0: int, T: int, m: int, lib=None):
    """Rows of the row functions above that stand for the decode queries:
    query i of batch b, at sequence position t0 + i, sees V = min(T,
    floor((t0+i+1)/m)) keys, which is what the row at position min(t0+i,
    m*T-1) of a sequence of m*T tokens (T keys) sees.  Returns (S, rows) to
    pass as the row functions' S and rows, with kc [B,T,D].  (lib: unused;
    present so every function of the module takes it.)"""
    S = m * T
    pos = np.minimum(t0 + np.arange(S_q, dtype=np.int64), S - 1)
    rows = (np.arange(B, dtype=np.int64)[:, None] * S + pos[None, :]).reshape(-1)
    return S, rows


def indexer_decode(q, w, kc, t0: int, m: int, k: int, lib=None):
    """Decode oracle: q [B,S_q,H,D] bf16 bits and w [B,S_q,H] at positions
    t0 .. t0+S_q-1 against kc [B,T,D].  Returns (idx, score, absmax) with one
    row per query, batch-major."""
    q, w = _c(q, np.uint16), _c(w, np.float32)
    B, S_q, H, D = q.shape
    S, rows = decode_rows(B, S_q, t0, kc.shape[1], m)
    return indexer_topk_rows_absmax(q.reshape(B * S_q, H, D), w.reshape(B * S_q, H), kc, S, m, k,
                                    rows, lib=lib)


def sparse_attention_rows(qa_rows, ka, va, idx_rows, batch, scale: float, lib=None):
    """Multi-query attention of each listed query row over its listed entries
    (see oracle_sparse_attention_rows): qa_rows [n,H,D] bf16 bits, ka and va
    [B,T,D] bf16 bits, idx_rows [n,k] int32, batch [n] (each row's batch).
    Returns (out [n,H,D], absw [n,H,D]) in fp64."""
    qa_rows, ka, va = _c(qa_rows, np.uint16), _c(ka, np.uint16), _c(va, np.uint16)
    idx_rows, batch = _c(idx_rows, np.int32), _c(batch, np.int64)
    n, H, D = qa_rows.shape
    B, T = ka.shape[0], ka.shape[1]
    k = idx_rows.shape[1]
    out = np.empty((n, H, D), dtype=np.float64)
    absw = np.empty((n, H, D), dtype=np.float64)
    rc = _use(lib).oracle_sparse_attention_rows(_p(qa_rows), _p(ka), _p(va), _p(idx_rows),
                                                _p(batch), n, B, T, H, D, k, float(scale),
                                                _p(out), _p(absw))
    if rc != 0:
        raise ValueError("oracle_sparse_attention_rows: bad arguments")
    return out, absw


def pivot_rows(q, w, kc, m: int, k: int, G: int, C: int, rows, lib=None):
    """Query-group candidate scan (the PIVOT news page: nearby queries share one
    prefix scan).  Reading used: the queries of a batch form groups of G
    consecutive positions; the group's last position (which sees the most keys)
    scans its visible keys once and keeps its C best by the exact score
    (score descending, index ascending); each query of the group then ranks
    only those candidates it can see, by its own exact score, and keeps its k
    best (padding -1 / -inf).

    q [B,S,H,D] bf16 bits, w [B,S,H], kc [B,T,D]; rows: flat rows b*S + t to
    evaluate.  Returns (idx [n,k], score [n,k] fp64, absmax [n]: the largest
    |score| over the row's visible candidates)."""
    q, w, kc = _c(q, np.uint16), _c(w, np.float32), _c(kc, np.uint16)
    B, S, H, D = q.shape
    T = kc.shape[1]
    rows = np.asarray(rows, dtype=np.int64)
    reps = np.unique((rows // S) * S + np.minimum((rows % S) // G * G + G - 1, S - 1))
    qf, wf = q.reshape(B * S, H, D), w.reshape(B * S, H)
    rep_idx, _ = indexer_topk_rows(qf[reps], wf[reps], kc, S, m, C, reps, lib=lib)
    cand = {int(r): c[c >= 0] for r, c in zip(reps, rep_idx)}
    out_i = np.full((rows.size, k), -1, dtype=np.int32)
    out_s = np.full((rows.size, k), -np.inf)
    amax = np.zeros(rows.size)
    for n, r in enumerate(rows):
        b, t = divmod(int(r), S)
        rep = b * S + min(t // G * G + G - 1, S - 1)
        V = min(T, (t + 1) // m)
        js = np.sort(cand[rep][cand[rep] < V]).astype(np.int32)
        if js.size == 0:
            continue
        sc = score_keys_rows(qf[r:r + 1], wf[r:r + 1], kc, S, m, np.array([r]), js[None, :],
                             lib=lib)[0]
        order = np.lexsort((js, -sc))[:k]
        out_i[n, :order.size] = js[order]
        out_s[n, :order.size] = sc[order]
        amax[n] = np.max(np.abs(sc))
    return out_i, out_s, amax


def topk_scores(X, m: int, k: int, rows=None, lib=None):
    """Selection alone on given fp32 scores X [B,S,T].
    Returns (idx [n,k] int32, score [n,k] float32 carrying the input bit patterns)."""
    X = _c(X, np.float32)
    B, S, T = X.shape
    rows = _c(np.arange(B * S) if rows is None else rows, np.int64)
    n = rows.size
    idx = np.empty((n, k), dtype=np.int32)
    sc = np.empty((n, k), dtype=np.float32)
    rc = _use(lib).oracle_topk_scores(_p(X), B, S, T, m, k, _p(rows), n, _p(idx), _p(sc))
    if rc != 0:
        raise ValueError("oracle_topk_scores: bad arguments")
    return idx, sc


def e4m3_decode(code: int, lib=None) -> float:
    return _use(lib).oracle_e4m3_decode(int(code))


def e4m3_encode(y: float, lib=None) -> int:
    return _use(lib).oracle_e4m3_encode(float(y))


def quantize_e4m3_rows(x, lib=None):
    """x [..., cols] uint16 bf16 bits -> (codes uint8 [..., cols], scale fp32 [...])."""
    x = _c(x, np.uint16)
    shp = x.shape
    x2 = x.reshape(-1, shp[-1])
    codes = np.empty(x2.shape, dtype=np.uint8)
    scale = np.empty(x2.shape[0], dtype=np.float32)
    _use(lib).oracle_quantize_e4m3_rows(_p(x2), x2.shape[0], x2.shape[1], _p(codes), _p(scale))
    return codes.reshape(shp), scale.reshape(shp[:-1])


def indexer_topk_fp8_rows(q8_rows, sq_rows, w_rows, k8, s_k, S: int, m: int, k: int, rows,
                          lib=None):
    """Oracle top-k of the FP8 score (codes decoded exactly, scales applied in fp64).

    q8_rows [n,H,D] uint8, sq_rows [n,H] fp32, w_rows [n,H] fp32 for the listed
    queries; k8 [B,T,D] uint8, s_k [B,T] fp32."""
    q8_rows, sq_rows = _c(q8_rows, np.uint8), _c(sq_rows, np.float32)
    w_rows = _c(w_rows, np.float32)
    k8, s_k, rows = _c(k8, np.uint8), _c(s_k, np.float32), _c(rows, np.int64)
    n, H, D = q8_rows.shape
    B = k8.shape[0]
    idx = np.empty((n, k), dtype=np.int32)
    sc = np.empty((n, k), dtype=np.float64)
    rc = _use(lib).oracle_indexer_topk_fp8_rows(_p(q8_rows), _p(sq_rows), _p(w_rows), _p(k8),
              _p(s_k), B, S, H, D, m, k, _p(rows), n, _p(idx), _p(sc))
    if rc != 0:
        raise ValueError("oracle_indexer_topk_fp8_rows: bad arguments")
    return idx, sc


def score_keys_fp8_rows(q8_rows, sq_rows, w_rows, k8, s_k, S: int, m: int, rows, js, lib=None):
    """FP8 scores of keys js[i, :] for the listed queries; keys a query cannot
    see give nan."""
    q8_rows, sq_rows = _c(q8_rows, np.uint8), _c(sq_rows, np.float32)
    w_rows = _c(w_rows, np.float32)
    k8, s_k, rows, js = _c(k8, np.uint8), _c(s_k, np.float32), _c(rows, np.int64), _c(js, np.int32)
    n, H, D = q8_rows.shape
    out = np.full(js.shape, np.nan, dtype=np.float64)
    _use(lib).oracle_score_keys_fp8_rows(_p(q8_rows), _p(sq_rows), _p(w_rows), _p(k8), _p(s_k), S,
         H, D, m, _p(rows), n, _p(js), js.shape[1], _p(out))
    return out


def mx_scale_byte(amax: float, lib=None) -> int:
    """E8M0 byte of an MX block whose largest magnitude is amax."""
    return _use(lib).oracle_mx_scale_byte(float(amax))


def quantize_mxfp8_rows(x, lib=None):
    """x [..., cols] uint16 bf16 bits, cols a multiple of 32 -> (codes uint8
    [..., cols], scale bytes uint8 [..., cols/32]): MX block scaling, one
    power-of-two scale per 32 consecutive elements."""
    x = _c(x, np.uint16)
    shp = x.shape
    x2 = x.reshape(-1, shp[-1])
    codes = np.empty(x2.shape, dtype=np.uint8)
    scales = np.empty((x2.shape[0], max(1, x2.shape[1] // 32)), dtype=np.uint8)
    if _use(lib).oracle_quantize_mxfp8_rows(_p(x2), x2.shape[0], x2.shape[1], _p(codes),
                                            _p(scales)) != 0:
        raise ValueError("oracle_quantize_mxfp8_rows: cols must be a positive multiple of 32")
    return codes.reshape(shp), scales.reshape(shp[:-1] + (shp[-1] // 32,))


def indexer_topk_mxfp8_rows(q8_rows, qs_rows, w_rows, k8, ks, S: int, m: int, k: int, rows,
                            lib=None):
    """Oracle top-k of the MXFP8 score (codes and block scales decoded exactly).

    q8_rows [n,H,D] uint8, qs_rows [n,H,D/32] uint8, w_rows [n,H] fp32 for the
    listed queries; k8 [B,T,D] uint8, ks [B,T,D/32] uint8."""
    q8_rows, qs_rows = _c(q8_rows, np.uint8), _c(qs_rows, np.uint8)
    w_rows = _c(w_rows, np.float32)
    k8, ks, rows = _c(k8, np.uint8), _c(ks, np.uint8), _c(rows, np.int64)
    n, H, D = q8_rows.shape
    B = k8.shape[0]
    idx = np.empty((n, k), dtype=np.int32)
    sc = np.empty((n, k), dtype=np.float64)
    rc = _use(lib).oracle_indexer_topk_mxfp8_rows(_p(q8_rows), _p(qs_rows), _p(w_rows), _p(k8),
              _p(ks), B, S, H, D, m, k, _p(rows), n, _p(idx), _p(sc))
    if rc != 0:
        raise ValueError("oracle_indexer_topk_mxfp8_rows: bad arguments")
    return idx, sc


_API = {name: globals()[name] for name in (
    "threads", "visible", "indexer_topk", "indexer_topk_rows", "indexer_topk_rows_absmax",
    "score_keys_rows", "row_absmax_rows", "topk_scores", "e4m3_decode", "e4m3_encode",
    "quantize_e4m3_rows", "indexer_topk_fp8_rows", "score_keys_fp8_rows", "decode_rows",
    "indexer_decode", "sparse_attention_rows", "pivot_rows", "mx_scale_byte",
    "quantize_mxfp8_rows", "indexer_topk_mxfp8_rows")}

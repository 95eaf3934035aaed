"""B200 (sm_100a) CSA lightning-indexer top-k.

Python face of libstreamindex.so.  It marshals torch CUDA tensors (device
pointers, the current stream) into the C ABI of include/streamindex.h; every
step of the computation runs in the library's CUDA kernels.  There is no CPU
path: the calls raise if the library is not built or no sm_100 GPU is present.

    idx, score = indexer_topk(q, w, kc, m=4, topk=512)

q [B,S,H_I,d_I] bf16, w [B,S,H_I] fp32, kc [B,S/m,d_I] bf16, all on one CUDA
device.  idx [B,S,topk] int32 (-1 padding), score [B,S,topk] fp32 (-inf padding).
"""

from __future__ import annotations

import ctypes

from . import _lib
from ._lib import SiOptions, SiPlanInfo, StreamIndexError  # noqa: F401

__all__ = [
    "indexer_topk", "indexer_topk_noalloc", "indexer_topk_fp8", "quantize_fp8_rows", "topk_scores",
    "workspace_size", "plan", "device_error", "options", "version", "StreamIndexError",
]


def _torch():
    import torch

    return torch


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None) -> ctypes.c_void_p:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, ndim, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def options(key_chunk: int = 0, scratch_mb: int = 0, grid_ctas: int = 0, timeout_ms: int = 0,
            debug_flags: int = 0, score_events=None, row_finish: int = 0,
            key_tile: int = 0, strip_slots: int = 0, score_event_list=None,
            plan_heads: int = 0, plan_dim: int = 0, plan_fp8: int = 0) -> SiOptions:
    """Tuning knobs of include/streamindex.h.  ``score_events`` is an optional
    pair of ``torch.cuda.Event(enable_timing=True)`` that the call records around
    its score-kernel launches (on the call's stream); ``score_event_list`` a
    list of such events, recorded in pairs around each query block's score
    launch.  ``row_finish``: 1 = rows finished in the fused kernel, 2 = by the
    merge kernel, 0 = the library's choice.  ``key_tile``: keys per score strip
    (128 .. 1024; 0 = the library's choice); ``strip_slots``: score strips in
    flight (2..4; 0 = the library's choice).  ``plan_heads``/``plan_dim``/
    ``plan_fp8``: make ``topk_scores`` select with the fused kernel's plan for
    that indexer shape."""
    o = SiOptions(key_chunk, scratch_mb, grid_ctas, timeout_ms, debug_flags)
    o.row_finish = row_finish
    o.key_tile = key_tile
    o.strip_slots = strip_slots
    o.plan_heads = plan_heads
    o.plan_dim = plan_dim
    o.plan_fp8 = plan_fp8
    if score_events is not None:
        a, b = score_events
        o.score_events[0] = a.cuda_event
        o.score_events[1] = b.cuda_event
    if score_event_list:
        arr = (ctypes.c_void_p * len(score_event_list))(*[e.cuda_event for e in score_event_list])
        o._event_array = arr  # keep the array alive as long as the options
        o.score_event_list = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
        o.score_event_count = len(score_event_list)
    return o


def version() -> int:
    return _lib.load().si_version()


def workspace_size(B: int, S: int, H: int, D: int, m: int, topk: int, opts: SiOptions | None = None) -> int:
    n = ctypes.c_size_t(0)
    lib = _lib.load()
    _lib.check("si_indexer_topk_workspace_size",
               lib.si_indexer_topk_workspace_size(B, S, H, D, m, topk,
                                                  ctypes.byref(opts) if opts else None,
                                                  ctypes.byref(n)))
    return n.value


def plan(B: int, S: int, H: int, D: int, m: int, topk: int, fp8: bool = False,
         opts: SiOptions | None = None) -> dict:
    """The plan the library would run for this problem (si_indexer_topk_plan):
    tile shape, shared-memory plan, key chunks, query blocks and launches."""
    info = SiPlanInfo()
    lib = _lib.load()
    _lib.check("si_indexer_topk_plan",
               lib.si_indexer_topk_plan(B, S, H, D, m, topk, 1 if fp8 else 0,
                                        ctypes.byref(opts) if opts else None,
                                        ctypes.byref(info)))
    return info.as_dict()


def _outputs(B, S, topk, device, out):
    torch = _torch()
    if out is not None:
        idx, score = out
        _need(idx, torch.int32, 3, "out_idx")
        _need(score, torch.float32, 3, "out_score")
        if tuple(idx.shape) != (B, S, topk) or tuple(score.shape) != (B, S, topk):
            raise ValueError("out tensors must be [B,S,topk]")
        return idx, score
    return (torch.empty((B, S, topk), dtype=torch.int32, device=device),
            torch.empty((B, S, topk), dtype=torch.float32, device=device))


def indexer_topk(q, w, kc, m: int, topk: int, *, out=None, opts: SiOptions | None = None,
                 workspace=None, stream=None):
    """Top-k compressed keys per query (bf16 score path).  Returns (idx, score)."""
    torch = _torch()
    _need(q, torch.bfloat16, 4, "q")
    _need(w, torch.float32, 3, "w")
    _need(kc, torch.bfloat16, 3, "kc")
    B, S, H, D = q.shape
    idx, score = _outputs(B, S, topk, q.device, out)
    lib = _lib.load()
    st = _stream(stream)
    if opts is None and workspace is None:
        rc = lib.si_indexer_topk(_ptr(q), _ptr(w), _ptr(kc), B, S, H, D, m, topk, _ptr(idx),
                                 _ptr(score), st)
        _lib.check("si_indexer_topk", rc)
        return idx, score
    need = workspace_size(B, S, H, D, m, topk, opts)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = lib.si_indexer_topk_ex(_ptr(q), _ptr(w), _ptr(kc), B, S, H, D, m, topk, _ptr(idx),
                                _ptr(score), ctypes.byref(opts) if opts else None,
                                _ptr(workspace), workspace.numel(), st)
    _lib.check("si_indexer_topk_ex", rc)
    return idx, score


def decode_workspace_size(B: int, S_q: int, t0: int, T: int, H: int, D: int, m: int, topk: int,
                          opts: SiOptions | None = None) -> int:
    n = ctypes.c_size_t(0)
    lib = _lib.load()
    _lib.check("si_indexer_decode_workspace_size",
               lib.si_indexer_decode_workspace_size(B, S_q, t0, T, H, D, m, topk,
                                                    ctypes.byref(opts) if opts else None,
                                                    ctypes.byref(n)))
    return n.value


def decode_plan(B: int, S_q: int, t0: int, T: int, H: int, D: int, m: int, topk: int,
                opts: SiOptions | None = None) -> dict:
    """The plan si_indexer_decode would run (tile shape, key chunks, launches)."""
    info = SiPlanInfo()
    lib = _lib.load()
    _lib.check("si_indexer_decode_plan",
               lib.si_indexer_decode_plan(B, S_q, t0, T, H, D, m, topk,
                                          ctypes.byref(opts) if opts else None,
                                          ctypes.byref(info)))
    return info.as_dict()


def indexer_decode(q, w, kc, t0: int, m: int, topk: int, *, out=None,
                   opts: SiOptions | None = None, workspace=None, stream=None):
    """Top-k compressed keys for the queries at sequence positions t0 ..
    t0 + S_q - 1 (q [B,S_q,H,D] bf16, w [B,S_q,H] fp32) against the keys kc
    [B,T,D] bf16 compressed so far (si_indexer_decode).  Returns (idx, score),
    each [B,S_q,topk]."""
    torch = _torch()
    _need(q, torch.bfloat16, 4, "q")
    _need(w, torch.float32, 3, "w")
    _need(kc, torch.bfloat16, 3, "kc")
    B, S, H, D = q.shape
    T = kc.shape[1]
    idx, score = _outputs(B, S, topk, q.device, out)
    need = decode_workspace_size(B, S, t0, T, H, D, m, topk, opts)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = _lib.load().si_indexer_decode(_ptr(q), _ptr(w), _ptr(kc), B, S, t0, T, H, D, m, topk,
                                       _ptr(idx), _ptr(score),
                                       ctypes.byref(opts) if opts else None, _ptr(workspace),
                                       workspace.numel(), _stream(stream))
    _lib.check("si_indexer_decode", rc)
    return idx, score


def pivot_workspace_size(B: int, S: int, H: int, D: int, m: int, topk: int, G: int, C: int,
                         opts: SiOptions | None = None) -> int:
    n = ctypes.c_size_t(0)
    lib = _lib.load()
    _lib.check("si_indexer_pivot_workspace_size",
               lib.si_indexer_pivot_workspace_size(B, S, H, D, m, topk, G, C,
                                                   ctypes.byref(opts) if opts else None,
                                                   ctypes.byref(n)))
    return n.value


def indexer_pivot(q, w, kc, m: int, topk: int, G: int, C: int, *, out=None,
                  opts: SiOptions | None = None, workspace=None, stream=None):
    """Query-group candidate scan (si_indexer_pivot): groups of G queries share
    their last query's C best keys as candidates.  Returns (idx, score)."""
    torch = _torch()
    _need(q, torch.bfloat16, 4, "q")
    _need(w, torch.float32, 3, "w")
    _need(kc, torch.bfloat16, 3, "kc")
    B, S, H, D = q.shape
    idx, score = _outputs(B, S, topk, q.device, out)
    need = pivot_workspace_size(B, S, H, D, m, topk, G, C, opts)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = _lib.load().si_indexer_pivot(_ptr(q), _ptr(w), _ptr(kc), B, S, H, D, m, topk, G, C,
                                      _ptr(idx), _ptr(score), ctypes.byref(opts) if opts else None,
                                      _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check("si_indexer_pivot", rc)
    return idx, score


def sparse_attention(qa, ka, va, idx, scale: float | None = None, *, out=None,
                     opts: SiOptions | None = None, stream=None):
    """Multi-query attention of each query's heads over the entries its row of
    ``idx`` lists (si_sparse_attention): qa [B,S,128,128] bf16, ka and va
    [B,T,128] bf16, idx [B,S,topk] int32 (-1 padding).  ``scale`` defaults to
    1/sqrt(128).  Returns out [B,S,128,128] fp32."""
    torch = _torch()
    _need(qa, torch.bfloat16, 4, "qa")
    _need(ka, torch.bfloat16, 3, "ka")
    _need(va, torch.bfloat16, 3, "va")
    _need(idx, torch.int32, 3, "idx")
    B, S, H, D = qa.shape
    T = ka.shape[1]
    if tuple(va.shape) != tuple(ka.shape) or idx.shape[0] != B or idx.shape[1] != S:
        raise ValueError("ka, va must be [B,T,D] and idx [B,S,topk]")
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty((B, S, H, D), dtype=torch.float32, device=qa.device)
    _need(out, torch.float32, 4, "out")
    rc = _lib.load().si_sparse_attention(_ptr(qa), _ptr(ka), _ptr(va), _ptr(idx), B, S, T, H, D,
                                         idx.shape[2], float(scale), _ptr(out),
                                         ctypes.byref(opts) if opts else None, _stream(stream))
    _lib.check("si_sparse_attention", rc)
    return out


def indexer_topk_noalloc(q, w, kc, m: int, topk: int, *, out=None, stream=None):
    """``indexer_topk`` through the entry point that allocates no device memory
    (its scratch is a fixed array inside the library; see
    si_indexer_topk_noalloc in include/streamindex.h).  Returns (idx, score);
    pass ``out`` to avoid allocating the outputs here as well."""
    torch = _torch()
    _need(q, torch.bfloat16, 4, "q")
    _need(w, torch.float32, 3, "w")
    _need(kc, torch.bfloat16, 3, "kc")
    B, S, H, D = q.shape
    idx, score = _outputs(B, S, topk, q.device, out)
    rc = _lib.load().si_indexer_topk_noalloc(_ptr(q), _ptr(w), _ptr(kc), B, S, H, D, m, topk,
                                             _ptr(idx), _ptr(score), _stream(stream))
    _lib.check("si_indexer_topk_noalloc", rc)
    return idx, score


def indexer_topk_fp8(q8, s_q, w, k8, s_k, m: int, topk: int, *, out=None,
                     opts: SiOptions | None = None, workspace=None, stream=None):
    """FP8 (E4M3) score path: q8 [B,S,H,D] and k8 [B,T,D] uint8 codes with
    per-row scales s_q [B,S,H], s_k [B,T].  Returns (idx, score)."""
    torch = _torch()
    _need(q8, torch.uint8, 4, "q8")
    _need(s_q, torch.float32, 3, "s_q")
    _need(w, torch.float32, 3, "w")
    _need(k8, torch.uint8, 3, "k8")
    _need(s_k, torch.float32, 2, "s_k")
    B, S, H, D = q8.shape
    idx, score = _outputs(B, S, topk, q8.device, out)
    need = workspace_size(B, S, H, D, m, topk, opts)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q8.device)
    lib = _lib.load()
    rc = lib.si_indexer_topk_fp8(_ptr(q8), _ptr(s_q), _ptr(w), _ptr(k8), _ptr(s_k), B, S, H, D, m,
                                 topk, _ptr(idx), _ptr(score),
                                 ctypes.byref(opts) if opts else None, _ptr(workspace),
                                 workspace.numel(), _stream(stream))
    _lib.check("si_indexer_topk_fp8", rc)
    return idx, score


def quantize_fp8_rows(x, stream=None):
    """Per-row E4M3 quantisation of a bf16 tensor [..., cols]: returns
    (codes uint8 [..., cols], scale fp32 [...])."""
    torch = _torch()
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    cols = x.shape[-1]
    rows = x.numel() // cols
    x8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    rc = _lib.load().si_quantize_fp8_rows(_ptr(x), rows, cols, _ptr(x8), _ptr(scale),
                                          _stream(stream))
    _lib.check("si_quantize_fp8_rows", rc)
    return x8, scale


def topk_scores(scores, m: int, topk: int, *, out=None, opts: SiOptions | None = None,
                stream=None):
    """Selection alone on given fp32 scores [B,S,T] (causal rule with ratio m)."""
    torch = _torch()
    _need(scores, torch.float32, 3, "scores")
    B, S, T = scores.shape
    idx, score = _outputs(B, S, topk, scores.device, out)
    rc = _lib.load().si_topk_scores(_ptr(scores), B, S, T, m, topk, _ptr(idx), _ptr(score),
                                    ctypes.byref(opts) if opts else None, _stream(stream))
    _lib.check("si_topk_scores", rc)
    return idx, score


def device_error(stream=None) -> int:
    """Synchronise and return the device status word as an SI status code."""
    return _lib.load().si_get_last_device_error(_stream(stream))

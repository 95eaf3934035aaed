"""ctypes loader for libstreamindex.so: declares the C ABI of include/streamindex.h.

There is no fallback: if the library is missing or cannot be loaded, importing
the calls raises.  Build it with ``python -m streaming_top_lightning_b200.build``.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libstreamindex.so")

SI_OK = 0
STATUS = {
    -1: "SI_ERR_NULL", -2: "SI_ERR_DIM", -3: "SI_ERR_TOPK", -4: "SI_ERR_ALIGN",
    -5: "SI_ERR_WORKSPACE", -6: "SI_ERR_CUDA", -7: "SI_ERR_DEVICE_TIMEOUT", -8: "SI_ERR_OPTIONS",
    -9: "SI_ERR_UNSUPPORTED",
}

# every symbol the header declares
EXPORTS = [
    "si_indexer_topk", "si_indexer_topk_workspace_size", "si_indexer_topk_ex",
    "si_indexer_topk_fp8", "si_quantize_fp8_rows", "si_topk_scores", "si_status_string",
    "si_get_last_device_error", "si_version", "si_indexer_topk_noalloc", "si_indexer_topk_plan",
    "si_role_cycles", "si_indexer_decode", "si_indexer_decode_workspace_size",
    "si_indexer_decode_plan", "si_sparse_attention", "si_indexer_pivot",
    "si_indexer_pivot_workspace_size",
]


class SiOptions(ctypes.Structure):
    _fields_ = [("key_chunk", ctypes.c_int), ("scratch_mb", ctypes.c_int),
                ("grid_ctas", ctypes.c_int), ("timeout_ms", ctypes.c_int),
                ("debug_flags", ctypes.c_int), ("score_events", ctypes.c_void_p * 2),
                ("row_finish", ctypes.c_int), ("key_tile", ctypes.c_int),
                ("strip_slots", ctypes.c_int), ("score_event_list", ctypes.POINTER(ctypes.c_void_p)),
                ("score_event_count", ctypes.c_int), ("plan_heads", ctypes.c_int),
                ("plan_dim", ctypes.c_int), ("plan_fp8", ctypes.c_int)]


class SiPlanInfo(ctypes.Structure):
    _fields_ = [("queries_per_tile", ctypes.c_int), ("mma_n", ctypes.c_int),
                ("key_tile", ctypes.c_int), ("stages", ctypes.c_int),
                ("strip_slots", ctypes.c_int), ("pool_keys", ctypes.c_int),
                ("partial_len", ctypes.c_int), ("key_chunks", ctypes.c_int),
                ("query_blocks", ctypes.c_int), ("launches", ctypes.c_int),
                ("workspace_bytes", ctypes.c_size_t), ("smem_bytes", ctypes.c_size_t)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


class StreamIndexError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({text})")
        self.status = status


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library (once) and declare argument types.  The first call
    fixes which build is used: the default one, or ``path`` (the profiling
    build, libstreamindex_roles.so)."""
    global _lib
    if _lib is not None:
        if path is not None and os.path.abspath(path) != os.path.abspath(_lib._name):
            raise RuntimeError(f"{_lib._name} is already loaded")
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run python -m streaming_top_lightning_b200.build")
    lib = ctypes.CDLL(path)
    P, I, L, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    OP = ctypes.POINTER(SiOptions)
    lib.si_indexer_topk.argtypes = [P, P, P, I, I, I, I, I, I, P, P, P]
    lib.si_indexer_topk_noalloc.argtypes = [P, P, P, I, I, I, I, I, I, P, P, P]
    lib.si_indexer_topk_workspace_size.argtypes = [I, I, I, I, I, I, OP, ctypes.POINTER(Z)]
    lib.si_indexer_topk_plan.argtypes = [I, I, I, I, I, I, I, OP, ctypes.POINTER(SiPlanInfo)]
    lib.si_indexer_topk_ex.argtypes = [P, P, P, I, I, I, I, I, I, P, P, OP, P, Z, P]
    lib.si_indexer_topk_fp8.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, OP, P, Z, P]
    lib.si_quantize_fp8_rows.argtypes = [P, L, I, P, P, P]
    lib.si_topk_scores.argtypes = [P, I, I, I, I, I, P, P, OP, P]
    lib.si_status_string.argtypes = [I]
    lib.si_status_string.restype = ctypes.c_char_p
    lib.si_get_last_device_error.argtypes = [P]
    lib.si_version.argtypes = []
    lib.si_role_cycles.argtypes = [P, I, I]
    lib.si_indexer_decode.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, P, OP, P, Z, P]
    lib.si_indexer_decode_workspace_size.argtypes = [I, I, I, I, I, I, I, I, OP,
                                                     ctypes.POINTER(Z)]
    lib.si_indexer_decode_plan.argtypes = [I, I, I, I, I, I, I, I, OP,
                                           ctypes.POINTER(SiPlanInfo)]
    lib.si_sparse_attention.argtypes = [P, P, P, P, I, I, I, I, I, I, ctypes.c_float, P, OP, P]
    lib.si_indexer_pivot.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, P, OP, P, Z, P]
    lib.si_indexer_pivot_workspace_size.argtypes = [I, I, I, I, I, I, I, I, OP,
                                                    ctypes.POINTER(Z)]
    for name in EXPORTS:
        if name != "si_status_string":
            getattr(lib, name).restype = I
    _lib = lib
    return lib


def check(fn: str, status: int) -> None:
    if status != SI_OK:
        raise StreamIndexError(fn, status, load().si_status_string(status).decode())

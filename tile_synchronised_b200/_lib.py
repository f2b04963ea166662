"""ctypes binding of libmk.so: the C ABI declared in include/mk.h, nothing else.

Loading fails loudly (RuntimeError) when the shared library is missing and
cannot be built: there is no CPU fallback anywhere on this path.
"""
from __future__ import annotations

import ctypes as C
import os

from . import build as _build

MK_OK, MK_ERR_INVALID, MK_ERR_CUDA, MK_ERR_TIMEOUT, MK_ERR_UNSUPPORTED, MK_ERR_STATE = 0, -1, -2, -3, -4, -5
MK_BF16 = 0
MK_MEGAKERNEL, MK_GRAPH, MK_GRAPH_PDL, MK_GRAPH_TILESYNC, MK_TENSOR_CORES = 0, 1, 2, 3, 4
MK_SWIGLU_AUTO, MK_SWIGLU_ROW, MK_SWIGLU_COL, MK_SWIGLU_TC = 0, 1, 2, 3
MK_SYNC_TAGS, MK_SYNC_COUNTERS = 0, 1
MK_PREFILL_AUTO, MK_PREFILL_STEPS, MK_PREFILL_TC = 0, 1, 2

STATUS_NAMES = {0: "MK_OK", -1: "MK_ERR_INVALID", -2: "MK_ERR_CUDA", -3: "MK_ERR_TIMEOUT",
                -4: "MK_ERR_UNSUPPORTED", -5: "MK_ERR_STATE"}

# Every symbol include/mk.h declares.
EXPORTS = ("mk_create", "mk_destroy", "mk_last_error", "mk_workspace_bytes", "mk_kv_cache_bytes",
           "mk_load_weights", "mk_prefill_kv", "mk_set_prefill", "mk_decode_step", "mk_get_status", "mk_reset",
           "mk_get_position", "mk_set_position", "mk_set_variant", "mk_tune", "mk_set_swiglu_tiling",
           "mk_get_swiglu_tiling", "mk_set_prefetch",
           "mk_set_timeout_ns", "mk_set_sync", "mk_set_ring_stages", "mk_debug_drop_signal",
           "mk_debug_shuffle_schedule", "mk_debug_poison_activations", "mk_set_trace",
           "mk_get_schedule", "mk_schedule_info", "mk_validate_schedule", "mk_swiglu_stage1",
           "mk_swiglu_tune", "mk_attention_decode", "mk_attention_scratch_bytes", "mk_attention_chunks",
           "mk_attention_decode_noalloc", "mk_attention_noalloc_limit_bytes", "mk_linear_tc",
           "mk_linear_tc_split", "mk_linear_tc_streamk", "mk_linear_tc_streamk_workspace_bytes",
           "mk_linear_tc_streamk_grid", "mk_tcdec_create", "mk_tcdec_workspace_bytes", "mk_tcdec_bind", "mk_tcdec_step",
           "mk_tcdec_status", "mk_tcdec_last_error", "mk_tcdec_destroy", "mk_tcdec_set_graph")


class MkConfig(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("n_layers", "hidden", "n_heads", "n_kv_heads", "head_dim",
                                       "intermediate", "vocab")] + \
               [("rms_eps", C.c_float), ("rope_theta", C.c_float)] + \
               [(n, C.c_int) for n in ("tied_embeddings", "qk_norm", "batch", "max_seq", "dtype", "variant",
                                       "num_sms")]


_PP = C.POINTER(C.c_void_p)


class MkWeights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p), ("lm_head", C.c_void_p)] + \
               [(n, _PP) for n in ("attn_norm", "wq", "wk", "wv", "wo", "q_norm", "k_norm", "mlp_norm",
                                   "wg", "wu", "wd")]


class MkError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def load() -> C.CDLL:
    """Load libmk.so (building it first only if it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if not os.path.exists(path):
        try:
            _build.build()
        except Exception as e:  # noqa: BLE001 - re-raised with context
            raise RuntimeError(f"libmk.so is missing and could not be built: {e}") from e
    L = C.CDLL(path)
    vp, i32, sz = C.c_void_p, C.c_int, C.c_size_t
    st = C.c_int
    sig = {
        "mk_create": ([C.POINTER(MkConfig), i32, C.POINTER(vp)], st),
        "mk_destroy": ([vp], st),
        "mk_last_error": ([vp], C.c_char_p),
        "mk_workspace_bytes": ([vp, C.POINTER(sz)], st),
        "mk_kv_cache_bytes": ([vp, C.POINTER(sz)], st),
        "mk_load_weights": ([vp, C.POINTER(MkWeights), vp, vp, vp], st),
        "mk_prefill_kv": ([vp, vp, i32, i32, vp], st),
        "mk_set_prefill": ([vp, i32], st),
        "mk_decode_step": ([vp, vp, vp, vp, vp], st),
        "mk_get_status": ([vp, vp], st),
        "mk_reset": ([vp, vp], st),
        "mk_get_position": ([vp, C.POINTER(i32)], st),
        "mk_set_position": ([vp, i32, vp], st),
        "mk_set_variant": ([vp, i32], st),
        "mk_tune": ([vp, vp, C.POINTER(i32)], st),
        "mk_set_swiglu_tiling": ([vp, i32, vp], st),
        "mk_get_swiglu_tiling": ([vp, C.POINTER(i32)], st),
        "mk_set_prefetch": ([vp, i32], st),
        "mk_set_timeout_ns": ([vp, C.c_ulonglong], st),
        "mk_set_sync": ([vp, i32], st),
        "mk_set_ring_stages": ([vp, i32], st),
        "mk_debug_drop_signal": ([vp, i32], st),
        "mk_debug_shuffle_schedule": ([vp, C.c_ulonglong], st),
        "mk_debug_poison_activations": ([vp, vp], st),
        "mk_set_trace": ([vp, vp, sz], st),
        "mk_get_schedule": ([vp, vp, sz, vp], st),
        "mk_schedule_info": ([vp, C.POINTER(C.c_longlong), i32], st),
        "mk_validate_schedule": ([vp], st),
        "mk_swiglu_stage1": ([vp, vp, vp, vp, i32, i32, i32, i32, vp], st),
        "mk_swiglu_tune": ([vp, vp, vp, vp, i32, i32, i32, vp, C.POINTER(i32), C.POINTER(C.c_float),
                            C.POINTER(C.c_float), C.POINTER(C.c_float)], st),
        "mk_attention_decode": ([vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp, sz, vp], st),
        "mk_attention_scratch_bytes": ([i32, i32, i32, i32], sz),
        "mk_attention_chunks": ([i32, i32, i32], i32),
        "mk_attention_decode_noalloc": ([vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp], st),
        "mk_attention_noalloc_limit_bytes": ([], sz),
        "mk_linear_tc": ([vp, vp, vp, i32, i32, i32, vp], st),
        "mk_linear_tc_split": ([i32, i32, i32, C.POINTER(i32)], st),
        "mk_linear_tc_streamk": ([vp, vp, vp, i32, i32, i32, vp, sz, vp], st),
        "mk_linear_tc_streamk_workspace_bytes": ([], sz),
        "mk_linear_tc_streamk_grid": ([i32, i32, i32], i32),
        "mk_tcdec_create": ([C.POINTER(MkConfig), C.POINTER(MkWeights), C.POINTER(vp)], st),
        "mk_tcdec_workspace_bytes": ([vp, C.POINTER(sz)], st),
        "mk_tcdec_bind": ([vp, vp, vp], st),
        "mk_tcdec_step": ([vp, vp, i32, vp, vp, vp], st),
        "mk_tcdec_status": ([vp, C.POINTER(i32), vp], st),
        "mk_tcdec_last_error": ([vp], C.c_char_p),
        "mk_tcdec_destroy": ([vp], st),
        "mk_tcdec_set_graph": ([vp, i32], st),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def check(status: int, ctx=None, what: str = "", op: bool = False) -> None:
    """Raise MkError for a failed call; the reason comes from the context, or,
    for a context-free call (op=True), from the calling thread's last error."""
    if status != MK_OK:
        msg = what
        if ctx is not None or op:
            msg = f"{what}: {load().mk_last_error(ctx).decode()}"
        raise MkError(status, msg)

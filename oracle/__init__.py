"""CPU oracle: a plain, slow reference of the decode step and the SwiGLU stage.

TEST INFRASTRUCTURE ONLY -- only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package.  The
product library never loads it and shares no code with it.

The arithmetic lives in ``mk_oracle.c`` (fp32 tensors, double sums, OpenMP
over output rows); this module compiles it with gcc on first use and
marshals numpy arrays through ctypes.  Every function here is argument
marshalling only.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mk_oracle.c")
_LIB = os.path.join(_HERE, "libmk_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libmk_oracle.so`` (gcc, -O3, OpenMP)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", "-O3", "-march=native", "-fopenmp", "-fPIC", "-shared",
                                   "-Wall", "-o", tmp, _SRC, "-lm"])
            os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_LIB)
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        L.orc_bf16_to_f32.argtypes = [C.c_uint16]
        L.orc_bf16_to_f32.restype = C.c_float
        L.orc_f16_to_f32.argtypes = [C.c_uint16]
        L.orc_f16_to_f32.restype = C.c_float
        L.orc_gemv_bf16.argtypes = [u16p, f32p, f32p, C.c_int64, C.c_int64]
        L.orc_rmsnorm.argtypes = [f32p, u16p, f32p, C.c_int64, C.c_float]
        L.orc_rope.argtypes = [f32p, C.c_int, C.c_int64, C.c_double]
        L.orc_silu.argtypes = [C.c_double]
        L.orc_silu.restype = C.c_double
        L.orc_attend.argtypes = [f32p, f32p, f32p, C.c_int64, C.c_int64, C.c_int, f32p]
        L.orc_argmax.argtypes = [f32p, C.c_int64]
        L.orc_argmax.restype = C.c_int64
        L.orc_decode_step.argtypes = [C.c_void_p, C.c_void_p, f32p, f32p, i32p, i32p, C.c_void_p, C.c_void_p]
        L.orc_decode_step.restype = C.c_int
        L.orc_forward_full.argtypes = [C.c_void_p, C.c_void_p, i32p, C.c_int64, f32p]
        L.orc_forward_full.restype = C.c_int
        L.orc_swiglu_stage1_f16.argtypes = [u16p, u16p, u16p, f32p, C.c_int64, C.c_int64, C.c_int64]
        L.orc_num_threads.restype = C.c_int
        L.orc_set_num_threads.argtypes = [C.c_int]
        _lib = L
    return _lib


# ---------------------------------------------------------------- building blocks
def bf16_to_f32(h: int) -> float:
    return lib().orc_bf16_to_f32(h)


def f16_to_f32(h: int) -> float:
    return lib().orc_f16_to_f32(h)


def gemv_bf16(W_u16: np.ndarray, x: np.ndarray) -> np.ndarray:
    N, K = W_u16.shape
    y = np.empty(N, np.float32)
    lib().orc_gemv_bf16(np.ascontiguousarray(W_u16), np.ascontiguousarray(x, np.float32), y, N, K)
    return y


def rmsnorm(x: np.ndarray, g_u16: np.ndarray, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty_like(x)
    lib().orc_rmsnorm(x, np.ascontiguousarray(g_u16), out, x.size, eps)
    return out


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    v = np.array(v, np.float32, copy=True)
    lib().orc_rope(v, v.size, pos, theta)
    return v


def silu(z: float) -> float:
    return lib().orc_silu(z)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    V = np.ascontiguousarray(V, np.float32)
    n, d = K.shape
    o = np.empty(d, np.float32)
    lib().orc_attend(q, K, V, d, n, d, o)
    return o


def argmax(v: np.ndarray) -> int:
    return int(lib().orc_argmax(np.ascontiguousarray(v, np.float32), v.size))


def swiglu_stage1_f16(x_u16: np.ndarray, wg_u16: np.ndarray, wu_u16: np.ndarray) -> np.ndarray:
    B, K = x_u16.shape
    K2, N = wg_u16.shape
    assert K2 == K and wu_u16.shape == (K, N)
    out = np.empty((B, N), np.float32)
    lib().orc_swiglu_stage1_f16(np.ascontiguousarray(x_u16), np.ascontiguousarray(wg_u16),
                                np.ascontiguousarray(wu_u16), out, B, K, N)
    return out


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of later oracle calls (n < 1: all processors)."""
    lib().orc_set_num_threads(int(n))


# ---------------------------------------------------------------- the decoder
class _Cfg(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("n_layers", "hidden", "n_heads", "n_kv_heads", "head_dim",
                                       "intermediate", "vocab")] + \
               [("rms_eps", C.c_float), ("rope_theta", C.c_float)] + \
               [(n, C.c_int) for n in ("tied", "qk_norm", "batch", "max_seq")]


_PP = C.POINTER(C.c_void_p)


class _W(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p), ("lm_head", C.c_void_p)] + \
               [(n, _PP) for n in ("attn_norm", "wq", "wk", "wv", "wo", "q_norm", "k_norm",
                                   "mlp_norm", "wg", "wu", "wd")]


class OracleModel:
    """The decoder over host bf16 weights (numpy uint16 arrays).

    ``weights`` has the structure ``synth.make_weights`` returns, with every
    tensor already converted to a host uint16 array (see ``from_torch``).
    The fp32 KV cache ``kc``/``vc`` [L][B][nkv][max_seq][d] and positions
    ``pos`` [B] are plain numpy arrays the caller may read or overwrite (for
    example to start from another implementation's cache).
    """

    def __init__(self, shape, weights: dict, batch: int | None = None, max_seq: int | None = None):
        self.shape = shape
        self.batch = shape.batch if batch is None else batch
        self.max_seq = shape.max_seq if max_seq is None else max_seq
        m = shape
        self.cfg = _Cfg(m.n_layers, m.hidden, m.n_heads, m.n_kv_heads, m.head_dim, m.intermediate,
                        m.vocab, m.rms_eps, m.rope_theta, int(m.tied), int(m.qk_norm), self.batch,
                        self.max_seq)
        self._keep = []

        def ptr(a):
            if a is None:
                return None
            a = np.ascontiguousarray(a, np.uint16)
            self._keep.append(a)
            return a.ctypes.data

        def arr(name):
            ps = (C.c_void_p * m.n_layers)(*[ptr(lw[name]) for lw in weights["layers"]])
            self._keep.append(ps)
            return C.cast(ps, _PP)

        self.w = _W(ptr(weights["embed"]), ptr(weights["final_norm"]), ptr(weights.get("lm_head")),
                    *[arr(n) for n in ("attn_norm", "wq", "wk", "wv", "wo", "q_norm", "k_norm",
                                       "mlp_norm", "wg", "wu", "wd")])
        kv_shape = (m.n_layers, self.batch, m.n_kv_heads, self.max_seq, m.head_dim)
        self.kc = np.zeros(kv_shape, np.float32)
        self.vc = np.zeros(kv_shape, np.float32)
        self.pos = np.zeros(self.batch, np.int32)

    @staticmethod
    def from_torch(shape, tw: dict, batch=None, max_seq=None) -> "OracleModel":
        from synth import to_u16
        hw = {k: (None if tw[k] is None else to_u16(tw[k])) for k in ("embed", "final_norm", "lm_head")}
        hw["layers"] = [{k: (None if v is None else to_u16(v)) for k, v in lw.items()} for lw in tw["layers"]]
        return OracleModel(shape, hw, batch, max_seq)

    def step(self, tokens, want_logits: bool = True):
        tok = np.ascontiguousarray(np.asarray(tokens, np.int32).reshape(self.batch))
        logits = np.empty((self.batch, self.shape.vocab), np.float32) if want_logits else None
        nxt = np.empty(self.batch, np.int32)
        rc = lib().orc_decode_step(C.byref(self.cfg), C.byref(self.w), self.kc, self.vc, self.pos, tok,
                                   None if logits is None else logits.ctypes.data, nxt.ctypes.data)
        if rc != 0:
            raise ValueError("oracle decode step: token or position out of range")
        return logits, nxt

    def prefill(self, tokens_bt) -> None:
        t = np.asarray(tokens_bt, np.int32).reshape(self.batch, -1)
        for s in range(t.shape[1]):
            self.step(t[:, s], want_logits=False)

    def forward_full(self, tokens) -> np.ndarray:
        tok = np.ascontiguousarray(np.asarray(tokens, np.int32).ravel())
        out = np.empty(self.shape.vocab, np.float32)
        rc = lib().orc_forward_full(C.byref(self.cfg), C.byref(self.w), tok, tok.size, out)
        if rc != 0:
            raise ValueError("oracle full forward: bad tokens")
        return out

"""B200 decode megakernel: one small-batch decode step of a dense
Llama-architecture decoder as a persistent, tile-synchronised kernel.

The work happens in libmk.so (CUDA for sm_100a, C ABI in include/mk.h).  This
module only marshals arguments: PyTorch provides device memory and streams.
"""
from __future__ import annotations

import ctypes as C

import torch

from ._lib import (MK_GRAPH, MK_GRAPH_PDL, MK_GRAPH_TILESYNC, MK_MEGAKERNEL, MK_TENSOR_CORES, MK_SWIGLU_AUTO, MK_SWIGLU_COL, MK_SWIGLU_ROW,
                   MK_SWIGLU_TC, MK_SYNC_COUNTERS, MK_SYNC_TAGS, MkConfig, MkError, MkWeights, check, load)

__all__ = ["Model", "TcDecoder", "swiglu_stage1", "swiglu_tune", "linear_tc", "linear_tc_split", "MkError", "VARIANTS",
           "MK_SWIGLU_AUTO", "MK_SWIGLU_ROW", "MK_SWIGLU_COL", "MK_SWIGLU_TC", "load"]

VARIANTS = {"megakernel": MK_MEGAKERNEL, "graph": MK_GRAPH, "graph_pdl": MK_GRAPH_PDL, "tilesync": MK_GRAPH_TILESYNC,
            "tensor_cores": MK_TENSOR_CORES}
SYNCS = {"tags": MK_SYNC_TAGS, "counters": MK_SYNC_COUNTERS}
PREFILLS = {"auto": 0, "steps": 1, "tc": 2}
SCHEDULE_FIELDS = ("n_instructions", "n_ctas", "n_counters", "n_phases", "batch_rows", "attention_chunks",
                   "ring_stages", "act_bytes", "swiglu_variant", "down_k_splits")


def _stream(stream) -> C.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def make_config(shape, batch: int, max_seq: int, variant: str = "megakernel", num_sms: int = 0) -> MkConfig:
    return MkConfig(shape.n_layers, shape.hidden, shape.n_heads, shape.n_kv_heads, shape.head_dim,
                    shape.intermediate, shape.vocab, shape.rms_eps, shape.rope_theta, int(shape.tied),
                    int(shape.qk_norm), batch, max_seq, 0, VARIANTS[variant], num_sms)


class Plan:
    """A host-only schedule (no device): for inspecting and validating plans on CPU."""

    def __init__(self, shape, batch: int, max_seq: int, num_sms: int = 148):
        self.lib = load()
        self.ctx = C.c_void_p()
        cfg = make_config(shape, batch, max_seq, "megakernel", num_sms)
        check(self.lib.mk_create(C.byref(cfg), -1, C.byref(self.ctx)), None, "mk_create")

    def info(self) -> dict:
        arr = (C.c_longlong * len(SCHEDULE_FIELDS))()
        check(self.lib.mk_schedule_info(self.ctx, arr, len(arr)), self.ctx, "mk_schedule_info")
        return dict(zip(SCHEDULE_FIELDS, list(arr)))

    def workspace_bytes(self) -> int:
        n = C.c_size_t()
        check(self.lib.mk_workspace_bytes(self.ctx, C.byref(n)), self.ctx, "mk_workspace_bytes")
        return n.value

    def kv_cache_bytes(self) -> int:
        n = C.c_size_t()
        check(self.lib.mk_kv_cache_bytes(self.ctx, C.byref(n)), self.ctx, "mk_kv_cache_bytes")
        return n.value

    def schedule(self):
        """The flattened instruction list as a numpy structured array, and CTA offsets."""
        import numpy as np
        n = self.info()["n_instructions"]
        dt = np.dtype([("op", "u1"), ("flags", "u1"), ("layer", "<u2"), ("tile", "<u4"), ("kb0", "<u2"),
                       ("kb1", "<u2"), ("b0", "<u2"), ("nb", "<u2"), ("wait_ctr", "<u2"), ("signal_ctr", "<u2"),
                       ("wait_count", "<u4"), ("signal2_ctr", "<u2"), ("ntiles", "<u2"), ("arrive_count", "<u4")])
        arr = np.zeros(n, dt)
        base = np.zeros(self.info()["n_ctas"] + 1, np.int32)
        check(self.lib.mk_get_schedule(self.ctx, C.c_void_p(arr.ctypes.data), arr.nbytes,
                                       C.c_void_p(base.ctypes.data)), self.ctx, "mk_get_schedule")
        return arr, base

    def shuffle_schedule(self, seed: int) -> None:
        """Reorder the schedule with a seeded dependency-preserving permutation (test hook)."""
        check(self.lib.mk_debug_shuffle_schedule(self.ctx, int(seed)), self.ctx, "mk_debug_shuffle_schedule")

    def validate(self) -> None:
        check(self.lib.mk_validate_schedule(self.ctx), self.ctx, "mk_validate_schedule")

    def close(self):
        ctx, self.ctx = self.ctx, None
        if ctx:
            try:
                self.lib.mk_destroy(ctx)
            except Exception:  # noqa: BLE001 - interpreter shutdown: the library may be gone
                pass

    __del__ = close


def _weights_struct(weights: dict, n_layers: int, keep: list) -> MkWeights:
    """The mk_weights struct of a ``synth.make_weights``-style dict; the host
    pointer arrays it refers to are appended to `keep`, which must outlive it."""
    def ptr(t):
        return None if t is None else t.data_ptr()

    def arr(name):
        a = (C.c_void_p * n_layers)(*[ptr(lw[name]) for lw in weights["layers"]])
        keep.append(a)
        return C.cast(a, C.POINTER(C.c_void_p))

    return MkWeights(ptr(weights["embed"]), ptr(weights["final_norm"]), ptr(weights.get("lm_head")),
                     *[arr(n) for n in ("attn_norm", "wq", "wk", "wv", "wo", "q_norm", "k_norm", "mlp_norm",
                                        "wg", "wu", "wd")])


class Model(Plan):
    """A decoder bound to device weights (``synth.make_weights`` structure, bf16 on CUDA)."""

    def __init__(self, shape, weights: dict, batch: int | None = None, max_seq: int | None = None,
                 variant: str = "megakernel", device: int | None = None, num_sms: int = 0, stream=None):
        self.lib = load()
        self.shape = shape
        self.batch = shape.batch if batch is None else batch
        self.max_seq = shape.max_seq if max_seq is None else max_seq
        dev = torch.cuda.current_device() if device is None else device
        self.device = torch.device("cuda", dev)
        self.ctx = C.c_void_p()
        cfg = make_config(shape, self.batch, self.max_seq, variant, num_sms)
        check(self.lib.mk_create(C.byref(cfg), dev, C.byref(self.ctx)), None, "mk_create")
        self.workspace = torch.empty(self.workspace_bytes(), dtype=torch.uint8, device=self.device)
        self.kv = torch.empty(self.kv_cache_bytes(), dtype=torch.uint8, device=self.device)
        self._weights = weights  # the embedding table must stay alive
        self._keep = []
        w = _weights_struct(weights, shape.n_layers, self._keep)
        check(self.lib.mk_load_weights(self.ctx, C.byref(w), C.c_void_p(self.workspace.data_ptr()),
                                       C.c_void_p(self.kv.data_ptr()), _stream(stream)), self.ctx, "mk_load_weights")
        self._next = torch.empty(self.batch, dtype=torch.int32, device=self.device)

    # ---------------------------------------------------------------- views
    def kv_views(self):
        """(K, V) bf16 views of the cache, each [L, B, nkv, max_seq, d]."""
        s = self.shape
        shp = (s.n_layers, self.batch, s.n_kv_heads, self.max_seq, s.head_dim)
        half = self.kv.numel() // 2
        k = self.kv[:half].view(torch.bfloat16).view(shp)
        v = self.kv[half:].view(torch.bfloat16).view(shp)
        return k, v

    @property
    def position(self) -> int:
        p = C.c_int()
        check(self.lib.mk_get_position(self.ctx, C.byref(p)), self.ctx, "mk_get_position")
        return p.value

    def set_trace(self, buf: torch.Tensor | None) -> None:
        """Trace into `buf` (int64 CUDA tensor of >= 8 * n_instructions), or None to stop."""
        if buf is None:
            check(self.lib.mk_set_trace(self.ctx, None, 0), self.ctx, "mk_set_trace")
        else:
            check(self.lib.mk_set_trace(self.ctx, C.c_void_p(buf.data_ptr()), buf.numel() * buf.element_size()),
                  self.ctx, "mk_set_trace")

    def set_position(self, pos: int, stream=None) -> None:
        check(self.lib.mk_set_position(self.ctx, int(pos), _stream(stream)), self.ctx, "mk_set_position")

    # ---------------------------------------------------------------- calls
    def prefill(self, tokens: torch.Tensor, stream=None) -> None:
        t = tokens.to(device=self.device, dtype=torch.int32).contiguous()
        assert t.dim() == 2 and t.shape[0] == self.batch
        check(self.lib.mk_prefill_kv(self.ctx, C.c_void_p(t.data_ptr()), self.batch, t.shape[1], _stream(stream)),
              self.ctx, "mk_prefill_kv")

    def set_prefill(self, mode: str) -> None:
        """How prefill runs: "auto" (tensor cores where the plan allows), "steps" or "tc"."""
        check(self.lib.mk_set_prefill(self.ctx, PREFILLS[mode]), self.ctx, "mk_set_prefill")

    def decode(self, tokens: torch.Tensor, logits: torch.Tensor | None = None, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        """One step; returns the next-token tensor (int32 [B]); fills `logits` if given (fp32 [B, V])."""
        assert tokens.dtype == torch.int32 and tokens.is_cuda and tokens.is_contiguous()
        nxt = self._next if out is None else out
        lp = C.c_void_p(logits.data_ptr()) if logits is not None else None
        check(self.lib.mk_decode_step(self.ctx, C.c_void_p(tokens.data_ptr()), C.c_void_p(nxt.data_ptr()), lp,
                                      _stream(stream)), self.ctx, "mk_decode_step")
        return nxt

    def status(self, stream=None) -> int:
        return self.lib.mk_get_status(self.ctx, _stream(stream))

    def reset(self, stream=None) -> None:
        check(self.lib.mk_reset(self.ctx, _stream(stream)), self.ctx, "mk_reset")

    def set_variant(self, name: str) -> None:
        check(self.lib.mk_set_variant(self.ctx, VARIANTS[name]), self.ctx, "mk_set_variant")

    def set_prefetch(self, blocks: int) -> None:
        check(self.lib.mk_set_prefetch(self.ctx, int(blocks)), self.ctx, "mk_set_prefetch")

    def set_sync(self, name: str) -> None:
        """Megakernel synchronisation: "tags" (readers spin on tagged
        activations, the default) or "counters" (tile-ready counters)."""
        check(self.lib.mk_set_sync(self.ctx, SYNCS[name]), self.ctx, "mk_set_sync")

    def set_ring_stages(self, stages: int) -> None:
        """Ring slots the producer may fill (0: as many as fit)."""
        check(self.lib.mk_set_ring_stages(self.ctx, int(stages)), self.ctx, "mk_set_ring_stages")

    def set_timeout_ns(self, ns: int) -> None:
        check(self.lib.mk_set_timeout_ns(self.ctx, int(ns)), self.ctx, "mk_set_timeout_ns")

    def drop_signal(self, instr: int) -> None:
        check(self.lib.mk_debug_drop_signal(self.ctx, int(instr)), self.ctx, "mk_debug_drop_signal")

    def poison_activations(self, stream=None) -> None:
        """Fill the buffers instructions hand to each other with NaN words under an unused tag (test hook)."""
        check(self.lib.mk_debug_poison_activations(self.ctx, _stream(stream)), self.ctx,
              "mk_debug_poison_activations")

    def tune(self, stream=None) -> int:
        ch = C.c_int()
        check(self.lib.mk_tune(self.ctx, _stream(stream), C.byref(ch)), self.ctx, "mk_tune")
        return ch.value

    def set_swiglu_tiling(self, variant: int, stream=None) -> None:
        """Pick the gate/up tiling (MK_SWIGLU_ROW or MK_SWIGLU_COL) without timing."""
        check(self.lib.mk_set_swiglu_tiling(self.ctx, int(variant), _stream(stream)), self.ctx,
              "mk_set_swiglu_tiling")

    def swiglu_tiling(self) -> int:
        v = C.c_int()
        check(self.lib.mk_get_swiglu_tiling(self.ctx, C.byref(v)), self.ctx, "mk_get_swiglu_tiling")
        return v.value

    def last_error(self) -> str:
        return self.lib.mk_last_error(self.ctx).decode()


def swiglu_stage1(x: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor, out: torch.Tensor | None = None,
                  variant: int = MK_SWIGLU_AUTO, stream=None) -> torch.Tensor:
    """out = SiLU(x @ w_gate) * (x @ w_up); fp16 x [B,K], w [K,N] -> out fp16 [B,N]."""
    B, K = x.shape
    N = w_gate.shape[1]
    if out is None:
        out = torch.empty((B, N), dtype=torch.float16, device=x.device)
    check(load().mk_swiglu_stage1(C.c_void_p(x.data_ptr()), C.c_void_p(w_gate.data_ptr()),
                                  C.c_void_p(w_up.data_ptr()), C.c_void_p(out.data_ptr()), B, K, N, variant,
                                  _stream(stream)), None, "mk_swiglu_stage1")
    return out


def swiglu_tune(x, w_gate, w_up, out, stream=None):
    """Time every applicable tiling once and remember the fastest; returns
    (chosen, us_row, us_col, us_tc) with us_tc 0 where the tensor-core variant
    does not apply."""
    B, K = x.shape
    N = w_gate.shape[1]
    ch, ur, uc, ut = C.c_int(), C.c_float(), C.c_float(), C.c_float()
    check(load().mk_swiglu_tune(C.c_void_p(x.data_ptr()), C.c_void_p(w_gate.data_ptr()), C.c_void_p(w_up.data_ptr()),
                                C.c_void_p(out.data_ptr()), B, K, N, _stream(stream), C.byref(ch), C.byref(ur),
                                C.byref(uc), C.byref(ut)), None, "mk_swiglu_tune")
    return ch.value, ur.value, uc.value, ut.value


def linear_tc(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x @ w.T on the tcgen05 tensor cores: bf16 x [B, K], bf16 w [M, K]
    (an [out, in] projection as given) -> fp32 y [B, M]."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16 or x.dim() != 2 or w.dim() != 2:
        raise ValueError("x must be bf16 [B, K] and w bf16 [M, K]")
    if not (x.is_contiguous() and w.is_contiguous()) or x.shape[1] != w.shape[1]:
        raise ValueError("x and w must be contiguous with the same K")
    B, K = x.shape
    M = w.shape[0]
    if out is None:
        out = torch.empty((B, M), dtype=torch.float32, device=x.device)
    check(load().mk_linear_tc(C.c_void_p(x.data_ptr()), C.c_void_p(w.data_ptr()), C.c_void_p(out.data_ptr()), B, K,
                              M, _stream(stream)), None, "mk_linear_tc")
    return out


_streamk_ws = {}


def linear_tc_streamk(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """linear_tc with stream-K work sharing (equal weight bytes per SM where
    the row tiles alone would not fill the SMs).  `workspace`: a zero-filled
    uint8 CUDA tensor of linear_tc_streamk_workspace_bytes() bytes, or None
    for one kept per device (calls sharing it must not overlap)."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16 or x.dim() != 2 or w.dim() != 2:
        raise ValueError("x must be bf16 [B, K] and w bf16 [M, K]")
    if not (x.is_contiguous() and w.is_contiguous()) or x.shape[1] != w.shape[1]:
        raise ValueError("x and w must be contiguous with the same K")
    B, K = x.shape
    M = w.shape[0]
    if out is None:
        out = torch.empty((B, M), dtype=torch.float32, device=x.device)
    if workspace is None:
        key = x.device.index
        if key not in _streamk_ws:
            _streamk_ws[key] = torch.zeros(linear_tc_streamk_workspace_bytes(), dtype=torch.uint8, device=x.device)
        workspace = _streamk_ws[key]
    check(load().mk_linear_tc_streamk(C.c_void_p(x.data_ptr()), C.c_void_p(w.data_ptr()),
                                      C.c_void_p(out.data_ptr()), B, K, M, C.c_void_p(workspace.data_ptr()),
                                      workspace.numel() * workspace.element_size(), _stream(stream)),
          None, "mk_linear_tc_streamk", op=True)
    return out


def linear_tc_streamk_workspace_bytes() -> int:
    return int(load().mk_linear_tc_streamk_workspace_bytes())


def linear_tc_streamk_grid(B: int, K: int, M: int) -> int:
    """CTAs of the stream-K launch for this shape, 0 where it falls back."""
    return int(load().mk_linear_tc_streamk_grid(B, K, M))


def linear_tc_split(B: int, K: int, M: int) -> int:
    """CTAs per row tile (K split) linear_tc uses for this shape."""
    s = C.c_int()
    check(load().mk_linear_tc_split(B, K, M, C.byref(s)), None, "mk_linear_tc_split")
    return s.value


class TcDecoder:
    """A batched decode step with every projection on the tensor cores
    (mk_tcdec_*): the caller's [out, in] bf16 weights are read at every step,
    so `weights` is kept alive here.  `kv_cache` is a uint8 CUDA tensor in the
    layout of ``Model.kv`` (pass a model's cache to decode on from its
    prefill), or None for a fresh one."""

    def __init__(self, shape, weights: dict, batch: int, max_seq: int, kv_cache: torch.Tensor | None = None,
                 device: int | None = None):
        self.lib = load()
        self.shape, self.batch, self.max_seq = shape, batch, max_seq
        dev = torch.cuda.current_device() if device is None else device
        self.device = torch.device("cuda", dev)
        self.dec = C.c_void_p()
        cfg = make_config(shape, batch, max_seq, "megakernel", 0)
        self._weights = weights
        self._keep = []
        w = _weights_struct(weights, shape.n_layers, self._keep)
        check(self.lib.mk_tcdec_create(C.byref(cfg), C.byref(w), C.byref(self.dec)), None, "mk_tcdec_create")
        n = C.c_size_t()
        check(self.lib.mk_tcdec_workspace_bytes(self.dec, C.byref(n)), None, "mk_tcdec_workspace_bytes")
        self.workspace = torch.empty(n.value, dtype=torch.uint8, device=self.device)
        if kv_cache is None:
            kv_bytes = 2 * shape.n_layers * batch * shape.n_kv_heads * max_seq * shape.head_dim * 2
            kv_cache = torch.zeros(kv_bytes, dtype=torch.uint8, device=self.device)
        self.kv = kv_cache
        self._check(self.lib.mk_tcdec_bind(self.dec, C.c_void_p(self.workspace.data_ptr()),
                                           C.c_void_p(self.kv.data_ptr())), "mk_tcdec_bind")
        self._next = torch.empty(batch, dtype=torch.int32, device=self.device)

    def _check(self, status: int, what: str) -> None:
        if status != 0:
            raise MkError(status, f"{what}: {self.lib.mk_tcdec_last_error(self.dec).decode()}")

    def step(self, tokens: torch.Tensor, pos: int, logits: torch.Tensor | None = None,
             out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Decode one token per sequence at position `pos`: int32 CUDA tokens
        [batch] -> next tokens [batch]; fills `logits` (fp32 [batch, vocab])
        if given."""
        assert tokens.dtype == torch.int32 and tokens.is_cuda and tokens.is_contiguous()
        nxt = self._next if out is None else out
        lp = None if logits is None else C.c_void_p(logits.data_ptr())
        self._check(self.lib.mk_tcdec_step(self.dec, C.c_void_p(tokens.data_ptr()), int(pos),
                                           C.c_void_p(nxt.data_ptr()), lp, _stream(stream)), "mk_tcdec_step")
        return nxt

    def set_graph(self, on: bool) -> None:
        """Replay the step from a CUDA graph (default) or launch its kernels one by one."""
        self._check(self.lib.mk_tcdec_set_graph(self.dec, int(bool(on))), "mk_tcdec_set_graph")

    def status(self, stream=None) -> int:
        v = C.c_int()
        self._check(self.lib.mk_tcdec_status(self.dec, C.byref(v), _stream(stream)), "mk_tcdec_status")
        return v.value

    def close(self):
        dec, self.dec = getattr(self, "dec", None), None
        if dec:
            try:
                self.lib.mk_tcdec_destroy(dec)
            except Exception:  # noqa: BLE001 - interpreter shutdown: the library may be gone
                pass

    __del__ = close


def _attn_shapes(q: torch.Tensor, k_cache: torch.Tensor):
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [batch, n_heads, head_dim] and the caches [batch, n_kv_heads, max_seq, head_dim]")
    if q.dtype != torch.float32 or k_cache.dtype != torch.bfloat16:
        raise TypeError("q must be float32 and the caches bfloat16")
    B, nq, d = q.shape
    return B, nq, k_cache.shape[1], d, k_cache.shape[2]


def attention_chunks(batch: int, n_kv_heads: int, n_pos: int) -> int:
    """The chunk count attention_decode picks for chunks=0 on the current device."""
    return int(load().mk_attention_chunks(batch, n_kv_heads, n_pos))


def attention_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, n_pos: int, chunks: int = 0,
                     out: torch.Tensor | None = None, scratch: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Split-KV decode attention over positions 0..n_pos-1 of one layer's cache:
    q fp32 [B, nq, d], caches bf16 [B, nkv, max_seq, d] -> out fp32 [B, nq, d]."""
    B, nq, nkv, d, max_seq = _attn_shapes(q, k_cache)
    if chunks == 0:
        chunks = attention_chunks(B, nkv, n_pos)
    if out is None:
        out = torch.empty((B, nq, d), dtype=torch.float32, device=q.device)
    need = int(load().mk_attention_scratch_bytes(B, nq, d, chunks))
    if scratch is None:
        scratch = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    check(load().mk_attention_decode(C.c_void_p(q.data_ptr()), C.c_void_p(k_cache.data_ptr()),
                                     C.c_void_p(v_cache.data_ptr()), B, nq, nkv, d, max_seq, n_pos, chunks,
                                     C.c_void_p(out.data_ptr()), C.c_void_p(scratch.data_ptr()),
                                     scratch.numel() * scratch.element_size(), _stream(stream)),
          None, "mk_attention_decode", op=True)
    return out


def attention_decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, n_pos: int,
                             out: torch.Tensor, chunks: int = 0, stream=None) -> torch.Tensor:
    """attention_decode with the library's fixed device scratch instead of a
    caller buffer; `out` (fp32 [B, nq, d]) must be given, nothing is allocated."""
    B, nq, nkv, d, max_seq = _attn_shapes(q, k_cache)
    check(load().mk_attention_decode_noalloc(C.c_void_p(q.data_ptr()), C.c_void_p(k_cache.data_ptr()),
                                             C.c_void_p(v_cache.data_ptr()), B, nq, nkv, d, max_seq, n_pos, chunks,
                                             C.c_void_p(out.data_ptr()), _stream(stream)),
          None, "mk_attention_decode_noalloc", op=True)
    return out

"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module holds workload shapes and random-number recipes only: none of the
decoder's arithmetic lives here.  Every tensor is drawn from a seeded
``torch.Generator`` on the device given, so one call yields the same bytes for
both sides of a parity check (values drawn on CPU and on CUDA differ from each
other; each is deterministic).

Workloads (the pages' named architectures with random-init weights; no
checkpoint or dataset is used anywhere):

* ``tiny``      -- 2 layers, hidden 256, 4/2 heads, head_dim 64, SwiGLU 688,
                   vocab 1024, untied head, batch 1, 64-token prefill, 32 steps.
* ``llama1b``   -- Llama-3.2-1B architecture ("Look Ma, No Bubbles!", intro:
                   a single sequence with Llama-3.2-1B), batch 1, prefill 1024,
                   256 teacher-forced steps.
* ``llama8b``   -- Llama-3.1-8B architecture, batch 1/8/32, prefill 512, 128 steps.
* ``qwen3_8b``  -- Qwen3-8B architecture (per-head q/k RMSNorm), batch 16,
                   KV grows from 1024 to 16384, checkpoints 1k/4k/16k.
* ``swiglu``    -- the fused SwiGLU first stage sized like one TP=4 shard of a
                   Llama-3.1-70B MLP ("Deep Kernel Fusion for Transformers",
                   Key points, "Setup"): x [B,8192], W_gate/W_up [8192,7168] fp16.

Recipe: weights ~ N(0, 0.02) rounded to bf16 (fp16 for ``swiglu``), RMSNorm
gains 1.0, seed 1000 + tensor index in a fixed order; tokens uniform in
[0, vocab) with seed 42; SwiGLU x ~ N(0, 1) with seed 7, W_gate seed 8, W_up
seed 9.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class ModelShape:
    name: str
    n_layers: int
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    intermediate: int
    vocab: int
    rms_eps: float
    rope_theta: float
    tied: bool
    qk_norm: bool
    batch: int
    prefill: int
    steps: int
    max_seq: int

    def replace(self, **kw) -> "ModelShape":
        return dataclasses.replace(self, **kw)

    @property
    def qkv_rows(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim

    def weight_bytes(self) -> int:
        """bf16 bytes of every weight the decode step streams once."""
        H, d, I = self.hidden, self.head_dim, self.intermediate
        per_layer = (self.qkv_rows * H + H * self.n_heads * d + 3 * I * H + 2 * H
                     + (2 * d if self.qk_norm else 0))
        return 2 * (self.n_layers * per_layer + self.vocab * H + H)


TINY = ModelShape("tiny", 2, 256, 4, 2, 64, 688, 1024, 1e-5, 500000.0, False, False,
                  batch=1, prefill=64, steps=32, max_seq=96)
LLAMA1B = ModelShape("llama1b", 16, 2048, 32, 8, 64, 8192, 128256, 1e-5, 500000.0, True, False,
                     batch=1, prefill=1024, steps=256, max_seq=1280)
LLAMA8B = ModelShape("llama8b", 32, 4096, 32, 8, 128, 14336, 128256, 1e-5, 500000.0, False, False,
                     batch=1, prefill=512, steps=128, max_seq=640)
QWEN3_8B = ModelShape("qwen3_8b", 36, 4096, 32, 8, 128, 12288, 151936, 1e-6, 1000000.0, False, True,
                      batch=16, prefill=1024, steps=15360, max_seq=16384)

MODELS = {m.name: m for m in (TINY, LLAMA1B, LLAMA8B, QWEN3_8B)}

SWIGLU_K, SWIGLU_N = 8192, 7168
SWIGLU_BATCHES = (1, 2, 4, 16, 64)
LLAMA8B_BATCHES = (1, 8, 32)
QWEN3_CHECKPOINTS = (1024, 4096, 16384)

TOKEN_SEED = 42
WEIGHT_SEED_BASE = 1000


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, seed: int, device, dtype, std: float) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=_gen(device, seed))
    return t.to(dtype)


def make_weights(m: ModelShape, device="cpu", dtype=torch.bfloat16) -> dict:
    """Random-init weights of architecture ``m`` in nn.Linear [out, in] layout.

    Returns ``{"embed", "final_norm", "lm_head" (None when tied), "layers": [...]}``
    where each layer is a dict with attn_norm, wq, wk, wv, wo, q_norm, k_norm
    (None without qk-norm), mlp_norm, wg, wu, wd.
    """
    H, d, I = m.hidden, m.head_dim, m.intermediate
    idx = [WEIGHT_SEED_BASE]

    def nxt(shape):
        s = idx[0]
        idx[0] += 1
        return _randn(shape, s, device, dtype, 0.02)

    def ones(n):
        idx[0] += 1
        return torch.ones(n, dtype=dtype, device=device)

    w = {"embed": nxt((m.vocab, H)), "layers": []}
    for _ in range(m.n_layers):
        lw = {
            "attn_norm": ones(H),
            "wq": nxt((m.n_heads * d, H)),
            "wk": nxt((m.n_kv_heads * d, H)),
            "wv": nxt((m.n_kv_heads * d, H)),
            "wo": nxt((H, m.n_heads * d)),
            "q_norm": ones(d) if m.qk_norm else None,
            "k_norm": ones(d) if m.qk_norm else None,
            "mlp_norm": ones(H),
            "wg": nxt((I, H)),
            "wu": nxt((I, H)),
            "wd": nxt((H, I)),
        }
        w["layers"].append(lw)
    w["final_norm"] = ones(H)
    w["lm_head"] = None if m.tied else nxt((m.vocab, H))
    return w


def make_tokens(m: ModelShape, n: int, batch: int | None = None, seed: int = TOKEN_SEED,
                device="cpu") -> torch.Tensor:
    """int32 tokens uniform in [0, vocab), shape [batch, n]."""
    b = m.batch if batch is None else batch
    t = torch.randint(0, m.vocab, (b, n), generator=_gen("cpu", seed), dtype=torch.int64)
    return t.to(torch.int32).to(device)


def make_swiglu_inputs(batch: int, K: int = SWIGLU_K, N: int = SWIGLU_N, device="cpu"):
    """x [B,K] ~ N(0,1), W_gate / W_up [K,N] ~ N(0,0.02), all fp16."""
    x = _randn((batch, K), 7, device, torch.float16, 1.0)
    wg = _randn((K, N), 8, device, torch.float16, 0.02)
    wu = _randn((K, N), 9, device, torch.float16, 0.02)
    return x, wg, wu


def make_linear_inputs(batch: int, K: int, M: int, device="cpu", seed: int = 21):
    """x [B,K] ~ N(0,1) and w [M,K] ~ N(0,0.02), both bf16 (one decoder
    projection in the [out, in] layout and a batch of input rows)."""
    x = _randn((batch, K), seed, device, torch.bfloat16, 1.0)
    w = _randn((M, K), seed + 1, device, torch.bfloat16, 0.02)
    return x, w


def to_u16(t: torch.Tensor):
    """Host numpy uint16 view of a 16-bit tensor's bytes (copies to CPU)."""
    import numpy as np
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def make_attention_inputs(batch: int, n_heads: int, n_kv_heads: int, head_dim: int, max_seq: int, n_pos: int,
                          seed: int = 11, q_std: float = 1.0, device="cpu"):
    """Decode-attention operands: q fp32 [B, nq, d] ~ N(0, q_std); K, V bf16
    [B, nkv, max_seq, d] ~ N(0, 1) at positions < n_pos and the bf16 NaN
    pattern 0xFFFF beyond, so that a read past n_pos poisons the result."""
    q = _randn((batch, n_heads, head_dim), seed, device, torch.float32, q_std)
    k = _randn((batch, n_kv_heads, max_seq, head_dim), seed + 1, device, torch.bfloat16, 1.0)
    v = _randn((batch, n_kv_heads, max_seq, head_dim), seed + 2, device, torch.bfloat16, 1.0)
    for t in (k, v):
        t.view(torch.int16)[:, :, n_pos:] = -1  # 0xFFFF
    return q, k, v

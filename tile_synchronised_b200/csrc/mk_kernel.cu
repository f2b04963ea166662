// mk_kernel.cu -- the decode-step interpreter for sm_100a.
//
// One CTA per SM runs its own instruction list (built on the host).  Warp 8 is
// the producer: one lane streams every instruction's weight tiles (and the
// split-KV chunks of the KV cache) from HBM into a ring of 32 KB shared-memory
// slots with 1-D TMA bulk copies.  Weights never depend on activations, so the
// producer runs ahead across instruction boundaries and keeps loads in flight
// while the consumers wait for their inputs ("MegaOps: A Kernel Overlapping
// Framework ...", "What the control can show": prefetch).  Warps 0..7 are the
// consumers: before an instruction they acquire-spin on one global counter
// until the producing instructions have released it ("In plain words": a
// consumer starts once the particular input tiles it needs are ready), then
// compute from the ring and release their own counter.
//
// The same kernel, launched once per phase with the counter waits turned off,
// is the separate-kernels variant replayed from a CUDA graph.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "mk_device.cuh"
#include "mk_kernel.h"

namespace mk {

// ------------------------------------------------------------------ shared memory
struct SmemLayout {
    uint8_t *ring;
    uint8_t *act;
    uint64_t *full;
    uint64_t *empty;
    volatile int *abort;
    volatile int *flag;
    float *rstd;   // [kMaxBatchRows]
    float2 *best;  // [64] (value, index bits)
    float *red;    // [8 warps][8 rows][kMaxBatchRows]
    float *mlc;    // m_run[8], l_run[8], corr[8]
};

__device__ __forceinline__ SmemLayout smem_layout(uint8_t *base, const KParams &P) {
    SmemLayout S;
    S.ring = base;
    S.act = base + (size_t)P.stages * kStageBytes;
    uint8_t *misc = S.act + P.act_bytes;
    S.full = reinterpret_cast<uint64_t *>(misc);
    S.empty = S.full + kMaxStages;
    S.abort = reinterpret_cast<volatile int *>(misc + 128);
    S.flag = reinterpret_cast<volatile int *>(misc + 132);
    S.rstd = reinterpret_cast<float *>(misc + 160);
    S.best = reinterpret_cast<float2 *>(misc + 256);
    S.red = reinterpret_cast<float *>(misc + 1024);
    S.mlc = reinterpret_cast<float *>(misc + 3072);
    return S;
}

__host__ int smem_bytes(const KParams &P) { return P.stages * kStageBytes + P.act_bytes + kSmemReserve; }

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ Instr load_instr(const KParams &P, int i) {
    const uint4 *p = reinterpret_cast<const uint4 *>(P.instrs + i);
    uint4 a = __ldg(p), b = __ldg(p + 1);
    Instr in;
    memcpy(reinterpret_cast<uint8_t *>(&in), &a, 16);
    memcpy(reinterpret_cast<uint8_t *>(&in) + 16, &b, 16);
    return in;
}

__device__ __forceinline__ void set_error(const KParams &P, uint32_t code, uint32_t instr, uint32_t ctr) {
    if (atomicCAS(&P.state->err, 0u, code) == 0u) {
        P.state->err_cta = blockIdx.x;
        P.state->err_instr = instr;
        P.state->err_ctr = ctr;
        __threadfence();
    }
}

// Acquire-spin until the counter reaches `target` (wrap-safe), bounded by the
// time limit; gives up early when another CTA has already reported an error.
__device__ bool wait_counter(const KParams &P, uint32_t ctr, uint32_t target, uint32_t instr) {
    const uint32_t *p = P.counters + ctr;
    uint64_t t0 = 0;
    for (uint32_t it = 1;; ++it) {
        uint32_t v = ld_acquire_gpu(p);
        if (static_cast<int32_t>(v - target) >= 0) return true;
        if ((it & 15u) == 0u) {
            if (ld_relaxed_gpu(&P.state->err) != 0u) return false;
            uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > P.timeout_ns) {
                set_error(P, 1u, instr, ctr);
                return false;
            }
        }
    }
}

// Bounded wait on a ring barrier; also returns false once the CTA aborts.
__device__ bool wait_bar(const KParams &P, uint64_t *bar, uint32_t parity, volatile int *abort, uint64_t limit_ns) {
    uint64_t t0 = 0;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 7u) == 0u) {
            if (*abort) return false;
            uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > limit_ns) return false;
        }
    }
}

__device__ __forceinline__ int token_of(const KParams &P, int b) {
    int t = P.tokens[(int64_t)b * P.tok_stride];
    return min(max(t, 0), P.vocab - 1);
}

struct MatRef {
    const uint8_t *base;
    int kc, nkb;
};

__device__ __forceinline__ MatRef mat_of(const KParams &P, const Instr &in) {
    MatRef m;
    const LayerW *L = P.layers + in.layer;
    switch (in.op) {
        case OP_QKV: m.base = (const uint8_t *)L->qkv; m.kc = P.qkv_kc; m.nkb = P.qkv_nkb; break;
        case OP_OPROJ: m.base = (const uint8_t *)L->o; m.kc = P.o_kc; m.nkb = P.o_nkb; break;
        case OP_GATEUP: m.base = (const uint8_t *)L->gu; m.kc = P.gu_kc; m.nkb = P.gu_nkb; break;
        case OP_DOWN: m.base = (const uint8_t *)L->down; m.kc = P.down_kc; m.nkb = P.down_nkb; break;
        default: m.base = (const uint8_t *)P.lm_w; m.kc = P.lm_kc; m.nkb = P.lm_nkb; break;
    }
    return m;
}

// Positions of one split-KV unit.  Chunk c of a (sequence, KV head) covers
// [p0, p1) of the C = pos + 1 attended positions; [p0, min(p1, pos)) was
// written by earlier steps and streams through the ring, position `pos` itself
// is produced by this step and handled from registers.
struct AttnGeom {
    int b, g, c, p0, p1, tma_end, nstages;
    bool has_cur;
};

__device__ __forceinline__ AttnGeom attn_geom(const KParams &P, const Instr &in, int pos) {
    AttnGeom a;
    const int unit = (int)in.tile;
    a.c = unit % P.chunks;
    const int bg = unit / P.chunks;
    a.g = bg % P.n_kv_heads;
    a.b = bg / P.n_kv_heads;
    const int C = pos + 1;
    int len = (C + P.chunks - 1) / P.chunks;
    len = (len + 7) & ~7;
    a.p0 = min(a.c * len, C);
    a.p1 = min(C, a.p0 + len);
    a.tma_end = max(a.p0, min(a.p1, pos));
    const int sp = kStageBytes / (4 * P.head_dim);
    a.nstages = (a.tma_end - a.p0 + sp - 1) / sp;
    a.has_cur = (pos >= a.p0 && pos < a.p1);
    return a;
}

__device__ __forceinline__ size_t kv_off(const KParams &P, int l, int b, int g, int p) {
    return ((((size_t)l * P.batch + b) * P.n_kv_heads + g) * (size_t)P.max_seq + p) * P.head_dim;
}

// ------------------------------------------------------------------ producer (one lane)
__device__ void producer(const KParams &P, const SmemLayout &S, int begin, int end, int pos) {
    const uint64_t pol = policy_evict_first();
    int slot = 0;
    uint32_t phase = 0, issued = 0, issued_par = 0;
    const uint64_t limit = 2ull * P.timeout_ns + 1000000ull;
    bool ok = true;
    for (int i = begin; i < end && ok; ++i) {
        const Instr in = load_instr(P, i);
        if (in.op == OP_ATTN) {
            const AttnGeom a = attn_geom(P, in, pos);
            const int d = P.head_dim, sp = kStageBytes / (4 * d);
            const uint16_t *kb = P.kcache + kv_off(P, in.layer, a.b, a.g, 0);
            const uint16_t *vb = P.vcache + kv_off(P, in.layer, a.b, a.g, 0);
            for (int s = 0; s < a.nstages; ++s) {
                const int p = a.p0 + s * sp;
                const int n = min(sp, a.tma_end - p);
                if (!wait_bar(P, &S.empty[slot], phase ^ 1u, S.abort, limit)) { ok = false; break; }
                const uint32_t bytes = (uint32_t)(n * d * 2);
                mbar_arrive_expect_tx(&S.full[slot], 2u * bytes);
                uint8_t *dst = S.ring + (size_t)slot * kStageBytes;
                bulk_g2s(dst, kb + (size_t)p * d, bytes, &S.full[slot], pol);
                bulk_g2s(dst + kStageBytes / 2, vb + (size_t)p * d, bytes, &S.full[slot], pol);
                issued |= 1u << slot;
                issued_par = (issued_par & ~(1u << slot)) | (phase << slot);
                if (++slot == P.stages) { slot = 0; phase ^= 1u; }
            }
        } else {
            const MatRef m = mat_of(P, in);
            const uint32_t bytes = (uint32_t)(kTileRows * m.kc * 2);
            for (int kb = in.kb0; kb < in.kb1; ++kb) {
                if (!wait_bar(P, &S.empty[slot], phase ^ 1u, S.abort, limit)) { ok = false; break; }
                mbar_arrive_expect_tx(&S.full[slot], bytes);
                const uint8_t *src = m.base + ((size_t)in.tile * m.nkb + kb) * bytes;
                bulk_g2s(S.ring + (size_t)slot * kStageBytes, src, bytes, &S.full[slot], pol);
                issued |= 1u << slot;
                issued_par = (issued_par & ~(1u << slot)) | (phase << slot);
                if (++slot == P.stages) { slot = 0; phase ^= 1u; }
            }
        }
    }
    if (!ok && !*S.abort) {
        set_error(P, 3u, (uint32_t)begin, 0u);
        *S.abort = 1;
    }
    // Never leave with a copy into this CTA's shared memory still in flight.
    for (int s = 0; s < P.stages; ++s)
        if (issued & (1u << s)) {
            volatile int never = 0;
            wait_bar(P, &S.full[s], (issued_par >> s) & 1u, &never, limit);
        }
}

// ------------------------------------------------------------------ consumer ring cursor
struct CRing {
    int slot;
    uint32_t phase;
};

__device__ __forceinline__ const uint8_t *c_wait(const KParams &P, const SmemLayout &S, CRing &r) {
    if (!wait_bar(P, &S.full[r.slot], r.phase, S.abort, P.timeout_ns)) {
        if (!*S.abort) set_error(P, 2u, blockIdx.x, 0u);
        *S.abort = 1;
    }
    return S.ring + (size_t)r.slot * kStageBytes;
}

__device__ __forceinline__ void c_release(const KParams &P, const SmemLayout &S, CRing &r) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&S.empty[r.slot]);
    if (++r.slot == P.stages) {
        r.slot = 0;
        r.phase ^= 1u;
    }
}

// ------------------------------------------------------------------ activation staging
// Writes the instruction's activations for batch rows [b0, b0+nb) as bf16
// [nb][klen] into shared memory: RMSNorm(x) * gain for QKV / gate-up / LM head,
// a plain copy of the attention output or of the SwiGLU product otherwise.
template <int BS>
__device__ void stage_act(const KParams &P, const SmemLayout &S, const Instr &in, const MatRef &m, int klen) {
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int nb = in.nb;
    uint16_t *act = reinterpret_cast<uint16_t *>(S.act);
    if (in.op == OP_OPROJ || in.op == OP_DOWN) {
        const uint16_t *src = in.op == OP_OPROJ ? P.attn : P.act_a;
        const int stride = in.op == OP_OPROJ ? P.o_nkb * P.o_kc : P.i_pad;
        const int k0 = in.kb0 * m.kc;
        for (int b = 0; b < nb; ++b) {
            const uint4 *s = reinterpret_cast<const uint4 *>(src + (size_t)(in.b0 + b) * stride + k0);
            uint4 *dst = reinterpret_cast<uint4 *>(act + (size_t)b * klen);
            for (int v = t; v < klen / 8; v += kConsumerThreads) dst[v] = __ldcg(s + v);
        }
        return;
    }
    const int H = P.hidden;
    const uint16_t *gain = reinterpret_cast<const uint16_t *>(
        in.op == OP_QKV ? P.layers[in.layer].attn_norm
                        : (in.op == OP_GATEUP ? P.layers[in.layer].mlp_norm : P.final_norm));
    const bool from_embed = (in.flags & F_EMBED_X) && in.op == OP_QKV;
    // pass 1: sum of squares per row
    float ss[BS];
#pragma unroll
    for (int b = 0; b < BS; ++b) ss[b] = 0.f;
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        if (b < nb) {
            const int row = in.b0 + b;
            if (from_embed) {
                const uint4 *e = reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(P.embed) +
                                                                 (size_t)token_of(P, row) * H);
                for (int v = t; v < H / 8; v += kConsumerThreads) {
                    float f[8];
                    unpack8(__ldg(e + v), f);
#pragma unroll
                    for (int q = 0; q < 8; ++q) ss[b] = fmaf(f[q], f[q], ss[b]);
                }
            } else {
                const float4 *x = reinterpret_cast<const float4 *>(P.x + (size_t)row * H);
                for (int v = t; v < H / 4; v += kConsumerThreads) {
                    float4 f = __ldcg(x + v);
                    ss[b] = fmaf(f.x, f.x, fmaf(f.y, f.y, fmaf(f.z, f.z, fmaf(f.w, f.w, ss[b]))));
                }
            }
        }
    }
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        float s = warp_sum(ss[b]);
        if (lane == 0) S.red[warp * kMaxBatchRows + b] = s;
    }
    consumer_sync();
    if (t < nb) {
        float s = 0.f;
        for (int w = 0; w < kConsumerWarps; ++w) s += S.red[w * kMaxBatchRows + t];
        S.rstd[t] = rsqrtf(s / (float)H + P.rms_eps);
    }
    consumer_sync();
    // pass 2: normalise, apply the gain, round to bf16
    const uint4 *g8 = reinterpret_cast<const uint4 *>(gain);
    for (int b = 0; b < nb; ++b) {
        const int row = in.b0 + b;
        const float r = S.rstd[b];
        uint4 *dst = reinterpret_cast<uint4 *>(act + (size_t)b * klen);
        for (int v = t; v < klen / 8; v += kConsumerThreads) {
            uint4 o = make_uint4(0, 0, 0, 0);
            if (v * 8 < H) {
                float f[8], g[8];
                if (from_embed) {
                    unpack8(__ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(P.embed) +
                                                                  (size_t)token_of(P, row) * H) + v), f);
                } else {
                    const float4 *x = reinterpret_cast<const float4 *>(P.x + (size_t)row * H) + 2 * v;
                    float4 a = __ldcg(x), c = __ldcg(x + 1);
                    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = c.x; f[5] = c.y; f[6] = c.z; f[7] = c.w;
                }
                unpack8(__ldg(g8 + v), g);
                o.x = pack_bf2(f[0] * r * g[0], f[1] * r * g[1]);
                o.y = pack_bf2(f[2] * r * g[2], f[3] * r * g[3]);
                o.z = pack_bf2(f[4] * r * g[4], f[5] * r * g[5]);
                o.w = pack_bf2(f[6] * r * g[6], f[7] * r * g[7]);
            }
            dst[v] = o;
        }
    }
}

// ------------------------------------------------------------------ GEMV over ring blocks
// Block = kTileRows rows x kc columns (CB = kc/8 chunks of 8).  Thread t owns
// chunk c = t % CB and rows rg + NRG*i (rg = t / CB), so one activation chunk
// load serves RPT rows; fp32 accumulation across all K blocks of the tile.
template <int BS, int RPT>
__device__ __forceinline__ void gemv_blocks(const KParams &P, const SmemLayout &S, CRing &ring, const uint8_t *act,
                                            int klen, int nb, int nblocks, float (&acc)[8][BS]) {
    constexpr int CB = RPT * 32;
    constexpr int NRG = 8 / RPT;
    constexpr int KC = CB * 8;
    const int t = threadIdx.x;
    const int c = t % CB, rg = t / CB;
    for (int j = 0; j < nblocks; ++j) {
        const uint8_t *blk = c_wait(P, S, ring);
        float af[BS][8];
#pragma unroll
        for (int b = 0; b < BS; ++b) {
            if (b < nb) {
                uint4 a = *reinterpret_cast<const uint4 *>(act + ((size_t)b * klen + j * KC + c * 8) * 2);
                unpack8(a, af[b]);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) af[b][q] = 0.f;
            }
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = rg + NRG * i;
            uint4 w = *reinterpret_cast<const uint4 *>(blk + ((size_t)r * KC + c * 8) * 2);
            float wf[8];
            unpack8(w, wf);
#pragma unroll
            for (int b = 0; b < BS; ++b)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[i][b] = fmaf(wf[q], af[b][q], acc[i][b]);
        }
        c_release(P, S, ring);
    }
}

template <int BS, int RPT>
__device__ __forceinline__ void reduce_rows(const SmemLayout &S, float (&acc)[8][BS]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int b = 0; b < BS; ++b) {
            float v = warp_sum(acc[i][b]);
            if (lane == 0) S.red[(warp * 8 + i) * kMaxBatchRows + b] = v;
        }
}

// Final dot product of tile row r (0..7), batch row b, after reduce_rows.
__device__ __forceinline__ float row_value(const SmemLayout &S, int kc, int r, int b) {
    const int CB = kc / 8, NRG = 256 / CB, wpr = CB / 32;
    const int rg = r % NRG, i = r / NRG;
    float s = 0.f;
    for (int w = rg * wpr; w < (rg + 1) * wpr; ++w) s += S.red[(w * 8 + i) * kMaxBatchRows + b];
    return s;
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) { return v > bv || (v == bv && i < bi); }

template <int BS>
__device__ void gemv_instr(const KParams &P, const SmemLayout &S, CRing &ring, const Instr &in, uint64_t &act_tag,
                           uint32_t gen, int pos) {
    const int t = threadIdx.x;
    const MatRef m = mat_of(P, in);
    const int nblocks = in.kb1 - in.kb0, klen = nblocks * m.kc, nb = in.nb;
    const uint64_t tag = ((uint64_t)in.op << 56) | ((uint64_t)in.layer << 40) | ((uint64_t)in.b0 << 24) |
                         ((uint64_t)in.kb0 << 12) | (uint64_t)in.kb1;
    if (tag != act_tag) {
        stage_act<BS>(P, S, in, m, klen);
        act_tag = tag;
        consumer_sync();
    }
    float acc[8][BS];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int b = 0; b < BS; ++b) acc[i][b] = 0.f;
    switch (m.kc) {
        case 256: gemv_blocks<BS, 1>(P, S, ring, S.act, klen, nb, nblocks, acc); reduce_rows<BS, 1>(S, acc); break;
        case 512: gemv_blocks<BS, 2>(P, S, ring, S.act, klen, nb, nblocks, acc); reduce_rows<BS, 2>(S, acc); break;
        case 1024: gemv_blocks<BS, 4>(P, S, ring, S.act, klen, nb, nblocks, acc); reduce_rows<BS, 4>(S, acc); break;
        default: gemv_blocks<BS, 8>(P, S, ring, S.act, klen, nb, nblocks, acc); reduce_rows<BS, 8>(S, acc); break;
    }
    consumer_sync();

    const int H = P.hidden;
    switch (in.op) {
        case OP_QKV:
            if (t < 8 * nb) {
                const int r = t & 7, b = t >> 3, n = (int)in.tile * 8 + r;
                if (n < P.qkv_rows) __stcg(P.qkv + (size_t)(in.b0 + b) * P.qkv_rows + n, row_value(S, m.kc, r, b));
            }
            break;
        case OP_OPROJ:
        case OP_DOWN:
            if (t < 8 * nb) {
                const int r = t & 7, b = t >> 3, n = (int)in.tile * 8 + r, row = in.b0 + b;
                if (n < H) {
                    const float v = row_value(S, m.kc, r, b);
                    float *xp = P.x + (size_t)row * H + n;
                    if (in.flags & F_ATOMIC) {
                        atomicAdd(xp, v);
                    } else {
                        float base = (in.flags & F_EMBED_X)
                                         ? bf2f(reinterpret_cast<const uint16_t *>(P.embed)[(size_t)token_of(P, row) * H + n])
                                         : __ldcg(xp);
                        __stcg(xp, base + v);
                    }
                }
            }
            break;
        case OP_GATEUP:
            if (t < 4 * nb) {
                const int r = t & 3, b = t >> 2, j = (int)in.tile * 4 + r;
                if (j < P.intermediate) {
                    const float gt = row_value(S, m.kc, r, b), up = row_value(S, m.kc, r + 4, b);
                    const float a = gt / (1.0f + __expf(-gt)) * up;
                    P.act_a[(size_t)(in.b0 + b) * P.i_pad + j] = f2bf(a);
                }
            }
            break;
        default: {  // OP_LMHEAD
            if (t < 64) {
                const int r = t & 7, b = t >> 3, n = (int)in.tile * 8 + r;
                float v = -CUDART_INF_F;
                int idx = 0x7fffffff;
                if (b < nb && n < P.vocab) {
                    v = row_value(S, m.kc, r, b);
                    idx = n;
                    if (P.logits) __stcg(P.logits + (size_t)(in.b0 + b) * P.vocab + n, v);
                }
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    float ov = __shfl_xor_sync(0xFFFFFFFFu, v, o);
                    int oi = __shfl_xor_sync(0xFFFFFFFFu, idx, o);
                    if (better(ov, oi, v, idx)) { v = ov; idx = oi; }
                }
                if (r == 0 && b < nb) {
                    float2 cur = S.best[in.b0 + b];
                    if (better(v, idx, cur.x, __float_as_int(cur.y))) S.best[in.b0 + b] = make_float2(v, __int_as_float(idx));
                }
            }
            if (in.flags & F_LAST_LM) {
                consumer_sync();
                if (t < P.batch) {
                    float2 cur = S.best[t];
                    LmBest e;
                    e.value = cur.x;
                    e.index = __float_as_int(cur.y);
                    e.gen = gen;
                    e.pad = 0;
                    P.lm_best[(size_t)t * P.n_ctas + blockIdx.x] = e;
                }
                consumer_sync();
                if (t == 0) {
                    __threadfence();
                    uint32_t old = atom_acq_rel_add(P.counters + in.signal_ctr, 1u);
                    *S.flag = (old + 1u == (gen + 1u) * in.arrive_count) ? 1 : 0;
                }
                consumer_sync();
                if (*S.flag) {
                    if (t < P.batch) {
                        float bv = -CUDART_INF_F;
                        int bi = 0x7fffffff;
                        for (int c = 0; c < P.n_ctas; ++c) {
                            const LmBest *e = P.lm_best + (size_t)t * P.n_ctas + c;
                            uint4 raw = __ldcg(reinterpret_cast<const uint4 *>(e));
                            if (raw.z == gen && better(__uint_as_float(raw.x), (int)raw.y, bv, bi)) {
                                bv = __uint_as_float(raw.x);
                                bi = (int)raw.y;
                            }
                        }
                        if (P.next) P.next[t] = bi;
                    }
                    consumer_sync();
                    if (t == 0) {
                        P.state->pos = pos + 1;
                        P.state->gen = gen + 1u;
                        __threadfence();
                    }
                }
            }
        } break;
    }
}

// ------------------------------------------------------------------ attention
// One warp prepares one head: optional per-head RMSNorm, rotate-half RoPE at
// `pos` (angles in double, reduced mod 2*pi before the fp32 sin/cos), scale.
__device__ void prep_head(const KParams &P, const float *src, const uint16_t *gain, int pos, float scale,
                          float *dst, uint16_t *cache_row) {
    const int lane = threadIdx.x & 31, d = P.head_dim, nj = d / 32, jh = nj / 2;
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = j < nj ? __ldcg(src + lane + 32 * j) : 0.f;
    if (gain) {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) s = fmaf(v[j], v[j], s);
        s = warp_sum(s);
        const float r = rsqrtf(s / (float)d + P.rms_eps);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j < nj) v[j] = v[j] * r * bf2f(gain[lane + 32 * j]);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        if (j < jh) {
            const int i = lane + 32 * j;
            double ang = (double)pos * P.rope_inv_freq[i];
            ang -= 6.283185307179586 * rint(ang * 0.15915494309189535);
            float sn, cs;
            sincosf((float)ang, &sn, &cs);
            const float a = v[j], b = v[j + jh];
            v[j] = a * cs - b * sn;
            v[j + jh] = b * cs + a * sn;
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j < nj) {
            float o = v[j];
            if (cache_row) {
                uint16_t h = f2bf(o);
                cache_row[lane + 32 * j] = h;
                o = bf2f(h);
            }
            dst[lane + 32 * j] = o * scale;
        }
    }
}

template <typename T>
__device__ __forceinline__ void load8(const T *p, float *f);
template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t *p, float *f) {
    unpack8(*reinterpret_cast<const uint4 *>(p), f);
}
template <>
__device__ __forceinline__ void load8<float>(const float *p, float *f) {
    float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ float ld1(const uint16_t *p) { return bf2f(*p); }
__device__ __forceinline__ float ld1(const float *p) { return *p; }

// Online-softmax update of the G heads of one KV head with n positions.
template <typename T>
__device__ void attn_block(const KParams &P, const SmemLayout &S, const T *K, const T *V, int n, int G,
                           const float *qs, float *sc, int sp, float (&o)[4]) {
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31, d = P.head_dim, CH = d / 8;
    float *mrun = S.mlc, *lrun = S.mlc + 8, *corr = S.mlc + 16;
    for (int base = 0; base < n * CH; base += kConsumerThreads) {
        const int idx = base + t, j = idx / CH, ch = idx % CH;
        const bool valid = j < n;
        float kf[8];
        if (valid) load8<T>(K + (size_t)j * d + ch * 8, kf);
        else {
#pragma unroll
            for (int q = 0; q < 8; ++q) kf[q] = 0.f;
        }
        float part[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            part[h] = 0.f;
            if (h < G) {
                const float *qh = qs + h * d + ch * 8;
#pragma unroll
                for (int q = 0; q < 8; ++q) part[h] = fmaf(qh[q], kf[q], part[h]);
            }
        }
        for (int off = 1; off < CH; off <<= 1)
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) part[h] += __shfl_xor_sync(0xFFFFFFFFu, part[h], off);
        if (valid && ch == 0)
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h)
                if (h < G) sc[h * sp + j] = part[h];
    }
    consumer_sync();
    if (warp < G) {
        float ml = -CUDART_INF_F;
        for (int j = lane; j < n; j += 32) ml = fmaxf(ml, sc[warp * sp + j]);
        ml = warp_max(ml);
        const float mold = mrun[warp];
        const float mnew = fmaxf(mold, ml);
        float s = 0.f;
        for (int j = lane; j < n; j += 32) {
            const float p = exp2f(sc[warp * sp + j] - mnew);
            sc[warp * sp + j] = p;
            s += p;
        }
        s = warp_sum(s);
        if (lane == 0) {
            const float cf = exp2f(mold - mnew);
            corr[warp] = cf;
            lrun[warp] = lrun[warp] * cf + s;
            mrun[warp] = mnew;
        }
    }
    consumer_sync();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int oi = t + kConsumerThreads * k;
        if (oi < G * d) {
            const int h = oi / d, e = oi % d;
            float acc = o[k] * corr[h];
            const float *ph = sc + h * sp;
            for (int j = 0; j < n; ++j) acc = fmaf(ph[j], ld1(V + (size_t)j * d + e), acc);
            o[k] = acc;
        }
    }
    consumer_sync();
}

__device__ void attn_instr(const KParams &P, const SmemLayout &S, CRing &ring, const Instr &in, uint32_t gen, int pos) {
    const int t = threadIdx.x, warp = t >> 5;
    const int d = P.head_dim, nkv = P.n_kv_heads, G = P.n_heads / nkv, l = in.layer;
    const AttnGeom a = attn_geom(P, in, pos);
    const int sp = kStageBytes / (4 * d);
    float *qs = reinterpret_cast<float *>(S.act);
    float *sc = qs + G * d;
    float *kpos = sc + G * sp;
    float *vpos = kpos + d;
    float *mrun = S.mlc, *lrun = S.mlc + 8;
    const float *qkv_b = P.qkv + (size_t)a.b * P.qkv_rows;
    const LayerW *LW = P.layers + l;
    const float qscale = 1.4426950408889634f * rsqrtf((float)d);  // log2(e)/sqrt(d): scores in the exp2 domain
    if (warp < G) {
        const int h = a.g * G + warp;
        prep_head(P, qkv_b + h * d, P.qk_norm ? reinterpret_cast<const uint16_t *>(LW->q_norm) : nullptr, pos, qscale,
                  qs + warp * d, nullptr);
    }
    if (t < 8) {
        mrun[t] = -CUDART_INF_F;
        lrun[t] = 0.f;
    }
    consumer_sync();
    if (a.has_cur) {
        uint16_t *krow = P.kcache + kv_off(P, l, a.b, a.g, pos);
        uint16_t *vrow = P.vcache + kv_off(P, l, a.b, a.g, pos);
        if (warp == 0) {
            prep_head(P, qkv_b + P.n_heads * d + a.g * d, P.qk_norm ? reinterpret_cast<const uint16_t *>(LW->k_norm) : nullptr,
                      pos, 1.0f, kpos, krow);
        } else if (warp == 1) {
            const float *vs = qkv_b + (P.n_heads + nkv) * d + a.g * d;
            for (int e = t - 32; e < d; e += 32) {
                const uint16_t h = f2bf(__ldcg(vs + e));
                vrow[e] = h;
                vpos[e] = bf2f(h);
            }
        }
        consumer_sync();
    }
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < a.nstages; ++s) {
        const int n = min(sp, a.tma_end - (a.p0 + s * sp));
        const uint8_t *slot = c_wait(P, S, ring);
        attn_block<uint16_t>(P, S, reinterpret_cast<const uint16_t *>(slot),
                             reinterpret_cast<const uint16_t *>(slot + kStageBytes / 2), n, G, qs, sc, sp, o);
        c_release(P, S, ring);
    }
    if (a.has_cur) attn_block<float>(P, S, kpos, vpos, 1, G, qs, sc, sp, o);

    // Partial result of this chunk: unnormalised o, running max m (log2 domain), sum l.
    const int NC = P.chunks, nq = P.n_heads;
    float *part = P.partials;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int oi = t + kConsumerThreads * k;
        if (oi < G * d) {
            const int h = oi / d, e = oi % d, hg = a.g * G + h;
            __stcg(part + (((size_t)a.b * nq + hg) * NC + a.c) * (d + 2) + e, o[k]);
        }
    }
    if (t < G) {
        const int hg = a.g * G + t;
        float *pm = part + (((size_t)a.b * nq + hg) * NC + a.c) * (d + 2) + d;
        __stcg(pm, mrun[t]);
        __stcg(pm + 1, lrun[t]);
    }
    consumer_sync();
    if (t == 0) {
        __threadfence();
        uint32_t old = atom_acq_rel_add(P.counters + in.signal_ctr, 1u);
        *S.flag = (old + 1u == (gen + 1u) * in.arrive_count) ? 1 : 0;
    }
    consumer_sync();
    if (*S.flag) {
        // Last chunk to finish for this (sequence, KV head): log-sum-exp combine.
        const int ostride = P.o_nkb * P.o_kc;
        for (int oi = t; oi < G * d; oi += kConsumerThreads) {
            const int h = oi / d, e = oi % d, hg = a.g * G + h;
            const float *ph = part + ((size_t)a.b * nq + hg) * NC * (d + 2);
            float M = -CUDART_INF_F;
            for (int c = 0; c < NC; ++c) M = fmaxf(M, __ldcg(ph + (size_t)c * (d + 2) + d));
            float Ls = 0.f, Os = 0.f;
            for (int c = 0; c < NC; ++c) {
                const float w = exp2f(__ldcg(ph + (size_t)c * (d + 2) + d) - M);
                Ls = fmaf(w, __ldcg(ph + (size_t)c * (d + 2) + d + 1), Ls);
                Os = fmaf(w, __ldcg(ph + (size_t)c * (d + 2) + e), Os);
            }
            P.attn[(size_t)a.b * ostride + hg * d + e] = f2bf(Os / Ls);
        }
        consumer_sync();
        if (t == 0 && !(in.flags & F_DROP_SIGNAL)) {
            __threadfence();
            red_release_add(P.counters + in.signal2_ctr, 1u);
        }
    }
}

// ------------------------------------------------------------------ consumer loop
template <int BS>
__device__ void consumer(const KParams &P, const SmemLayout &S, int begin, int end, uint32_t gen, int pos) {
    const int t = threadIdx.x;
    CRing ring{0, 0u};
    uint64_t act_tag = ~0ull;
    if (t < 64) S.best[t] = make_float2(-CUDART_INF_F, __int_as_float(0x7fffffff));
    if (P.pdl) pdl_wait();
    consumer_sync();
    for (int i = begin; i < end; ++i) {
        if (*S.abort) break;
        const Instr in = load_instr(P, i);
        if (P.use_waits && in.wait_ctr != kNoCounter) {
            if (t == 0 && !wait_counter(P, in.wait_ctr, (gen + 1u) * in.wait_count, (uint32_t)i)) *S.abort = 1;
            consumer_sync();
            if (*S.abort) break;
        }
        if (in.op == OP_ATTN) {
            attn_instr(P, S, ring, in, gen, pos);
            act_tag = ~0ull;
        } else {
            gemv_instr<BS>(P, S, ring, in, act_tag, gen, pos);
        }
        consumer_sync();
        if (t == 0 && in.op != OP_ATTN && in.op != OP_LMHEAD && !(in.flags & F_DROP_SIGNAL) && !*S.abort) {
            __threadfence();
            red_release_add(P.counters + in.signal_ctr, 1u);
        }
    }
}

template <int BS>
__global__ void __launch_bounds__(kThreads, 1) step_kernel(const __grid_constant__ KParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const SmemLayout S = smem_layout(smem_raw, P);
    const int t = threadIdx.x;
    if (P.pdl) pdl_launch_dependents();
    if (t == 0) {
        for (int s = 0; s < P.stages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], kConsumerWarps);
        }
        *S.abort = 0;
        *S.flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const int begin = P.cta_begin[blockIdx.x], end = P.cta_end[blockIdx.x];
    const uint32_t gen = *reinterpret_cast<volatile const uint32_t *>(&P.state->gen);
    const int pos = *reinterpret_cast<volatile const int32_t *>(&P.state->pos);
    if (t >= kConsumerThreads) {
        if ((t & 31) == 0) producer(P, S, begin, end, pos);
        __syncwarp();
    } else {
        consumer<BS>(P, S, begin, end, gen, pos);
    }
    __syncthreads();
}

// ------------------------------------------------------------------ packing
// dst block (t, kb) row r column col  <-  source row, column kb*kc + col.
// mode 0: source row t*8 + r of src; mode 1 (gate/up): rows r < 4 are gate
// row 4t + r, rows r >= 4 are up row 4t + r - 4.
__global__ void pack_kernel(const uint16_t *src, const uint16_t *src2, uint16_t *dst, int n_rows, int k, int kc,
                            int nkb, int tiles, int mode) {
    const size_t total8 = (size_t)tiles * nkb * kTileRows * kc / 8;
    for (size_t v = (size_t)blockIdx.x * blockDim.x + threadIdx.x; v < total8; v += (size_t)gridDim.x * blockDim.x) {
        const size_t e = v * 8;
        const int col = (int)(e % kc);
        size_t rest = e / kc;
        const int r = (int)(rest % kTileRows);
        rest /= kTileRows;
        const int kb = (int)(rest % nkb);
        const int t = (int)(rest / nkb);
        const int kk = kb * kc + col;
        const uint16_t *s = src;
        int row = t * kTileRows + r;
        if (mode == 1) {
            row = t * 4 + (r & 3);
            s = r < 4 ? src : src2;
        }
        uint16_t out[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) out[q] = (row < n_rows && kk + q < k) ? s[(size_t)row * k + kk + q] : (uint16_t)0;
        *reinterpret_cast<uint4 *>(dst + e) = *reinterpret_cast<uint4 *>(out);
    }
}

// ------------------------------------------------------------------ host launchers
template <int BS>
static cudaError_t launch_bs(const KParams &P, int n_ctas, cudaStream_t s, bool cooperative, bool pdl_attr) {
    const int smem = smem_bytes(P);
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(step_kernel<BS>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (cooperative) {
        attr[na].id = cudaLaunchAttributeCooperative;
        attr[na].val.cooperative = 1;
        ++na;
    }
    if (pdl_attr) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, step_kernel<BS>, P);
}

const void *step_kernel_func(int bs) {
    if (bs <= 1) return reinterpret_cast<const void *>(step_kernel<1>);
    if (bs <= 2) return reinterpret_cast<const void *>(step_kernel<2>);
    if (bs <= 4) return reinterpret_cast<const void *>(step_kernel<4>);
    return reinterpret_cast<const void *>(step_kernel<8>);
}

cudaError_t launch_step(const KParams &P, int bs, int n_ctas, cudaStream_t s, bool cooperative, bool pdl_attr) {
    if (bs <= 1) return launch_bs<1>(P, n_ctas, s, cooperative, pdl_attr);
    if (bs <= 2) return launch_bs<2>(P, n_ctas, s, cooperative, pdl_attr);
    if (bs <= 4) return launch_bs<4>(P, n_ctas, s, cooperative, pdl_attr);
    return launch_bs<8>(P, n_ctas, s, cooperative, pdl_attr);
}

__global__ void set_position_kernel(State *state, int pos) { state->pos = pos; }

cudaError_t launch_set_position(State *state, int pos, cudaStream_t s) {
    set_position_kernel<<<1, 1, 0, s>>>(state, pos);
    return cudaGetLastError();
}

cudaError_t launch_pack(const void *src, const void *src2, void *dst, int n_rows, int k, int kc, int nkb, int tiles,
                        int mode, cudaStream_t s) {
    pack_kernel<<<1184, 256, 0, s>>>(static_cast<const uint16_t *>(src), static_cast<const uint16_t *>(src2),
                                     static_cast<uint16_t *>(dst), n_rows, k, kc, nkb, tiles, mode);
    return cudaGetLastError();
}

}  // namespace mk

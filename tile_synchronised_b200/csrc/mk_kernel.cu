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
// [ring: stages x 32 KB][activations: act_bytes][misc: misc_bytes(bs, stages)]
struct SmemLayout {
    uint8_t *ring;
    uint8_t *act;
    uint64_t *full;
    uint64_t *empty;
    volatile int *abort;
    volatile int *flag;
    float *rstd;              // [8] RMSNorm scale per batch row
    float *mlc;               // [24] attention m, l, correction per head
    float *ssq;               // [8 warps][8] sums of squares
    unsigned long long *best; // [64] argmax keys per batch row
    int *rcnt;                // [slots][8] warps that delivered each output
    float *rsum;              // [slots][8 warps][8 rows][bs] per-warp partial dot products
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
    S.mlc = reinterpret_cast<float *>(misc + 192);
    S.ssq = reinterpret_cast<float *>(misc + 320);
    S.best = reinterpret_cast<unsigned long long *>(misc + 576);
    S.rcnt = reinterpret_cast<int *>(misc + 1088);
    S.rsum = reinterpret_cast<float *>(misc + 1536);
    return S;
}

__host__ int smem_bytes(const KParams &P) { return P.stages * kStageBytes + P.act_bytes + misc_bytes(P.bs, P.stages); }

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
        unsigned long long pw = 0;
        if (P.trace) P.trace[8 * (size_t)i + 3] = 0ull;
        if (in.op == OP_ATTN) {
            const AttnGeom a = attn_geom(P, in, pos);
            const int d = P.head_dim, sp = kStageBytes / (4 * d);
            const uint16_t *kb = P.kcache + kv_off(P, in.layer, a.b, a.g, 0);
            const uint16_t *vb = P.vcache + kv_off(P, in.layer, a.b, a.g, 0);
            for (int s = 0; s < a.nstages; ++s) {
                const int p = a.p0 + s * sp;
                const int n = min(sp, a.tma_end - p);
                const unsigned long long w0 = P.trace ? globaltimer_ns() : 0ull;
                if (!wait_bar(P, &S.empty[slot], phase ^ 1u, S.abort, limit)) { ok = false; break; }
                if (P.trace) pw += globaltimer_ns() - w0;
                const uint32_t bytes = (uint32_t)(n * d * 2);
                if (P.trace && s == 0) P.trace[8 * (size_t)i + 3] = globaltimer_ns();
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
                const unsigned long long w0 = P.trace ? globaltimer_ns() : 0ull;
                if (!wait_bar(P, &S.empty[slot], phase ^ 1u, S.abort, limit)) { ok = false; break; }
                if (P.trace) pw += globaltimer_ns() - w0;
                if (P.trace && kb == in.kb0) P.trace[8 * (size_t)i + 3] = globaltimer_ns();
                mbar_arrive_expect_tx(&S.full[slot], bytes);
                const uint8_t *src = m.base + ((size_t)in.tile * m.nkb + kb) * bytes;
                bulk_g2s(S.ring + (size_t)slot * kStageBytes, src, bytes, &S.full[slot], pol);
                issued |= 1u << slot;
                issued_par = (issued_par & ~(1u << slot)) | (phase << slot);
                if (++slot == P.stages) { slot = 0; phase ^= 1u; }
            }
        }
        if (P.trace) {
            P.trace[8 * (size_t)i + 5] = pw;
            P.trace[8 * (size_t)i + 6] = globaltimer_ns();
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
    unsigned long long waited;  // ns spent waiting for ring data (thread 0, tracing only)
};

__device__ __forceinline__ const uint8_t *c_wait(const KParams &P, const SmemLayout &S, CRing &r) {
    if (P.trace && threadIdx.x == 0 && !mbar_try_wait(&S.full[r.slot], r.phase)) {
        const unsigned long long w0 = globaltimer_ns();
        wait_bar(P, &S.full[r.slot], r.phase, S.abort, P.timeout_ns);
        r.waited += globaltimer_ns() - w0;
    }
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
// Writes the instruction's activations for batch rows [b0, b0+nb) as fp32
// [nb][klen] into shared memory: RMSNorm(x) * gain for QKV / gate-up / LM head,
// a plain copy of the attention output or of the SwiGLU product otherwise.
template <int BS>
__device__ void stage_act(const KParams &P, const SmemLayout &S, const Instr &in, const MatRef &m, int klen,
                          float *red) {
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int nb = in.nb;
    float *act = reinterpret_cast<float *>(S.act);
    if (in.op == OP_OPROJ || in.op == OP_DOWN) {
        const float *src = in.op == OP_OPROJ ? P.attn : P.act_a;
        const int stride = in.op == OP_OPROJ ? P.o_nkb * P.o_kc : P.i_pad;
        const int k0 = in.kb0 * m.kc;
        for (int b = 0; b < nb; ++b) {
            const float4 *s = reinterpret_cast<const float4 *>(src + (size_t)(in.b0 + b) * stride + k0);
            float4 *dst = reinterpret_cast<float4 *>(act + (size_t)b * klen);
            for (int v = t; v < klen / 4; v += kConsumerThreads) dst[v] = __ldcg(s + v);
        }
        return;
    }
    const int H = P.hidden;
    const uint16_t *gain = reinterpret_cast<const uint16_t *>(
        in.op == OP_QKV ? P.layers[in.layer].attn_norm
                        : (in.op == OP_GATEUP ? P.layers[in.layer].mlp_norm : P.final_norm));
    const bool from_embed = (in.flags & F_EMBED_X) && in.op == OP_QKV;
    const uint16_t *emb = reinterpret_cast<const uint16_t *>(P.embed);
    // pass 1: sum of squares per row
    float ss[BS];
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        ss[b] = 0.f;
        if (b < nb) {
            const int row = in.b0 + b;
            if (from_embed) {
                const uint4 *e = reinterpret_cast<const uint4 *>(emb + (size_t)token_of(P, row) * H);
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
        if (lane == 0) red[warp * BS + b] = s;
    }
    consumer_sync();
    if (t < nb) {
        float s = 0.f;
        for (int w = 0; w < kConsumerWarps; ++w) s += red[w * BS + t];
        S.rstd[t] = rsqrtf(s / (float)H + P.rms_eps);
    }
    consumer_sync();
    // pass 2: normalise and apply the gain (fp32)
    const uint4 *g8 = reinterpret_cast<const uint4 *>(gain);
    for (int b = 0; b < nb; ++b) {
        const int row = in.b0 + b;
        const float r = S.rstd[b];
        float4 *dst = reinterpret_cast<float4 *>(act + (size_t)b * klen);
        for (int v = t; v < klen / 8; v += kConsumerThreads) {
            float4 o0 = make_float4(0.f, 0.f, 0.f, 0.f), o1 = o0;
            if (v * 8 < H) {
                float f[8], g[8];
                if (from_embed) {
                    unpack8(__ldg(reinterpret_cast<const uint4 *>(emb + (size_t)token_of(P, row) * H) + v), f);
                } else {
                    const float4 *x = reinterpret_cast<const float4 *>(P.x + (size_t)row * H) + 2 * v;
                    float4 a = __ldcg(x), c = __ldcg(x + 1);
                    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = c.x; f[5] = c.y; f[6] = c.z; f[7] = c.w;
                }
                unpack8(__ldg(g8 + v), g);
                o0 = make_float4(f[0] * r * g[0], f[1] * r * g[1], f[2] * r * g[2], f[3] * r * g[3]);
                o1 = make_float4(f[4] * r * g[4], f[5] * r * g[5], f[6] * r * g[6], f[7] * r * g[7]);
            }
            dst[2 * v] = o0;
            dst[2 * v + 1] = o1;
        }
    }
}

// ------------------------------------------------------------------ GEMV over ring blocks
// Block = kTileRows rows x KC columns (CB = KC/8 chunks of 8).  Thread t owns
// chunk c = t % CB and rows rg + NRG*i (rg = t / CB), so one activation chunk
// load serves RPT rows; fp32 accumulation across all K blocks of the tile.
template <int BS, int RPT>
__device__ __forceinline__ void gemv_blocks(const KParams &P, const SmemLayout &S, CRing &ring, const float *act,
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
                const float4 *a4 = reinterpret_cast<const float4 *>(act + (size_t)b * klen + j * KC + c * 8);
                const float4 x0 = a4[0], x1 = a4[1];
                af[b][0] = x0.x; af[b][1] = x0.y; af[b][2] = x0.z; af[b][3] = x0.w;
                af[b][4] = x1.x; af[b][5] = x1.y; af[b][6] = x1.z; af[b][7] = x1.w;
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) af[b][q] = 0.f;
            }
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = rg + NRG * i;
            const uint4 w = *reinterpret_cast<const uint4 *>(blk + ((size_t)r * KC + c * 8) * 2);
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

// Fold N per-lane values across lanes `o` apart: each lane keeps half of them
// (the upper half when its `o` bit is set), added to its partner's copy.
template <int N>
__device__ __forceinline__ void fold_rows(float *v, int lane, int o) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        const float send = upper ? v[i] : v[i + N / 2];
        const float keep = upper ? v[i + N / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) { return v > bv || (v == bv && i < bi); }

// (value, index) as one 64-bit key whose unsigned order is "larger value,
// then lower index": the sign-flipped float bits above the inverted index.
__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}
__device__ __forceinline__ float key_value(unsigned long long k) {
    uint32_t u = (uint32_t)(k >> 32);
    u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
    return __uint_as_float(u);
}
__device__ __forceinline__ int key_index(unsigned long long k) { return (int)(0xFFFFFFFFu - (uint32_t)k); }

// Epilogue of one finished output (tile row r, or gate/up pair r) for all
// batch rows: v0 = the row's dot products, v1 = the up row's for gate/up.
template <int BS>
__device__ void gemv_epilogue(const KParams &P, const SmemLayout &S, const Instr &in, int r, const float (&v0)[BS],
                              const float (&v1)[BS]) {
    const int H = P.hidden, nb = in.nb;
    switch (in.op) {
        case OP_QKV: {
            const int n = (int)in.tile * 8 + r;
            if (n < P.qkv_rows)
#pragma unroll
                for (int b = 0; b < BS; ++b)
                    if (b < nb) __stcg(P.qkv + (size_t)(in.b0 + b) * P.qkv_rows + n, v0[b]);
        } break;
        case OP_OPROJ:
        case OP_DOWN: {
            const int n = (int)in.tile * 8 + r;
            if (n < H)
#pragma unroll
                for (int b = 0; b < BS; ++b) {
                    if (b >= nb) break;
                    const int row = in.b0 + b;
                    float *xp = P.x + (size_t)row * H + n;
                    if (in.flags & F_ATOMIC) {
                        atomicAdd(xp, v0[b]);
                    } else {
                        const float base =
                            (in.flags & F_EMBED_X)
                                ? bf2f(reinterpret_cast<const uint16_t *>(P.embed)[(size_t)token_of(P, row) * H + n])
                                : __ldcg(xp);
                        __stcg(xp, base + v0[b]);
                    }
                }
        } break;
        case OP_GATEUP: {
            const int j = (int)in.tile * 4 + r;
            if (j < P.intermediate)
#pragma unroll
                for (int b = 0; b < BS; ++b)
                    if (b < nb)
                        __stcg(P.act_a + (size_t)(in.b0 + b) * P.i_pad + j, v0[b] / (1.0f + __expf(-v0[b])) * v1[b]);
        } break;
        default: {  // OP_LMHEAD
            const int n = (int)in.tile * 8 + r;
            if (n < P.vocab)
#pragma unroll
                for (int b = 0; b < BS; ++b) {
                    if (b >= nb) break;
                    if (P.logits) __stcg(P.logits + (size_t)(in.b0 + b) * P.vocab + n, v0[b]);
                    atomicMax(S.best + in.b0 + b, argmax_key(v0[b], n));
                }
        } break;
    }
}

// One GEMV tile.  No CTA-wide barrier on the common path: each warp folds its
// row partials and stores them in its own entries of rotating slot q; the
// warp whose store completes a row (or gate/up pair), counted with a
// shared-memory atomic, adds the row's partials in fixed warp order -- so the
// result does not depend on which warp came last -- and runs the epilogue.
// Warps run ahead of each other by at most the ring depth, fewer instructions
// than there are slots.
template <int BS, int RPT>
__device__ __forceinline__ void gemv_tile(const KParams &P, const SmemLayout &S, CRing &ring, const Instr &in,
                                          const MatRef &m, int nblocks, int klen, int q) {
    constexpr int NRG = 8 / RPT;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    float acc[8][BS];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int b = 0; b < BS; ++b) acc[i][b] = 0.f;
    gemv_blocks<BS, RPT>(P, S, ring, reinterpret_cast<const float *>(S.act), klen, in.nb, nblocks, acc);
    // warp sums of the RPT rows: log2(RPT) folding steps, then plain butterflies
    float v[BS];
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        float w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = acc[i][b];
        int o = 16;
        if constexpr (RPT >= 8) { fold_rows<8>(w, lane, o); o >>= 1; }
        if constexpr (RPT >= 4) { fold_rows<4>(w, lane, o); o >>= 1; }
        if constexpr (RPT >= 2) { fold_rows<2>(w, lane, o); o >>= 1; }
        for (; o >= 1; o >>= 1) w[0] += __shfl_xor_sync(0xFFFFFFFFu, w[0], o);
        v[b] = w[0];
    }
    int fi = 0;
    if constexpr (RPT == 8) fi = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
    if constexpr (RPT == 4) fi = ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
    if constexpr (RPT == 2) fi = (lane >> 4) & 1;
    if ((lane & (32 / RPT - 1)) != 0) return;
    const int rg = warp / RPT;
    const int r = rg + NRG * fi;  // the tile row whose warp sum this lane holds
    float *part = S.rsum + (size_t)q * 64 * BS;  // [warp][row][b]
    volatile float *vpart = part;
#pragma unroll
    for (int b = 0; b < BS; ++b) vpart[(warp * 8 + r) * BS + b] = v[b];
    __threadfence_block();
    const bool pair = in.op == OP_GATEUP;
    const int ci = pair ? (r & 3) : r;
    int *cnt = S.rcnt + q * 8;
    if (atomicAdd(cnt + ci, 1) != (pair ? 2 * RPT : RPT) - 1) return;
    __threadfence_block();
    cnt[ci] = 0;
    const int r0 = ci;
    float v0[BS], v1[BS];
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        v0[b] = 0.f;
        v1[b] = 0.f;
    }
    // row x was delivered by the RPT warps of its row group x % NRG, in warp order
    const int w0 = (r0 % NRG) * RPT, w1 = ((r0 + 4) % NRG) * RPT;
#pragma unroll
    for (int k = 0; k < RPT; ++k)
#pragma unroll
        for (int b = 0; b < BS; ++b) {
            v0[b] += vpart[((w0 + k) * 8 + r0) * BS + b];
            if (pair) v1[b] += vpart[((w1 + k) * 8 + r0 + 4) * BS + b];
        }
    gemv_epilogue<BS>(P, S, in, r0, v0, v1);
}

template <int BS>
__device__ void gemv_instr(const KParams &P, const SmemLayout &S, CRing &ring, const Instr &in, uint64_t &act_tag,
                           uint32_t gen, int pos, int q) {
    const int t = threadIdx.x;
    const MatRef m = mat_of(P, in);
    const int nblocks = in.kb1 - in.kb0, klen = nblocks * m.kc;
    const uint64_t tag = ((uint64_t)in.op << 56) | ((uint64_t)in.layer << 40) | ((uint64_t)in.b0 << 24) |
                         ((uint64_t)in.kb0 << 12) | (uint64_t)in.kb1;
    if (tag != act_tag) {
        consumer_sync();  // no warp still reads the previous activations
        stage_act<BS>(P, S, in, m, klen, S.ssq);
        act_tag = tag;
        consumer_sync();
    }
    switch (m.kc) {
        case 256: gemv_tile<BS, 1>(P, S, ring, in, m, nblocks, klen, q); break;
        case 512: gemv_tile<BS, 2>(P, S, ring, in, m, nblocks, klen, q); break;
        case 1024: gemv_tile<BS, 4>(P, S, ring, in, m, nblocks, klen, q); break;
        default: gemv_tile<BS, 8>(P, S, ring, in, m, nblocks, klen, q); break;
    }
    if (in.op == OP_LMHEAD && (in.flags & F_LAST_LM)) {
        consumer_sync();  // every row of every LM tile of this CTA is folded into best[]
        if (t < P.batch) {
            const unsigned long long k = S.best[t];
            LmBest e;
            e.value = key_value(k);
            e.index = key_index(k);
            e.gen = gen;
            e.pad = 0;
            P.lm_best[(size_t)t * P.n_ctas + blockIdx.x] = e;
        }
        consumer_sync();
        if (t == 0) {
            __threadfence();
            const uint32_t old = atom_acq_rel_add(P.counters + in.signal_ctr, 1u);
            *S.flag = (old + 1u == (gen + 1u) * in.arrive_count) ? 1 : 0;
        }
        consumer_sync();
        if (*S.flag) {
            if (t < P.batch) {
                float bv = -CUDART_INF_F;
                int bi = 0x7fffffff;
                for (int c = 0; c < P.n_ctas; ++c) {
                    const uint4 raw = __ldcg(reinterpret_cast<const uint4 *>(P.lm_best + (size_t)t * P.n_ctas + c));
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

// Online-softmax update of the G heads of one KV head over n positions from a
// ring slot (bf16 K rows, then V rows 16 KB further), plus, when `extra`, the
// position decoded in this step from fp32 rows kx / vx.
__device__ void attn_block(const KParams &P, const SmemLayout &S, const uint16_t *K, const uint16_t *V, int n,
                           const float *kx, const float *vx, bool extra, int G, const float *qs, float *sc, int scs,
                           float (&o)[4]) {
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31, d = P.head_dim, CH = d / 8;
    float *mrun = S.mlc, *lrun = S.mlc + 8, *corr = S.mlc + 16;
    const int rows = n + (extra ? 1 : 0);
    for (int base = 0; base < rows * CH; base += kConsumerThreads) {
        const int idx = base + t, j = idx / CH, ch = idx % CH;
        float kf[8];
        if (j < n) {
            unpack8(*reinterpret_cast<const uint4 *>(K + (size_t)j * d + ch * 8), kf);
        } else if (j < rows) {
            const float4 a = *reinterpret_cast<const float4 *>(kx + ch * 8);
            const float4 b = *reinterpret_cast<const float4 *>(kx + ch * 8 + 4);
            kf[0] = a.x; kf[1] = a.y; kf[2] = a.z; kf[3] = a.w; kf[4] = b.x; kf[5] = b.y; kf[6] = b.z; kf[7] = b.w;
        } else {
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
            for (int h = 0; h < kMaxGroup; ++h)
                if (h < G) part[h] += __shfl_xor_sync(0xFFFFFFFFu, part[h], off);
        if (j < rows && ch == 0)
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h)
                if (h < G) sc[h * scs + j] = part[h];
    }
    consumer_sync();
    if (warp < G) {
        float *sh = sc + warp * scs;
        float ml = -CUDART_INF_F;
        for (int j = lane; j < rows; j += 32) ml = fmaxf(ml, sh[j]);
        ml = warp_max(ml);
        const float mold = mrun[warp];
        const float mnew = fmaxf(mold, ml);
        float s = 0.f;
        for (int j = lane; j < rows; j += 32) {
            const float p = exp2f(sh[j] - mnew);
            sh[j] = p;
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
            const float *ph = sc + h * scs;
            float acc = o[k] * corr[h];
            float a2 = 0.f;
            int j = 0;
            for (; j + 1 < n; j += 2) {
                acc = fmaf(ph[j], bf2f(V[(size_t)j * d + e]), acc);
                a2 = fmaf(ph[j + 1], bf2f(V[(size_t)(j + 1) * d + e]), a2);
            }
            for (; j < n; ++j) acc = fmaf(ph[j], bf2f(V[(size_t)j * d + e]), acc);
            if (extra) acc = fmaf(ph[n], vx[e], acc);
            o[k] = acc + a2;
        }
    }
    consumer_sync();
}

__device__ bool attn_instr(const KParams &P, const SmemLayout &S, CRing &ring, const Instr &in, uint32_t gen, int pos) {
    const int t = threadIdx.x, warp = t >> 5;
    const int d = P.head_dim, nkv = P.n_kv_heads, G = P.n_heads / nkv, l = in.layer;
    const int NC = P.chunks, nq = P.n_heads;
    const AttnGeom a = attn_geom(P, in, pos);
    const int sp = kStageBytes / (4 * d);
    float *qs = reinterpret_cast<float *>(S.act);  // [G][d] rotated, scaled queries
    const int scs = score_stride(d);
    float *sc = qs + G * d;                         // [G][scs] scores / probabilities
    float *kpos = sc + G * scs;                     // [d] key of this step's position
    float *vpos = kpos + d;                         // [d] value of this step's position
    float *mrun = S.mlc, *lrun = S.mlc + 8;
    const float *qkv_b = P.qkv + (size_t)a.b * P.qkv_rows;
    const LayerW *LW = P.layers + l;
    const float qscale = 1.4426950408889634f * rsqrtf((float)d);  // log2(e)/sqrt(d): scores in the exp2 domain
    consumer_sync();  // the previous instruction's readers of the activation region are done
    if (warp < G) {
        const int h = a.g * G + warp;
        prep_head(P, qkv_b + h * d, P.qk_norm ? reinterpret_cast<const uint16_t *>(LW->q_norm) : nullptr, pos, qscale,
                  qs + warp * d, nullptr);
    } else if (a.has_cur && warp == G) {
        prep_head(P, qkv_b + nq * d + a.g * d, P.qk_norm ? reinterpret_cast<const uint16_t *>(LW->k_norm) : nullptr,
                  pos, 1.0f, kpos, P.kcache + kv_off(P, l, a.b, a.g, pos));
    }
    if (a.has_cur && warp == kConsumerWarps - 1) {
        // with G == 8 every warp holds a query head; the key then follows below
        const float *vs = qkv_b + (nq + nkv) * d + a.g * d;
        uint16_t *vrow = P.vcache + kv_off(P, l, a.b, a.g, pos);
        for (int e = t & 31; e < d; e += 32) {
            const uint16_t h = f2bf(__ldcg(vs + e));
            vrow[e] = h;
            vpos[e] = bf2f(h);
        }
    }
    if (t < 8) {
        mrun[t] = -CUDART_INF_F;
        lrun[t] = 0.f;
    }
    consumer_sync();
    if (a.has_cur && G == kConsumerWarps) {
        if (warp == 0)
            prep_head(P, qkv_b + nq * d + a.g * d, P.qk_norm ? reinterpret_cast<const uint16_t *>(LW->k_norm) : nullptr,
                      pos, 1.0f, kpos, P.kcache + kv_off(P, l, a.b, a.g, pos));
        consumer_sync();
    }
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < a.nstages; ++s) {
        const int n = min(sp, a.tma_end - (a.p0 + s * sp));
        const uint8_t *slot = c_wait(P, S, ring);
        const bool last = s == a.nstages - 1;
        attn_block(P, S, reinterpret_cast<const uint16_t *>(slot), reinterpret_cast<const uint16_t *>(slot + kStageBytes / 2),
                   n, kpos, vpos, last && a.has_cur, G, qs, sc, scs, o);
        c_release(P, S, ring);
    }
    if (a.nstages == 0 && a.has_cur) attn_block(P, S, nullptr, nullptr, 0, kpos, vpos, true, G, qs, sc, scs, o);

    // Partial result of this chunk: unnormalised o, running max m (log2 domain), sum l.
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
        const uint32_t old = atom_acq_rel_add(P.counters + in.signal_ctr, 1u);
        *S.flag = (old + 1u == (gen + 1u) * in.arrive_count) ? 1 : 0;
    }
    consumer_sync();
    if (*S.flag) {
        // Last chunk to finish for this (sequence, KV head): log-sum-exp combine.
        // The group's partials are one contiguous [G][NC][d + 2] range: gather it
        // into shared memory with independent loads, then reduce there.
        float *co = reinterpret_cast<float *>(S.act);  // [G][NC][d]
        float *cm = co + G * NC * d;                    // [G][NC] chunk maxima -> weights
        float *cl = cm + G * NC;                        // [G][NC] chunk sums; cl[h*NC] <- 1 / L
        const float *src = part + ((size_t)a.b * nq + a.g * G) * NC * (d + 2);
        const int total = G * NC * (d + 2);
#pragma unroll 4
        for (int i = t; i < total; i += kConsumerThreads) {
            const float val = __ldcg(src + i);
            const int hc = i / (d + 2), e = i % (d + 2);
            if (e < d) co[hc * d + e] = val;
            else if (e == d) cm[hc] = val;
            else cl[hc] = val;
        }
        consumer_sync();
        if (t < G) {  // per head: M = max_c m_c, w_c = 2^(m_c - M), L = sum_c w_c l_c
            float M = -CUDART_INF_F;
            for (int c = 0; c < NC; ++c) M = fmaxf(M, cm[t * NC + c]);
            float L = 0.f;
            for (int c = 0; c < NC; ++c) {
                const float w = exp2f(cm[t * NC + c] - M);
                cm[t * NC + c] = w;
                L = fmaf(w, cl[t * NC + c], L);
            }
            cl[t * NC] = 1.0f / L;
        }
        consumer_sync();
        const int ostride = P.o_nkb * P.o_kc;
        for (int oi = t; oi < G * d; oi += kConsumerThreads) {
            const int h = oi / d, e = oi % d, hg = a.g * G + h;
            const float *ph = co + (size_t)h * NC * d + e;
            float acc = 0.f;
            for (int c = 0; c < NC; ++c) acc = fmaf(cm[h * NC + c], ph[(size_t)c * d], acc);
            __stcg(P.attn + (size_t)a.b * ostride + hg * d + e, acc * cl[h * NC]);
        }
        consumer_sync();
        if (t == 0 && !(in.flags & F_DROP_SIGNAL)) red_release_add(P.counters + in.signal2_ctr, 1u);
    }
    return consumer_sync_or(*S.abort != 0);
}

// ------------------------------------------------------------------ consumer loop
// Signals are batched: a CTA adds the number of instructions it finished for a
// counter in one release when it moves on to another counter, and always
// before it blocks on a wait, so it never holds back a signal it (through
// others) might be waiting for.  A wait already satisfied for this step is not
// re-checked.  Every stop decision comes out of an OR-reducing barrier.
template <int BS>
__device__ void consumer(const KParams &P, const SmemLayout &S, int begin, int end, uint32_t gen, int pos) {
    const int t = threadIdx.x;
    CRing ring{0, 0u, 0ull};
    uint64_t act_tag = ~0ull;
    uint32_t sat_ctr = 0xFFFFFFFFu, sat_target = 0u;
    uint32_t pend_ctr = kNoCounter, pend_n = 0u;
    int q = 0;
    bool stop = false;
    if (P.pdl) pdl_wait();
    consumer_sync();
    Instr nxt;
    if (begin < end) nxt = load_instr(P, begin);
    for (int i = begin; i < end && !stop; ++i) {
        const Instr in = nxt;
        if (i + 1 < end) nxt = load_instr(P, i + 1);
        unsigned long long t_start = 0;
        if (P.trace && t == 0) t_start = globaltimer_ns();
        if (P.use_waits && in.wait_ctr != kNoCounter) {
            const uint32_t target = (gen + 1u) * in.wait_count;
            if (in.wait_ctr != sat_ctr || target != sat_target) {
                if (pend_n) consumer_sync();  // this CTA's earlier writes are complete
                if (t == 0) {
                    if (pend_n) red_release_add(P.counters + pend_ctr, pend_n);
                    if (!wait_counter(P, in.wait_ctr, target, (uint32_t)i)) *S.abort = 1;
                }
                pend_n = 0u;
                pend_ctr = kNoCounter;
                if (consumer_sync_or(*S.abort != 0)) break;
                sat_ctr = in.wait_ctr;
                sat_target = target;
            }
        }
        if (P.trace && t == 0) {
            P.trace[8 * (size_t)i + 0] = t_start;
            P.trace[8 * (size_t)i + 1] = globaltimer_ns();
        }
        if (in.op == OP_ATTN) {
            stop = attn_instr(P, S, ring, in, gen, pos);
            act_tag = ~0ull;
        } else {
            gemv_instr<BS>(P, S, ring, in, act_tag, gen, pos, q);
            if (++q == reduce_slots(P.stages)) q = 0;
            if (in.op != OP_LMHEAD && !(in.flags & F_DROP_SIGNAL)) {
                if (pend_ctr != in.signal_ctr) {
                    if (pend_n) {
                        consumer_sync();
                        if (t == 0) red_release_add(P.counters + pend_ctr, pend_n);
                    }
                    pend_ctr = in.signal_ctr;
                    pend_n = 0u;
                }
                ++pend_n;
            }
        }
        if (P.trace && t == 0) {
            P.trace[8 * (size_t)i + 2] = globaltimer_ns();
            P.trace[8 * (size_t)i + 4] = ring.waited;
            ring.waited = 0;
        }
    }
    if (!stop && pend_n) {
        consumer_sync();
        if (t == 0) red_release_add(P.counters + pend_ctr, pend_n);
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
    for (int i = t; i < reduce_slots(P.stages) * 8; i += kThreads) S.rcnt[i] = 0;
    if (t < 64) S.best[t] = argmax_key(-CUDART_INF_F, 0x7fffffff);
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

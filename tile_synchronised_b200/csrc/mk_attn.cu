// mk_attn.cu -- split-KV decode attention with a log-sum-exp combine, as an
// operation of its own (the attention of one layer of one decode step).
//
// The decode step's attention reads every cached K/V position of a sequence
// for a handful of query heads, so one (sequence, KV head) alone cannot keep
// the GPU busy.  The positions are therefore cut into chunks; each CTA turns
// one chunk into an unnormalised partial (o, m, l) for the G query heads that
// share the KV head, and a second kernel combines the chunks:
//     M = max_c m_c,   out = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c
// (scores kept in the base-2 domain).  This is the split-KV attention plus
// LSE combine of the decode step ("Look Ma, No Bubbles! Designing a
// Low-Latency Megakernel for Llama-1B", introduction: one sequence generated
// with Llama-3.2-1B; the megakernel runs the same split inside its
// interpreter).
//
// Layouts: q fp32 [B][nq][d] (already rotated); K/V bf16 [B][nkv][max_seq][d]
// (one layer of the model's KV cache); out fp32 [B][nq][d]; partial records
// fp32 [B][nq][chunks][d + 2] = (o[0..d), m, l).
#include <cuda_runtime.h>
#include <math_constants.h>

#include <atomic>
#include <cstdio>
#include <mutex>

#include "../../include/mk.h"
#include "mk_device.cuh"
#include "mk_kernel.h"

namespace mk {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;

// Positions per shared-memory tile: K and V tiles together take 32 KB
// (16 KB at d = 256), leaving the whole CTA under the 48 KB static limit.
__host__ __device__ constexpr int attn_tile_positions(int d) { return d == 256 ? 16 : 8192 / d; }

__host__ __device__ inline int attn_smem_bytes(int G, int d) {
    return G * d * 4 + 2 * attn_tile_positions(d) * d * 2 + kAttnWarps * (d + 2) * 4;
}

struct AttnArgs {
    const float *q;
    const uint16_t *k, *v;
    float *out, *part;
    int B, nq, nkv, d, max_seq, n_pos, chunks;
    const int *n_pos_dev;  // if set, the attended length is read here (a captured graph's step)
    // if set, row b of q / out is a query of sequence row_seq[b] over its
    // positions 0 .. row_len[b] - 1 (a prefill chunk: several positions of one
    // sequence, each attending causally); else row b is sequence b
    const int *row_seq, *row_len;
    int pdl;  // launch both kernels with programmatic dependent launch (a step's chain of kernels)
    // if set, the combine writes bf16 hi / lo pairs here (rows b and B + b,
    // nq * d wide) instead of fp32 to out
    uint16_t *hilo;
};

// One CTA = one (chunk, KV head, sequence).  Warps split the G heads
// (kAttnWarps / G warps per head, interleaving the tile's positions); each
// keeps an online softmax over its positions with lane l owning dimensions
// l*DPL .. l*DPL + DPL - 1.  The warps' states are merged in shared memory.
template <int DPL>
__global__ void __launch_bounds__(kAttnThreads) attn_partial_kernel(AttnArgs a) {
    pdl_wait();  // no-ops unless launched with programmatic dependent launch
    pdl_launch_dependents();
    constexpr int d = 32 * DPL;
    constexpr int TP = attn_tile_positions(d);
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int G = a.nq / a.nkv;
    const int wph = G >= kAttnWarps ? 1 : kAttnWarps / G;
    const int h = warp / wph, sl = warp % wph;
    const bool active = h < G;
    extern __shared__ __align__(16) uint8_t smem[];
    float *qs = reinterpret_cast<float *>(smem);                    // [G][d], scaled by log2(e)/sqrt(d)
    uint16_t *kt = reinterpret_cast<uint16_t *>(qs + G * d);        // [TP][d]
    uint16_t *vt = kt + TP * d;                                     // [TP][d]
    float *mrg = reinterpret_cast<float *>(vt + TP * d);            // [warps][d + 2]
    const int n_pos = a.row_len ? a.row_len[b] : (a.n_pos_dev ? *a.n_pos_dev : a.n_pos);  // empty chunks write empty records
    const int seq = a.row_seq ? a.row_seq[b] : b;
    const long long p0 = (long long)c * n_pos / a.chunks, p1 = (long long)(c + 1) * n_pos / a.chunks;
    const float qscale = 1.4426950408889634f * rsqrtf((float)d);
    const float *qb = a.q + ((size_t)b * a.nq + (size_t)g * G) * d;
    for (int i = t; i < G * d; i += kAttnThreads) qs[i] = qb[i] * qscale;
    const size_t head = ((size_t)seq * a.nkv + g) * (size_t)a.max_seq;
    float m = -CUDART_INF_F, l = 0.f, o[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[e] = 0.f;
    for (long long t0 = p0; t0 < p1; t0 += TP) {
        const int n = (int)min((long long)TP, p1 - t0);
        __syncthreads();  // the previous tile is consumed (and q is staged)
        const uint4 *ks = reinterpret_cast<const uint4 *>(a.k + (head + t0) * d);
        const uint4 *vs = reinterpret_cast<const uint4 *>(a.v + (head + t0) * d);
        for (int i = t; i < n * d / 8; i += kAttnThreads) {
            reinterpret_cast<uint4 *>(kt)[i] = __ldg(ks + i);
            reinterpret_cast<uint4 *>(vt)[i] = __ldg(vs + i);
        }
        __syncthreads();
        if (active) {
            float qr[DPL];
#pragma unroll
            for (int e = 0; e < DPL; ++e) qr[e] = qs[h * d + lane * DPL + e];
            for (int j = sl; j < n; j += wph) {
                const uint16_t *kr = kt + j * d + lane * DPL;
                const uint16_t *vr = vt + j * d + lane * DPL;
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e) s = fmaf(qr[e], bf2f(kr[e]), s);
                s = warp_sum(s);
                const float mn = fmaxf(m, s);
                const float sc = exp2f(m - mn), p = exp2f(s - mn);
                l = l * sc + p;
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[e] = fmaf(p, bf2f(vr[e]), o[e] * sc);
                m = mn;
            }
        }
    }
    __syncthreads();
    if (active) {
#pragma unroll
        for (int e = 0; e < DPL; ++e) mrg[warp * (d + 2) + lane * DPL + e] = o[e];
        if (lane == 0) {
            mrg[warp * (d + 2) + d] = m;
            mrg[warp * (d + 2) + d + 1] = l;
        }
    }
    __syncthreads();
    for (int i = t; i < G * d; i += kAttnThreads) {
        const int hh = i / d, e = i % d;
        float M = -CUDART_INF_F;
        for (int w = hh * wph; w < (hh + 1) * wph; ++w) M = fmaxf(M, mrg[w * (d + 2) + d]);
        float O = 0.f, L = 0.f;
        if (M != -CUDART_INF_F)
            for (int w = hh * wph; w < (hh + 1) * wph; ++w) {
                const float mw = mrg[w * (d + 2) + d];
                if (mw == -CUDART_INF_F) continue;
                const float f = exp2f(mw - M);
                O = fmaf(f, mrg[w * (d + 2) + e], O);
                L = fmaf(f, mrg[w * (d + 2) + d + 1], L);
            }
        float *rec = a.part + (((size_t)b * a.nq + (size_t)g * G + hh) * a.chunks + c) * (d + 2);
        rec[e] = O;
        if (e == 0) {
            rec[d] = M;
            rec[d + 1] = L;
        }
    }
}

// Raise a kernel's dynamic shared-memory limit once per device (bit d of
// `done` records device d).
static cudaError_t allow_smem(const void *fn, int bytes, std::atomic<unsigned long long> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// ------------------------------------------------------------------ tiles through a TMA ring
// The same partials for head_dim 64 and 128 and G = 8 query heads per KV head
// (attn_wide_kernel below serves G = 2 and 4 with the same ring and
// records), with the cache streamed by 1-D bulk copies (TMA) through a ring of
// kTileStages shared-memory stages, so that the next tiles are in flight
// while one is consumed.  A stage holds the K rows and then the V rows of
// kTileBytes / (2 d) consecutive positions.
//
// Every warp serves all G heads, so each K and V row is read from shared
// memory once per CTA.  Lane l owns dimensions l*DPL .. l*DPL + DPL - 1 and
// keeps q and the output of every head for them in registers.  A warp takes
// 32 / G positions at a time (32 (position, head) pairs): each lane forms its
// partial dot products for all 32 pairs, and a transposing butterfly over the
// lanes (16 + 8 + 4 + 2 + 1 shuffles) leaves lane l with the whole score of
// pair l (position l / G, head l % G).  The online softmax runs on those
// lanes; the probabilities go through shared memory to the lanes that apply
// them to the V rows.  The eight warps take alternate groups of positions and
// merge at the end, through the drained ring.
constexpr int kTileStages = 3;
constexpr int kTileBytes = 16384;  // one stage's K rows; its V rows as many

__host__ __device__ inline int attn_tile_smem_bytes() {
    return kTileStages * 2 * kTileBytes + kAttnWarps * 40 * 4 + kTileStages * 8;
}

__device__ __forceinline__ void load_bf16_row_part(const uint16_t *p, float *f, int n) {
    if (n == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        f[0] = __uint_as_float(u.x << 16);
        f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16);
        f[3] = __uint_as_float(u.y & 0xffff0000u);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
        f[0] = __uint_as_float(u << 16);
        f[1] = __uint_as_float(u & 0xffff0000u);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kAttnThreads, 2) attn_tile_kernel(AttnArgs a) {
    pdl_wait();  // no-ops unless launched with programmatic dependent launch
    pdl_launch_dependents();
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(G == 2 || G == 4 || G == 8, "query heads per KV head");
    constexpr int TP = kTileBytes / (2 * D);  // positions per stage
    constexpr int DPL = D / 32;               // dimensions per lane
    constexpr int P = 32 / G;                 // positions per warp group
    constexpr unsigned FULL = 0xffffffffu;
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t *ring = smem;                                                            // [stages][K | V]
    float *pw = reinterpret_cast<float *>(smem + kTileStages * 2 * kTileBytes) + warp * 40;  // [32] p, [8] corr
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kTileStages * 2 * kTileBytes + kAttnWarps * 40 * 4);
    const int n_pos = a.row_len ? a.row_len[b] : (a.n_pos_dev ? *a.n_pos_dev : a.n_pos);  // empty chunks write empty records
    const int seq = a.row_seq ? a.row_seq[b] : b;
    const int p0 = (int)((long long)c * n_pos / a.chunks), p1 = (int)((long long)(c + 1) * n_pos / a.chunks);
    const int ntiles = p1 > p0 ? (p1 - p0 + TP - 1) / TP : 0;
    const size_t head = ((size_t)seq * a.nkv + g) * (size_t)a.max_seq;
    if (t == 0) {
        for (int s = 0; s < kTileStages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncthreads();
    const uint64_t pol = policy_evict_first();
    auto issue = [&](int i) {
        const int s = i % kTileStages, pos = p0 + i * TP, n = min(TP, p1 - pos);
        const uint32_t bytes = (uint32_t)(n * D * 2);
        uint8_t *dst = ring + (size_t)s * 2 * kTileBytes;
        mbar_arrive_expect_tx(&full[s], 2 * bytes);
        bulk_g2s(dst, a.k + (head + pos) * D, bytes, &full[s], pol);
        bulk_g2s(dst + kTileBytes, a.v + (head + pos) * D, bytes, &full[s], pol);
    };
    if (t == 0)
        for (int i = 0; i < ntiles && i < kTileStages; ++i) issue(i);

    // q of the G heads for this lane's dimensions, scaled by log2(e)/sqrt(d)
    const float qscale = 1.4426950408889634f * rsqrtf((float)D);
    float q[G][DPL], o[G][DPL];
    {
        const float *qb = a.q + ((size_t)b * a.nq + (size_t)g * G) * D + lane * DPL;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < DPL; ++e) {
                q[h][e] = qb[h * D + e] * qscale;
                o[h][e] = 0.f;
            }
    }
    float m = -CUDART_INF_F, l = 0.f;  // running max and sum of head lane % G
    bool bad = false;
    int i = 0;
    for (; i < ntiles; ++i) {
        const int s = i % kTileStages;
        const uint32_t par = (uint32_t)(i / kTileStages) & 1u;
        if (!mbar_try_wait(&full[s], par)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(&full[s], par, 10000u))
                if (globaltimer_ns() - t0 > 2000000000ull) {
                    bad = true;
                    break;
                }
        }
        if (!bad) {
            const int n = min(TP, p1 - (p0 + i * TP));
            const uint16_t *K = reinterpret_cast<const uint16_t *>(ring + (size_t)s * 2 * kTileBytes);
            const uint16_t *V = K + kTileBytes / 2;
            for (int base = warp * P; base < n; base += kAttnWarps * P) {
                const int cnt = min(P, n - base);
                float acc[32];
#pragma unroll
                for (int j = 0; j < P; ++j) {
                    float kf[DPL];
                    load_bf16_row_part(K + (size_t)(base + min(j, cnt - 1)) * D + lane * DPL, kf, DPL);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float x = q[h][0] * kf[0];
#pragma unroll
                        for (int e = 1; e < DPL; ++e) x = fmaf(q[h][e], kf[e], x);
                        acc[j * G + h] = x;
                    }
                }
                // transposing butterfly: lane l ends with the full sum of pair l
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) {
                    const bool up = lane & off;
#pragma unroll
                    for (int r = 0; r < off; ++r) {
                        const float send = up ? acc[r] : acc[r + off];
                        const float keep = up ? acc[r + off] : acc[r];
                        acc[r] = keep + __shfl_xor_sync(FULL, send, off);
                    }
                }
                const bool valid = lane / G < cnt;
                const float sc = valid ? acc[0] : -CUDART_INF_F;
                float gm = sc;
#pragma unroll
                for (int off = G; off < 32; off <<= 1) gm = fmaxf(gm, __shfl_xor_sync(FULL, gm, off));
                const float mnew = fmaxf(m, gm);
                const float corr = exp2f(m - mnew);
                const float p = valid ? exp2f(sc - mnew) : 0.f;
                float ps = p;
#pragma unroll
                for (int off = G; off < 32; off <<= 1) ps += __shfl_xor_sync(FULL, ps, off);
                l = l * corr + ps;
                m = mnew;
                pw[lane] = p;
                if (lane < G) pw[32 + lane] = corr;
                __syncwarp();
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float cr = pw[32 + h];
#pragma unroll
                    for (int e = 0; e < DPL; ++e) o[h][e] *= cr;
                }
#pragma unroll
                for (int j = 0; j < P; ++j) {
                    if (j < cnt) {
                        float vf[DPL];
                        load_bf16_row_part(V + (size_t)(base + j) * D + lane * DPL, vf, DPL);
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float pj = pw[j * G + h];
#pragma unroll
                            for (int e = 0; e < DPL; ++e) o[h][e] = fmaf(pj, vf[e], o[h][e]);
                        }
                    }
                }
                __syncwarp();  // pw is rewritten by the next group
            }
        }
        if (__syncthreads_or(bad)) break;  // every warp is done with stage s (or some wait gave up)
        if (t == 0 && i + kTileStages < ntiles) issue(i + kTileStages);
    }
    const bool aborted = i < ntiles;
    if (aborted) {
        // never leave with a copy into this CTA's shared memory in flight
        if (t == 0)
            for (int k = i; k < ntiles && k < i + kTileStages; ++k) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait_sleep(&full[k % kTileStages], (uint32_t)(k / kTileStages) & 1u, 10000u))
                    if (globaltimer_ns() - t0 > 2000000000ull) break;
            }
        for (int x = t; x < G * D; x += kAttnThreads) {
            const int hh = x / D, e = x % D;
            float *rec = a.part + (((size_t)b * a.nq + (size_t)g * G + hh) * a.chunks + c) * (D + 2);
            rec[e] = CUDART_NAN_F;
            if (e == 0) rec[D] = rec[D + 1] = CUDART_NAN_F;
        }
        return;
    }
    // merge the warps through the ring (every copy into it has landed and been read)
    float *mo = reinterpret_cast<float *>(ring);         // [warp][G][D]
    float *ml = mo + kAttnWarps * G * D;                 // [warp][G][2]
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < DPL; ++e) mo[(warp * G + h) * D + lane * DPL + e] = o[h][e];
    if (lane < G) {
        ml[(warp * G + lane) * 2] = m;
        ml[(warp * G + lane) * 2 + 1] = l;
    }
    __syncthreads();
    for (int x = t; x < G * D; x += kAttnThreads) {
        const int hh = x / D, e = x % D;
        float M = -CUDART_INF_F;
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, ml[(w * G + hh) * 2]);
        float O = 0.f, L = 0.f;
        if (M != -CUDART_INF_F)
            for (int w = 0; w < kAttnWarps; ++w) {
                const float mw = ml[(w * G + hh) * 2];
                if (mw == -CUDART_INF_F) continue;
                const float f = exp2f(mw - M);
                O = fmaf(f, mo[(w * G + hh) * D + e], O);
                L = fmaf(f, ml[(w * G + hh) * 2 + 1], L);
            }
        float *rec = a.part + (((size_t)b * a.nq + (size_t)g * G + hh) * a.chunks + c) * (D + 2);
        rec[e] = O;
        if (e == 0) {
            rec[D] = M;
            rec[D + 1] = L;
        }
    }
}

// The same partials with 8 dimensions per lane, for G <= 4: a cache row is
// read by d / 8 lanes (16 bytes each, one load), so a warp reads 32 / (d / 8)
// rows at once (its sub-warps).  Each sub-warp forms the partial dot
// products of its positions for all G heads, and a transposing butterfly
// over its d / 8 lanes leaves lane l of the sub-warp with the whole score of
// pair l (position l / G of the sub-warp, head l % G); the online softmax
// runs over the whole warp as above, each sub-warp applies the probabilities
// of its own positions to their V rows, and the sub-warps' outputs are added
// once at the end.  About two thirds of the instructions of the 4-dimension
// layout per cache byte (that kernel is issue-bound).
template <int D, int G>
__global__ void __launch_bounds__(kAttnThreads, 2) attn_wide_kernel(AttnArgs a) {
    pdl_wait();  // no-ops unless launched with programmatic dependent launch
    pdl_launch_dependents();
    static_assert(D == 64 || D == 128, "head_dim");
    constexpr int TP = kTileBytes / (2 * D);  // positions per stage
    constexpr int LPR = D / 8;                // lanes per cache row
    constexpr int SUBS = 32 / LPR;            // sub-warps (rows read at once)
    static_assert(LPR % G == 0, "G must divide d / 8");
    constexpr int PPS = LPR / G;              // positions per sub-warp per group
    constexpr int P = SUBS * PPS;             // positions per warp per group (32 / G)
    constexpr unsigned FULL = 0xffffffffu;
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31, sub = lane / LPR, li = lane % LPR;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t *ring = smem;
    float *pw = reinterpret_cast<float *>(smem + kTileStages * 2 * kTileBytes) + warp * 40;  // [32] p, [8] corr
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kTileStages * 2 * kTileBytes + kAttnWarps * 40 * 4);
    const int n_pos = a.row_len ? a.row_len[b] : (a.n_pos_dev ? *a.n_pos_dev : a.n_pos);
    const int seq = a.row_seq ? a.row_seq[b] : b;
    const int p0 = (int)((long long)c * n_pos / a.chunks), p1 = (int)((long long)(c + 1) * n_pos / a.chunks);
    const int ntiles = p1 > p0 ? (p1 - p0 + TP - 1) / TP : 0;
    const size_t head = ((size_t)seq * a.nkv + g) * (size_t)a.max_seq;
    if (t == 0) {
        for (int s = 0; s < kTileStages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncthreads();
    const uint64_t pol = policy_evict_first();
    auto issue = [&](int i) {
        const int s = i % kTileStages, pos = p0 + i * TP, n = min(TP, p1 - pos);
        const uint32_t bytes = (uint32_t)(n * D * 2);
        uint8_t *dst = ring + (size_t)s * 2 * kTileBytes;
        mbar_arrive_expect_tx(&full[s], 2 * bytes);
        bulk_g2s(dst, a.k + (head + pos) * D, bytes, &full[s], pol);
        bulk_g2s(dst + kTileBytes, a.v + (head + pos) * D, bytes, &full[s], pol);
    };
    if (t == 0)
        for (int i = 0; i < ntiles && i < kTileStages; ++i) issue(i);

    const float qscale = 1.4426950408889634f * rsqrtf((float)D);
    float q[G][8], o[G][8];
    {
        const float *qb = a.q + ((size_t)b * a.nq + (size_t)g * G) * D + li * 8;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float4 x0 = *reinterpret_cast<const float4 *>(qb + h * D);
            const float4 x1 = *reinterpret_cast<const float4 *>(qb + h * D + 4);
            q[h][0] = x0.x * qscale; q[h][1] = x0.y * qscale; q[h][2] = x0.z * qscale; q[h][3] = x0.w * qscale;
            q[h][4] = x1.x * qscale; q[h][5] = x1.y * qscale; q[h][6] = x1.z * qscale; q[h][7] = x1.w * qscale;
#pragma unroll
            for (int e = 0; e < 8; ++e) o[h][e] = 0.f;
        }
    }
    float m = -CUDART_INF_F, l = 0.f;  // running max and sum of head lane % G
    bool bad = false;
    int i = 0;
    for (; i < ntiles; ++i) {
        const int s = i % kTileStages;
        const uint32_t par = (uint32_t)(i / kTileStages) & 1u;
        if (!mbar_try_wait(&full[s], par)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(&full[s], par, 10000u))
                if (globaltimer_ns() - t0 > 2000000000ull) {
                    bad = true;
                    break;
                }
        }
        if (!bad) {
            const int n = min(TP, p1 - (p0 + i * TP));
            const uint16_t *K = reinterpret_cast<const uint16_t *>(ring + (size_t)s * 2 * kTileBytes);
            const uint16_t *V = K + kTileBytes / 2;
            for (int base = warp * P; base < n; base += kAttnWarps * P) {
                const int cnt = min(P, n - base);
                float acc[LPR];
#pragma unroll
                for (int jj = 0; jj < PPS; ++jj) {
                    const int row = base + min(sub * PPS + jj, cnt - 1);
                    float kf[8];
                    unpack8(*reinterpret_cast<const uint4 *>(K + (size_t)row * D + li * 8), kf);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float x = q[h][0] * kf[0];
#pragma unroll
                        for (int e = 1; e < 8; ++e) x = fmaf(q[h][e], kf[e], x);
                        acc[jj * G + h] = x;
                    }
                }
                // transposing butterfly within the sub-warp: lane li ends with pair li
#pragma unroll
                for (int off = LPR / 2; off >= 1; off >>= 1) {
                    const bool up = li & off;
#pragma unroll
                    for (int r = 0; r < off; ++r) {
                        const float send = up ? acc[r] : acc[r + off];
                        const float keep = up ? acc[r + off] : acc[r];
                        acc[r] = keep + __shfl_xor_sync(FULL, send, off);
                    }
                }
                const int mypos = sub * PPS + li / G;  // this lane's position in the group
                const bool valid = mypos < cnt;
                const float sc = valid ? acc[0] : -CUDART_INF_F;
                float gm = sc;
#pragma unroll
                for (int off = G; off < 32; off <<= 1) gm = fmaxf(gm, __shfl_xor_sync(FULL, gm, off));
                const float mnew = fmaxf(m, gm);
                const float corr = exp2f(m - mnew);
                const float p = valid ? exp2f(sc - mnew) : 0.f;
                float ps = p;
#pragma unroll
                for (int off = G; off < 32; off <<= 1) ps += __shfl_xor_sync(FULL, ps, off);
                l = l * corr + ps;
                m = mnew;
                pw[sub * PPS * G + li] = p;  // index = position * G + head
                if (lane < G) pw[32 + lane] = corr;
                __syncwarp();
                if (__any_sync(FULL, corr != 1.0f)) {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float cr = pw[32 + h];
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[h][e] *= cr;
                    }
                }
#pragma unroll
                for (int jj = 0; jj < PPS; ++jj) {
                    const int pos = sub * PPS + jj;
                    if (pos < cnt) {
                        float vf[8];
                        unpack8(*reinterpret_cast<const uint4 *>(V + (size_t)(base + pos) * D + li * 8), vf);
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float pj = pw[pos * G + h];
#pragma unroll
                            for (int e = 0; e < 8; ++e) o[h][e] = fmaf(pj, vf[e], o[h][e]);
                        }
                    }
                }
                __syncwarp();  // pw is rewritten by the next group
            }
        }
        if (__syncthreads_or(bad)) break;  // every warp is done with stage s (or some wait gave up)
        if (t == 0 && i + kTileStages < ntiles) issue(i + kTileStages);
    }
    if (i < ntiles) {
        // never leave with a copy into this CTA's shared memory in flight
        if (t == 0)
            for (int k = i; k < ntiles && k < i + kTileStages; ++k) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait_sleep(&full[k % kTileStages], (uint32_t)(k / kTileStages) & 1u, 10000u))
                    if (globaltimer_ns() - t0 > 2000000000ull) break;
            }
        for (int x = t; x < G * D; x += kAttnThreads) {
            const int hh = x / D, e = x % D;
            float *rec = a.part + (((size_t)b * a.nq + (size_t)g * G + hh) * a.chunks + c) * (D + 2);
            rec[e] = CUDART_NAN_F;
            if (e == 0) rec[D] = rec[D + 1] = CUDART_NAN_F;
        }
        return;
    }
    // the sub-warps hold the same running max per head: their outputs add
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) o[h][e] += __shfl_xor_sync(FULL, o[h][e], off);
    // merge the warps through the ring (every copy into it has landed and been read)
    float *mo = reinterpret_cast<float *>(ring);  // [warp][G][D]
    float *ml = mo + kAttnWarps * G * D;          // [warp][G][2]
    if (sub == 0)
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) mo[(warp * G + h) * D + li * 8 + e] = o[h][e];
    if (lane < G) {
        ml[(warp * G + lane) * 2] = m;
        ml[(warp * G + lane) * 2 + 1] = l;
    }
    __syncthreads();
    for (int x = t; x < G * D; x += kAttnThreads) {
        const int hh = x / D, e = x % D;
        float M = -CUDART_INF_F;
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, ml[(w * G + hh) * 2]);
        float O = 0.f, L = 0.f;
        if (M != -CUDART_INF_F)
            for (int w = 0; w < kAttnWarps; ++w) {
                const float mw = ml[(w * G + hh) * 2];
                if (mw == -CUDART_INF_F) continue;
                const float f = exp2f(mw - M);
                O = fmaf(f, mo[(w * G + hh) * D + e], O);
                L = fmaf(f, ml[(w * G + hh) * 2 + 1], L);
            }
        float *rec = a.part + (((size_t)b * a.nq + (size_t)g * G + hh) * a.chunks + c) * (D + 2);
        rec[e] = O;
        if (e == 0) {
            rec[D] = M;
            rec[D + 1] = L;
        }
    }
}

template <int D, int G>
static cudaError_t launch_tile(cudaLaunchConfig_t &cfg, const AttnArgs &a) {
    static std::atomic<unsigned long long> configured{0};
    const int smem = attn_tile_smem_bytes();
    cfg.dynamicSmemBytes = (size_t)smem;
    // 8 dimensions per lane where q and the outputs of the G heads fit the
    // registers of two CTAs per SM; 4 per lane for G = 8
    if constexpr (G <= 4) {
        const cudaError_t e = allow_smem(reinterpret_cast<const void *>(attn_wide_kernel<D, G>), smem, configured);
        return e == cudaSuccess ? cudaLaunchKernelEx(&cfg, attn_wide_kernel<D, G>, a) : e;
    } else {
        const cudaError_t e = allow_smem(reinterpret_cast<const void *>(attn_tile_kernel<D, G>), smem, configured);
        return e == cudaSuccess ? cudaLaunchKernelEx(&cfg, attn_tile_kernel<D, G>, a) : e;
    }
}

// One CTA per (query head, sequence), one thread per output dimension.
__global__ void attn_combine_kernel(AttnArgs a) {
    pdl_wait();
    pdl_launch_dependents();
    const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x, d = a.d;
    const float *rec = a.part + ((size_t)b * a.nq + h) * a.chunks * (size_t)(d + 2);
    float M = -CUDART_INF_F;
    for (int c = 0; c < a.chunks; ++c) M = fmaxf(M, rec[(size_t)c * (d + 2) + d]);
    float O = 0.f, L = 0.f;
    for (int c = 0; c < a.chunks; ++c) {
        const float mc = rec[(size_t)c * (d + 2) + d];
        if (mc == -CUDART_INF_F) continue;
        const float f = exp2f(mc - M);
        O = fmaf(f, rec[(size_t)c * (d + 2) + e], O);
        L = fmaf(f, rec[(size_t)c * (d + 2) + d + 1], L);
    }
    const float o = O / L;
    if (a.hilo) {
        const uint16_t hi = f2bf(o);
        a.hilo[((size_t)b * a.nq + h) * d + e] = hi;
        a.hilo[((size_t)(a.B + b) * a.nq + h) * d + e] = f2bf(o - bf2f(hi));
    } else {
        a.out[((size_t)b * a.nq + h) * d + e] = o;
    }
}

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t s) {
    const int G = a.nq / a.nkv;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.chunks, a.nkv, a.B);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = (size_t)attn_smem_bytes(G, a.d);
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = a.pdl ? 1 : 0;
    cudaError_t e;
    if ((a.d == 64 || a.d == 128) && (G == 2 || G == 4 || G == 8)) {
        // the TMA-ring kernel (~97 KB of shared memory, two CTAs per SM)
        if (a.d == 64)
            e = G == 2 ? launch_tile<64, 2>(cfg, a) : G == 4 ? launch_tile<64, 4>(cfg, a) : launch_tile<64, 8>(cfg, a);
        else
            e = G == 2 ? launch_tile<128, 2>(cfg, a) : G == 4 ? launch_tile<128, 4>(cfg, a)
                                                           : launch_tile<128, 8>(cfg, a);
    } else {
        switch (a.d) {
            case 64: e = cudaLaunchKernelEx(&cfg, attn_partial_kernel<2>, a); break;
            case 128: e = cudaLaunchKernelEx(&cfg, attn_partial_kernel<4>, a); break;
            default: e = cudaLaunchKernelEx(&cfg, attn_partial_kernel<8>, a); break;
        }
    }
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(a.nq, a.B);
    cfg.blockDim = dim3(a.d);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, attn_combine_kernel, a);
}

// The decode attention with the attended length read from device memory at
// run time (n_pos_dev, between 1 and max_seq) over a fixed number of chunks,
// for a step that is captured once in a CUDA graph and replayed at every
// position.  `part` holds batch * nq * chunks * (d + 2) floats.
cudaError_t launch_attention_dev(const float *q, const void *k, const void *v, int B, int nq, int nkv, int d,
                                 int max_seq, const int *n_pos_dev, int chunks, float *out, float *part,
                                 cudaStream_t s) {
    AttnArgs a{q, static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(v), out, part, B, nq, nkv, d,
               max_seq, max_seq, chunks, n_pos_dev, nullptr, nullptr, 0};
    return launch_attention(a, s);
}

// Causal attention of `rows` query rows over one layer's cache: row r is a
// query of sequence row_seq[r] over its positions 0 .. row_len[r] - 1 (the
// rows of a prefill chunk), `chunks` split-KV chunks per row.
cudaError_t launch_attention_rows(const float *q, const void *k, const void *v, int rows, int nq, int nkv, int d,
                                  int max_seq, const int *row_seq, const int *row_len, int chunks, float *out,
                                  float *part, cudaStream_t s, bool pdl, void *hilo) {
    AttnArgs a{q, static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(v), out, part, rows, nq, nkv, d,
               max_seq, max_seq, chunks, nullptr, row_seq, row_len, pdl ? 1 : 0, static_cast<uint16_t *>(hilo)};
    return launch_attention(a, s);
}

// ------------------------------------------------------------------ host side
static thread_local char g_op_error[256] = "";

void set_op_error(const char *msg) { snprintf(g_op_error, sizeof(g_op_error), "%s", msg); }
const char *op_error() { return g_op_error[0] ? g_op_error : "null context"; }

int attention_auto_chunks(int B, int nkv, int n_pos, int sms) {
    // about one CTA per SM over the (sequence, KV head) pairs, at least 16 positions per chunk
    int c = sms / (B * nkv);
    if (c < 1) c = 1;
    if (c > 64) c = 64;
    const int by_len = n_pos / 16 > 0 ? n_pos / 16 : 1;
    if (c > by_len) c = by_len;
    // long caches: chunks of at least 512 positions, as many as fill the
    // two-per-SM slots in whole waves (the first count reaching 90 % of its
    // last wave, else the best one)
    const long long pairs = (long long)B * nkv, slots = 2LL * (sms > 0 ? sms : 1);
    const int hi = n_pos / 512 < 64 ? n_pos / 512 : 64;
    int best = 0;
    double best_eff = 0.0;
    for (int k = 1; k <= hi; ++k) {
        const long long ctas = pairs * k, waves = (ctas + slots - 1) / slots;
        const double eff = (double)ctas / (double)(waves * slots);
        if (eff > best_eff + 1e-9) {
            best = k;
            best_eff = eff;
        }
        if (eff >= 0.9) break;
    }
    return best > c ? best : c;
}

// Checks shared by every attention entry point; fills a.chunks when it is 0.
mk_status attention_args(AttnArgs &a, const void *q, const void *k, const void *v, const float *out) {
    char msg[200];
    if (!q || !k || !v || !out) {
        set_op_error("attention: null pointer");
        return MK_ERR_INVALID;
    }
    if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out) & 15u) {
        set_op_error("attention: q, k_cache, v_cache and out must be 16-byte aligned");
        return MK_ERR_INVALID;
    }
    if (a.d != 64 && a.d != 128 && a.d != 256) {
        snprintf(msg, sizeof msg, "attention: head_dim %d not in {64, 128, 256}", a.d);
        set_op_error(msg);
        return MK_ERR_UNSUPPORTED;
    }
    if (a.B < 1 || a.nkv < 1 || a.nq < a.nkv || a.nq % a.nkv || a.nq / a.nkv > kAttnWarps || a.max_seq < 1 ||
        a.n_pos < 1 || a.n_pos > a.max_seq || a.chunks < 0 || a.B > 65535 || a.nkv > 65535 || a.nq > 65535) {
        snprintf(msg, sizeof msg,
                 "attention: bad sizes (batch %d, heads %d/%d, max_seq %d, n_pos %d, chunks %d)", a.B, a.nq, a.nkv,
                 a.max_seq, a.n_pos, a.chunks);
        set_op_error(msg);
        return MK_ERR_INVALID;
    }
    if (a.chunks == 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        a.chunks = attention_auto_chunks(a.B, a.nkv, a.n_pos, sms);
    }
    if (a.chunks > a.n_pos || a.chunks > 65535) {
        snprintf(msg, sizeof msg, "attention: %d chunks for %d positions", a.chunks, a.n_pos);
        set_op_error(msg);
        return MK_ERR_INVALID;
    }
    return MK_OK;
}


}  // namespace mk

using namespace mk;

extern "C" size_t mk_attention_scratch_bytes(int batch, int n_heads, int head_dim, int chunks) {
    if (batch < 1 || n_heads < 1 || head_dim < 1 || chunks < 1) return 0;
    return (size_t)batch * n_heads * chunks * (head_dim + 2) * sizeof(float);
}

extern "C" int mk_attention_chunks(int batch, int n_kv_heads, int n_pos) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (batch < 1 || n_kv_heads < 1 || n_pos < 1) return 0;
    return attention_auto_chunks(batch, n_kv_heads, n_pos, sms);
}

extern "C" mk_status mk_attention_decode(const float *q, const void *k_cache, const void *v_cache, int batch,
                                         int n_heads, int n_kv_heads, int head_dim, int max_seq, int n_pos,
                                         int chunks, float *out, void *scratch, size_t scratch_bytes,
                                         void *stream) {
    AttnArgs a{q, static_cast<const uint16_t *>(k_cache), static_cast<const uint16_t *>(v_cache), out, nullptr,
               batch, n_heads, n_kv_heads, head_dim, max_seq, n_pos, chunks, nullptr, nullptr, nullptr, 0};
    mk_status st = attention_args(a, q, k_cache, v_cache, out);
    if (st != MK_OK) return st;
    const size_t need = mk_attention_scratch_bytes(batch, n_heads, head_dim, a.chunks);
    if (!scratch || ((uintptr_t)scratch & 15u) || scratch_bytes < need) {
        char msg[160];
        snprintf(msg, sizeof msg, "attention: scratch must be 16-byte aligned and hold %zu bytes (got %zu)", need,
                 scratch_bytes);
        set_op_error(msg);
        return MK_ERR_INVALID;
    }
    a.part = static_cast<float *>(scratch);
    cudaError_t e = launch_attention(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        set_op_error(cudaGetErrorString(e));
        return MK_ERR_CUDA;
    }
    return MK_OK;
}

// ------------------------------------------------------------------ no-allocation variant
// The same two kernels with their partials in a fixed array of device memory
// owned by this library, for callers that cannot allocate, or be handed, a
// scratch buffer: code that runs after the caching allocator that owns the
// device's memory has reported it full (an out-of-memory handler that still
// needs attention outputs), code that may not take the allocator's lock
// (callbacks of the allocator itself), and C callers without an allocator of
// their own.  The pages have no counterpart of this entry point.
namespace mk {
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // 4 MiB of partial records
static __device__ __align__(256) float g_noalloc_partials[kNoAllocScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
static std::mutex g_noalloc_mu;
static void *g_noalloc_addr[kMaxDevices];  // device address of g_noalloc_partials, per device ordinal
}  // namespace mk

extern "C" size_t mk_attention_noalloc_limit_bytes(void) { return kNoAllocScratchBytes; }

extern "C" mk_status mk_attention_decode_noalloc(const float *q, const void *k_cache, const void *v_cache, int batch,
                                                 int n_heads, int n_kv_heads, int head_dim, int max_seq, int n_pos,
                                                 int chunks, float *out, void *stream) {
    AttnArgs a{q, static_cast<const uint16_t *>(k_cache), static_cast<const uint16_t *>(v_cache), out, nullptr,
               batch, n_heads, n_kv_heads, head_dim, max_seq, n_pos, chunks, nullptr, nullptr, nullptr, 0};
    const bool auto_chunks = chunks == 0;
    mk_status st = attention_args(a, q, k_cache, v_cache, out);
    if (st != MK_OK) return st;
    char msg[200];
    const size_t per_chunk = mk_attention_scratch_bytes(batch, n_heads, head_dim, 1);
    if (auto_chunks && per_chunk * (size_t)a.chunks > kNoAllocScratchBytes)
        a.chunks = (int)(kNoAllocScratchBytes / per_chunk);  // fewer chunks, if even one fits
    if (a.chunks < 1 || per_chunk * (size_t)a.chunks > kNoAllocScratchBytes) {
        snprintf(msg, sizeof msg,
                 "attention (no-alloc): partials need %zu bytes (batch %d x %d heads x %d chunks x (d + 2) floats), "
                 "above the fixed %zu-byte scratch",
                 per_chunk * (size_t)(a.chunks < 1 ? 1 : a.chunks), batch, n_heads, a.chunks < 1 ? 1 : a.chunks,
                 kNoAllocScratchBytes);
        set_op_error(msg);
        return MK_ERR_INVALID;
    }
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        set_op_error(e != cudaSuccess ? cudaGetErrorString(e) : "attention (no-alloc): device ordinal out of range");
        return e != cudaSuccess ? MK_ERR_CUDA : MK_ERR_UNSUPPORTED;
    }
    void *addr;
    {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        if (!g_noalloc_addr[dev]) {  // first call on this device (which is current): look the array up once
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_partials);
            if (e != cudaSuccess || !p) {
                snprintf(msg, sizeof msg, "attention (no-alloc): cudaGetSymbolAddress: %s",
                         e != cudaSuccess ? cudaGetErrorString(e) : "null address");
                set_op_error(msg);
                return MK_ERR_CUDA;
            }
            g_noalloc_addr[dev] = p;
        }
        addr = g_noalloc_addr[dev];
    }
    a.part = static_cast<float *>(addr);
    e = launch_attention(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        set_op_error(cudaGetErrorString(e));
        return MK_ERR_CUDA;
    }
    return MK_OK;
}

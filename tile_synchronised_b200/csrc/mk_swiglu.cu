// mk_swiglu.cu -- the fused SwiGLU first stage on its own
// ("Deep Kernel Fusion for Transformers", Summary and Key points, "Fusion
// scope"): out = SiLU(x W_gate) * (x W_up) in one kernel, with no
// intermediate written to HBM.
//
// x [B, K] fp16, W_gate / W_up [K, N] fp16 (N contiguous), out [B, N] fp16.
// A CTA owns a slab of kSlab output columns of both matrices and streams the
// slab's K rows once per batch group of up to 8 rows; fp32 accumulation.
//   column-tiled (MK_SWIGLU_COL): one CTA per slab loops over all batch groups,
//       so each weight byte leaves HBM once and later groups re-read it from L2.
//   row-tiled    (MK_SWIGLU_ROW): one CTA per (slab, batch group), so a batch
//       group's activations stay resident while the weights are re-read per group.
// At B <= 8 both are the same single pass.  For B <= 8 (K a multiple of 128,
// N of 128) the column tiling runs instead on the TMA pipeline of
// mk_swiglu_tc.cu, and MK_SWIGLU_TC runs on the tensor cores at any batch
// (rounded up to 16 with zero rows).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <tuple>

#include "../../include/mk.h"
#include "mk_kernel.h"

namespace mk {

constexpr int kSlab = 32;      // output columns per CTA
constexpr int kChunkK = 512;   // K rows of x staged per pass
constexpr int kSwThreads = 256;

template <int BG>
__global__ void __launch_bounds__(kSwThreads) swiglu_kernel(const __half *__restrict__ x, const __half *__restrict__ wg,
                                                            const __half *__restrict__ wu, __half *__restrict__ out,
                                                            int B, int K, int N, int groups_per_cta) {
    __shared__ float xs[BG][kChunkK];
    __shared__ float red[2][8][BG][kSlab];
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int cg = t & 7, ks = t >> 3;  // 8 column groups of 4, 32 K slices
    const int n0 = blockIdx.x * kSlab;
    const int g_first = blockIdx.y * groups_per_cta;
    const int n_groups = (B + BG - 1) / BG;
    for (int grp = g_first; grp < min(n_groups, g_first + groups_per_cta); ++grp) {
        const int b0 = grp * BG, nb = min(BG, B - b0);
        float ag[BG][4], au[BG][4];
#pragma unroll
        for (int b = 0; b < BG; ++b)
#pragma unroll
            for (int q = 0; q < 4; ++q) ag[b][q] = au[b][q] = 0.f;
        for (int k0 = 0; k0 < K; k0 += kChunkK) {
            __syncthreads();
            for (int i = t; i < BG * kChunkK; i += kSwThreads) {
                const int b = i / kChunkK, k = i % kChunkK;
                xs[b][k] = (b < nb && k0 + k < K) ? __half2float(x[(size_t)(b0 + b) * K + k0 + k]) : 0.f;
            }
            __syncthreads();
            const int kend = min(kChunkK, K - k0);
#pragma unroll 8
            for (int kk = ks; kk < kend; kk += 32) {
                const size_t off = (size_t)(k0 + kk) * N + n0 + cg * 4;
                const uint2 g2 = __ldg(reinterpret_cast<const uint2 *>(wg + off));
                const uint2 u2 = __ldg(reinterpret_cast<const uint2 *>(wu + off));
                const float2 g01 = __half22float2(*reinterpret_cast<const __half2 *>(&g2.x));
                const float2 g23 = __half22float2(*reinterpret_cast<const __half2 *>(&g2.y));
                const float2 u01 = __half22float2(*reinterpret_cast<const __half2 *>(&u2.x));
                const float2 u23 = __half22float2(*reinterpret_cast<const __half2 *>(&u2.y));
#pragma unroll
                for (int b = 0; b < BG; ++b) {
                    const float xv = xs[b][kk];
                    ag[b][0] = fmaf(xv, g01.x, ag[b][0]);
                    ag[b][1] = fmaf(xv, g01.y, ag[b][1]);
                    ag[b][2] = fmaf(xv, g23.x, ag[b][2]);
                    ag[b][3] = fmaf(xv, g23.y, ag[b][3]);
                    au[b][0] = fmaf(xv, u01.x, au[b][0]);
                    au[b][1] = fmaf(xv, u01.y, au[b][1]);
                    au[b][2] = fmaf(xv, u23.x, au[b][2]);
                    au[b][3] = fmaf(xv, u23.y, au[b][3]);
                }
            }
        }
        // reduce the 4 K slices inside each warp (lanes 8 apart), then across warps
#pragma unroll
        for (int b = 0; b < BG; ++b)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float g = ag[b][q], u = au[b][q];
                g += __shfl_xor_sync(0xFFFFFFFFu, g, 8);
                g += __shfl_xor_sync(0xFFFFFFFFu, g, 16);
                u += __shfl_xor_sync(0xFFFFFFFFu, u, 8);
                u += __shfl_xor_sync(0xFFFFFFFFu, u, 16);
                if (lane < 8) {
                    red[0][warp][b][cg * 4 + q] = g;
                    red[1][warp][b][cg * 4 + q] = u;
                }
            }
        __syncthreads();
        for (int i = t; i < BG * kSlab; i += kSwThreads) {
            const int b = i / kSlab, col = i % kSlab;
            if (b < nb) {
                float g = 0.f, u = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    g += red[0][w][b][col];
                    u += red[1][w][b][col];
                }
                const float a = g / (1.0f + __expf(-g)) * u;
                out[(size_t)(b0 + b) * N + n0 + col] = __float2half_rn(a);
            }
        }
    }
}

cudaError_t launch_swiglu(const void *x, const void *wg, const void *wu, void *out, int B, int K, int N, int variant,
                          cudaStream_t s) {
    const int BG = B >= 8 ? 8 : (B >= 4 ? 4 : (B >= 2 ? 2 : 1));
    const int n_groups = (B + BG - 1) / BG;
    const int gpc = variant == MK_SWIGLU_ROW ? 1 : n_groups;
    dim3 grid(N / kSlab, (n_groups + gpc - 1) / gpc);
    auto X = static_cast<const __half *>(x);
    auto G = static_cast<const __half *>(wg);
    auto U = static_cast<const __half *>(wu);
    auto O = static_cast<__half *>(out);
    switch (BG) {
        case 1: swiglu_kernel<1><<<grid, kSwThreads, 0, s>>>(X, G, U, O, B, K, N, gpc); break;
        case 2: swiglu_kernel<2><<<grid, kSwThreads, 0, s>>>(X, G, U, O, B, K, N, gpc); break;
        case 4: swiglu_kernel<4><<<grid, kSwThreads, 0, s>>>(X, G, U, O, B, K, N, gpc); break;
        default: swiglu_kernel<8><<<grid, kSwThreads, 0, s>>>(X, G, U, O, B, K, N, gpc); break;
    }
    return cudaGetLastError();
}

}  // namespace mk

using namespace mk;

static std::mutex g_tune_mu;
static std::map<std::tuple<int, int, int>, int> g_tuned;

static bool swiglu_args_ok(const void *x, const void *wg, const void *wu, const void *out, int B, int K, int N) {
    if (!x || !wg || !wu || !out) return false;
    if (B < 1 || B > 64 || K < 64 || N < 64 || K % 64 || N % 64) return false;
    for (const void *p : {x, wg, wu, out})
        if ((uintptr_t)p & 15) return false;
    return true;
}

static cudaError_t run_variant(const void *x, const void *wg, const void *wu, void *out, int B, int K, int N,
                               int variant, cudaStream_t s) {
    if (variant == MK_SWIGLU_TC) return launch_swiglu_tc(x, wg, wu, out, B, K, N, s);
    if (variant == MK_SWIGLU_COL && swiglu_col_tma_supported(B, K, N))
        return launch_swiglu_col_tma(x, wg, wu, out, B, K, N, s);
    return launch_swiglu(x, wg, wu, out, B, K, N, variant, s);
}

extern "C" mk_status mk_swiglu_stage1(const void *x, const void *w_gate, const void *w_up, void *out, int B, int K,
                                      int N, int variant, void *stream) {
    if (!swiglu_args_ok(x, w_gate, w_up, out, B, K, N)) return MK_ERR_INVALID;
    if (variant == MK_SWIGLU_AUTO) {
        std::lock_guard<std::mutex> lk(g_tune_mu);
        auto it = g_tuned.find({B, K, N});
        variant = it != g_tuned.end() ? it->second
                                      : (swiglu_tc_supported(B, K, N) ? MK_SWIGLU_TC
                                                                      : (B <= 8 ? MK_SWIGLU_COL : MK_SWIGLU_ROW));
    }
    if (variant != MK_SWIGLU_ROW && variant != MK_SWIGLU_COL && variant != MK_SWIGLU_TC) return MK_ERR_INVALID;
    if (variant == MK_SWIGLU_TC && !swiglu_tc_supported(B, K, N)) return MK_ERR_UNSUPPORTED;
    cudaError_t e = run_variant(x, w_gate, w_up, out, B, K, N, variant, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}

extern "C" mk_status mk_swiglu_tune(const void *x, const void *w_gate, const void *w_up, void *out, int B, int K,
                                    int N, void *stream, int *chosen, float *us_row, float *us_col, float *us_tc) {
    if (!swiglu_args_ok(x, w_gate, w_up, out, B, K, N)) return MK_ERR_INVALID;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return MK_ERR_CUDA;
    const int reps = 20;
    const int vs[3] = {MK_SWIGLU_ROW, MK_SWIGLU_COL, MK_SWIGLU_TC};
    float us[3] = {0.f, 0.f, 0.f};
    const int nv = swiglu_tc_supported(B, K, N) ? 3 : 2;
    int best = MK_SWIGLU_COL;
    float best_us = 0.f;
    for (int i = 0; i < nv; ++i) {
        if (run_variant(x, w_gate, w_up, out, B, K, N, vs[i], s) != cudaSuccess) return MK_ERR_CUDA;
        cudaEventRecord(e0, s);
        for (int r = 0; r < reps; ++r) run_variant(x, w_gate, w_up, out, B, K, N, vs[i], s);
        cudaEventRecord(e1, s);
        if (cudaEventSynchronize(e1) != cudaSuccess) return MK_ERR_CUDA;
        float ms = 0.f;
        cudaEventElapsedTime(&ms, e0, e1);
        us[i] = ms * 1000.f / reps;
        if (i == 0 || us[i] < best_us) {
            best_us = us[i];
            best = vs[i];
        }
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    {
        std::lock_guard<std::mutex> lk(g_tune_mu);
        g_tuned[{B, K, N}] = best;
    }
    if (chosen) *chosen = best;
    if (us_row) *us_row = us[0];
    if (us_col) *us_col = us[1];
    if (us_tc) *us_tc = us[2];
    return cudaGetLastError() == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}

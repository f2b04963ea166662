// mk_swiglu_tc.cu -- the fused SwiGLU first stage on the 5th-generation tensor
// cores (tcgen05) at any batch up to 128 (rounded up to 16 with zero rows:
// the stage is bound by the weight stream, so the padding costs nothing), and
// the CUDA-core column tiling on the same TMA pipeline for batches up to 8
// ("Deep Kernel Fusion for Transformers", Key points, "Fusion scope": Up and
// Gate GEMMs, SiLU and the product in one kernel).
//
//   out[b][n] = SiLU(sum_k x[b][k] Wg[k][n]) * sum_k x[b][k] Wu[k][n]
//
// A cluster of two CTAs owns 128 output features n0 .. n0+127 and the whole
// batch; each CTA of the pair takes half of K, so twice as many SMs stream
// the weights.  The MMA computes D[m][b] = sum_k W[k][n0+m] x[b][k] with the
// weights as operand A (M = 128, MN-major: n is contiguous in W) and x as
// operand B (N = batch rounded up to 16, K-major), both staged by TMA with
// 128-byte swizzling, fp32 accumulators for gate and up in tensor memory.
// Warp 0 lane 0 issues the TMA loads of a 4..6-stage ring, warp 1 lane 0
// issues the MMAs and commits each stage back to its "empty" barrier.  Then
// the second CTA of the pair reads its accumulators out of tensor memory (one
// row per thread) and stores them into the first CTA's shared memory over the
// cluster; the first adds them to its own and writes SiLU(g) * u as fp16.
// Every barrier wait is bounded; a wait that runs out stops the CTA and its
// outputs are written as NaN so that the failure cannot pass for a result.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/mk.h"
#include "mk_device.cuh"
#include "mk_kernel.h"
#include "mk_tc.cuh"

namespace mk {

constexpr int kTcM = 128;           // output features per CTA (MMA M)
constexpr int kTcBK = 64;           // K per stage: one 128-byte swizzle row of fp16
constexpr int kTcThreads = 128;

constexpr int kTcSplit = 2;         // CTAs per cluster, each on its share of K

struct TcShape {
    int B, K, N, stages;
    int rows;  // batch rows written; the tensor-core form rounds B up to 16 with zero rows
    uint32_t stage_bytes, a_bytes, x_bytes;
    uint32_t tx_bytes;  // bytes the TMA loads of one stage deliver
};

// Instruction descriptor of kind::f16: fp32 accumulate, fp16 A and B, A
// MN-major, B K-major, M = 128, N = batch.
__host__ __device__ constexpr uint32_t tc_idesc(int n) {
    return (1u << 4)                    // D format: F32
           | (0u << 7) | (0u << 10)     // A, B format: F16
           | (1u << 15)                 // A MN-major
           | (0u << 16)                 // B K-major
           | ((uint32_t)(n >> 3) << 17) // N >> 3
           | ((uint32_t)(kTcM >> 4) << 24);
}


__global__ void __launch_bounds__(kTcThreads, 1)
    swiglu_tc_kernel(const __grid_constant__ CUtensorMap map_g, const __grid_constant__ CUtensorMap map_u,
                     const __grid_constant__ CUtensorMap map_x, __half *__restrict__ out, TcShape sh) {
    extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
    // stages start on a 1024-byte boundary (128-byte swizzle atoms)
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int S = sh.stages, B = sh.B;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)S * sh.stage_bytes);
    uint64_t *empty = full + S;
    uint64_t *done = empty + S;
    volatile uint32_t *tmem_base = reinterpret_cast<volatile uint32_t *>(done + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    const uint32_t rank = cluster_rank();
    const int n0 = (blockIdx.x / kTcSplit) * kTcM;
    const int nkb_all = sh.K / kTcBK;
    const int kb_first = (int)rank * nkb_all / kTcSplit, nkb = (int)(rank + 1) * nkb_all / kTcSplit - kb_first;
    const uint32_t ncols = B <= 16 ? 32u : (B <= 32 ? 64u : (B <= 64 ? 128u : 256u));  // gate + up, power of two

    if (t == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {  // the whole warp allocates the accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(const_cast<uint32_t *>(tmem_base))),
                     "r"(ncols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_base;

    if (warp == 0 && lane == 0) {
        // producer: W_gate and W_up as two 64-feature boxes each, x as one box
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % S;
            if (kb >= S && !tc_wait(&empty[s], ((kb / S) - 1) & 1u, abort)) break;
            uint8_t *st = smem + (size_t)s * sh.stage_bytes;
            mbar_arrive_expect_tx(&full[s], sh.tx_bytes);
            const int k0 = (kb_first + kb) * kTcBK;
            tma_load_2d(st, &map_g, n0, k0, &full[s]);
            tma_load_2d(st + sh.a_bytes / 2, &map_g, n0 + 64, k0, &full[s]);
            tma_load_2d(st + sh.a_bytes, &map_u, n0, k0, &full[s]);
            tma_load_2d(st + sh.a_bytes + sh.a_bytes / 2, &map_u, n0 + 64, k0, &full[s]);
            tma_load_2d(st + 2 * sh.a_bytes, &map_x, k0, 0, &full[s]);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer.  A (weights, MN-major): two 64-feature atoms 8 KB apart
        // (LBO), 8 k-rows of 128 B per swizzle group (SBO 1 KB); a K step of
        // 16 is two groups, 2 KB.  B (x, K-major): 8 rows per group (SBO
        // 1 KB); a K step of 16 is 32 bytes along the row.
        const uint32_t idesc = tc_idesc(B);
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % S;
            if (!tc_wait(&full[s], (kb / S) & 1u, abort)) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint8_t *st = smem + (size_t)s * sh.stage_bytes;
#pragma unroll
            for (int ks = 0; ks < kTcBK / 16; ++ks) {
                const uint64_t ag = smem_desc_sw128(st + ks * 2048, sh.a_bytes / 2, 1024);
                const uint64_t au = smem_desc_sw128(st + sh.a_bytes + ks * 2048, sh.a_bytes / 2, 1024);
                const uint64_t bx = smem_desc_sw128(st + 2 * sh.a_bytes + ks * 32, 16, 1024);
                const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
                tc_mma(tmem, ag, bx, idesc, acc);
                tc_mma(tmem + (uint32_t)B, au, bx, idesc, acc);
            }
            tc_commit(&empty[s]);
        }
        tc_commit(done);
    }
    __syncwarp();
    // epilogue: thread t holds row m = t of both accumulators (tensor-memory
    // lane t; warp w may read lanes 32w .. 32w+31)
    const bool ok = tc_wait(done, 0u, abort) && !*abort;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    // The first CTA's stage memory is free once both CTAs are past their
    // final MMA; it then receives the second CTA's accumulators, column-major
    // [2B][128], and its "ok" word after them.
    float *part = reinterpret_cast<float *>(smem);
    volatile int *part_ok = reinterpret_cast<volatile int *>(part + 2 * B * kTcM);
    cluster_sync_all();
    if (rank == 1) {
        const uint32_t remote = cluster_map(part, 0);
        for (int c0 = 0; c0 < 2 * B; c0 += 16) {
            float v[16];
            tmem_ld16(lane_addr + (uint32_t)c0, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) st_cluster_f32(remote + (uint32_t)(((c0 + i) * kTcM + t) * 4), v[i]);
        }
        if (t == 0) st_cluster_f32(cluster_map((const void *)part_ok, 0), ok ? 1.f : 0.f);
    }
    cluster_sync_all();
    if (rank == 0) {
        const bool all_ok = ok && *reinterpret_cast<volatile float *>(part_ok) != 0.f;
        const int n = n0 + t;
        for (int c0 = 0; c0 < B; c0 += 16) {
            float g[16], u[16];
            tmem_ld16(lane_addr + (uint32_t)c0, g);
            tmem_ld16(lane_addr + (uint32_t)(B + c0), u);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float gs = g[i] + part[(c0 + i) * kTcM + t], us = u[i] + part[(B + c0 + i) * kTcM + t];
                const float r = all_ok ? gs / (1.0f + __expf(-gs)) * us : __int_as_float(0x7fc00000);
                if (c0 + i < sh.rows) out[(size_t)(c0 + i) * sh.N + n] = __float2half_rn(r);
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
}

// ------------------------------------------------------------------ column tiling on CUDA cores
// The column-tiled form for small batches (B <= 8): the same cluster pair,
// TMA ring and split of K, but the arithmetic on CUDA cores.  Each of the 256
// threads of the eight compute warps owns a pair of adjacent output columns
// (a 4-byte word of every weight row, so a warp reads 128 consecutive bytes)
// and a quarter of each stage's 64 k-rows; a ninth warp issues the TMA loads.
// The quarters are summed through shared memory at the end.  Each weight byte
// leaves HBM once.
constexpr int kCcWarps = 8;
constexpr int kCcThreads = (kCcWarps + 1) * 32;

template <int BS>
__global__ void __launch_bounds__(kCcThreads, 1)
    swiglu_col_kernel(const __grid_constant__ CUtensorMap map_g, const __grid_constant__ CUtensorMap map_u,
                      const __grid_constant__ CUtensorMap map_x, __half *__restrict__ out, TcShape sh) {
    extern __shared__ __align__(1024) uint8_t cc_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(cc_smem_raw) + 1023) & ~uintptr_t(1023));
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int S = sh.stages, B = sh.B;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)S * sh.stage_bytes);
    uint64_t *empty = full + S;
    volatile int *abort = reinterpret_cast<volatile int *>(empty + S);
    const uint32_t rank = cluster_rank();
    const int n0 = (blockIdx.x / kTcSplit) * kTcM;
    const int nkb_all = sh.K / kTcBK;
    const int kb_first = (int)rank * nkb_all / kTcSplit, nkb = (int)(rank + 1) * nkb_all / kTcSplit - kb_first;
    if (t == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCcWarps);  // one arrival per compute warp
        }
        *abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const int p = t % 64, q = t / 64;  // column pair 2p, 2p+1; k-rows 16q .. 16q+15 of each stage
    float ag[2][BS], au[2][BS];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int b = 0; b < BS; ++b) ag[c][b] = au[c][b] = 0.f;
    bool ok = true;
    if (warp == kCcWarps) {
        if (lane == 0) {
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % S;
                if (kb >= S && !tc_wait(&empty[s], ((kb / S) - 1) & 1u, abort)) break;
                uint8_t *st = smem + (size_t)s * sh.stage_bytes;
                mbar_arrive_expect_tx(&full[s], sh.tx_bytes);
                const int k0 = (kb_first + kb) * kTcBK;
                tma_load_2d(st, &map_g, n0, k0, &full[s]);
                tma_load_2d(st + sh.a_bytes / 2, &map_g, n0 + 64, k0, &full[s]);
                tma_load_2d(st + sh.a_bytes, &map_u, n0, k0, &full[s]);
                tma_load_2d(st + sh.a_bytes + sh.a_bytes / 2, &map_u, n0 + 64, k0, &full[s]);
                tma_load_2d(st + 2 * sh.a_bytes, &map_x, k0, 0, &full[s]);
            }
        }
        __syncwarp();
    } else {
        // the pair sits in the 64-column atom p / 32, at byte 4 * (p % 32) of every 128-byte k-row
        const int col_off = (p / 32) * (kTcBK * 128) + (p % 32) * 4;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % S;
            if (!tc_wait(&full[s], (kb / S) & 1u, abort)) {
                ok = false;
                break;
            }
            const uint8_t *st = smem + (size_t)s * sh.stage_bytes;
            const uint8_t *wg = st + col_off, *wu = st + sh.a_bytes + col_off;
            const __half *xs = reinterpret_cast<const __half *>(st + 2 * sh.a_bytes);  // [B][64]
#pragma unroll
            for (int k = 16 * q; k < 16 * q + 16; k += 2) {
                const float2 g0 = __half22float2(*reinterpret_cast<const __half2 *>(wg + k * 128));
                const float2 g1 = __half22float2(*reinterpret_cast<const __half2 *>(wg + (k + 1) * 128));
                const float2 u0 = __half22float2(*reinterpret_cast<const __half2 *>(wu + k * 128));
                const float2 u1 = __half22float2(*reinterpret_cast<const __half2 *>(wu + (k + 1) * 128));
#pragma unroll
                for (int b = 0; b < BS; ++b) {
                    if (b >= B) break;
                    const float2 xv = __half22float2(*reinterpret_cast<const __half2 *>(xs + b * kTcBK + k));
                    ag[0][b] = fmaf(g0.x, xv.x, fmaf(g1.x, xv.y, ag[0][b]));
                    ag[1][b] = fmaf(g0.y, xv.x, fmaf(g1.y, xv.y, ag[1][b]));
                    au[0][b] = fmaf(u0.x, xv.x, fmaf(u1.x, xv.y, au[0][b]));
                    au[1][b] = fmaf(u0.y, xv.x, fmaf(u1.y, xv.y, au[1][b]));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
    // Sum the four k-quarters: red[q][v][c] with v = (matrix, column, row) and
    // c = the 128 columns; then the second CTA of the pair hands its sums to
    // the first over the cluster.  Both reuse the stage memory, which is idle
    // once both CTAs are past their loops.
    float *red = reinterpret_cast<float *>(smem);
    float *part = red + 4 * 2 * BS * kTcM;  // [2 * BS][128]
    volatile float *part_ok = reinterpret_cast<volatile float *>(part + 2 * BS * kTcM);
    cluster_sync_all();
    if (warp < kCcWarps)
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int b = 0; b < BS; ++b) {
                red[((q * 2 + 0) * BS + b) * kTcM + 2 * p + c] = ag[c][b];
                red[((q * 2 + 1) * BS + b) * kTcM + 2 * p + c] = au[c][b];
            }
    __syncthreads();
    const int col = t;  // threads 0..127 finish one column each
    float g[BS], u[BS];
    if (col < kTcM)
#pragma unroll
        for (int b = 0; b < BS; ++b) {
            g[b] = red[(0 * BS + b) * kTcM + col] + red[(2 * BS + b) * kTcM + col] + red[(4 * BS + b) * kTcM + col] +
                   red[(6 * BS + b) * kTcM + col];
            u[b] = red[(1 * BS + b) * kTcM + col] + red[(3 * BS + b) * kTcM + col] + red[(5 * BS + b) * kTcM + col] +
                   red[(7 * BS + b) * kTcM + col];
        }
    if (rank == 1 && col < kTcM) {
        const uint32_t remote = cluster_map(part, 0);
#pragma unroll
        for (int b = 0; b < BS; ++b) {
            st_cluster_f32(remote + (uint32_t)((b * kTcM + col) * 4), g[b]);
            st_cluster_f32(remote + (uint32_t)(((BS + b) * kTcM + col) * 4), u[b]);
        }
    }
    if (rank == 1 && t == 0) st_cluster_f32(cluster_map((const void *)part_ok, 0), (ok && !*abort) ? 1.f : 0.f);
    cluster_sync_all();
    if (rank == 0 && col < kTcM) {
        const bool all_ok = ok && !*abort && *part_ok != 0.f;
#pragma unroll
        for (int b = 0; b < BS; ++b) {
            if (b >= B) break;
            const float gs = g[b] + part[b * kTcM + col], us = u[b] + part[(BS + b) * kTcM + col];
            const float r = all_ok ? gs / (1.0f + __expf(-gs)) * us : __int_as_float(0x7fc00000);
            out[(size_t)b * sh.N + n0 + col] = __float2half_rn(r);
        }
    }
}

bool swiglu_col_tma_supported(int B, int K, int N) {
    return B >= 1 && B <= 8 && K % (kTcBK * kTcSplit) == 0 && N % kTcM == 0;
}

// ------------------------------------------------------------------ host side
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_fn() {
    static std::once_flag once;
    static EncodeTiled fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

bool tc_make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows, bool swizzle) {
    EncodeTiled enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_make_map_packed(CUtensorMap *m, const void *base, uint64_t tiles, uint32_t nkb, uint32_t rows, uint32_t kc) {
    EncodeTiled enc = encode_fn();
    if (!enc || rows < 1 || rows > 128 || 128 % rows || kc % 64) return false;
    const cuuint64_t dims[4] = {kc, rows, nkb, tiles};
    const cuuint64_t strides[3] = {(cuuint64_t)kc * 2, (cuuint64_t)rows * kc * 2, (cuuint64_t)nkb * rows * kc * 2};
    const cuuint32_t box[4] = {64, rows, 1, 128 / rows};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool swiglu_tc_supported(int B, int K, int N) {
    return B >= 1 && B <= 128 && K % (kTcBK * kTcSplit) == 0 && N % kTcM == 0;
}

cudaError_t launch_swiglu_tc(const void *x, const void *wg, const void *wu, void *out, int B, int K, int N,
                             cudaStream_t s) {
    // The MMA's N (the batch) is a multiple of 16: the x box is that many rows
    // high and the rows past B arrive as zeros (out-of-bounds fill), which the
    // transaction count includes.
    const int Bp = (B + 15) / 16 * 16;
    CUtensorMap mg, mu, mx;
    if (!tc_make_map(&mg, wg, (uint64_t)K, (uint64_t)N, 64, kTcBK) ||
        !tc_make_map(&mu, wu, (uint64_t)K, (uint64_t)N, 64, kTcBK) ||
        !tc_make_map(&mx, x, (uint64_t)B, (uint64_t)K, kTcBK, (uint32_t)Bp))
        return cudaErrorInvalidValue;
    TcShape sh;
    sh.B = Bp;
    sh.rows = B;
    sh.K = K;
    sh.N = N;
    sh.a_bytes = (uint32_t)kTcM * kTcBK * 2;  // one matrix's stage: 2 atoms of 64 features x 64 k
    sh.x_bytes = (uint32_t)Bp * kTcBK * 2;
    sh.stage_bytes = 2 * sh.a_bytes + sh.x_bytes;
    sh.tx_bytes = sh.stage_bytes;
    const int budget = 227 * 1024 - 1024 - 256;  // alignment slack and the barriers
    sh.stages = budget / (int)sh.stage_bytes;
    if (sh.stages > 6) sh.stages = 6;
    if (sh.stages < 2) return cudaErrorInvalidValue;
    const int smem = sh.stages * (int)sh.stage_bytes + 1024 + 256;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t ce = tc_allow_smem(reinterpret_cast<const void *>(swiglu_tc_kernel), 227 * 1024, configured);
    if (ce != cudaSuccess) return ce;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((N / kTcM) * kTcSplit);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kTcSplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, swiglu_tc_kernel, mg, mu, mx, static_cast<__half *>(out), sh);
}

cudaError_t launch_swiglu_col_tma(const void *x, const void *wg, const void *wu, void *out, int B, int K, int N,
                                  cudaStream_t s) {
    // x box rows: the batch rounded up to a multiple of 2 (rows past B read as zeros)
    const int xb = (B + 1) / 2 * 2;
    CUtensorMap mg, mu, mx;
    if (!tc_make_map(&mg, wg, (uint64_t)K, (uint64_t)N, 64, kTcBK, false) ||
        !tc_make_map(&mu, wu, (uint64_t)K, (uint64_t)N, 64, kTcBK, false) ||
        !tc_make_map(&mx, x, (uint64_t)B, (uint64_t)K, kTcBK, (uint32_t)xb, false))
        return cudaErrorInvalidValue;
    TcShape sh;
    sh.B = B;
    sh.rows = B;
    sh.K = K;
    sh.N = N;
    sh.a_bytes = (uint32_t)kTcM * kTcBK * 2;
    sh.x_bytes = ((uint32_t)xb * kTcBK * 2 + 1023) / 1024 * 1024;  // stage stride keeps 1 KB alignment
    sh.stage_bytes = 2 * sh.a_bytes + sh.x_bytes;
    sh.tx_bytes = 2 * sh.a_bytes + (uint32_t)xb * kTcBK * 2;
    const int budget = 227 * 1024 - 1024 - 256;
    sh.stages = budget / (int)sh.stage_bytes;
    if (sh.stages > 6) sh.stages = 6;
    if (sh.stages < 2) return cudaErrorInvalidValue;
    const int smem = sh.stages * (int)sh.stage_bytes + 1024 + 256;
    const void *fn = B <= 1 ? (const void *)swiglu_col_kernel<1>
                   : B <= 2 ? (const void *)swiglu_col_kernel<2>
                   : B <= 4 ? (const void *)swiglu_col_kernel<4>
                            : (const void *)swiglu_col_kernel<8>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((N / kTcM) * kTcSplit);
    cfg.blockDim = dim3(kCcThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kTcSplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    __half *o = static_cast<__half *>(out);
    if (B <= 1) return cudaLaunchKernelEx(&cfg, swiglu_col_kernel<1>, mg, mu, mx, o, sh);
    if (B <= 2) return cudaLaunchKernelEx(&cfg, swiglu_col_kernel<2>, mg, mu, mx, o, sh);
    if (B <= 4) return cudaLaunchKernelEx(&cfg, swiglu_col_kernel<4>, mg, mu, mx, o, sh);
    return cudaLaunchKernelEx(&cfg, swiglu_col_kernel<8>, mg, mu, mx, o, sh);
}

}  // namespace mk

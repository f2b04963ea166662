// mk_linear_tc.cu -- one decode projection on the 5th-generation tensor cores
// (tcgen05): y[b][m] = sum_k W[m][k] x[b][k] for the batched decode, where a
// projection of a whole batch is a dense GEMM with the batch as its narrow
// side.  W is a model matrix as given ([out, in] row-major bf16, the layout
// of every projection of the decoder: QKV, O, gate, up, down, LM head), x is
// the batch of input rows (bf16, [B, in]), y is fp32 [B, out].
//
// Swap-AB: the weights are operand A (M = 128 output rows per CTA, K-major,
// a row of W is contiguous in K), the batch is operand B (N = B rounded up
// to 16, K-major), so every weight byte leaves HBM once for the whole batch
// and the accumulator (128 lanes x N fp32 columns) lives in tensor memory.
// Both operands are staged by TMA with 128-byte swizzling into a ring of up
// to 6 stages; warp 0 lane 0 issues the loads, warp 1 lane 0 the MMAs, and
// each stage goes back to the producer through tcgen05.commit.
//
// When there are few output tiles (a 4096-row projection has 32), a cluster
// of 2 or 4 CTAs shares one tile and splits K, so that more SMs stream the
// weights; the other CTAs of the cluster then store their accumulators into
// the first one's idle stage memory over the cluster (mapa +
// st.shared::cluster), and the first adds them in rank order and writes y.
// Every wait is bounded; a wait that runs out stops the CTA and its outputs
// are written as NaN so that the failure cannot pass for a result.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "../../include/mk.h"
#include "mk_device.cuh"
#include "mk_kernel.h"
#include "mk_tc.cuh"

namespace mk {

constexpr int kLinM = 128;    // output rows per CTA (MMA M)
constexpr int kLinBK = 64;    // K per stage: one 128-byte swizzle row of bf16
constexpr int kLinThreads = 128;
constexpr int kLinMaxSplit = 4;
constexpr int kLinMaxB = 256;  // the MMA's N limit at M = 128
constexpr int kLinMaxStages = 6;
constexpr int kSkMaxCtas = 256;  // stream-K CTAs at most (the workspace is sized for this many)
static_assert(kSkWorkspaceFloats >= (size_t)kSkMaxCtas * kLinMaxB * kLinM && kSkWorkspaceFlags >= kSkMaxCtas,
              "stream-K workspace");

struct LinShape {
    int Bp, rows, K, M, stages;      // Bp: the MMA's N (B rounded up to 16); rows: B
    uint32_t stage_bytes, a_bytes;  // a stage is the W box then the x box
    int w_kc, w_rows;               // W packed as [tiles][K / w_kc][w_rows][w_kc] (4-D map), or w_kc = 0: row-major
};

// Instruction descriptor of kind::f16: fp32 accumulate, bf16 A and B, both
// K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t lin_idesc(int n) {
    return (1u << 4)                     // D format: F32
           | (1u << 7) | (1u << 10)      // A, B format: BF16
           | (0u << 15) | (0u << 16)     // A, B K-major
           | ((uint32_t)(n >> 3) << 17)  // N >> 3
           | ((uint32_t)(kLinM >> 4) << 24);
}

__global__ void __launch_bounds__(kLinThreads, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                     float *__restrict__ y, LinShape sh) {
    extern __shared__ __align__(1024) uint8_t lin_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(lin_smem_raw) + 1023) & ~uintptr_t(1023));
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int S = sh.stages, Bp = sh.Bp;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)S * sh.stage_bytes);
    uint64_t *empty = full + S;
    uint64_t *done = empty + S;
    volatile uint32_t *tmem_base = reinterpret_cast<volatile uint32_t *>(done + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    const uint32_t rank = cluster_rank(), nrank = cluster_size();
    const int m0 = (int)(blockIdx.x / nrank) * kLinM;
    const int nkb_all = sh.K / kLinBK;
    const int kb_first = (int)rank * nkb_all / (int)nrank;
    const int nkb = (int)(rank + 1) * nkb_all / (int)nrank - kb_first;
    uint32_t ncols = 32;  // a power of two >= 32 that holds N columns
    while (ncols < (uint32_t)Bp) ncols <<= 1;

    if (t == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {  // the whole warp allocates the accumulator columns
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
    // Launched with programmatic dependent launch (a step's chain of kernels),
    // the next kernel may now start its own set-up; without it this is a no-op.
    pdl_launch_dependents();

    int issued = 0;  // K blocks whose copies the producer (warp 0 lane 0) has issued
    if (warp == 0 && lane == 0) {
        auto load_w = [&](int kb) {
            const int s = kb % S, k0 = (kb_first + kb) * kLinBK;
            uint8_t *st = smem + (size_t)s * sh.stage_bytes;
            mbar_arrive_expect_tx(&full[s], sh.stage_bytes);  // rows past M or B arrive as zeros and count
            if (sh.w_kc)
                tma_load_4d(st, &map_w, k0 % sh.w_kc, 0, k0 / sh.w_kc, m0 / sh.w_rows, &full[s]);
            else
                tma_load_2d(st, &map_w, k0, m0, &full[s]);
        };
        auto load_x = [&](int kb) {
            const int s = kb % S, k0 = (kb_first + kb) * kLinBK;
            tma_load_2d(smem + (size_t)s * sh.stage_bytes + sh.a_bytes, &map_x, k0, 0, &full[s]);
        };
        // The weights do not depend on the kernel before this one: the first
        // stages' weight boxes go out before the wait for its results (x).
        const int pre = nkb < S ? nkb : S;
        for (int kb = 0; kb < pre; ++kb) load_w(kb);
        pdl_wait();
        for (int kb = 0; kb < pre; ++kb) load_x(kb);
        issued = pre;
        for (int kb = pre; kb < nkb; ++kb) {
            const int s = kb % S;
            if (!tc_wait(&empty[s], ((kb / S) - 1) & 1u, abort)) break;
            load_w(kb);
            load_x(kb);
            issued = kb + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // Both operands K-major, 128-byte swizzle: 8 rows of 128 bytes per
        // 1 KB group (SBO), a K step of 16 is 32 bytes along the rows.
        const uint32_t idesc = lin_idesc(Bp);
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % S;
            if (!tc_wait(&full[s], (kb / S) & 1u, abort)) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint8_t *st = smem + (size_t)s * sh.stage_bytes;
#pragma unroll
            for (int ks = 0; ks < kLinBK / 16; ++ks) {
                const uint64_t a = smem_desc_sw128(st + ks * 32, 16, 1024);
                const uint64_t b = smem_desc_sw128(st + sh.a_bytes + ks * 32, 16, 1024);
                tc_mma(tmem, a, b, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
            }
            tc_commit(&empty[s]);
        }
        tc_commit(done);
    }
    __syncwarp();
    // epilogue: thread t holds output row m0 + t (tensor-memory lane t; warp w
    // may read lanes 32w .. 32w+31), one column per batch row
    const bool ok = tc_wait(done, 0u, abort) && !*abort;
    // After an abort some copies may never have been waited for.  A stage
    // holds at most one copy in flight, so the producer lets the last copy of
    // every stage land before this CTA's stage memory is reused (by the
    // cluster reduction below) or freed; the other threads wait for it at the
    // next CTA or cluster barrier.
    if (warp == 0 && lane == 0 && *abort)
        for (int kb = issued > S ? issued - S : 0; kb < issued; ++kb)
            tc_drain(&full[kb % S], (uint32_t)(kb / S) & 1u, kTcTimeoutNs);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    // Once every CTA of the cluster is past its last MMA, the first CTA's
    // stage memory receives the others' accumulators, [rank - 1][Bp][128],
    // and their "ok" words after them.
    float *part = reinterpret_cast<float *>(smem);
    float *part_ok = part + (size_t)(nrank - 1) * Bp * kLinM;
    if (nrank > 1) cluster_sync_all();
    if (rank != 0) {
        const uint32_t remote = cluster_map(part, 0) + (rank - 1) * (uint32_t)(Bp * kLinM * 4);
        for (int c0 = 0; c0 < Bp; c0 += 16) {
            float v[16];
            tmem_ld16(lane_addr + (uint32_t)c0, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) st_cluster_f32(remote + (uint32_t)(((c0 + i) * kLinM + t) * 4), v[i]);
        }
        if (t == 0) st_cluster_f32(cluster_map(part_ok + (rank - 1), 0), ok ? 1.f : 0.f);
    }
    if (nrank > 1) cluster_sync_all();
    if (rank == 0) {
        bool all_ok = ok;
        for (uint32_t r = 1; r < nrank; ++r) all_ok = all_ok && part_ok[r - 1] != 0.f;
        const int m = m0 + t;
        for (int c0 = 0; c0 < Bp; c0 += 16) {
            float v[16];
            tmem_ld16(lane_addr + (uint32_t)c0, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int b = c0 + i;
                float acc = v[i];
                for (uint32_t r = 1; r < nrank; ++r) acc += part[((size_t)(r - 1) * Bp + b) * kLinM + t];
                if (b < sh.rows && m < sh.M) y[(size_t)b * sh.M + m] = all_ok ? acc : __int_as_float(0x7fc00000);
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
}

// ------------------------------------------------------------------ stream-K
// The same product for projections with too few 128-row tiles to give every
// SM an equal share (a 4096-row projection has 32 tiles, a 28672-row one 224,
// i.e. 1.5 waves): the work is cut into units of one tile x one K block,
// tiles x K/64 of them, and CTA i of G (G <= the SM count, all resident)
// takes the contiguous units [i U / G, (i + 1) U / G).  A CTA's range
// therefore covers at most kSkMaxSeg pieces (segments) of consecutive tiles:
// possibly the tail of one tile, whole tiles, and the head of a last one,
// each accumulated in its own tensor-memory columns.  A segment that holds
// its tile's first K block belongs to that CTA (the tile's owner); a segment
// without it (at most one per CTA, its first) is a contribution: after the
// main loop the CTA stores that accumulator in its slot of `ws` and raises
// its flag, before it waits for anyone.  The owner then adds the
// contributions of the CTAs after it that hold the rest of its tile, in CTA
// order (deterministic), writes y and lowers their flags for the next
// launch.  Waits only run towards higher CTA indices and every CTA publishes
// before it waits, so they always end.  The roles are the plain kernel's:
// warp 0 lane 0 issues the copies, warp 1 lane 0 the MMAs, and all four
// warps run the epilogue.
constexpr int kSkMaxSeg = 4;

struct SkArgs {
    int G, U, nkb;    // CTAs, units (tiles x K blocks), K blocks per tile
    float *ws;        // [G][Bp][128]: a CTA's contribution, row-contiguous
    uint32_t *flags;  // [G]: 1 while CTA i's contribution waits in ws; zero between launches
};

__host__ __device__ inline int sk_first(const SkArgs &k, int i) { return (int)((long long)i * k.U / k.G); }

__global__ void __launch_bounds__(kLinThreads, 1)
    linear_sk_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                     float *__restrict__ y, LinShape sh, SkArgs sk) {
    extern __shared__ __align__(1024) uint8_t lin_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(lin_smem_raw) + 1023) & ~uintptr_t(1023));
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int S = sh.stages, Bp = sh.Bp, nkb = sk.nkb;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)S * sh.stage_bytes);
    uint64_t *empty = full + S;
    uint64_t *done = empty + S;
    volatile uint32_t *tmem_base = reinterpret_cast<volatile uint32_t *>(done + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    const int i = blockIdx.x;
    const int u0 = sk_first(sk, i), u1 = sk_first(sk, i + 1), n = u1 - u0;
    const int t_first = u0 / nkb, nseg = (u1 - 1) / nkb - t_first + 1;
    uint32_t ncols = 32;
    while (ncols < (uint32_t)(nseg * Bp)) ncols <<= 1;

    if (t == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
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
    pdl_launch_dependents();

    int issued = 0;
    if (warp == 0 && lane == 0) {
        // unit j of this CTA: tile (u0 + j) / nkb, K block (u0 + j) % nkb,
        // stepped without divisions
        int tile = t_first, kb = u0 - t_first * nkb;
        auto load = [&](int j, int tl, int k, bool w_only, bool x_only) {
            const int s = j % S, k0 = k * kLinBK;
            uint8_t *st = smem + (size_t)s * sh.stage_bytes;
            if (!x_only) {
                mbar_arrive_expect_tx(&full[s], sh.stage_bytes);
                if (sh.w_kc)
                    tma_load_4d(st, &map_w, k0 % sh.w_kc, 0, k0 / sh.w_kc, tl * kLinM / sh.w_rows, &full[s]);
                else
                    tma_load_2d(st, &map_w, k0, tl * kLinM, &full[s]);
            }
            if (!w_only) tma_load_2d(st + sh.a_bytes, &map_x, k0, 0, &full[s]);
        };
        const int pre = n < S ? n : S;
        {
            int tl = tile, k = kb;
            for (int j = 0; j < pre; ++j) {
                load(j, tl, k, true, false);
                if (++k == nkb) k = 0, ++tl;
            }
        }
        pdl_wait();
        for (int j = 0; j < pre; ++j) {
            load(j, tile, kb, false, true);
            if (++kb == nkb) kb = 0, ++tile;
        }
        issued = pre;
        for (int j = pre; j < n; ++j) {
            const int s = j % S;
            if (!tc_wait(&empty[s], ((j / S) - 1) & 1u, abort)) break;
            load(j, tile, kb, false, false);
            if (++kb == nkb) kb = 0, ++tile;
            issued = j + 1;
        }
    } else if (warp == 1 && lane == 0) {
        const uint32_t idesc = lin_idesc(Bp);
        int seg = 0, kb = u0 - t_first * nkb;
        for (int j = 0; j < n; ++j) {
            const int s = j % S;
            if (!tc_wait(&full[s], (j / S) & 1u, abort)) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint8_t *st = smem + (size_t)s * sh.stage_bytes;
            const bool first = j == 0 || kb == 0;
            const uint32_t d = tmem + (uint32_t)(seg * Bp);
#pragma unroll
            for (int ks = 0; ks < kLinBK / 16; ++ks) {
                const uint64_t a = smem_desc_sw128(st + ks * 32, 16, 1024);
                const uint64_t b = smem_desc_sw128(st + sh.a_bytes + ks * 32, 16, 1024);
                tc_mma(d, a, b, idesc, (!first || ks > 0) ? 1u : 0u);
            }
            tc_commit(&empty[s]);
            if (++kb == nkb) kb = 0, ++seg;
        }
        tc_commit(done);
    }
    __syncwarp();
    bool ok = tc_wait(done, 0u, abort) && !*abort;
    if (warp == 0 && lane == 0 && *abort)
        for (int j = issued > S ? issued - S : 0; j < issued; ++j)
            tc_drain(&full[j % S], (uint32_t)(j / S) & 1u, kTcTimeoutNs);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // epilogue: thread t holds row t of a tile (tensor-memory lane t)
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const float nan = __int_as_float(0x7fc00000);
    for (int seg = 0; seg < nseg; ++seg) {
        const int T = t_first + seg, tu0 = T * nkb, tu1 = tu0 + nkb;
        const bool head = u0 <= tu0, whole = head && u1 >= tu1;
        const int m = T * kLinM + t;
        if (!head) {  // a contribution to tile T, this CTA's first segment
            float *slot = sk.ws + (size_t)i * Bp * kLinM + t;
            for (int c0 = 0; c0 < Bp; c0 += 16) {
                float v[16];
                tmem_ld16(lane_addr + (uint32_t)(seg * Bp + c0), v);
#pragma unroll
                for (int c = 0; c < 16; ++c) slot[(size_t)(c0 + c) * kLinM] = ok ? v[c] : nan;
            }
            __threadfence();
            __syncthreads();
            if (t == 0) red_release_add(&sk.flags[i], 1u);
            continue;
        }
        // the owner: contributions from CTAs i+1, i+2, ... while they start inside T
        int jend = i + 1;
        if (!whole)
            while (jend < sk.G && sk_first(sk, jend) < tu1) ++jend;
        bool got = ok;
        for (int j = i + 1; j < jend && got; ++j) {
            const uint64_t t0 = globaltimer_ns();
            uint32_t it = 0;
            while (ld_acquire_gpu(&sk.flags[j]) == 0u) {
                __nanosleep(32);
                if ((++it & 15u) == 0u && globaltimer_ns() - t0 > kTcTimeoutNs) {
                    got = false;
                    break;
                }
            }
        }
        for (int c0 = 0; c0 < Bp; c0 += 16) {
            float v[16];
            tmem_ld16(lane_addr + (uint32_t)(seg * Bp + c0), v);
            if (got)
                for (int j = i + 1; j < jend; ++j) {
                    const float *slot = sk.ws + (size_t)j * Bp * kLinM + t;
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] += slot[(size_t)(c0 + c) * kLinM];
                }
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int b = c0 + c;
                if (b < sh.rows && m < sh.M) y[(size_t)b * sh.M + m] = got ? v[c] : nan;
            }
        }
        if (jend > i + 1) {
            __syncthreads();  // every thread has read the contributions
            if (t == 0)
                for (int j = i + 1; j < jend; ++j) sk.flags[j] = 0u;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
}

// Launch geometry of one call, worked out on the host.
struct LinPlan {
    LinShape sh;
    int split, tiles, smem;
};

static bool lin_plan(int B, int K, int M, LinPlan &p) {
    if (B < 1 || B > kLinMaxB || K < kLinBK || K % kLinBK || M < 1) return false;
    LinShape &sh = p.sh;
    sh.Bp = (B + 15) / 16 * 16;
    sh.rows = B;
    sh.K = K;
    sh.M = M;
    sh.a_bytes = (uint32_t)kLinM * kLinBK * 2;                      // 16 KB of W
    sh.stage_bytes = sh.a_bytes + (uint32_t)sh.Bp * kLinBK * 2;     // + Bp rows of x, a multiple of 2 KB
    const int budget = 227 * 1024 - 1024 - 256;                    // alignment slack and the barriers
    p.tiles = (M + kLinM - 1) / kLinM;
    const int nkb = K / kLinBK;
    // up to 6 stages (96 KB of weights in flight; 12 measured slower, the LM
    // head at 0.76 of HBM against 0.96), never more than the K blocks there are
    sh.stages = budget / (int)sh.stage_bytes;
    if (sh.stages > kLinMaxStages) sh.stages = kLinMaxStages;
    if (sh.stages > nkb) sh.stages = nkb;
    if (sh.stages < 2) return false;
    // K split across a cluster while the grid stays within one wave of SMs,
    // every CTA keeps at least two K blocks, and the first CTA's stage
    // memory holds the other CTAs' accumulators.
    p.split = 1;
    for (int s = kLinMaxSplit; s > 1; s /= 2)
        if (p.tiles * s <= 148 && nkb >= 2 * s &&
            (size_t)(s - 1) * sh.Bp * kLinM * 4 + 16 <= (size_t)sh.stages * sh.stage_bytes) {
            p.split = s;
            break;
        }
    p.smem = sh.stages * (int)sh.stage_bytes + 1024 + 256;
    return true;
}

// w_kc > 0: W is packed as [tiles][K / w_kc][w_rows][w_kc] (tiles = M / w_rows
// rounded up), read through a 4-D tensor map; else W is row-major [M, K].
static cudaError_t launch_linear(const void *x, const void *w, float *y, int B, int K, int M, int w_kc, int w_rows,
                                 cudaStream_t s, bool pdl) {
    LinPlan p;
    if (!lin_plan(B, K, M, p)) return cudaErrorInvalidValue;
    if (w_kc && (w_kc % kLinBK || K % w_kc || w_rows < 1 || kLinM % w_rows)) return cudaErrorInvalidValue;
    p.sh.w_kc = w_kc;
    p.sh.w_rows = w_rows;
    CUtensorMap mw, mx;
    const bool wmap = w_kc ? tc_make_map_packed(&mw, w, (uint64_t)((M + w_rows - 1) / w_rows), (uint32_t)(K / w_kc),
                                                (uint32_t)w_rows, (uint32_t)w_kc)
                           : tc_make_map(&mw, w, (uint64_t)M, (uint64_t)K, kLinBK, kLinM);
    if (!wmap || !tc_make_map(&mx, x, (uint64_t)B, (uint64_t)K, kLinBK, (uint32_t)p.sh.Bp))
        return cudaErrorInvalidValue;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t ce = tc_allow_smem(reinterpret_cast<const void *>(linear_tc_kernel), 227 * 1024, configured);
    if (ce != cudaSuccess) return ce;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.tiles * p.split));
    cfg.blockDim = dim3(kLinThreads);
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, linear_tc_kernel, mw, mx, y, p.sh);
}

cudaError_t launch_linear_tc(const void *x, const void *w, float *y, int B, int K, int M, cudaStream_t s) {
    return launch_linear(x, w, y, B, K, M, 0, 0, s, false);
}

cudaError_t launch_linear_tc_packed(const void *x, const void *w, float *y, int B, int K, int M, int kc, int rows,
                                    cudaStream_t s, bool pdl) {
    return launch_linear(x, w, y, B, K, M, kc, rows, s, pdl);
}

// Stream-K geometry: G CTAs (at most the SM count, at least 4 units each)
// over tiles x K blocks; false when a CTA's range would span more than
// kSkMaxSeg tiles (many tiles: the one-tile-per-CTA kernel then already
// fills the SMs in several waves).
static bool sk_plan(int B, int K, int M, int sms, LinPlan &p, SkArgs &sk) {
    if (!lin_plan(B, K, M, p)) return false;
    sk.nkb = K / kLinBK;
    sk.U = p.tiles * sk.nkb;
    sk.G = sms < sk.U / 4 ? sms : sk.U / 4;
    if (sk.G > kSkMaxCtas) sk.G = kSkMaxCtas;
    if (sk.G < 2) return false;
    const int per = (sk.U + sk.G - 1) / sk.G;  // the longest range
    const int segs = (per + sk.nkb - 1) / sk.nkb + 1;
    if (segs > kSkMaxSeg || segs * p.sh.Bp > 512) return false;  // every segment's columns in tensor memory
    p.smem = p.sh.stages * (int)p.sh.stage_bytes + 1024 + 256;
    return true;
}

static int device_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// The stream-K grid for (B, K, M), or 0 where the one-tile-per-CTA kernel
// does as well: one full wave with its K split, or 1.5 waves of tiles and
// more (its later CTAs then start out of step with the first ones; a
// 28672-row projection of 224 tiles measured 46 us plain, 48 us stream-K).
static int sk_grid(int B, int K, int M, int sms, LinPlan &p, SkArgs &sk) {
    if (!lin_plan(B, K, M, p)) return 0;
    if (p.tiles * p.split == sms || 2 * p.tiles >= 3 * sms) return 0;
    // above 64 columns a contribution (128 rows x Bp fp32) costs more than an
    // uneven wave unless the tiles fill at most half the SMs (at 256 columns
    // the 128-tile gate/up of a 1B model took 34 us plain, 46 us stream-K)
    if (p.sh.Bp > 64 && 2 * p.tiles * p.split > sms) return 0;
    return sk_plan(B, K, M, sms, p, sk) ? sk.G : 0;
}

cudaError_t launch_linear_tc_packed_sk(const void *x, const void *w, float *y, int B, int K, int M, int kc, int rows,
                                       float *ws, uint32_t *flags, cudaStream_t s, bool pdl) {
    LinPlan p;
    SkArgs sk{};
    if (!ws || !flags || sk_grid(B, K, M, device_sms(), p, sk) == 0)
        return launch_linear(x, w, y, B, K, M, kc, rows, s, pdl);
    if (kc && (kc % kLinBK || K % kc || rows < 1 || kLinM % rows)) return cudaErrorInvalidValue;
    p.sh.w_kc = kc;
    p.sh.w_rows = rows;
    sk.ws = ws;
    sk.flags = flags;
    CUtensorMap mw, mx;
    const bool wmap = kc ? tc_make_map_packed(&mw, w, (uint64_t)((M + rows - 1) / rows), (uint32_t)(K / kc),
                                              (uint32_t)rows, (uint32_t)kc)
                         : tc_make_map(&mw, w, (uint64_t)M, (uint64_t)K, kLinBK, kLinM);
    if (!wmap || !tc_make_map(&mx, x, (uint64_t)B, (uint64_t)K, kLinBK, (uint32_t)p.sh.Bp))
        return cudaErrorInvalidValue;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t ce = tc_allow_smem(reinterpret_cast<const void *>(linear_sk_kernel), 227 * 1024, configured);
    if (ce != cudaSuccess) return ce;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sk.G);
    cfg.blockDim = dim3(kLinThreads);
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, linear_sk_kernel, mw, mx, y, p.sh, sk);
}

}  // namespace mk

using namespace mk;

extern "C" mk_status mk_linear_tc(const void *x, const void *w, float *y, int B, int K, int M, void *stream) {
    if (!x || !w || !y) {
        set_op_error("linear_tc: null pointer");
        return MK_ERR_INVALID;
    }
    if (B < 1 || K < 1 || M < 1) {
        set_op_error("linear_tc: B, K and M must be positive");
        return MK_ERR_INVALID;
    }
    for (const void *p : {x, w, static_cast<const void *>(y)})
        if ((uintptr_t)p & 15) {
            set_op_error("linear_tc: x, w and y must be 16-byte aligned");
            return MK_ERR_INVALID;
        }
    LinPlan p;
    if (!lin_plan(B, K, M, p)) {
        set_op_error("linear_tc: needs B <= 256 and K a multiple of 64");
        return MK_ERR_UNSUPPORTED;
    }
    const cudaError_t e = launch_linear_tc(x, w, y, B, K, M, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        char msg[160];
        snprintf(msg, sizeof(msg), "linear_tc: launch failed: %s", cudaGetErrorString(e));
        set_op_error(msg);
        return MK_ERR_CUDA;
    }
    return MK_OK;
}

extern "C" mk_status mk_linear_tc_split(int B, int K, int M, int *split) {
    if (!split) return MK_ERR_INVALID;
    LinPlan p;
    if (!lin_plan(B, K, M, p)) return MK_ERR_UNSUPPORTED;
    *split = p.split;
    return MK_OK;
}

extern "C" size_t mk_linear_tc_streamk_workspace_bytes(void) {
    return kSkWorkspaceFloats * sizeof(float) + kSkWorkspaceFlags * sizeof(uint32_t);
}

extern "C" int mk_linear_tc_streamk_grid(int B, int K, int M) {
    LinPlan p;
    SkArgs sk{};
    return sk_grid(B, K, M, device_sms(), p, sk);
}

extern "C" mk_status mk_linear_tc_streamk(const void *x, const void *w, float *y, int B, int K, int M,
                                          void *workspace, size_t workspace_bytes, void *stream) {
    if (!x || !w || !y || !workspace) {
        set_op_error("linear_tc_streamk: null pointer");
        return MK_ERR_INVALID;
    }
    if (B < 1 || K < 1 || M < 1) {
        set_op_error("linear_tc_streamk: B, K and M must be positive");
        return MK_ERR_INVALID;
    }
    for (const void *p : {x, w, static_cast<const void *>(y), static_cast<const void *>(workspace)})
        if ((uintptr_t)p & 15) {
            set_op_error("linear_tc_streamk: x, w, y and the workspace must be 16-byte aligned");
            return MK_ERR_INVALID;
        }
    if (workspace_bytes < mk_linear_tc_streamk_workspace_bytes()) {
        char msg[160];
        snprintf(msg, sizeof(msg), "linear_tc_streamk: the workspace needs %zu bytes (got %zu)",
                 mk_linear_tc_streamk_workspace_bytes(), workspace_bytes);
        set_op_error(msg);
        return MK_ERR_INVALID;
    }
    LinPlan p;
    if (!lin_plan(B, K, M, p)) {
        set_op_error("linear_tc_streamk: needs B <= 256 and K a multiple of 64");
        return MK_ERR_UNSUPPORTED;
    }
    float *ws = static_cast<float *>(workspace);
    uint32_t *flags = reinterpret_cast<uint32_t *>(ws + kSkWorkspaceFloats);
    const cudaError_t e =
        launch_linear_tc_packed_sk(x, w, y, B, K, M, 0, 0, ws, flags, static_cast<cudaStream_t>(stream), false);
    if (e != cudaSuccess) {
        char msg[160];
        snprintf(msg, sizeof(msg), "linear_tc_streamk: launch failed: %s", cudaGetErrorString(e));
        set_op_error(msg);
        return MK_ERR_CUDA;
    }
    return MK_OK;
}

// mk_tc.cuh -- pieces shared by the tcgen05 kernels (the SwiGLU stage and the
// decode projection): cluster and TMA helpers, bounded mbarrier waits, the
// shared-memory descriptor of a 128-byte-swizzled operand, the MMA issue and
// commit, tensor-memory loads, and the tensor-map encoder.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "mk_device.cuh"

namespace mk {

constexpr uint64_t kTcTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t cluster_map(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}

// 4-D tile of a tensor map: coordinates innermost first.
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(smem_addr(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_addr(bar))
        : "memory");
}

// Bounded wait for the phase `parity` of an mbarrier; false after the time
// limit or once another role of the CTA has given up.
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 10000u)) return true;
        if ((it & 7u) == 0u) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > kTcTimeoutNs) {
                *abort = 1;
                return false;
            }
        }
    }
}

// After a CTA gave up: wait (bounded by `limit_ns`, ignoring the abort flag)
// until the phase `parity` of `bar` -- the last copy issued into that stage --
// has landed, so that no copy into this CTA's shared memory is still in
// flight when it frees its resources and exits.  False if it did not land.
__device__ __forceinline__ bool tc_drain(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 10000u))
        if (globaltimer_ns() - t0 > limit_ns) return false;
    return true;
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2,
// descriptor version 1): start address, leading and stride byte offsets, all
// in 16-byte units.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void *p, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    const uint64_t start = (smem_addr(p) >> 4) & 0x3FFFu;
    return start | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) | ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) |
           (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// 16 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per device (bit d of `done` records device d; the attribute
// is per device, so a second device gets its own call).
inline cudaError_t tc_allow_smem(const void *fn, int bytes, std::atomic<unsigned long long> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// 2-D tensor of 2-byte elements [rows][cols] (cols contiguous, row stride
// cols * 2 bytes), box box_cols x box_rows, 128-byte swizzle (or none);
// reads outside the tensor return zeros.  False if the driver entry point is
// missing or refuses the map.
bool tc_make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows, bool swizzle = true);
// A matrix packed as [tiles][nkb][rows][kc] 2-byte elements (the decode
// megakernel's weight tiles: `rows` rows of K block kb of tile t contiguous)
// as a 4-D tensor (kc, rows, nkb, tiles), with a box of 64 columns of 128 /
// rows consecutive tiles, i.e. 128 consecutive matrix rows x 64 columns laid
// out in shared memory exactly as a 2-D box of a row-major matrix, 128-byte
// swizzled.  kc a multiple of 64, rows a power of two <= 128.
bool tc_make_map_packed(CUtensorMap *m, const void *base, uint64_t tiles, uint32_t nkb, uint32_t rows, uint32_t kc);

}  // namespace mk

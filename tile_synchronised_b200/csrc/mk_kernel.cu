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
    volatile uint32_t *seq;   // [kMaxStages] ring block index each slot currently holds
    float *ssq;               // [consumer warps][8] sums of squares
    unsigned long long *best; // [64] argmax keys per batch row
    float2 *rope;             // [64] (cos, sin) of the RoPE angles at this step's position
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
    S.seq = reinterpret_cast<volatile uint32_t *>(misc + 384);  // 8 words
    S.best = reinterpret_cast<unsigned long long *>(misc + 512);
    S.ssq = reinterpret_cast<float *>(misc + 1024);   // [16 warps][8]
    S.rope = reinterpret_cast<float2 *>(misc + 2048); // [64]
    return S;
}

__host__ int smem_bytes(const KParams &P) { return P.stages * kStageBytes + P.act_bytes + misc_bytes(P.bs, P.stages); }

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ Instr load_instr(const KParams &P, int i) {
    // field-by-field from two 16-byte loads (no address-taken copy, so the
    // instruction stays in registers)
    const uint4 *p = reinterpret_cast<const uint4 *>(P.instrs + i);
    const uint4 a = __ldg(p), b = __ldg(p + 1);
    Instr in;
    in.op = (uint8_t)(a.x & 0xFFu);
    in.flags = (uint8_t)((a.x >> 8) & 0xFFu);
    in.layer = (uint16_t)(a.x >> 16);
    in.tile = a.y;
    in.kb0 = (uint16_t)(a.z & 0xFFFFu);
    in.kb1 = (uint16_t)(a.z >> 16);
    in.b0 = (uint16_t)(a.w & 0xFFFFu);
    in.nb = (uint16_t)(a.w >> 16);
    in.wait_ctr = (uint16_t)(b.x & 0xFFFFu);
    in.signal_ctr = (uint16_t)(b.x >> 16);
    in.wait_count = b.y;
    in.signal2_ctr = (uint16_t)(b.z & 0xFFFFu);
    in.ntiles = (uint16_t)(b.z >> 16);
    in.arrive_count = b.w;
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
        __nanosleep(32);
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

// Bounded wait on a ring barrier; also returns false once the CTA aborts.  The
// thread sleeps in hardware between checks (woken when the phase completes),
// so a waiting producer does not take issue slots from the consumer warps.
__device__ bool wait_bar(const KParams &P, uint64_t *bar, uint32_t parity, volatile int *abort, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = 0;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if ((it & 3u) == 0u) {
            if (*abort) return false;
            uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > limit_ns) return false;
        }
    }
}

// The token of sequence b, with one outside [0, vocab) replaced by 0 so that
// every read stays inside the embedding table (check_tokens has recorded it;
// the step still runs to the end, so no wait is cut short).
__device__ __forceinline__ int token_of(const KParams &P, int b) {
    const int t = P.tokens[(int64_t)b * P.tok_stride];
    return (unsigned)t < (unsigned)P.vocab ? t : 0;
}

// At the start of a launch, thread b of CTA 0 checks the token of sequence b
// and records one outside [0, vocab) in the step state (the first such
// sequence and its value; mk_get_status reports it as an invalid argument).
__device__ __forceinline__ void check_tokens(const KParams &P) {
    const int b = threadIdx.x;
    if (blockIdx.x != 0 || b >= P.batch) return;
    const int t = P.tokens[(int64_t)b * P.tok_stride];
    if ((unsigned)t >= (unsigned)P.vocab && atomicCAS(&P.state->tok_err, 0u, (uint32_t)b + 1u) == 0u)
        P.state->tok_bad = t;
}

struct MatRef {
    const uint8_t *base;
    int kc, nkb, rows;
};

__device__ __forceinline__ MatRef mat_of(const KParams &P, const Instr &in) {
    MatRef m;
    const LayerW *L = P.layers + in.layer;
    switch (in.op) {
        case OP_QKV: m.base = (const uint8_t *)L->qkv; m.kc = P.qkv_kc; m.nkb = P.qkv_nkb; m.rows = P.qkv_rt; break;
        case OP_OPROJ: m.base = (const uint8_t *)L->o; m.kc = P.o_kc; m.nkb = P.o_nkb; m.rows = P.o_rt; break;
        case OP_GATEUP: m.base = (const uint8_t *)L->gu; m.kc = P.gu_kc; m.nkb = P.gu_nkb; m.rows = P.gu_rt; break;
        case OP_DOWN: m.base = (const uint8_t *)L->down; m.kc = P.down_kc; m.nkb = P.down_nkb; m.rows = P.down_rt; break;
        default: m.base = (const uint8_t *)P.lm_w; m.kc = P.lm_kc; m.nkb = P.lm_nkb; m.rows = P.lm_rt; break;
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
// A cursor over the ring blocks of a CTA's instruction list: GEMV weight
// blocks, or (K, V) chunks of one split-KV unit.  Instructions that stream
// nothing are skipped.
struct BlockCursor {
    int i, end, j, n;
    Instr in;
    AttnGeom a;
    MatRef m;
};

__device__ __forceinline__ void cursor_settle(const KParams &P, BlockCursor &c, int pos) {
    while (c.i < c.end) {
        c.in = load_instr(P, c.i);
        c.j = 0;
        if (c.in.op == OP_ATTN) {
            c.a = attn_geom(P, c.in, pos);
            c.n = c.a.nstages;
        } else {
            c.m = mat_of(P, c.in);
            c.n = (c.in.kb1 - c.in.kb0) * c.in.ntiles;
        }
        if (c.n > 0) return;
        ++c.i;
    }
}

__device__ __forceinline__ void cursor_next(const KParams &P, BlockCursor &c, int pos) {
    if (++c.j >= c.n) {
        ++c.i;
        cursor_settle(P, c, pos);
    }
}

// Source of the cursor's block: src2 is the V half of an attention chunk
// (null for weights); `bytes` is per half.
__device__ __forceinline__ void cursor_block(const KParams &P, const BlockCursor &c, const void *&src1,
                                             const void *&src2, uint32_t &bytes) {
    if (c.in.op == OP_ATTN) {
        const int d = P.head_dim, sp = kStageBytes / (4 * d);
        const int p = c.a.p0 + c.j * sp;
        const int n = min(sp, c.a.tma_end - p);
        bytes = (uint32_t)(n * d * 2);
        src1 = P.kcache + kv_off(P, c.in.layer, c.a.b, c.a.g, p);
        src2 = P.vcache + kv_off(P, c.in.layer, c.a.b, c.a.g, p);
    } else {
        const int nkr = c.in.kb1 - c.in.kb0;  // blocks of one tile in this run
        bytes = (uint32_t)(c.m.rows * c.m.kc * 2);
        src1 = c.m.base + ((size_t)(c.in.tile + c.j / nkr) * c.m.nkb + c.in.kb0 + c.j % nkr) * bytes;
        src2 = nullptr;
    }
}

// The producer fills the ring in instruction order.  A second cursor pulls
// blocks further ahead into L2 with bulk prefetches: it always keeps a short
// base distance, and while the next slot is still in use (the consumers are
// waiting on an input, so HBM would otherwise idle) it runs on up to
// P.prefetch blocks ahead.  Prefetching only while stalled keeps the far-ahead
// traffic from competing with blocks the consumers need now.
constexpr uint32_t kPrefetchBase = 4;

__device__ void producer(const KParams &P, const SmemLayout &S, int begin, int end, int pos) {
    const uint64_t pol = policy_evict_first();
    const uint64_t pol_pf = policy_evict_normal();
    int slot = 0;
    uint32_t phase = 0, issued = 0, issued_par = 0, bi = 0;
    const uint64_t limit = 2ull * P.timeout_ns + 1000000ull;
    bool ok = true;
    BlockCursor cur{begin, end, 0, 0}, pf{begin, end, 0, 0};
    cursor_settle(P, cur, pos);
    cursor_settle(P, pf, pos);
    const uint32_t maxd = (uint32_t)P.prefetch, base = maxd < kPrefetchBase ? maxd : kPrefetchBase;
    uint32_t pf_n = 0;  // blocks from cur (included) to the prefetch cursor (excluded)
    auto prefetch_one = [&]() {
        const void *p1, *p2;
        uint32_t pb;
        cursor_block(P, pf, p1, p2, pb);
        bulk_prefetch_l2(p1, pb, pol_pf);
        if (p2) bulk_prefetch_l2(p2, pb, pol_pf);
        cursor_next(P, pf, pos);
        ++pf_n;
    };
    while (pf_n < base && pf.i < end) prefetch_one();
    unsigned long long pw = 0;
    while (cur.i < end) {
        const void *s1, *s2;
        uint32_t bytes;
        cursor_block(P, cur, s1, s2, bytes);
        const unsigned long long w0 = P.trace ? globaltimer_ns() : 0ull;
        if (!mbar_try_wait(&S.empty[slot], phase ^ 1u)) {
            while (pf_n < maxd && pf.i < end) {
                prefetch_one();
                if (mbar_try_wait(&S.empty[slot], phase ^ 1u)) break;
            }
            if (!wait_bar(P, &S.empty[slot], phase ^ 1u, S.abort, limit)) {
                ok = false;
                break;
            }
        }
        if (P.trace) {
            pw += globaltimer_ns() - w0;
            if (cur.j == 0) P.trace[8 * (size_t)cur.i + 3] = globaltimer_ns();
        }
        uint8_t *dst = S.ring + (size_t)slot * kStageBytes;
        S.seq[slot] = bi++;  // the slot is free: announce which block it will hold
        mbar_arrive_expect_tx(&S.full[slot], s2 ? 2u * bytes : bytes);
        bulk_g2s(dst, s1, bytes, &S.full[slot], pol);
        if (s2) bulk_g2s(dst + kStageBytes / 2, s2, bytes, &S.full[slot], pol);
        issued |= 1u << slot;
        issued_par = (issued_par & ~(1u << slot)) | (phase << slot);
        if (++slot == P.stages) {
            slot = 0;
            phase ^= 1u;
        }
        if (P.trace && cur.j == cur.n - 1) {
            P.trace[8 * (size_t)cur.i + 5] = pw;
            P.trace[8 * (size_t)cur.i + 6] = globaltimer_ns();
            pw = 0;
        }
        cursor_next(P, cur, pos);
        if (pf_n > 0)
            --pf_n;  // cur moved into the prefetched window
        else
            cursor_next(P, pf, pos);  // the prefetch cursor never falls behind cur
        while (pf_n < base && pf.i < end) prefetch_one();
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

// ------------------------------------------------------------------ consumer side of the ring
// Blocks are numbered per CTA in the order the producer loads them; block bi
// sits in slot bi % stages during its (bi / stages)-th use of that slot.
struct CRing {
    unsigned long long waited;  // SM cycles spent waiting for ring data (thread 0, tracing only)
};

// Wait until block bi is in shared memory.  Warps consume blocks out of
// order (each GEMV tile belongs to one warp), so a warp may reach slot s for
// use u while s is still on use u - 1; the parity of u then matches the long
// completed use u - 2.  So first wait until the producer has stamped the slot
// with bi (it does so only after use u - 1 was released, i.e. its data phase
// completed), and only then test the phase parity.
__device__ __forceinline__ const uint8_t *ring_wait(const KParams &P, const SmemLayout &S, CRing &r, uint32_t bi) {
    const uint32_t slot = bi % (uint32_t)P.stages, par = (bi / (uint32_t)P.stages) & 1u;
    const long long c0 = (P.trace && threadIdx.x == 0) ? clock64() : 0;
    bool ok = true;
    if (S.seq[slot] != bi) {
        uint64_t t0 = 0;
        for (uint32_t it = 1; S.seq[slot] != bi; ++it) {
            __nanosleep(20);
            if ((it & 15u) == 0u) {
                if (*S.abort) { ok = false; break; }
                const uint64_t now = globaltimer_ns();
                if (t0 == 0) t0 = now;
                else if (now - t0 > P.timeout_ns) { ok = false; break; }
            }
        }
    }
    if (!ok || !wait_bar(P, &S.full[slot], par, S.abort, P.timeout_ns)) {
        if (!*S.abort) set_error(P, 2u, blockIdx.x, bi);
        *S.abort = 1;
    }
    if (P.trace && threadIdx.x == 0) r.waited += (unsigned long long)(clock64() - c0);
    return S.ring + (size_t)slot * kStageBytes;
}

// Hand block bi's slot back to the producer.  A slot is free once it has
// kConsumerWarps arrivals: every warp arrives once for a block they all read
// (attention), the one consuming warp arrives for all of them (GEMV tiles).
__device__ __forceinline__ void ring_release(const SmemLayout &S, const KParams &P, uint32_t bi, uint32_t count) {
    mbar_arrive_cnt(&S.empty[bi % (uint32_t)P.stages], count);
}

// ------------------------------------------------------------------ tagged reads
// Bounded spin for a reader whose words do not carry the expected tag yet.
struct LlSpin {
    uint64_t t0;
    uint32_t it;
};
__device__ __forceinline__ bool ll_spin(const KParams &P, const SmemLayout &S, LlSpin &sp, uint32_t who,
                                        uint32_t tag) {
    if ((++sp.it & 15u) == 0u) {
        if (*S.abort) return false;
        const uint64_t now = globaltimer_ns();
        if (sp.t0 == 0) {
            sp.t0 = now;
        } else if (now - sp.t0 > P.timeout_ns) {
            set_error(P, 4u, who, tag);
            *S.abort = 1;
            return false;
        }
    }
    return true;
}

// Slow path of the tagged reads: re-read the chunks (8 words each, chunk j
// at base[j]) that did not all carry `tag` yet until they do.  Kept out of
// line so the wait state costs the fast path no registers; it only runs while
// a producer has not published yet.
__device__ __noinline__ bool ll_spin_chunks(const KParams &P, const SmemLayout &S, const uint64_t *const *base,
                                            int m, uint32_t pending, uint32_t tag, float *vals, uint32_t who) {
    LlSpin sp{0ull, 0u};
    while (pending) {
        __nanosleep(16);
        for (int j = 0; j < m; ++j) {
            if (!((pending >> j) & 1u)) continue;
            // the chunk's four loads go out together, before any value is kept
            ulonglong2 w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) w[q] = ll_ld2(base[j] + 2 * q);
            bool all = true;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                all = all && ll_tag(w[q].x) == tag && ll_tag(w[q].y) == tag;
                vals[8 * j + 2 * q] = ll_value(w[q].x);
                vals[8 * j + 2 * q + 1] = ll_value(w[q].y);
            }
            if (all) pending &= ~(1u << j);
        }
        if (pending && !ll_spin(P, S, sp, who, tag)) return false;
    }
    return true;
}

// Read m <= M chunks of 8 tagged words (chunk j at ptr[j], 16-byte aligned),
// all loads in flight together; if any word does not carry `tag` yet, spin
// until all do.  The values go to f[j][0..7].  False when the wait gave up (f
// is then junk).
template <int M>
__device__ __forceinline__ bool ll_chunks(const KParams &P, const SmemLayout &S, const uint64_t *const (&ptr)[M],
                                          int m, uint32_t tag, float (&f)[M][8], uint32_t who) {
    uint32_t pending = 0;
#pragma unroll
    for (int j = 0; j < M; ++j)
        if (j < m) {
            bool ok = true;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const ulonglong2 w = ll_ld2(ptr[j] + 2 * q);
                ok = ok && ll_tag(w.x) == tag && ll_tag(w.y) == tag;
                f[j][2 * q] = ll_value(w.x);
                f[j][2 * q + 1] = ll_value(w.y);
            }
            if (!ok) pending |= 1u << j;
        }
    if (!pending) return true;
    return ll_spin_chunks(P, S, ptr, m, pending, tag, &f[0][0], who);
}

// One tagged word, spinning until it carries `tag`.
__device__ __forceinline__ bool ll_word(const KParams &P, const SmemLayout &S, const uint64_t *p, uint32_t tag,
                                        float &v, uint32_t who) {
    const uint64_t w = ll_ld(p);
    if (ll_tag(w) == tag) {
        v = ll_value(w);
        return true;
    }
    LlSpin sp{0ull, 0u};
    for (;;) {
        __nanosleep(16);
        if (!ll_spin(P, S, sp, who, tag)) return false;
        const uint64_t w2 = ll_ld(p);
        if (ll_tag(w2) == tag) {
            v = ll_value(w2);
            return true;
        }
    }
}

__device__ __forceinline__ uint32_t who_of(const Instr &in) { return ((uint32_t)in.op << 16) | in.layer; }

// The residual stream leaving layer l, x = x_end(l) + the outputs of the down
// projection's further K ranges (only plans whose batch rows exceed the
// activation budget have any), for 8 columns starting at col of sequence
// `row`; the same additions, in the same order, wherever x is formed.
__device__ __forceinline__ bool residual8(const KParams &P, const SmemLayout &S, int row, int col, uint32_t tag,
                                          float (&x)[8], uint32_t who) {
    const size_t H = (size_t)P.hidden, rows = (size_t)P.batch;
    const uint64_t *ptr[1] = {P.xe + (size_t)row * H + col};
    float f[1][8];
    bool ok = ll_chunks<1>(P, S, ptr, 1, tag, f, who);
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = f[0][q];
    for (int k = 1; k < P.down_ranges; ++k) {
        ptr[0] = P.dpart + ((size_t)(k - 1) * rows + row) * H + col;
        ok = ll_chunks<1>(P, S, ptr, 1, tag, f, who) && ok;
#pragma unroll
        for (int q = 0; q < 8; ++q) x[q] += f[0][q];
    }
    return ok;
}

// ------------------------------------------------------------------ activation staging
// Shared-memory position of the first of the 8 values of chunk c (values
// c*8 .. c*8+7 of a staged row); the other four sit 128 floats further.  A
// lane multiplies 8 consecutive columns of a 256-column chunk by the
// activations staged here: split into two float4 that the warp's 32 lanes
// read as two contiguous 512-byte runs, those reads are free of shared-memory
// bank conflicts (8 consecutive floats per lane would be 32 bytes apart,
// two lanes per bank group).
__device__ __forceinline__ int act_slot(int c) { return (c >> 5) * 256 + (c & 31) * 4; }

// Writes the instruction's activations for batch rows [b0, b0+nb) as fp32
// [nb][klen] into shared memory (each 256-value group in the act_slot order):
// RMSNorm(x) * gain for QKV / gate-up / LM head,
// a plain copy of the attention output or of the SwiGLU product otherwise.
// Each thread reads tagged words and spins until they carry the producing
// layer's tag.  Returns false if a wait gave up; every thread still reaches
// every barrier.
template <int BS>
__device__ __forceinline__ bool stage_act(const KParams &P, const SmemLayout &S, const Instr &in, const MatRef &m,
                                          int klen, float *red, uint32_t gen) {
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int nb = in.nb;
    float *act = reinterpret_cast<float *>(S.act);
    const uint32_t who = who_of(in);
    bool ok = true;
    if (in.op == OP_DOWN || in.op == OP_OPROJ) {
        // copy of the SwiGLU product or of the attention output; columns past
        // the logical row (block padding) are zero
        const int k0 = in.kb0 * m.kc, nch = klen / 8;
        const uint64_t *src = in.op == OP_DOWN ? P.act_a : P.attn;
        const int len = in.op == OP_DOWN ? P.intermediate : P.n_heads * P.head_dim;
        const uint32_t tag = act_tag(gen, P.n_layers, in.layer);
        for (int b = 0; b < nb; ++b) {
            const uint64_t *row = src + (size_t)(in.b0 + b) * len;
            float *dst = act + (size_t)b * klen;
            for (int c0 = t; c0 < nch; c0 += 4 * kConsumerThreads) {
                const uint64_t *ptr[4];
                int mm = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = c0 + j * kConsumerThreads;
                    ptr[j] = row + k0 + (size_t)c * 8;
                    if (c < nch && k0 + c * 8 < len) mm = j + 1;
                }
                float f[4][8];
                ok = ll_chunks<4>(P, S, ptr, mm, tag, f, who) && ok;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = c0 + j * kConsumerThreads;
                    if (c < nch) {
                        float4 *d0 = reinterpret_cast<float4 *>(dst + act_slot(c));
                        float4 *d1 = reinterpret_cast<float4 *>(dst + act_slot(c) + 128);
                        if (j < mm) {
                            *d0 = make_float4(f[j][0], f[j][1], f[j][2], f[j][3]);
                            *d1 = make_float4(f[j][4], f[j][5], f[j][6], f[j][7]);
                        } else {
                            *d0 = make_float4(0.f, 0.f, 0.f, 0.f);
                            *d1 = *d0;
                        }
                    }
                }
            }
        }
        return ok;
    }
    // RMSNorm(x) * gain with one pass over global memory: every thread reads
    // its chunks of x (all batch rows) together with the gains, accumulates
    // sum(x^2) and keeps x * gain in shared memory, then multiplies by the
    // per-row 1/rms once the sums are known (the gain and 1/rms commute).
    // Gate/up reads x_mid of its own layer; QKV (layer > 0) and the LM head
    // read x_mid plus the down parts of the previous layer.
    const int H = P.hidden;
    const uint16_t *gain = reinterpret_cast<const uint16_t *>(
        in.op == OP_QKV ? P.layers[in.layer].attn_norm
                        : (in.op == OP_GATEUP ? P.layers[in.layer].mlp_norm : P.final_norm));
    const bool from_embed = (in.flags & F_EMBED_X) && in.op == OP_QKV;
    const bool with_down = in.op != OP_GATEUP;
    const int xl = in.op == OP_GATEUP ? in.layer : (in.op == OP_LMHEAD ? P.n_layers - 1 : in.layer - 1);
    const uint32_t xtag = act_tag(gen, P.n_layers, xl);
    const uint16_t *emb = reinterpret_cast<const uint16_t *>(P.embed);
    float ss[BS];
#pragma unroll
    for (int b = 0; b < BS; ++b) ss[b] = 0.f;
    const int nch = klen / 8;
    const uint4 *g8 = reinterpret_cast<const uint4 *>(gain);
    // one batch row at a time keeps a single row's chunk in registers
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        if (b >= nb) break;
        const int row = in.b0 + b;
        for (int c = t; c < nch; c += kConsumerThreads) {
            float4 *d0 = reinterpret_cast<float4 *>(act + (size_t)b * klen + act_slot(c));
            float4 *d1 = reinterpret_cast<float4 *>(act + (size_t)b * klen + act_slot(c) + 128);
            if (c * 8 >= H) {
                *d0 = make_float4(0.f, 0.f, 0.f, 0.f);
                *d1 = *d0;
                continue;
            }
            float f[8], g[8];
            unpack8(__ldg(g8 + c), g);
            if (from_embed) {
                unpack8(__ldg(reinterpret_cast<const uint4 *>(emb + (size_t)token_of(P, row) * H) + c), f);
            } else if (with_down) {
                ok = residual8(P, S, row, c * 8, xtag, f, who) && ok;
            } else {
                const uint64_t *ptr[1] = {P.xm + (size_t)row * H + c * 8};
                float f1[1][8];
                ok = ll_chunks<1>(P, S, ptr, 1, xtag, f1, who) && ok;
#pragma unroll
                for (int q = 0; q < 8; ++q) f[q] = f1[0][q];
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) ss[b] = fmaf(f[q], f[q], ss[b]);
            *d0 = make_float4(f[0] * g[0], f[1] * g[1], f[2] * g[2], f[3] * g[3]);
            *d1 = make_float4(f[4] * g[4], f[5] * g[5], f[6] * g[6], f[7] * g[7]);
        }
    }
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        const float s = warp_sum(ss[b]);
        if (lane == 0) red[warp * BS + b] = s;
    }
    consumer_sync();
    float rs[BS];
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        float s = 0.f;
        for (int w = 0; w < kConsumerWarps; ++w) s += red[w * BS + b];
        rs[b] = rsqrtf(s / (float)H + P.rms_eps);
    }
    for (int c = t; c < nch; c += kConsumerThreads) {
        if (c * 8 >= H) continue;
#pragma unroll
        for (int b = 0; b < BS; ++b) {
            if (b < nb) {
                float4 *d0 = reinterpret_cast<float4 *>(act + (size_t)b * klen + act_slot(c));
                float4 *d1 = reinterpret_cast<float4 *>(act + (size_t)b * klen + act_slot(c) + 128);
                const float4 x0 = *d0, x1 = *d1;
                const float r = rs[b];
                *d0 = make_float4(x0.x * r, x0.y * r, x0.z * r, x0.w * r);
                *d1 = make_float4(x1.x * r, x1.y * r, x1.z * r, x1.w * r);
            }
        }
    }
    return ok;
}

// ------------------------------------------------------------------ GEMV: one warp per tile
// A tile is RT rows x (nkr blocks of kc columns) of one matrix, one ring slot
// per block.  Lane l owns columns c*256 + l*8 .. +8 of every block (kc/256
// chunks), accumulates RT x BS fp32 dot products, then the warp folds the RT
// rows across its lanes (log2(RT) halving steps, then butterflies) and the
// lanes holding a row's total run its epilogue.  No other warp takes part, so
// warps never wait for each other on GEMV work.

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

template <int BS, int RT>
__device__ __forceinline__ bool gemv_warp_tile(const KParams &P, const SmemLayout &S, CRing &ring, const Instr &in,
                                               const MatRef &m, int tile, uint32_t bi0, int klen, uint32_t gen) {
    const int lane = threadIdx.x & 31;
    const int nkr = in.kb1 - in.kb0, kc = m.kc, nch = kc / 256, nb = in.nb;
    const float *act = reinterpret_cast<const float *>(S.act);
    // row held by this lane after the fold: bit 4 is the top row bit, then bits 3, 2
    int fr = 0;
    if constexpr (RT == 8) fr = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
    if constexpr (RT == 4) fr = ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
    if constexpr (RT == 2) fr = (lane >> 4) & 1;
    const bool holder = (lane & (32 / RT - 1)) == 0;
    const int H = P.hidden;
    // The residual-stream word an epilogue adds to is read now, ahead of the
    // dot products, so its round trip overlaps them: x_end of the previous
    // layer for the O-projection, x_mid of this layer for the down
    // projection's first K range.
    const int n_out = tile * RT + fr;
    const bool early = holder && n_out < H &&
                       ((in.op == OP_OPROJ && !(in.flags & F_EMBED_X)) || (in.op == OP_DOWN && in.kb0 < P.down_per));
    const uint64_t *early_src = in.op == OP_OPROJ ? P.xe : P.xm;
    uint64_t pre[BS];
#pragma unroll
    for (int b = 0; b < BS; ++b) pre[b] = (early && b < nb) ? ll_ld(early_src + (size_t)(in.b0 + b) * H + n_out) : 0ull;
    float acc[RT][BS];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int b = 0; b < BS; ++b) acc[r][b] = 0.f;
    for (int j = 0; j < nkr; ++j) {
        const uint8_t *blk = ring_wait(P, S, ring, bi0 + j);
        for (int c = 0; c < nch; ++c) {
            const int col = c * 256 + lane * 8;
            float af[BS][8];
#pragma unroll
            for (int b = 0; b < BS; ++b) {
                if (b < nb) {
                    const float *ab = act + (size_t)b * klen + j * kc + c * 256 + lane * 4;
                    const float4 x0 = *reinterpret_cast<const float4 *>(ab);
                    const float4 x1 = *reinterpret_cast<const float4 *>(ab + 128);
                    af[b][0] = x0.x; af[b][1] = x0.y; af[b][2] = x0.z; af[b][3] = x0.w;
                    af[b][4] = x1.x; af[b][5] = x1.y; af[b][6] = x1.z; af[b][7] = x1.w;
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) af[b][q] = 0.f;
                }
            }
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                const uint4 w = *reinterpret_cast<const uint4 *>(blk + ((size_t)r * kc + col) * 2);
                float wf[8];
                unpack8(w, wf);
#pragma unroll
                for (int b = 0; b < BS; ++b)
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[r][b] = fmaf(wf[q], af[b][q], acc[r][b]);
            }
        }
        __syncwarp();
        if (lane == 0) ring_release(S, P, bi0 + j, kConsumerWarps);
    }
    float v[BS];
#pragma unroll
    for (int b = 0; b < BS; ++b) {
        float w[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) w[r] = r < RT ? acc[r < RT ? r : 0][b] : 0.f;
        int o = 16;
        if constexpr (RT >= 8) { fold_rows<8>(w, lane, o); o >>= 1; }
        if constexpr (RT >= 4) { fold_rows<4>(w, lane, o); o >>= 1; }
        if constexpr (RT >= 2) { fold_rows<2>(w, lane, o); o >>= 1; }
        for (; o >= 1; o >>= 1) w[0] += __shfl_xor_sync(0xFFFFFFFFu, w[0], o);
        v[b] = w[0];
    }
    // outputs carry this layer's tag (a stale one for the timeout test hook)
    const uint32_t tag = act_tag(gen, P.n_layers, in.layer) - ((in.flags & F_DROP_SIGNAL) ? 1u : 0u);
    bool ok = true;
    switch (in.op) {
        case OP_QKV: {
            const int n = tile * RT + fr;
            if (holder && n < P.qkv_rows)
#pragma unroll
                for (int b = 0; b < BS; ++b)
                    if (b < nb) ll_st(P.qkv + (size_t)(in.b0 + b) * P.qkv_rows + n, ll_pack(v[b], tag));
        } break;
        case OP_OPROJ: {
            // x_mid = x + attn . W_o^T, x being the embedding row (layer 0) or
            // the residual leaving the previous layer
            if (holder && n_out < H)
#pragma unroll
                for (int b = 0; b < BS; ++b) {
                    if (b >= nb) break;
                    const int row = in.b0 + b;
                    float base;
                    if (in.flags & F_EMBED_X) {
                        base = bf2f(reinterpret_cast<const uint16_t *>(P.embed)[(size_t)token_of(P, row) * H + n_out]);
                    } else {
                        const uint32_t xtag = act_tag(gen, P.n_layers, in.layer - 1);
                        const uint32_t who = who_of(in);
                        if (ll_tag(pre[b]) == xtag) base = ll_value(pre[b]);
                        else ok = ll_word(P, S, P.xe + (size_t)row * H + n_out, xtag, base, who) && ok;
                        for (int k = 1; k < P.down_ranges; ++k) {
                            float dv = 0.f;
                            ok = ll_word(P, S, P.dpart + ((size_t)(k - 1) * P.batch + row) * H + n_out, xtag, dv, who) &&
                                 ok;
                            base += dv;
                        }
                    }
                    ll_st(P.xm + (size_t)row * H + n_out, ll_pack(base + v[b], tag));
                }
        } break;
        case OP_DOWN: {
            // the first K range completes x_end = x_mid + its output; further
            // ranges publish their outputs on their own
            const int k = in.kb0 / P.down_per;
            if (holder && n_out < H)
#pragma unroll
                for (int b = 0; b < BS; ++b) {
                    if (b >= nb) break;
                    const int row = in.b0 + b;
                    if (k == 0) {
                        const uint32_t mtag = act_tag(gen, P.n_layers, in.layer);
                        float base;
                        if (ll_tag(pre[b]) == mtag) base = ll_value(pre[b]);
                        else ok = ll_word(P, S, P.xm + (size_t)row * H + n_out, mtag, base, who_of(in)) && ok;
                        ll_st(P.xe + (size_t)row * H + n_out, ll_pack(base + v[b], tag));
                    } else {
                        ll_st(P.dpart + ((size_t)(k - 1) * P.batch + row) * H + n_out, ll_pack(v[b], tag));
                    }
                }
        } break;
        case OP_GATEUP: {
            // gate rows 0..RT/2-1, up rows RT/2..RT-1: the up partner is lane ^ 16
            float up[BS];
#pragma unroll
            for (int b = 0; b < BS; ++b) up[b] = __shfl_xor_sync(0xFFFFFFFFu, v[b], 16);
            const int j = tile * (RT / 2) + fr;
            if (RT >= 2 && holder && (lane & 16) == 0 && j < P.intermediate)
#pragma unroll
                for (int b = 0; b < BS; ++b)
                    if (b < nb)
                        ll_st(P.act_a + (size_t)(in.b0 + b) * P.intermediate + j,
                              ll_pack(v[b] / (1.0f + __expf(-v[b])) * up[b], tag));
        } break;
        default: {  // OP_LMHEAD: logits, then the warp's best of this tile folded into the CTA's
            const int n = tile * RT + fr;
            const bool valid = holder && n < P.vocab;
#pragma unroll
            for (int b = 0; b < BS; ++b) {
                if (b >= nb) break;
                if (valid && P.logits) __stcg(P.logits + (size_t)(in.b0 + b) * P.vocab + n, v[b]);
                unsigned long long key = valid ? argmax_key(v[b], n) : 0ull;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, key, o);
                    key = other > key ? other : key;
                }
                if (lane == 0) atomicMax(S.best + in.b0 + b, key);
            }
        } break;
    }
    return ok;
}

// Publish this CTA's best (value, index) per sequence; the last CTA to do so
// picks the token and advances the step state.
__device__ __forceinline__ void lm_publish(const KParams &P, const SmemLayout &S, const Instr &in, uint32_t gen, int pos) {
    const int t = threadIdx.x;
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

// One GEMV instruction: a run of consecutive tiles.  Tile k goes to warp
// (tc + k) % warps (tc counts this CTA's tiles so far) and uses ring blocks
// bc + k*nkr .. bc + (k+1)*nkr - 1 (bc counts this CTA's ring blocks so far).
// Returns true when the CTA must stop (a wait gave up).
template <int BS>
__device__ __forceinline__ bool gemv_instr(const KParams &P, const SmemLayout &S, CRing &ring, const Instr &in,
                                           uint64_t &staged_key, uint32_t gen, int pos, uint32_t &bc, uint32_t &tc,
                                           int ii) {
    const int warp = threadIdx.x >> 5;
    const MatRef m = mat_of(P, in);
    const int nkr = in.kb1 - in.kb0, klen = nkr * m.kc;
    const uint64_t key = ((uint64_t)in.op << 56) | ((uint64_t)in.layer << 40) | ((uint64_t)in.b0 << 24) |
                         ((uint64_t)in.kb0 << 12) | (uint64_t)in.kb1;
    if (key != staged_key) {
        consumer_sync();  // no warp still reads the previous activations
        const bool ok = stage_act<BS>(P, S, in, m, klen, S.ssq, gen);
        staged_key = key;
        if (consumer_sync_or(!ok || *S.abort != 0)) return true;
    }
    if (P.trace && threadIdx.x == 0) P.trace[8 * (size_t)ii + 7] = globaltimer_ns();  // activations staged
    const int T = (int)in.ntiles;
    bool ok = true;
    for (int k = (int)((warp - tc % kConsumerWarps + kConsumerWarps) % kConsumerWarps); k < T; k += kConsumerWarps) {
        const uint32_t bi0 = bc + (uint32_t)(k * nkr);
        switch (m.rows) {
            case 8: ok = gemv_warp_tile<BS, 8>(P, S, ring, in, m, (int)in.tile + k, bi0, klen, gen) && ok; break;
            case 4: ok = gemv_warp_tile<BS, 4>(P, S, ring, in, m, (int)in.tile + k, bi0, klen, gen) && ok; break;
            case 2: ok = gemv_warp_tile<BS, 2>(P, S, ring, in, m, (int)in.tile + k, bi0, klen, gen) && ok; break;
            default: ok = gemv_warp_tile<BS, 1>(P, S, ring, in, m, (int)in.tile + k, bi0, klen, gen) && ok; break;
        }
    }
    bc += (uint32_t)(T * nkr);
    tc += (uint32_t)T;
    if ((in.op == OP_OPROJ || in.op == OP_DOWN) && consumer_sync_or(!ok || *S.abort != 0)) return true;  // epilogues read x
    if (in.op == OP_LMHEAD && (in.flags & F_LAST_LM)) lm_publish(P, S, in, gen, pos);
    return false;
}

// ------------------------------------------------------------------ attention
// One warp prepares one head: optional per-head RMSNorm, rotate-half RoPE at
// `pos` (from the step's cos/sin table), scale.
__device__ __forceinline__ bool prep_head(const KParams &P, const SmemLayout &S, const uint64_t *src, uint32_t tag,
                                          const uint16_t *gain, int pos, float scale, float *dst, uint16_t *cache_row) {
    const int lane = threadIdx.x & 31, d = P.head_dim, nj = d / 32, jh = nj / 2;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    bool ok = true;
    {
        uint64_t w[4];
        LlSpin sp{0ull, 0u};
        for (;;) {
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = j < nj ? ll_ld(src + lane + 32 * j) : ll_pack(0.f, tag);
            bool all = true;
#pragma unroll
            for (int j = 0; j < 4; ++j) all = all && ll_tag(w[j]) == tag;
            if (all) break;
            __nanosleep(16);
            if (!ll_spin(P, S, sp, ((uint32_t)OP_ATTN << 16), tag)) {
                ok = false;
                break;
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = ll_value(w[j]);
    }
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
    // rotate-half pairs (i, i + d/2): d = 64 -> (v0, v1); d = 128 -> (v0, v2), (v1, v3)
    auto rot = [&](float &x, float &y, int i) {
        const float2 cs = S.rope[i];
        const float a = x, b = y;
        x = a * cs.x - b * cs.y;
        y = b * cs.x + a * cs.y;
    };
    if (jh == 1) {
        rot(v[0], v[1], lane);
    } else {
        rot(v[0], v[2], lane);
        rot(v[1], v[3], lane + 32);
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
    return ok;
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

// One split-KV unit: the G query heads of KV head g over positions [p0, p1).
// Warps are split into G groups of wph = 8 / G; warp (h, s) takes positions
// s*32 + k*wph*32 + lane of every ring stage, one position per lane, and keeps
// its own online-softmax state (running max m, sum l, unnormalised output o)
// in registers, so a stage needs no CTA barrier.  The warps of a head merge at
// the end and write the chunk's partial (o, m, l) as tagged words; a combine
// instruction later merges the group's chunks.
constexpr int kAttnStop = 1;

// DPL consecutive bf16 values (2 or 4) of one V row, widened.
template <int DPL>
__device__ __forceinline__ void load_dpl(const uint16_t *p, float *v) {
    if constexpr (DPL == 2) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
        v[0] = bf_lo(w);
        v[1] = bf_hi(w);
    } else {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        v[0] = bf_lo(w.x);
        v[1] = bf_hi(w.x);
        v[2] = bf_lo(w.y);
        v[3] = bf_hi(w.y);
    }
}

template <int D>
__device__ __forceinline__ int attn_instr(const KParams &P, const SmemLayout &S, CRing &ring, const Instr &in,
                                          uint32_t gen, int pos, uint32_t &bc, int ii) {
    constexpr int NCH = D / 8, DPL = D / 32;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int d = D, nkv = P.n_kv_heads, G = P.n_heads / nkv, l = in.layer;
    const int NC = P.chunks, nq = P.n_heads;
    const AttnGeom a = attn_geom(P, in, pos);
    const int sp = kStageBytes / (4 * d);
    const int wph = kConsumerWarps / G, h = warp / wph, sl = warp % wph;
    const bool active = h < G;
    const int dpl = d / 32;  // output dimensions per lane: lane*dpl .. lane*dpl + dpl - 1
    float *qs = reinterpret_cast<float *>(S.act);  // [G][d] rotated, scaled queries
    float *kpos = qs + G * d;                       // [d] key of this step's position
    float *vpos = kpos + d;                         // [d] value of this step's position
    float *mrg = vpos + d;                          // [8 warps][d + 2] per-warp states
    float *pbuf = mrg + kConsumerWarps * (d + 2);   // [8 warps][64] probabilities
    const uint64_t *qkv_b = P.qkv + (size_t)a.b * P.qkv_rows;
    const uint32_t tag = act_tag(gen, P.n_layers, l);
    const LayerW *LW = P.layers + l;
    const float qscale = 1.4426950408889634f * rsqrtf((float)d);  // log2(e)/sqrt(d): scores in the exp2 domain
    bool ok = true;
    consumer_sync();  // the previous instruction's readers of the activation region are done
    if (warp < G) {
        ok = prep_head(P, S, qkv_b + (a.g * G + warp) * d, tag,
                       P.qk_norm ? reinterpret_cast<const uint16_t *>(LW->q_norm) : nullptr, pos, qscale,
                       qs + warp * d, nullptr);
    } else if (a.has_cur && warp == G) {
        ok = prep_head(P, S, qkv_b + nq * d + a.g * d, tag,
                       P.qk_norm ? reinterpret_cast<const uint16_t *>(LW->k_norm) : nullptr, pos, 1.0f, kpos,
                       P.kcache + kv_off(P, l, a.b, a.g, pos));
    }
    if (a.has_cur && warp == kConsumerWarps - 1) {
        // this step's V row: a lane's d/32 words are loaded together and
        // re-read together until all carry the tag (one round trip, not one
        // per word)
        const uint64_t *vs = qkv_b + (nq + nkv) * d + a.g * d;
        uint16_t *vrow = P.vcache + kv_off(P, l, a.b, a.g, pos);
        const int nj = d / 32;
        uint64_t w[4];
        LlSpin sp{0ull, 0u};
        for (;;) {
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = j < nj ? ll_ld(vs + lane + 32 * j) : ll_pack(0.f, tag);
            bool all = true;
#pragma unroll
            for (int j = 0; j < 4; ++j) all = all && ll_tag(w[j]) == tag;
            if (all) break;
            __nanosleep(16);
            if (!ll_spin(P, S, sp, (uint32_t)OP_ATTN << 16, tag)) {
                ok = false;
                break;
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j < nj) {
                const uint16_t hv = f2bf(ll_value(w[j]));
                vrow[lane + 32 * j] = hv;
                vpos[lane + 32 * j] = bf2f(hv);
            }
    }
    if (consumer_sync_or(!ok || *S.abort != 0)) return kAttnStop;
    if (a.has_cur && G == kConsumerWarps) {  // every warp held a query head: the key comes now
        if (warp == 0)
            ok = prep_head(P, S, qkv_b + nq * d + a.g * d, tag,
                           P.qk_norm ? reinterpret_cast<const uint16_t *>(LW->k_norm) : nullptr, pos, 1.0f, kpos,
                           P.kcache + kv_off(P, l, a.b, a.g, pos));
        if (consumer_sync_or(!ok || *S.abort != 0)) return kAttnStop;
    }
    if (P.trace && t == 0) P.trace[8 * (size_t)ii + 7] = globaltimer_ns();  // heads prepared
    float m = -CUDART_INF_F, lsum = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    const float *qh = qs + (active ? h : 0) * d;
    float *pw = pbuf + warp * 64;  // this warp's probabilities, broadcast to all lanes for P.V
    for (int st = 0; st < a.nstages; ++st) {
        const int n = min(sp, a.tma_end - (a.p0 + st * sp));
        const uint8_t *slot = ring_wait(P, S, ring, bc + st);
        if (active) {
            const uint16_t *K = reinterpret_cast<const uint16_t *>(slot);
            const uint16_t *V = reinterpret_cast<const uint16_t *>(slot + kStageBytes / 2);
            // Each pass takes two 32-position groups of this warp's share
            // (base and base + 32 * wph), one position of each per lane, so
            // every q load and every reduction serves two positions.
            for (int base = sl * 32; base < n; base += 2 * wph * 32) {
                const int j0 = base + lane, j1 = base + wph * 32 + lane;
                const bool v0 = j0 < n, v1 = j1 < n;
                float a0 = 0.f, b0 = 0.f, a1 = 0.f, b1 = 0.f;
                const uint16_t *kr0 = K + (size_t)(v0 ? j0 : 0) * D, *kr1 = K + (size_t)(v1 ? j1 : 0) * D;
#pragma unroll
                for (int k = 0; k < NCH; ++k) {
                    // rotated chunk order: the lanes' 16-byte reads hit different banks
                    const int cc = (k + lane) & (NCH - 1);
                    float k0[8], k1[8];
                    unpack8(*reinterpret_cast<const uint4 *>(kr0 + cc * 8), k0);
                    unpack8(*reinterpret_cast<const uint4 *>(kr1 + cc * 8), k1);
                    const float4 q0 = *reinterpret_cast<const float4 *>(qh + cc * 8);
                    const float4 q1 = *reinterpret_cast<const float4 *>(qh + cc * 8 + 4);
                    a0 = fmaf(q0.x, k0[0], a0); b0 = fmaf(q0.y, k0[1], b0);
                    a1 = fmaf(q0.x, k1[0], a1); b1 = fmaf(q0.y, k1[1], b1);
                    a0 = fmaf(q0.z, k0[2], a0); b0 = fmaf(q0.w, k0[3], b0);
                    a1 = fmaf(q0.z, k1[2], a1); b1 = fmaf(q0.w, k1[3], b1);
                    a0 = fmaf(q1.x, k0[4], a0); b0 = fmaf(q1.y, k0[5], b0);
                    a1 = fmaf(q1.x, k1[4], a1); b1 = fmaf(q1.y, k1[5], b1);
                    a0 = fmaf(q1.z, k0[6], a0); b0 = fmaf(q1.w, k0[7], b0);
                    a1 = fmaf(q1.z, k1[6], a1); b1 = fmaf(q1.w, k1[7], b1);
                }
                const float sc0 = v0 ? a0 + b0 : -CUDART_INF_F, sc1 = v1 ? a1 + b1 : -CUDART_INF_F;
                const float mb = warp_max(fmaxf(sc0, sc1));
                const float mnew = fmaxf(m, mb);
                const float corr = exp2f(m - mnew);
                const float p0 = v0 ? exp2f(sc0 - mnew) : 0.f, p1 = v1 ? exp2f(sc1 - mnew) : 0.f;
                lsum = lsum * corr + warp_sum(p0 + p1);
                m = mnew;
                pw[lane] = p0;
                pw[32 + lane] = p1;
                __syncwarp();
                // P.V: lane owns DPL dimensions; rows four at a time, two
                // accumulator sets so consecutive FMAs do not depend on each other
                float oa[DPL], ob[DPL];
#pragma unroll
                for (int e = 0; e < DPL; ++e) oa[e] = ob[e] = 0.f;
#pragma unroll
                for (int grp = 0; grp < 2; ++grp) {
                    const int gbase = base + grp * wph * 32;
                    const int cnt = max(0, min(32, n - gbase));
                    const float *pg = pw + grp * 32;
                    const uint16_t *vb = V + (size_t)gbase * D + lane * DPL;
                    int jj = 0;
                    for (; jj + 4 <= cnt; jj += 4) {
                        const float4 p4 = *reinterpret_cast<const float4 *>(pg + jj);
                        float w0[DPL], w1[DPL], w2[DPL], w3[DPL];
                        load_dpl<DPL>(vb + (size_t)(jj + 0) * D, w0);
                        load_dpl<DPL>(vb + (size_t)(jj + 1) * D, w1);
                        load_dpl<DPL>(vb + (size_t)(jj + 2) * D, w2);
                        load_dpl<DPL>(vb + (size_t)(jj + 3) * D, w3);
#pragma unroll
                        for (int e = 0; e < DPL; ++e) {
                            oa[e] = fmaf(p4.x, w0[e], oa[e]);
                            ob[e] = fmaf(p4.y, w1[e], ob[e]);
                            oa[e] = fmaf(p4.z, w2[e], oa[e]);
                            ob[e] = fmaf(p4.w, w3[e], ob[e]);
                        }
                    }
                    for (; jj < cnt; ++jj) {
                        float w0[DPL];
                        load_dpl<DPL>(vb + (size_t)jj * D, w0);
#pragma unroll
                        for (int e = 0; e < DPL; ++e) oa[e] = fmaf(pg[jj], w0[e], oa[e]);
                    }
                }
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[e] = fmaf(o[e], corr, oa[e] + ob[e]);
                __syncwarp();  // pw is rewritten by the next pass
            }
        }
        __syncwarp();
        if (lane == 0) ring_release(S, P, bc + st, 1);
    }
    bc += (uint32_t)a.nstages;
    if (a.has_cur && active && sl == 0) {  // this step's own position, from fp32 rows
        float part = 0.f;
        for (int e = lane; e < d; e += 32) part = fmaf(qh[e], kpos[e], part);
        const float sc = warp_sum(part);
        const float mnew = fmaxf(m, sc);
        const float corr = exp2f(m - mnew);
        const float p = exp2f(sc - mnew);
        lsum = lsum * corr + p;
        m = mnew;
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (e < dpl) o[e] = o[e] * corr + p * vpos[lane * dpl + e];
    }
    // merge the warps of each head
    if (active) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (e < dpl) mrg[warp * (d + 2) + lane * dpl + e] = o[e];
        if (lane == 0) {
            mrg[warp * (d + 2) + d] = m;
            mrg[warp * (d + 2) + d + 1] = lsum;
        }
    }
    consumer_sync();
    uint64_t *part = P.partials;
    if (active && sl == 0) {
        const int w0 = h * wph;
        float M = -CUDART_INF_F;
        for (int k = 0; k < wph; ++k) M = fmaxf(M, mrg[(w0 + k) * (d + 2) + d]);
        float L = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < wph; ++k) {
            const float mk = mrg[(w0 + k) * (d + 2) + d];
            const float wk = (mk == -CUDART_INF_F) ? 0.f : exp2f(mk - M);
            L = fmaf(wk, mrg[(w0 + k) * (d + 2) + d + 1], L);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (e < dpl) O[e] = fmaf(wk, mrg[(w0 + k) * (d + 2) + lane * dpl + e], O[e]);
        }
        const int hg = a.g * G + h;
        uint64_t *pd = part + (((size_t)a.b * nq + hg) * NC + a.c) * partial_stride(d);
        const uint32_t ptag = tag - ((in.flags & F_DROP_SIGNAL) ? 1u : 0u);
        ll_st2(pd + lane * dpl, ll_pack(O[0], ptag), ll_pack(O[1], ptag));
        if (dpl == 4) ll_st2(pd + lane * dpl + 2, ll_pack(O[2], ptag), ll_pack(O[3], ptag));
        if (lane == 0) ll_st2(pd + d, ll_pack(M, ptag), ll_pack(L, ptag));
    }
    return consumer_sync_or(*S.abort != 0) ? kAttnStop : 0;
}

// ------------------------------------------------------------------ split-KV combine
// Merge the chunk partials of one (sequence, KV head) into its G heads'
// attention output: attn[h*d + e] = sum_c 2^(m_c - M) o_c[e] / sum_c 2^(m_c - M) l_c,
// M = max_c m_c (scores are in the base-2 domain).  tpi threads of one warp
// share a float4 of output and take every tpi-th chunk, so each thread has at
// most four chunks' loads in flight; they merge their (max, sum, vector) by
// shuffles.  Returns true when the CTA must stop.
__device__ __forceinline__ bool acomb_instr(const KParams &P, const SmemLayout &S, const Instr &in, uint32_t gen) {
    const int t = threadIdx.x;
    const int d = P.head_dim, nkv = P.n_kv_heads, G = P.n_heads / nkv, nq = P.n_heads, NC = P.chunks;
    const int b = (int)in.tile / nkv, g = (int)in.tile % nkv;
    const uint32_t tag = act_tag(gen, P.n_layers, in.layer);
    const uint32_t otag = tag - ((in.flags & F_DROP_SIGNAL) ? 1u : 0u);
    const int ps = partial_stride(d), items = G * d / 4;
    int tpi = 1;
    while (tpi < 16 && tpi < NC && 2 * tpi * items <= kConsumerThreads) tpi *= 2;
    const int per_pass = kConsumerThreads / tpi, q = t % tpi;
    uint64_t *dst = P.attn + (size_t)b * nq * d + (size_t)g * G * d;
    bool ok = true;
    for (int i0 = 0; i0 < items; i0 += per_pass) {
        const int it = i0 + t / tpi;
        const bool mine = it < items;
        const int h = mine ? (4 * it) / d : 0, e = mine ? (4 * it) % d : 0;
        const uint64_t *pc = P.partials + (((size_t)b * nq + g * G + h) * NC) * ps;
        float M = -CUDART_INF_F, L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c0 = q; c0 < NC; c0 += 2 * tpi) {
            ulonglong2 ml[2], o01[2], o23[2];
            LlSpin sp{0ull, 0u};
                for (;;) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = c0 + u * tpi;
                    if (mine && c < NC) {
                        const uint64_t *r = pc + (size_t)c * ps;
                        ml[u] = ll_ld2(r + d);
                        o01[u] = ll_ld2(r + e);
                        o23[u] = ll_ld2(r + e + 2);
                    }
                }
                bool all = true;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = c0 + u * tpi;
                    if (mine && c < NC)
                        all = all && ll_tag(ml[u].x) == tag && ll_tag(ml[u].y) == tag && ll_tag(o01[u].x) == tag &&
                              ll_tag(o01[u].y) == tag && ll_tag(o23[u].x) == tag && ll_tag(o23[u].y) == tag;
                }
                if (all) break;
                __nanosleep(16);
                if (!ll_spin(P, S, sp, who_of(in), tag)) {
                    ok = false;
                    break;
                }
            }
            float Mn = M;
#pragma unroll
            for (int u = 0; u < 2; ++u)
                if (mine && c0 + u * tpi < NC) Mn = fmaxf(Mn, ll_value(ml[u].x));
            const float r = (M == -CUDART_INF_F) ? 0.f : exp2f(M - Mn);
            L *= r;
            acc.x *= r; acc.y *= r; acc.z *= r; acc.w *= r;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (!(mine && c0 + u * tpi < NC)) continue;
                const float mu = ll_value(ml[u].x);
                const float w = (mu == -CUDART_INF_F) ? 0.f : exp2f(mu - Mn);
                L = fmaf(w, ll_value(ml[u].y), L);
                acc.x = fmaf(w, ll_value(o01[u].x), acc.x);
                acc.y = fmaf(w, ll_value(o01[u].y), acc.y);
                acc.z = fmaf(w, ll_value(o23[u].x), acc.z);
                acc.w = fmaf(w, ll_value(o23[u].y), acc.w);
            }
            M = Mn;
        }
        // merge the tpi partial states of this float4 (lanes q = 0 .. tpi-1)
        for (int o2 = 1; o2 < tpi; o2 <<= 1) {
            const float Mo = __shfl_xor_sync(0xFFFFFFFFu, M, o2);
            const float Lo = __shfl_xor_sync(0xFFFFFFFFu, L, o2);
            const float ax = __shfl_xor_sync(0xFFFFFFFFu, acc.x, o2), ay = __shfl_xor_sync(0xFFFFFFFFu, acc.y, o2);
            const float az = __shfl_xor_sync(0xFFFFFFFFu, acc.z, o2), aw = __shfl_xor_sync(0xFFFFFFFFu, acc.w, o2);
            const float Mn = fmaxf(M, Mo);
            const float ra = (M == -CUDART_INF_F) ? 0.f : exp2f(M - Mn);
            const float rb = (Mo == -CUDART_INF_F) ? 0.f : exp2f(Mo - Mn);
            L = L * ra + Lo * rb;
            acc = make_float4(acc.x * ra + ax * rb, acc.y * ra + ay * rb, acc.z * ra + az * rb, acc.w * ra + aw * rb);
            M = Mn;
        }
        if (mine && q == 0) {
            const float inv = 1.0f / L;
            ll_st2(dst + h * d + e, ll_pack(acc.x * inv, otag), ll_pack(acc.y * inv, otag));
            ll_st2(dst + h * d + e + 2, ll_pack(acc.z * inv, otag), ll_pack(acc.w * inv, otag));
        }
    }
    return consumer_sync_or(!ok || *S.abort != 0);
}

// Counter increment after an instruction's outputs are stored: a release,
// so a reader that acquires the counter sees the data.
__device__ __forceinline__ void signal_counter(const KParams &P, uint32_t ctr, uint32_t n) {
    red_release_add(P.counters + ctr, n);
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
    CRing ring{0ull};
    uint32_t bc = 0, tc = 0;  // ring blocks and GEMV tiles of this CTA consumed so far
    uint64_t staged_key = ~0ull;  // which activations the shared-memory region holds
    uint32_t sat_ctr = 0xFFFFFFFFu, sat_target = 0u;
    uint32_t pend_ctr = kNoCounter, pend_n = 0u;
    bool stop = false;
    if (P.pdl == 1) pdl_wait();  // 2: start on the tiles read, not on the previous kernel's end
    consumer_sync();
    // instructions are fetched three ahead: an L2 round trip is longer than
    // one instruction's work, and L1 is nearly all given to shared memory
    Instr q1, q2, q3;
    if (begin < end) q1 = load_instr(P, begin);
    if (begin + 1 < end) q2 = load_instr(P, begin + 1);
    if (begin + 2 < end) q3 = load_instr(P, begin + 2);
    for (int i = begin; i < end && !stop; ++i) {
        const Instr in = q1;
        q1 = q2;
        q2 = q3;
        if (i + 3 < end) q3 = load_instr(P, i + 3);
        unsigned long long t_start = 0;
        if (P.trace && t == 0) t_start = globaltimer_ns();
        if (P.use_waits && in.wait_ctr != kNoCounter) {
            const uint32_t target = (gen + 1u) * in.wait_count;
            if (in.wait_ctr != sat_ctr || target != sat_target) {
                if (pend_n) consumer_sync();  // this CTA's earlier writes are complete
                if (t == 0) {
                    if (pend_n) signal_counter(P, pend_ctr, pend_n);
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
        const bool signal = P.use_signals && in.op != OP_LMHEAD && !(in.flags & F_DROP_SIGNAL);
        if (in.op == OP_ATTN) {
            const int r = P.head_dim == 64 ? attn_instr<64>(P, S, ring, in, gen, pos, bc, i)
                                           : attn_instr<128>(P, S, ring, in, gen, pos, bc, i);
            stop = (r & kAttnStop) != 0;
            staged_key = ~0ull;
        } else if (in.op == OP_ACOMB) {
            stop = acomb_instr(P, S, in, gen);
        } else {
            stop = gemv_instr<BS>(P, S, ring, in, staged_key, gen, pos, bc, tc, i);
        }
        if (!stop) {
            if (signal) {
                if (pend_ctr != in.signal_ctr) {
                    if (pend_n) {
                        consumer_sync();
                        if (t == 0) signal_counter(P, pend_ctr, pend_n);
                    }
                    pend_ctr = in.signal_ctr;
                    pend_n = 0u;
                }
                ++pend_n;
            }
        }
        if (P.trace) consumer_sync();  // "done" means every warp is done (tracing only)
        if (P.trace && t == 0) {
            P.trace[8 * (size_t)i + 2] = globaltimer_ns();
            P.trace[8 * (size_t)i + 4] = ring.waited;
            ring.waited = 0;
        }
    }
    if (!stop && pend_n) {
        consumer_sync();
        if (t == 0) signal_counter(P, pend_ctr, pend_n);
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
            S.seq[s] = 0xFFFFFFFFu;
        }
        *S.abort = 0;
        *S.flag = 0;
        fence_barrier_init();
    }
    // Position and step of this launch (the step state changes only in the
    // last phase of a step, after every other phase of it has finished).
    const uint32_t gen = *reinterpret_cast<volatile const uint32_t *>(&P.state->gen);
    const int pos = *reinterpret_cast<volatile const int32_t *>(&P.state->pos);
    // RoPE angles pos * theta^(-2i/d) in double, reduced mod 2*pi, then the
    // fp32 sine and cosine of the reduced angle (|angle| <= pi).
    for (int i = t; i < P.head_dim / 2; i += kThreads) {
        double ang = (double)pos * P.rope_inv_freq[i];
        ang -= 6.283185307179586 * rint(ang * 0.15915494309189535);
        float sn, cs;
        __sincosf((float)ang, &sn, &cs);
        S.rope[i] = make_float2(cs, sn);
    }
    if (t < 64) S.best[t] = argmax_key(-CUDART_INF_F, 0x7fffffff);
    check_tokens(P);
    __syncthreads();
    const int begin = P.cta_begin[blockIdx.x], end = P.cta_end[blockIdx.x];
    if (t >= kConsumerThreads) {
        if ((t & 31) == 0) producer(P, S, begin, end, pos);
        __syncwarp();
    } else {
        consumer<BS>(P, S, begin, end, gen, pos);
    }
    __syncthreads();
}

// ------------------------------------------------------------------ packing
// dst block (t, kb), row r, column col  <-  source row, column kb*kc + col.
// mode 0: source row t*rows + r of src; mode 1 (gate/up): rows r < rows/2 are
// gate row t*rows/2 + r, the others up row t*rows/2 + r - rows/2.
__global__ void pack_kernel(const uint16_t *src, const uint16_t *src2, uint16_t *dst, int n_rows, int k, int kc,
                            int nkb, int tiles, int rows, int mode) {
    const size_t total8 = (size_t)tiles * nkb * rows * kc / 8;
    for (size_t v = (size_t)blockIdx.x * blockDim.x + threadIdx.x; v < total8; v += (size_t)gridDim.x * blockDim.x) {
        const size_t e = v * 8;
        const int col = (int)(e % kc);
        size_t rest = e / kc;
        const int r = (int)(rest % rows);
        rest /= rows;
        const int kb = (int)(rest % nkb);
        const int t = (int)(rest / nkb);
        const int kk = kb * kc + col;
        const uint16_t *s = src;
        int row = t * rows + r;
        if (mode == 1) {
            const int half = rows / 2;
            row = t * half + (r % half);
            s = r < half ? src : src2;
        }
        uint16_t out[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) out[q] = (row < n_rows && kk + q < k) ? s[(size_t)row * k + kk + q] : (uint16_t)0;
        *reinterpret_cast<uint4 *>(dst + e) = *reinterpret_cast<uint4 *>(out);
    }
}

__global__ void set_position_kernel(State *state, int pos) { state->pos = pos; }

cudaError_t launch_set_position(State *state, int pos, cudaStream_t s) {
    set_position_kernel<<<1, 1, 0, s>>>(state, pos);
    return cudaGetLastError();
}

cudaError_t launch_pack(const void *src, const void *src2, void *dst, int n_rows, int k, int kc, int nkb, int tiles,
                        int rows, int mode, cudaStream_t s) {
    pack_kernel<<<1184, 256, 0, s>>>(static_cast<const uint16_t *>(src), static_cast<const uint16_t *>(src2),
                                     static_cast<uint16_t *>(dst), n_rows, k, kc, nkb, tiles, rows, mode);
    return cudaGetLastError();
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

const void *step_kernel_func(const KParams &P) {
    if (P.bs <= 1) return reinterpret_cast<const void *>(step_kernel<1>);
    if (P.bs <= 2) return reinterpret_cast<const void *>(step_kernel<2>);
    return reinterpret_cast<const void *>(step_kernel<4>);
}

cudaError_t launch_step(const KParams &P, int bs, int n_ctas, cudaStream_t s, bool cooperative, bool pdl_attr) {
    if (bs <= 1) return launch_bs<1>(P, n_ctas, s, cooperative, pdl_attr);
    if (bs <= 2) return launch_bs<2>(P, n_ctas, s, cooperative, pdl_attr);
    return launch_bs<4>(P, n_ctas, s, cooperative, pdl_attr);
}

}  // namespace mk

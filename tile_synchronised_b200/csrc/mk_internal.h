// mk_internal.h -- structures shared by the host scheduler and the device
// interpreter of the decode megakernel.  Plain C++ (no CUDA types) so the
// scheduler compiles with the host compiler as well.
#pragma once
#include <stdint.h>

namespace mk {

// ---------------------------------------------------------------- constants
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;   // 256
constexpr int kThreads = kConsumerThreads + 32;         // + one producer warp
constexpr int kStageBytes = 32768;                      // one ring slot
constexpr int kMaxStages = 8;
constexpr int kMaxTileRows = 8;                         // weight rows per GEMV tile (fewer for long rows)
constexpr int kMaxBatchRows = 4;                        // batch rows one GEMV instruction carries
constexpr int kMaxSmem = 232448;                        // opt-in dynamic smem per CTA on sm_100
// shared memory after the ring and the activations: barriers, flags, two reduction buffers
// Batch rows of the kernel instance that runs a plan carrying `bs` rows per
// instruction (instances exist for 1, 2 and 4).
constexpr int kernel_bs(int bs) { return bs <= 1 ? 1 : (bs <= 2 ? 2 : 4); }
// Bytes after the ring and the activation region: barriers, flags, small
// arrays and the RoPE table.
constexpr int misc_bytes(int bs, int stages) { return 2560 + 0 * bs * stages; }
constexpr int kMaxAttnChunks = 16;  // split-KV chunks per (sequence, KV head); one combine instruction gathers them
// Tagged words per split-KV partial record: o[d], m, l.
constexpr int partial_stride(int head_dim) { return head_dim + 2; }
constexpr int kMaxGroup = 8;                            // query heads per KV head
constexpr int kPrefillRows = 128;     // positions of one sequence per tensor-core prefill chunk (hi/lo: 256 MMA columns)
constexpr int kPrefillChunks = 16;    // most split-KV chunks per row in the prefill's causal attention
constexpr uint16_t kNoCounter = 0xFFFF;

// ---------------------------------------------------------------- opcodes
// Every activation that crosses an instruction boundary is a tagged word:
// the fp32 value in the low half, the tag of the (step, layer) that wrote it in
// the high half, stored and loaded as one 64-bit access.  A reader knows the
// tag it expects, so a stale word can never pass for a fresh one.
enum Op : uint8_t {
    OP_QKV = 1,     // RMSNorm(x) . W_qkv^T                      -> qkv
    OP_ATTN = 2,    // RoPE/qk-norm, KV append, one split-KV chunk -> partial (o, m, l)
    OP_OPROJ = 3,   // x_mid = x + attn . W_o^T        (x = x_end + further down parts of the previous layer)
    OP_GATEUP = 4,  // RMSNorm(x_mid) . [W_g;W_u]^T, SiLU(g)*u   -> a
    OP_DOWN = 5,    // a . W_d^T over one K range: x_end = x_mid + range 0, further ranges -> down parts
    OP_LMHEAD = 6,  // RMSNorm(x) . W_head^T -> logits, running argmax; last arriver picks the token
    OP_ACOMB = 7,   // log-sum-exp combine of one (sequence, KV head)'s chunk partials -> attn
};

enum Flags : uint8_t {
    F_EMBED_X = 1,    // layer 0: the residual stream before the O-projection is the embedding row
    F_LAST_LM = 2,    // last LM-head instruction of this CTA: publish the CTA's best
    F_DROP_SIGNAL = 8 // test hook: publish nothing (no counter signal, outputs keep a stale tag)
};

#ifdef __CUDACC__
#define MK_HD __host__ __device__
#else
#define MK_HD
#endif
// Tag of every activation a layer writes in a step (never 0, so zeroed
// buffers hold no valid word).
MK_HD inline uint32_t act_tag(uint32_t gen, int n_layers, int layer) {
    return gen * (uint32_t)n_layers + (uint32_t)layer + 1u;
}

// One instruction: 32 bytes, read by both the producer and the consumer warps.
struct Instr {
    uint8_t op;
    uint8_t flags;
    uint16_t layer;
    uint32_t tile;        // GEMV: first row tile of the run; ATTN: (b * nkv + g) * chunks + c
    uint16_t kb0, kb1;    // K block range [kb0, kb1)
    uint16_t b0, nb;      // batch rows [b0, b0 + nb)
    uint16_t wait_ctr;    // counter to wait on (kNoCounter: none)
    uint16_t signal_ctr;  // counter to increment when done
    uint32_t wait_count;  // increments the waited counter receives per step
    uint16_t signal2_ctr; // ATTN: split-KV arrival counter of its (sequence, KV head)
    uint16_t ntiles;      // GEMV: consecutive row tiles in this run (>= 1)
    uint32_t arrive_count;// LM: arrivals per step on signal_ctr; ATTN: chunks per (sequence, KV head)
};
static_assert(sizeof(Instr) == 32, "Instr must be 32 bytes");

// A weight matrix repacked into tiles of `rows` rows x kc columns; the
// (tile, kblock) blocks are contiguous, kblock fastest, each block row-major.
// rows * kc * 2 <= 32 KB: one block fills at most one ring slot.
struct PackedMat {
    uint64_t offset;   // byte offset in the workspace
    int32_t n_rows;    // logical rows (N)
    int32_t k;         // logical columns (K)
    int32_t kc;        // block width (columns, a multiple of 256)
    int32_t nkb;       // blocks along K
    int32_t tiles;     // row tiles
    int32_t rows;      // rows per tile (1, 2, 4 or 8)
};

// Per-layer device pointers (in the workspace; filled by the host after packing).
struct LayerW {
    const void *qkv;       // packed [(nq+2nkv)d, H]
    const void *o;         // packed [H, nq d]
    const void *gu;        // packed, tile t = gate rows 4t..4t+3 then up rows 4t..4t+3
    const void *down;      // packed [H, I]
    const void *attn_norm; // bf16 [H]
    const void *mlp_norm;  // bf16 [H]
    const void *q_norm;    // bf16 [d] or null
    const void *k_norm;    // bf16 [d] or null
};

// Device-resident step state.
struct State {
    uint32_t gen;      // steps completed since the last reset
    int32_t pos;       // position of the token decoded by the next step
    uint32_t err;      // 0 or an error code (1 = wait timeout)
    uint32_t err_cta;
    uint32_t err_instr;
    uint32_t err_ctr;
    uint32_t tok_err;  // 0, or 1 + the first sequence whose token was outside [0, vocab)
    int32_t tok_bad;   // that token
};

struct LmBest {
    float value;
    int32_t index;
    uint32_t gen;
    uint32_t pad;
};

// Kernel parameters (passed by value).
struct KParams {
    const Instr *instrs;
    const int32_t *cta_begin;   // [n_ctas] first instruction of each CTA in this launch
    const int32_t *cta_end;     // [n_ctas] one past the last
    const LayerW *layers;
    const void *lm_w;           // packed LM head
    const void *final_norm;     // bf16 [H]
    const void *embed;          // bf16 [V, H] (caller's)
    // tagged activations (see act_tag)
    uint64_t *xm;               // [B, H] residual stream after the layer's O-projection
    uint64_t *xe;               // [B, H] x_mid + the down projection's first K range
    uint64_t *dpart;            // [down K ranges - 1, B, H] outputs of the further K ranges
    uint64_t *qkv;              // [B, qkv_rows]
    uint64_t *attn;             // [B, nq * d] attention output (combined split-KV partials)
    uint64_t *act_a;            // [B, I] SwiGLU product
    uint64_t *partials;         // [B, nq, chunks, d + 2]: o[d], m, l
    uint16_t *kcache;           // bf16 [L, B, nkv, max_seq, d]
    uint16_t *vcache;
    uint32_t *counters;
    State *state;
    LmBest *lm_best;            // [B, n_ctas]
    const int32_t *tokens;      // token of sequence b at tokens[b * tok_stride]
    int32_t *next;              // [B] or null
    float *logits;              // [B, V] or null
    int64_t tok_stride;
    unsigned long long timeout_ns;
    // shapes
    int32_t n_layers, hidden, n_heads, n_kv_heads, head_dim, intermediate, vocab, batch, max_seq;
    int32_t qkv_rows, i_pad, chunks, n_ctas, stages, act_bytes, qk_norm, bs, down_ranges, down_per;
    float rms_eps;
    int32_t qkv_kc, qkv_nkb, o_kc, o_nkb, gu_kc, gu_nkb, down_kc, down_nkb, lm_kc, lm_nkb;
    int32_t qkv_rt, o_rt, gu_rt, down_rt, lm_rt;  // rows per tile
    int32_t use_waits;          // 1: acquire-spin on the tile-ready counters before each instruction
    int32_t use_signals;        // 1: release-increment the counters after each instruction
    int32_t pdl;                // 1: trigger dependents, wait on the previous grid; 2: trigger only
    unsigned long long *trace;  // [n_instr][8] globaltimer stamps and waits, or null
    int32_t prefetch;           // ring blocks the L2 prefetch cursor runs ahead of the TMA loads
    double rope_inv_freq[64];   // theta^(-2i/d), i < d/2
};

}  // namespace mk

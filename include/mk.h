/*
 * mk.h -- C ABI of the B200 decode megakernel library (libmk.so).
 *
 * One call of mk_decode_step computes the next token of every sequence in a
 * small batch from the previous token, the weights and the KV cache -- the
 * workload of "Look Ma, No Bubbles! Designing a Low-Latency Megakernel for
 * Llama-1B" (Hazy Research), introduction: a single sequence generated with
 * Llama-3.2-1B, bound by how fast the weights stream from HBM.  It runs as one
 * persistent kernel whose dependent operations start as soon as the tiles
 * they read are ready ("MegaOps: A Kernel Overlapping Framework ...",
 * "In plain words" and "Keep kernels separate": a consumer starts once the
 * particular input tiles it needs are ready), or, for comparison, as the same
 * operations launched as separate kernels inside one CUDA graph (the
 * megakernel-versus-graph argument of "Megakernel Debate Sparks CUDA
 * Infrastructure Community Feud", "Confirmed").
 *
 * Conventions
 *  - Every call returns an mk_status.  MK_OK is 0; errors are negative.
 *    mk_last_error() gives a one-line reason for the last failure on a ctx;
 *    mk_last_error(NULL) gives the calling thread's last failure of a
 *    context-free call (mk_attention_decode and the like).
 *  - All device memory is owned by the caller (for example allocated through
 *    PyTorch) and passed as raw device pointers; the library allocates host
 *    memory only and never frees caller memory.  mk_swiglu_stage1 is
 *    stateless and allocates nothing.
 *  - `stream` arguments are cudaStream_t values passed as void* (NULL = the
 *    legacy default stream).  Calls are asynchronous on that stream unless
 *    stated otherwise.
 *  - All sequences of a context sit at the same position; mk_prefill_kv sets
 *    it to T and every decode step advances it by one.
 *  - Not thread-safe per context.  Different contexts are independent.
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MK_OK = 0,
    MK_ERR_INVALID = -1,     /* bad argument: null pointer, size or position out of range */
    MK_ERR_CUDA = -2,        /* a CUDA runtime call failed (message in mk_last_error) */
    MK_ERR_TIMEOUT = -3,     /* a device-side dependency wait ran past its time limit */
    MK_ERR_UNSUPPORTED = -4, /* a shape the kernels do not handle (see mk_create) */
    MK_ERR_STATE = -5        /* call out of order (e.g. decode before load), or the
                                context is poisoned by an earlier device error */
} mk_status;

enum { MK_BF16 = 0 };
/* Execution variants of one decode step. */
enum {
    MK_MEGAKERNEL = 0, /* one persistent launch, tile-ready counters between ops */
    MK_GRAPH = 1,      /* the same ops as one launch per op, replayed from a CUDA graph */
    MK_GRAPH_PDL = 2,  /* as MK_GRAPH, launches chained by programmatic dependent launch so
                          each op streams its weights while the previous op finishes */
    MK_GRAPH_TILESYNC = 3, /* the ops as separate kernels in the same CUDA graph, each
                          launched early by programmatic dependent launch and started
                          on the tiles it reads instead of on the previous kernel's
                          end ("MegaOps: A Kernel Overlapping Framework ...", "In plain
                          words" and "Keep kernels separate"): a kernel's CTAs occupy
                          SMs as the previous kernel's CTAs leave them, stream their
                          weights at once and wait on the tagged words (or, with
                          MK_SYNC_COUNTERS, the tile-ready counters) of the data they
                          read.  A kernel launches only after every CTA of the one
                          before it has started, so what it waits for is always
                          running; every wait is bounded. */
    MK_TENSOR_CORES = 4   /* the same step with every projection a tcgen05 GEMM over the
                          packed weights (up to 32 sequences a pass, each activation row
                          a hi/lo pair of bf16 rows), attention per sequence, the LM
                          head and the argmax; replayed from a CUDA graph.  The batched
                          counterpart of the megakernel, whose CUDA-core GEMVs turn
                          arithmetic-bound as the batch grows. */
};
/* How the megakernel's dependent instructions learn that their inputs are
 * ready ("MegaOps: A Kernel Overlapping Framework ...", "In plain words": a
 * consumer starts once the particular input tiles it needs are ready).  Every
 * activation word carries the tag of the (step, layer) that wrote it in the
 * same 64-bit store in both modes. */
enum {
    MK_SYNC_TAGS = 0,    /* readers spin on the tagged words they read (no fence,
                            no separate flag; the default) */
    MK_SYNC_COUNTERS = 1 /* tile-ready counters: each instruction release-increments
                            its phase counter, consumers acquire-spin on it before
                            reading (tags are then only verified) */
};
/* Tilings of the fused SwiGLU first stage ("Deep Kernel Fusion for
 * Transformers", Key points, "Fusion scope": row-major tiling reuses the
 * activations, column-major tiling reuses the weights).  MK_SWIGLU_TC runs
 * both projections as tcgen05 MMAs with tensor-memory accumulators (the
 * batch is the MMA's N, rounded up to 16 with zero rows in shared memory). */
enum { MK_SWIGLU_AUTO = 0, MK_SWIGLU_ROW = 1, MK_SWIGLU_COL = 2, MK_SWIGLU_TC = 3 };

/* Architecture and limits of one context. */
typedef struct {
    int n_layers, hidden, n_heads, n_kv_heads, head_dim, intermediate, vocab;
    float rms_eps, rope_theta;
    int tied_embeddings; /* 1: the LM head is the embedding table */
    int qk_norm;         /* 1: per-head RMSNorm of q and k before RoPE (Qwen3) */
    int batch;           /* sequences decoded together, 1..64 */
    int max_seq;         /* KV cache positions per sequence */
    int dtype;           /* MK_BF16 (the only one) */
    int variant;         /* MK_MEGAKERNEL | MK_GRAPH | MK_GRAPH_PDL | MK_GRAPH_TILESYNC | MK_TENSOR_CORES */
    int num_sms;         /* CTAs of the persistent kernel; 0 = the device's SM count */
} mk_config;

/* Device pointers to the caller's bf16 weights in nn.Linear layout
 * [out_features, in_features], row-major.  The per-layer members are HOST
 * arrays of n_layers DEVICE pointers.  q_norm/k_norm are read only when
 * qk_norm is set; lm_head is ignored when tied_embeddings is set. */
typedef struct {
    const void *embed;      /* [vocab, hidden]; must stay alive while the ctx decodes */
    const void *final_norm; /* [hidden] */
    const void *lm_head;    /* [vocab, hidden] */
    const void *const *attn_norm; /* [hidden] */
    const void *const *wq;  /* [n_heads*head_dim, hidden] */
    const void *const *wk;  /* [n_kv_heads*head_dim, hidden] */
    const void *const *wv;  /* [n_kv_heads*head_dim, hidden] */
    const void *const *wo;  /* [hidden, n_heads*head_dim] */
    const void *const *q_norm; /* [head_dim] */
    const void *const *k_norm; /* [head_dim] */
    const void *const *mlp_norm; /* [hidden] */
    const void *const *wg;  /* [intermediate, hidden] (gate) */
    const void *const *wu;  /* [intermediate, hidden] (up) */
    const void *const *wd;  /* [hidden, intermediate] (down) */
} mk_weights;

typedef struct mk_ctx mk_ctx;

/* Validate `cfg`, build the per-SM instruction lists and counter targets on
 * the host, and check that schedule for deadlock and producer/consumer count
 * mismatches.  `device` is the CUDA device ordinal, or -1 to plan without a
 * device (then cfg->num_sms must be > 0; only the planning calls below work).
 * Shapes handled: head_dim 64 or 128, n_heads a multiple of n_kv_heads with at
 * most 8 query heads per KV head, hidden/intermediate multiples of 8,
 * hidden <= 8192.  Errors: MK_ERR_INVALID (null/negative), MK_ERR_UNSUPPORTED. */
mk_status mk_create(const mk_config *cfg, int device, mk_ctx **out);
mk_status mk_destroy(mk_ctx *ctx);
const char *mk_last_error(const mk_ctx *ctx);

/* Bytes of the caller-allocated device workspace (256-byte aligned base):
 * repacked weights, activations, partial sums, counters, instruction lists. */
mk_status mk_workspace_bytes(const mk_ctx *ctx, size_t *bytes);
/* Bytes of the caller-allocated KV cache: bf16 K then V, each
 * [n_layers][batch][n_kv_heads][max_seq][head_dim]. */
mk_status mk_kv_cache_bytes(const mk_ctx *ctx, size_t *bytes);

/* Repack the weights into the workspace in the tile order the kernels stream
 * (one pass, synchronous on `stream`), upload the instruction lists, zero the
 * counters and the KV cache, and set the position to 0.  The caller's weight
 * buffers other than `embed` may be freed afterwards. */
mk_status mk_load_weights(mk_ctx *ctx, const mk_weights *w, void *workspace, void *kv_cache, void *stream);

/* Fill the KV cache from a prompt: `d_tokens` is a device int32 [batch, T]
 * row-major array; positions restart at 0 and end at T.  With the tensor-core
 * prefill (the default, see mk_set_prefill) the prompt goes through the
 * decoder 128 positions of one sequence at a time: every projection is one
 * tcgen05 GEMM reading the packed weight tiles of mk_load_weights in place,
 * with each activation row entering as a hi/lo pair of bf16 rows, and
 * position t attends causally to positions 0 .. t; only the KV cache is kept
 * (the last layer stops after its K/V rows).  Otherwise it runs T decode
 * steps whose outputs are discarded.  A token outside [0, vocab) is reported by
 * mk_get_status as for mk_decode_step.  MK_ERR_INVALID if T < 1 or
 * T > max_seq. */
mk_status mk_prefill_kv(mk_ctx *ctx, const int32_t *d_tokens, int batch, int T, void *stream);
/* How mk_prefill_kv runs: MK_PREFILL_AUTO (default) and MK_PREFILL_TC, the
 * tensor cores; MK_PREFILL_STEPS, one decode step per position.  Host only. */
enum { MK_PREFILL_AUTO = 0, MK_PREFILL_STEPS = 1, MK_PREFILL_TC = 2 };
mk_status mk_set_prefill(mk_ctx *ctx, int mode);

/* One decode step at the current position p: `d_tokens` is a device int32
 * [batch]; the K/V rows of those tokens are written at position p, every
 * sequence attends to positions 0..p, and the argmax over the vocabulary
 * (lowest index on ties) goes to `d_next` (device int32 [batch], may be NULL).
 * If `d_logits` is not NULL it receives the fp32 logits [batch, vocab] the
 * argmax was taken over.  Advances the position.  MK_ERR_INVALID if p ==
 * max_seq.  The tokens live in device memory, so their range is checked on the
 * device: a token outside [0, vocab) is recorded (the step decodes token 0 in
 * its place so that no read leaves the embedding table) and the next
 * mk_get_status returns MK_ERR_INVALID naming the sequence and the token; a
 * device wait timeout is reported by mk_get_status too. */
mk_status mk_decode_step(mk_ctx *ctx, const int32_t *d_tokens, int32_t *d_next, float *d_logits, void *stream);

/* Synchronize `stream` and return MK_ERR_TIMEOUT if a device wait gave up
 * during any earlier step, MK_ERR_INVALID if an earlier step (or prefill) was
 * given a token outside [0, vocab) -- in both cases the context is poisoned
 * until mk_reset, and the KV rows written at the positions of those steps hold
 * no valid result -- MK_ERR_CUDA on a CUDA error, else MK_OK. */
mk_status mk_get_status(mk_ctx *ctx, void *stream);
/* Clear counters, error word and position (KV cache contents are kept). */
mk_status mk_reset(mk_ctx *ctx, void *stream);
mk_status mk_get_position(const mk_ctx *ctx, int *pos);
/* Rewind (or advance) the position to `pos` (0 <= pos <= max_seq), for
 * example to decode another continuation of a shared prompt.  KV slots at
 * and after `pos` are treated as free and are overwritten by later steps;
 * slots before it must have been written.  One tiny kernel on `stream`. */
mk_status mk_set_position(mk_ctx *ctx, int pos, void *stream);

/* Select the execution variant for later decode steps (MK_MEGAKERNEL,
 * MK_GRAPH, MK_GRAPH_PDL, MK_GRAPH_TILESYNC or MK_TENSOR_CORES). */
mk_status mk_set_variant(mk_ctx *ctx, int variant);

/* One-time profiling pass ("Deep Kernel Fusion for Transformers", Summary and
 * Key points: a profiler-based scheduler benchmarks the tiling variants on
 * the target GPU before inference and keeps the fastest, with no dispatch
 * cost at run time).  Times the row-tiled and column-tiled forms of the fused
 * gate/up stage inside the step and keeps the faster; the KV cache and the
 * position are restored afterwards.  Synchronous.  *chosen (may be NULL)
 * receives MK_SWIGLU_ROW or MK_SWIGLU_COL. */
mk_status mk_tune(mk_ctx *ctx, void *stream, int *chosen);

/* Select the gate/up tiling of later steps without timing it (what mk_tune
 * would otherwise pick): MK_SWIGLU_COL, every gate/up instruction carries all
 * of its batch rows and streams its weight tiles once; MK_SWIGLU_ROW, an
 * instruction carries at most half of them (rounded up), so each weight tile
 * streams once per row group.  Both give bit-identical results.  Synchronous
 * on `stream`; the KV cache and the position are kept.  MK_ERR_INVALID for
 * another value, MK_ERR_STATE before mk_load_weights or on a poisoned
 * context.  mk_get_swiglu_tiling reports the active one. */
mk_status mk_set_swiglu_tiling(mk_ctx *ctx, int variant, void *stream);
mk_status mk_get_swiglu_tiling(const mk_ctx *ctx, int *variant);

/* How far, in 32 KB ring blocks, the producer's L2 prefetches may run ahead of
 * its shared-memory loads.  It keeps min(4, blocks) ahead at all times and
 * runs on up to `blocks` while the ring is full (the consumers are waiting on
 * an input).  Default 10; 0 disables prefetching.  0..64. */
mk_status mk_set_prefetch(mk_ctx *ctx, int blocks);

/* Shared-memory ring slots (32 KB each) the producer may fill: 0 (default)
 * uses as many as the plan's shared memory allows, otherwise the smaller of
 * `stages` and that.  Fewer slots keep fewer weight loads in flight per SM
 * ahead of the consumers' activation reads.  0 or 2..8; MK_ERR_INVALID
 * otherwise. */
mk_status mk_set_ring_stages(mk_ctx *ctx, int stages);

/* Device wait limit in nanoseconds (default 1e9).  A wait that runs out sets
 * the context's error word and makes every CTA return early. */
mk_status mk_set_timeout_ns(mk_ctx *ctx, unsigned long long ns);
/* Synchronisation of the megakernel variant: MK_SYNC_TAGS (default) or
 * MK_SYNC_COUNTERS.  Results are bit-identical; only the waiting differs.
 * Host-only, takes effect at the next launch.  MK_ERR_INVALID otherwise. */
mk_status mk_set_sync(mk_ctx *ctx, int mode);

/* Test hook: when set, the instruction at index `instr` of the flattened
 * schedule does its work but publishes nothing (no counter signal, and its
 * outputs keep a stale tag), so its consumers' waits run out in either sync
 * mode; -1 clears it.  Used to test timeout reporting. */
mk_status mk_debug_drop_signal(mk_ctx *ctx, int instr);

/* Test hook: fill every buffer the step's instructions hand to each other
 * (the tagged activation words: residual stream, q/k/v, split-KV partials,
 * attention output, SwiGLU product, down-projection partial outputs, and the
 * per-CTA argmax records) with 0xFF bytes -- NaN values under a tag no step
 * writes -- so that a read of a word its producer has not written this step
 * cannot pass for data.  Synchronous on `stream`.  MK_ERR_STATE before
 * mk_load_weights. */
mk_status mk_debug_poison_activations(mk_ctx *ctx, void *stream);

/* Test hook: reorder the active schedule with the seeded permutation that
 * keeps every dependency (for each phase, the CTAs' groups of instructions
 * are dealt to the CTAs in a random order and each group is shuffled; every
 * CTA's list stays in phase order), re-check it as mk_validate_schedule does
 * and, when weights are loaded, upload it (synchronous).  Each instruction
 * computes the same values wherever it runs, so results must be
 * bit-identical to the unshuffled schedule's; a dependency the planner failed
 * to express would show up as a difference or a timeout.  It stays in effect
 * until the gate/up tiling is switched (mk_set_swiglu_tiling, mk_tune), which
 * installs that tiling's unshuffled plan.  MK_ERR_STATE if the check fails. */
mk_status mk_debug_shuffle_schedule(mk_ctx *ctx, unsigned long long seed);

/* Per-instruction timing trace for the following steps: `d_trace` is a
 * device buffer of at least 8 * n_instructions uint64 (64 bytes per
 * instruction; see mk_schedule_info).  For instruction i of the flattened
 * schedule, entries [8i..8i+7] receive, in %globaltimer nanoseconds: when its
 * CTA starts it, when its dependency wait is satisfied, when it is done, when
 * the producer issued its first copy (0 if it streams nothing), the SM clock
 * cycles the consumer spent waiting for ring data, the time the producer spent waiting
 * for a free ring slot, when the producer issued its last copy, and when the
 * instruction's inputs were in shared memory (activations staged, or
 * attention heads rotated).  "Done" is taken after every consumer warp has
 * finished, so tracing adds one CTA barrier per instruction.  Each step
 * overwrites the buffer.  NULL turns tracing off.  MK_ERR_INVALID if the
 * buffer is too small. */
mk_status mk_set_trace(mk_ctx *ctx, void *d_trace, size_t bytes);
/* Copy the flattened schedule to host memory: 32 bytes per instruction
 * (uint8 op, uint8 flags, uint16 layer, uint32 tile, uint16 kb0, kb1, b0, nb,
 * then counter fields), CTA-major; `cta_base` (may be NULL) receives
 * n_ctas + 1 int32 offsets of each CTA's first instruction. */
mk_status mk_get_schedule(const mk_ctx *ctx, void *host_instrs, size_t bytes, int32_t *cta_base);

/* Introspection of the host-built schedule (CPU-testable with device -1).
 * info[] receives, in order: n_instructions, n_ctas, n_counters, n_phases,
 * batch_rows_per_instruction, attention_chunks, ring_stages,
 * act_bytes, swiglu_variant, down_k_splits.  `n` is the capacity of info[]. */
mk_status mk_schedule_info(const mk_ctx *ctx, long long *info, int n);
/* Re-run the host-side schedule check: simulates every CTA executing its list
 * in order against the counters and fails (MK_ERR_STATE, reason in
 * mk_last_error) on a deadlock, a counter whose producers do not match its
 * consumers' expected count, or an index outside its buffer. */
mk_status mk_validate_schedule(const mk_ctx *ctx);

/* Fused SwiGLU first stage on its own ("Deep Kernel Fusion for
 * Transformers", Summary and Key points, "Fusion scope"):
 *   out[b][n] = SiLU(sum_k x[b][k] w_gate[k][n]) * sum_k x[b][k] w_up[k][n]
 * x: device fp16 [B, K] row-major; w_gate, w_up: device fp16 [K, N] row-major
 * (N contiguous); out: device fp16 [B, N].  fp32 accumulation, SiLU in fp32,
 * one rounding to fp16 at the end.  variant: MK_SWIGLU_ROW, MK_SWIGLU_COL,
 * MK_SWIGLU_TC or MK_SWIGLU_AUTO (the variant mk_swiglu_tune picked for this
 * (B, K, N), else MK_SWIGLU_TC where it applies, COL for B <= 8 and ROW
 * above).  Needs K % 64 == 0, N % 64 == 0, 1 <= B <= 64, all pointers 16-byte
 * aligned; MK_SWIGLU_TC also needs K % 128 == 0 and N % 128 == 0
 * (MK_ERR_UNSUPPORTED otherwise).  MK_ERR_INVALID on bad arguments.
 * Allocates nothing. */
mk_status mk_swiglu_stage1(const void *x, const void *w_gate, const void *w_up, void *out, int B, int K, int N,
                           int variant, void *stream);
/* Time every applicable variant on the given buffers (synchronous; `out` is
 * overwritten), remember the fastest for (B, K, N) in a process-wide table
 * and return it in *chosen.  Mean microseconds go to us_row, us_col and
 * us_tc (each may be NULL; us_tc gets 0 when the tensor-core variant does not
 * apply). */
mk_status mk_swiglu_tune(const void *x, const void *w_gate, const void *w_up, void *out, int B, int K, int N,
                         void *stream, int *chosen, float *us_row, float *us_col, float *us_tc);

/* One projection of a batched decode step on the tcgen05 tensor cores (the
 * matrix-vector products of "Look Ma, No Bubbles! Designing a Low-Latency
 * Megakernel for Llama-1B", where a batch of B sequences makes each one a GEMM
 * with the batch as its narrow side):
 *   y[b][m] = sum_k w[m][k] x[b][k]
 * w: device bf16 [M, K] row-major (the [out, in] layout of every decoder
 * projection, as given); x: device bf16 [B, K] row-major; y: device fp32
 * [B, M].  Swap-AB: 128 rows of w per CTA are the MMA's M, the batch
 * (rounded up to 16 with zero rows) its N, fp32 accumulators in tensor
 * memory (up to 256 columns); every weight byte is read once for the whole
 * batch.  With few row tiles a cluster of 2 or 4 CTAs splits K
 * (mk_linear_tc_split) and sums in a
 * fixed order, so results are deterministic.  Needs 1 <= B <= 256,
 * K % 64 == 0 (MK_ERR_UNSUPPORTED otherwise), M >= 1, all pointers 16-byte
 * aligned (MK_ERR_INVALID).  Asynchronous on `stream`; a device-side wait
 * that runs out (2 s) writes NaN outputs rather than hanging.  Allocates
 * nothing. */
mk_status mk_linear_tc(const void *x, const void *w, float *y, int B, int K, int M, void *stream);
/* The K split (1, 2 or 4 CTAs per row tile) mk_linear_tc uses for this shape;
 * host only.  MK_ERR_UNSUPPORTED for shapes mk_linear_tc refuses. */
mk_status mk_linear_tc_split(int B, int K, int M, int *split);
/* The same product as stream-K work sharing, for projections whose row tiles
 * do not fill the SMs evenly (a 4096-row projection has 32 tiles of 128
 * rows, a 28672-row one 224, one and a half waves): the tiles x K/64 units
 * are cut into one contiguous range per CTA, at most one CTA per SM, so
 * every SM streams the same number of weight bytes.  A tile split between
 * CTAs is finished by the CTA holding its first K block, which adds the
 * other CTAs' partial sums in CTA order after they raise a flag (the sum is
 * deterministic).  `workspace` is device memory of
 * mk_linear_tc_streamk_workspace_bytes() bytes, 16-byte aligned, zero-filled
 * before its first use; every call that completes leaves it as it found it
 * (zero flags); after a call whose device-side wait ran out (NaN outputs)
 * zero it again.  Calls sharing a workspace must not run concurrently.  Falls
 * back to mk_linear_tc's launch where one tile per CTA already fills the
 * SMs (mk_linear_tc_streamk_grid returns 0 then).  Arguments and errors as
 * mk_linear_tc; NULL or short workspace: MK_ERR_INVALID. */
size_t mk_linear_tc_streamk_workspace_bytes(void);
mk_status mk_linear_tc_streamk(const void *x, const void *w, float *y, int B, int K, int M, void *workspace,
                               size_t workspace_bytes, void *stream);
/* CTAs the stream-K launch of (B, K, M) uses on the current device, 0 when
 * mk_linear_tc_streamk runs the one-tile-per-CTA kernel instead. */
int mk_linear_tc_streamk_grid(int B, int K, int M);

/* A batched decode step whose projections all run on the tensor cores
 * (mk_linear_tc) and whose attention is the split-KV pair of kernels above
 * (mk_attention_decode), for the batches where the megakernel's CUDA-core
 * GEMV becomes arithmetic-bound ("Look Ma, No Bubbles! Designing a
 * Low-Latency Megakernel for Llama-1B" for the step; the same plain decoder
 * math as mk_decode_step).  Every activation row enters each projection as
 * two bf16 rows (hi = bf16(x), lo = bf16(x - hi)), so the MMA's bf16 inputs
 * keep about 16 significant bits.
 * mk_tcdec_create checks `cfg` (batch <= 32; hidden, intermediate and
 * n_heads*head_dim multiples of 64; head_dim 64 or 128; at most 8 query heads
 * per KV head) and records the weight pointers of `w`, which are READ AT EVERY
 * STEP: they must stay alive (unlike mk_load_weights, nothing is repacked).
 * mk_tcdec_bind gives it the caller's workspace (mk_tcdec_workspace_bytes,
 * 256-byte aligned) and KV cache (the layout of mk_kv_cache_bytes, so a
 * context's prefilled cache can be shared).  mk_tcdec_step decodes one token
 * per sequence at position `pos` (all sequences share it): it writes K/V at
 * `pos`, attends to 0 .. pos, writes d_next (device int32 [batch]) and, if
 * d_logits is set, the fp32 logits [batch, vocab].  Asynchronous on `stream`.
 * Device-side failures are ORed into a status word that mk_tcdec_status reads
 * (synchronous; 0 = none): bit 0, a token outside [0, vocab) (its row decodes
 * from zeros); bit 1, a sequence with no finite logit, which happens when a
 * projection's bounded wait ran out and wrote NaN (d_next then holds 0 for
 * it).  The word is cleared by mk_tcdec_bind only.
 * Errors: MK_ERR_INVALID, MK_ERR_UNSUPPORTED, MK_ERR_STATE (step before
 * bind), MK_ERR_CUDA; the reason is in mk_tcdec_last_error.  A step that
 * returns an error may have queued part of its work: the K/V rows at `pos`
 * of some layers can already be written, so the cache at `pos` is undefined
 * until a step at the same `pos` succeeds. */
typedef struct mk_tcdec mk_tcdec;
mk_status mk_tcdec_create(const mk_config *cfg, const mk_weights *w, mk_tcdec **out);
mk_status mk_tcdec_workspace_bytes(const mk_tcdec *dec, size_t *bytes);
mk_status mk_tcdec_bind(mk_tcdec *dec, void *workspace, void *kv_cache);
mk_status mk_tcdec_step(mk_tcdec *dec, const int32_t *d_tokens, int pos, int32_t *d_next, float *d_logits,
                        void *stream);
mk_status mk_tcdec_status(mk_tcdec *dec, int *status, void *stream);
const char *mk_tcdec_last_error(const mk_tcdec *dec);
mk_status mk_tcdec_destroy(mk_tcdec *dec);
/* Replay the step from a CUDA graph (on = 1, the default) or launch its
 * ~16-per-layer kernels one by one (on = 0).  Every kernel of the step reads
 * the position and the tokens from the workspace, so the first step runs
 * eagerly and the next one captures the whole step once (once more the first
 * time logits are asked for, or not) into a graph that every later step
 * replays: mk_tcdec_step then queues a 4-byte-per-sequence token copy, a
 * one-thread position write, the graph launch and the output copies.  The
 * results are bit-identical either way (the split-KV chunk count is fixed by
 * max_seq in both).  Rebinding drops the captured graphs.  Host only. */
mk_status mk_tcdec_set_graph(mk_tcdec *dec, int on);

/* Split-KV decode attention with a log-sum-exp combine, on its own: the
 * attention of one layer of one decode step ("Look Ma, No Bubbles! Designing
 * a Low-Latency Megakernel for Llama-1B", introduction: generating one
 * sequence with Llama-3.2-1B; the megakernel runs the same split inside its
 * interpreter).  For every sequence b and query head h (KV head
 * g = h / (n_heads / n_kv_heads)):
 *   out[b][h] = sum_j softmax_j(q[b][h] . K[b][g][j] / sqrt(d)) V[b][g][j],
 *   j = 0 .. n_pos - 1.
 * q: device fp32 [batch][n_heads][head_dim] (already rotated);
 * k_cache, v_cache: device bf16 [batch][n_kv_heads][max_seq][head_dim], the
 * layout of one layer of the decode cache; out: device fp32
 * [batch][n_heads][head_dim].  The positions are cut into `chunks` equal
 * ranges (0 = pick from the SM count, see mk_attention_chunks; at most n_pos);
 * one CTA per (chunk, KV head, sequence) writes an unnormalised partial
 * (o, max, sum) to `scratch`, and a second kernel combines them.  scratch is
 * caller-owned device memory of at least mk_attention_scratch_bytes(batch,
 * n_heads, head_dim, chunks) bytes; it needs no initialisation and is fully
 * rewritten by every call, so calls that share a scratch buffer must not
 * overlap.  head_dim in {64, 128, 256}; n_heads a multiple of n_kv_heads with at
 * most 8 query heads per KV head; 1 <= n_pos <= max_seq; all pointers 16-byte
 * aligned.  MK_ERR_INVALID / MK_ERR_UNSUPPORTED otherwise (reason in
 * mk_last_error(NULL)).  fp32 accumulation, softmax in base 2.  Allocates
 * nothing; asynchronous on `stream`. */
mk_status mk_attention_decode(const float *q, const void *k_cache, const void *v_cache, int batch, int n_heads,
                              int n_kv_heads, int head_dim, int max_seq, int n_pos, int chunks, float *out,
                              void *scratch, size_t scratch_bytes, void *stream);
/* Bytes of scratch mk_attention_decode needs (0 for non-positive arguments). */
size_t mk_attention_scratch_bytes(int batch, int n_heads, int head_dim, int chunks);
/* The chunk count mk_attention_decode picks for chunks = 0 on the current
 * device: about one CTA per SM over (sequence, KV head) pairs, at most 64, and
 * at least 16 positions per chunk; for caches of 1024 positions and more, as
 * many chunks of at least 512 positions as fill two CTAs per SM in whole
 * waves (the first count whose last wave is 90 % full), when that is more. */
int mk_attention_chunks(int batch, int n_kv_heads, int n_pos);

/* mk_attention_decode without a scratch argument: the partial records live in
 * a fixed 4 MiB array of device memory inside libmk.so (one per device), so
 * the call allocates nothing and needs no buffer from the caller.  It serves
 * callers that cannot allocate or be handed scratch: code running after the
 * allocator that owns the device's memory has reported it full, callbacks of
 * that allocator (which may not re-enter it), and C callers without a device
 * allocator.  The pages have no counterpart of this entry point.
 *   Limit: batch * n_heads * chunks * (head_dim + 2) * 4 bytes must fit in
 * mk_attention_noalloc_limit_bytes() (4 MiB).  With chunks = 0 the automatic
 * count is lowered until it fits; an explicit `chunks`, or a shape where not
 * even one chunk fits, is refused with MK_ERR_INVALID and the needed size in
 * mk_last_error(NULL).  Other arguments as mk_attention_decode.
 *   Set-up: the first call on a device looks up that device's copy of the
 * array (cudaGetSymbolAddress, with the device current) and keeps it; make that
 * first call before any stream capture on the device.
 *   Nothing has to start at zero: every partial record is written by the
 * first kernel of a call before the second kernel reads it.
 *   Calls that overlap on the device (other streams or threads with work in
 * flight at the same time) race on the one array and corrupt each other's
 * results; calls issued in order on one stream are safe. */
mk_status mk_attention_decode_noalloc(const float *q, const void *k_cache, const void *v_cache, int batch,
                                      int n_heads, int n_kv_heads, int head_dim, int max_seq, int n_pos, int chunks,
                                      float *out, void *stream);
/* Bytes of the fixed scratch behind mk_attention_decode_noalloc (4 MiB). */
size_t mk_attention_noalloc_limit_bytes(void);

#ifdef __cplusplus
}
#endif
#endif /* MK_H */

// mk_api.cu -- the C ABI of libmk.so (see include/mk.h for the contract).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_kernel.h"
#include "mk_sched.h"

using namespace mk;

struct mk_ctx {
    Plan plan;            // active plan
    Plan plan_alt;        // the other gate/up tiling (same workspace layout)
    int device = -1;
    std::string err;
    uint8_t *ws = nullptr;
    uint8_t *kv = nullptr;
    bool loaded = false;
    bool poisoned = false;
    int pos = 0;
    int variant = MK_MEGAKERNEL;
    unsigned long long timeout_ns = 1000000000ull;
    int drop_instr = -1;
    unsigned long long *trace = nullptr;
    int prefetch = 10;  // furthest L2 prefetch distance in ring blocks
    int sync = MK_SYNC_TAGS;
    int stages = 0;  // ring slots in use (0: all the plan's shared memory allows)
    const void *embed = nullptr;
    std::vector<LayerW> lw;  // host copy of the per-layer device pointers (packed weights, norms)
    int prefill = MK_PREFILL_AUTO;
    // captured graph of the separate-kernels variant
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t gexec = nullptr;
    std::vector<cudaGraphNode_t> gnodes;  // kernel node of each phase
    const void *g_tok = nullptr, *g_next = nullptr, *g_logits = nullptr;
    int g_variant = -1;
    // captured decode step on the tensor cores (MK_TENSOR_CORES)
    cudaGraphExec_t tc_exec = nullptr;
    const float *tc_logits = nullptr;
    bool tc_warmed = false;
};

static mk_status fail(mk_ctx *c, mk_status s, const std::string &msg) {
    if (c) c->err = msg;
    return s;
}
static mk_status cuda_fail(mk_ctx *c, cudaError_t e, const char *where) {
    return fail(c, MK_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}
#define CK(call)                                             \
    do {                                                     \
        cudaError_t e_ = (call);                             \
        if (e_ != cudaSuccess) return cuda_fail(c, e_, #call); \
    } while (0)

static void drop_graph(mk_ctx *c) {
    if (c->tc_exec) cudaGraphExecDestroy(c->tc_exec);
    c->tc_exec = nullptr;
    if (c->gexec) cudaGraphExecDestroy(c->gexec);
    if (c->graph) cudaGraphDestroy(c->graph);
    c->gexec = nullptr;
    c->graph = nullptr;
    c->gnodes.clear();
    c->g_variant = -1;
}

// Build both gate/up tilings with the same instruction capacity so that the
// workspace layout does not depend on which one is active.
static mk_status plan_both(mk_ctx *c, const mk_config &cfg, int n_ctas, int active) {
    Plan a, b;
    mk_status s = build_plan(cfg, n_ctas, MK_SWIGLU_COL, a, c->err);
    if (s != MK_OK) return s;
    s = build_plan(cfg, n_ctas, MK_SWIGLU_ROW, b, c->err);
    if (s != MK_OK) return s;
    // Give both the larger instruction region: shift every later offset.
    size_t need = std::max(a.instrs.size(), b.instrs.size()) * sizeof(Instr);
    for (Plan *p : {&a, &b}) {
        size_t have = p->off_ranges - p->off_instrs;
        size_t grow = need > have ? ((need - have + 255) / 256) * 256 : 0;
        if (grow) {
            for (size_t *o : {&p->off_ranges, &p->off_layers, &p->off_rope, &p->off_x, &p->off_xe, &p->off_dpart, &p->off_qkv, &p->off_attn,
                              &p->off_act_a, &p->off_partials, &p->off_lm_best, &p->off_next_scratch, &p->off_norms,
                              &p->off_weights, &p->off_lm, &p->off_prefill, &p->workspace_bytes})
                *o += grow;
            p->lm.offset = p->off_lm;
        }
    }
    // Align both layouts to the same (larger) offsets.
    if (a.workspace_bytes != b.workspace_bytes) {
        Plan &small = a.workspace_bytes < b.workspace_bytes ? a : b;
        const Plan &big = a.workspace_bytes < b.workspace_bytes ? b : a;
        small.off_ranges = big.off_ranges; small.off_layers = big.off_layers; small.off_rope = big.off_rope;
        small.off_x = big.off_x; small.off_xe = big.off_xe; small.off_dpart = big.off_dpart; small.off_qkv = big.off_qkv; small.off_attn = big.off_attn;
        small.off_act_a = big.off_act_a; small.off_partials = big.off_partials; small.off_lm_best = big.off_lm_best;
        small.off_next_scratch = big.off_next_scratch; small.off_norms = big.off_norms;
        small.off_weights = big.off_weights; small.off_lm = big.off_lm; small.lm.offset = big.lm.offset;
        small.off_prefill = big.off_prefill;
        small.workspace_bytes = big.workspace_bytes;
    }
    s = validate_plan(a, c->err);
    if (s != MK_OK) return s;
    s = validate_plan(b, c->err);
    if (s != MK_OK) return s;
    if (active == MK_SWIGLU_ROW) {
        c->plan = b;
        c->plan_alt = a;
    } else {
        c->plan = a;
        c->plan_alt = b;
    }
    return MK_OK;
}

extern "C" {

mk_status mk_create(const mk_config *cfg, int device, mk_ctx **out) {
    if (!cfg || !out) return MK_ERR_INVALID;
    *out = nullptr;
    mk_ctx *c = new mk_ctx();
    int n_ctas = cfg->num_sms;
    if (device >= 0) {
        cudaError_t e = cudaSetDevice(device);
        if (e != cudaSuccess) {
            delete c;
            return MK_ERR_CUDA;
        }
        cudaDeviceProp prop;
        e = cudaGetDeviceProperties(&prop, device);
        if (e != cudaSuccess) {
            delete c;
            return MK_ERR_CUDA;
        }
        if (prop.major < 10) {
            delete c;
            return MK_ERR_UNSUPPORTED;
        }
        if (n_ctas <= 0 || n_ctas > prop.multiProcessorCount) n_ctas = prop.multiProcessorCount;
    } else if (n_ctas <= 0) {
        delete c;
        return MK_ERR_INVALID;
    }
    mk_status s = plan_both(c, *cfg, n_ctas, MK_SWIGLU_COL);
    if (s != MK_OK) {
        fprintf(stderr, "mk_create: %s\n", c->err.c_str());
        delete c;
        return s;
    }
    c->device = device;
    c->variant = cfg->variant;
    *out = c;
    return MK_OK;
}

mk_status mk_destroy(mk_ctx *c) {
    if (!c) return MK_ERR_INVALID;
    drop_graph(c);
    delete c;
    return MK_OK;
}

const char *mk_last_error(const mk_ctx *c) { return c ? c->err.c_str() : op_error(); }

mk_status mk_workspace_bytes(const mk_ctx *c, size_t *bytes) {
    if (!c || !bytes) return MK_ERR_INVALID;
    *bytes = c->plan.workspace_bytes;
    return MK_OK;
}

mk_status mk_kv_cache_bytes(const mk_ctx *c, size_t *bytes) {
    if (!c || !bytes) return MK_ERR_INVALID;
    *bytes = c->plan.kv_bytes;
    return MK_OK;
}

mk_status mk_schedule_info(const mk_ctx *c, long long *info, int n) {
    if (!c || !info) return MK_ERR_INVALID;
    const Plan &p = c->plan;
    long long v[10] = {(long long)p.instrs.size(), p.n_ctas, p.n_counters, p.n_phases, p.bs, p.chunks,
                       p.stages, p.act_bytes, p.swiglu_variant, p.down_ksplit};
    for (int i = 0; i < n && i < 10; ++i) info[i] = v[i];
    return MK_OK;
}

mk_status mk_set_trace(mk_ctx *c, void *d_trace, size_t bytes) {
    if (!c) return MK_ERR_INVALID;
    if (d_trace && bytes < c->plan.instrs.size() * 64) return fail(c, MK_ERR_INVALID, "trace buffer too small");
    c->trace = static_cast<unsigned long long *>(d_trace);
    drop_graph(c);
    return MK_OK;
}

mk_status mk_get_schedule(const mk_ctx *c, void *host_instrs, size_t bytes, int32_t *cta_base) {
    if (!c || !host_instrs) return MK_ERR_INVALID;
    const Plan &p = c->plan;
    if (bytes < p.instrs.size() * sizeof(Instr)) return MK_ERR_INVALID;
    memcpy(host_instrs, p.instrs.data(), p.instrs.size() * sizeof(Instr));
    if (cta_base) memcpy(cta_base, p.cta_base.data(), p.cta_base.size() * sizeof(int32_t));
    return MK_OK;
}

mk_status mk_validate_schedule(const mk_ctx *c) {
    if (!c) return MK_ERR_INVALID;
    return validate_plan(c->plan, const_cast<mk_ctx *>(c)->err);
}

static KParams make_params(mk_ctx *c, const int32_t *tokens, int64_t tok_stride, int32_t *next, float *logits) {
    const Plan &p = c->plan;
    const mk_config &g = p.cfg;
    KParams P{};
    uint8_t *ws = c->ws;
    P.instrs = reinterpret_cast<const Instr *>(ws + p.off_instrs);
    P.layers = reinterpret_cast<const LayerW *>(ws + p.off_layers);
    P.lm_w = ws + p.lm.offset;
    P.final_norm = ws + p.off_norms + (size_t)g.n_layers * (2 * g.hidden + 2 * g.head_dim) * 2;
    P.embed = c->embed;
    for (int i = 0; i < g.head_dim / 2 && i < 64; ++i) P.rope_inv_freq[i] = std::pow((double)g.rope_theta, -2.0 * i / g.head_dim);
    P.xm = reinterpret_cast<uint64_t *>(ws + p.off_x);
    P.xe = reinterpret_cast<uint64_t *>(ws + p.off_xe);
    P.dpart = reinterpret_cast<uint64_t *>(ws + p.off_dpart);
    P.qkv = reinterpret_cast<uint64_t *>(ws + p.off_qkv);
    P.attn = reinterpret_cast<uint64_t *>(ws + p.off_attn);
    P.act_a = reinterpret_cast<uint64_t *>(ws + p.off_act_a);
    P.partials = reinterpret_cast<uint64_t *>(ws + p.off_partials);
    P.down_ranges = p.down_ksplit;
    P.down_per = p.down_per;
    P.kcache = reinterpret_cast<uint16_t *>(c->kv);
    P.vcache = reinterpret_cast<uint16_t *>(c->kv + p.kv_bytes / 2);
    P.counters = reinterpret_cast<uint32_t *>(ws + p.off_counters);
    P.state = reinterpret_cast<State *>(ws + p.off_state);
    P.lm_best = reinterpret_cast<LmBest *>(ws + p.off_lm_best);
    P.tokens = tokens;
    P.next = next;
    P.logits = logits;
    P.tok_stride = tok_stride;
    P.timeout_ns = c->timeout_ns;
    P.trace = c->trace;
    P.prefetch = c->prefetch;
    P.n_layers = g.n_layers;
    P.hidden = g.hidden;
    P.n_heads = g.n_heads;
    P.n_kv_heads = g.n_kv_heads;
    P.head_dim = g.head_dim;
    P.intermediate = g.intermediate;
    P.vocab = g.vocab;
    P.batch = g.batch;
    P.max_seq = g.max_seq;
    P.qkv_rows = p.qkv_rows;
    P.i_pad = p.i_pad;
    P.chunks = p.chunks;
    P.n_ctas = p.n_ctas;
    P.stages = (c->stages > 0 && c->stages < p.stages) ? c->stages : p.stages;
    P.act_bytes = p.act_bytes;
    P.qk_norm = g.qk_norm;
    P.bs = p.bs;
    P.rms_eps = g.rms_eps;
    P.qkv_kc = p.qkv.kc; P.qkv_nkb = p.qkv.nkb;
    P.o_kc = p.o.kc; P.o_nkb = p.o.nkb;
    P.gu_kc = p.gu.kc; P.gu_nkb = p.gu.nkb;
    P.down_kc = p.down.kc; P.down_nkb = p.down.nkb;
    P.lm_kc = p.lm.kc; P.lm_nkb = p.lm.nkb;
    P.qkv_rt = p.qkv.rows; P.o_rt = p.o.rows; P.gu_rt = p.gu.rows; P.down_rt = p.down.rows; P.lm_rt = p.lm.rows;
    return P;
}

// Upload the active plan's instructions and launch ranges.
static mk_status upload_schedule(mk_ctx *c, cudaStream_t s) {
    const Plan &p = c->plan;
    std::vector<Instr> ins = p.instrs;
    if (c->drop_instr >= 0 && c->drop_instr < (int)ins.size()) ins[c->drop_instr].flags |= F_DROP_SIGNAL;
    CK(cudaMemcpyAsync(c->ws + p.off_instrs, ins.data(), ins.size() * sizeof(Instr), cudaMemcpyHostToDevice, s));
    // ranges: [0]: megakernel begin, [1]: megakernel end, then per phase k: begin(k), end(k) = begin(k+1)
    std::vector<int32_t> r((size_t)(p.n_phases + 2) * 2 * p.n_ctas);
    for (int i = 0; i < p.n_ctas; ++i) {
        r[i] = p.cta_base[i];
        r[p.n_ctas + i] = p.cta_base[i + 1];
    }
    for (int k = 0; k <= p.n_phases; ++k)
        for (int i = 0; i < p.n_ctas; ++i) r[(size_t)(2 + k) * p.n_ctas + i] = p.phase_begin[(size_t)k * p.n_ctas + i];
    CK(cudaMemcpyAsync(c->ws + p.off_ranges, r.data(), r.size() * 4, cudaMemcpyHostToDevice, s));
    CK(cudaStreamSynchronize(s));
    return MK_OK;
}

static mk_status reset_device_state(mk_ctx *c, cudaStream_t s) {
    const Plan &p = c->plan;
    // the step count restarts, so no tagged activation may keep a tag of the
    // new count's range: zero them (tag 0 is never valid)
    CK(cudaMemsetAsync(c->ws + p.off_x, 0, p.off_lm_best - p.off_x, s));
    CK(cudaMemsetAsync(c->ws + p.off_state, 0, sizeof(State), s));
    CK(cudaMemsetAsync(c->ws + p.off_counters, 0, (size_t)p.n_counters * 4, s));
    CK(cudaMemsetAsync(c->ws + p.off_lm_best, 0, (size_t)p.B * p.n_ctas * sizeof(LmBest), s));
    c->pos = 0;
    c->poisoned = false;
    return MK_OK;
}

mk_status mk_load_weights(mk_ctx *c, const mk_weights *w, void *workspace, void *kv_cache, void *stream) {
    if (!c) return MK_ERR_INVALID;
    if (c->device < 0) return fail(c, MK_ERR_STATE, "context was created without a device");
    if (!w || !workspace || !kv_cache || !w->embed || !w->final_norm || !w->attn_norm || !w->wq || !w->wk ||
        !w->wv || !w->wo || !w->mlp_norm || !w->wg || !w->wu || !w->wd)
        return fail(c, MK_ERR_INVALID, "mk_load_weights: null pointer");
    if (((uintptr_t)workspace & 255) || ((uintptr_t)kv_cache & 255))
        return fail(c, MK_ERR_INVALID, "workspace and kv_cache must be 256-byte aligned");
    const Plan &p = c->plan;
    const mk_config &g = p.cfg;
    if (!g.tied_embeddings && !w->lm_head) return fail(c, MK_ERR_INVALID, "lm_head is null for an untied model");
    if (g.qk_norm && (!w->q_norm || !w->k_norm)) return fail(c, MK_ERR_INVALID, "q_norm/k_norm null with qk_norm set");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CK(cudaSetDevice(c->device));
    c->ws = static_cast<uint8_t *>(workspace);
    c->kv = static_cast<uint8_t *>(kv_cache);
    c->embed = w->embed;
    drop_graph(c);
    const int L = g.n_layers, H = g.hidden, d = g.head_dim, I = g.intermediate;
    std::vector<LayerW> lw(L);
    uint8_t *norms = c->ws + p.off_norms;
    for (int l = 0; l < L; ++l) {
        if (!w->wq[l] || !w->wk[l] || !w->wv[l] || !w->wo[l] || !w->wg[l] || !w->wu[l] || !w->wd[l] ||
            !w->attn_norm[l] || !w->mlp_norm[l] || (g.qk_norm && (!w->q_norm[l] || !w->k_norm[l])))
            return fail(c, MK_ERR_INVALID, "mk_load_weights: null per-layer pointer");
        uint8_t *base = c->ws + p.off_weights + (size_t)l * p.layer_weight_bytes;
        // QKV: q, k and v rows packed into consecutive tile ranges (each count
        // is a multiple of the tile height)
        const int nqd = g.n_heads * d, nkd = g.n_kv_heads * d;
        const PackedMat &Q = p.qkv;
        const size_t tile_bytes = (size_t)Q.nkb * Q.rows * Q.kc * 2;
        CK(launch_pack(w->wq[l], nullptr, base + Q.offset, nqd, H, Q.kc, Q.nkb, nqd / Q.rows, Q.rows, 0, s));
        CK(launch_pack(w->wk[l], nullptr, base + Q.offset + tile_bytes * (nqd / Q.rows), nkd, H, Q.kc, Q.nkb,
                       nkd / Q.rows, Q.rows, 0, s));
        CK(launch_pack(w->wv[l], nullptr, base + Q.offset + tile_bytes * ((nqd + nkd) / Q.rows), nkd, H, Q.kc, Q.nkb,
                       nkd / Q.rows, Q.rows, 0, s));
        CK(launch_pack(w->wo[l], nullptr, base + p.o.offset, H, nqd, p.o.kc, p.o.nkb, p.o.tiles, p.o.rows, 0, s));
        CK(launch_pack(w->wg[l], w->wu[l], base + p.gu.offset, I, H, p.gu.kc, p.gu.nkb, p.gu.tiles, p.gu.rows, 1, s));
        CK(launch_pack(w->wd[l], nullptr, base + p.down.offset, H, I, p.down.kc, p.down.nkb, p.down.tiles, p.down.rows, 0, s));
        uint8_t *nl = norms + (size_t)l * (2 * H + 2 * d) * 2;
        CK(cudaMemcpyAsync(nl, w->attn_norm[l], (size_t)H * 2, cudaMemcpyDeviceToDevice, s));
        CK(cudaMemcpyAsync(nl + (size_t)H * 2, w->mlp_norm[l], (size_t)H * 2, cudaMemcpyDeviceToDevice, s));
        if (g.qk_norm) {
            CK(cudaMemcpyAsync(nl + (size_t)4 * H, w->q_norm[l], (size_t)d * 2, cudaMemcpyDeviceToDevice, s));
            CK(cudaMemcpyAsync(nl + (size_t)4 * H + 2 * d, w->k_norm[l], (size_t)d * 2, cudaMemcpyDeviceToDevice, s));
        }
        lw[l].qkv = base + p.qkv.offset;
        lw[l].o = base + p.o.offset;
        lw[l].gu = base + p.gu.offset;
        lw[l].down = base + p.down.offset;
        lw[l].attn_norm = nl;
        lw[l].mlp_norm = nl + (size_t)H * 2;
        lw[l].q_norm = g.qk_norm ? nl + (size_t)4 * H : nullptr;
        lw[l].k_norm = g.qk_norm ? nl + (size_t)4 * H + 2 * d : nullptr;
    }
    const void *head = g.tied_embeddings ? w->embed : w->lm_head;
    CK(launch_pack(head, nullptr, c->ws + p.lm.offset, g.vocab, H, p.lm.kc, p.lm.nkb, p.lm.tiles, p.lm.rows, 0, s));
    CK(cudaMemcpyAsync(norms + (size_t)L * (2 * H + 2 * d) * 2, w->final_norm, (size_t)H * 2,
                       cudaMemcpyDeviceToDevice, s));
    CK(cudaMemcpyAsync(c->ws + p.off_layers, lw.data(), lw.size() * sizeof(LayerW), cudaMemcpyHostToDevice, s));
    c->lw = lw;
    std::vector<double> inv(d / 2);
    for (int i = 0; i < d / 2; ++i) inv[i] = std::pow((double)g.rope_theta, -2.0 * i / d);
    CK(cudaMemcpyAsync(c->ws + p.off_rope, inv.data(), inv.size() * 8, cudaMemcpyHostToDevice, s));
    CK(cudaStreamSynchronize(s));  // the host vectors above must outlive the copies
    mk_status st = upload_schedule(c, s);
    if (st != MK_OK) return st;
    st = reset_device_state(c, s);
    if (st != MK_OK) return st;
    CK(cudaStreamSynchronize(s));
    c->loaded = true;
    return MK_OK;
}

static mk_status launch_megakernel(mk_ctx *c, const int32_t *tok, int64_t stride, int32_t *next, float *logits,
                                   cudaStream_t s) {
    KParams P = make_params(c, tok, stride, next, logits);
    const Plan &p = c->plan;
    const int32_t *ranges = reinterpret_cast<const int32_t *>(c->ws + p.off_ranges);
    P.cta_begin = ranges;
    P.cta_end = ranges + p.n_ctas;
    // tags: readers spin on the tagged activations themselves; counters:
    // acquire-spin / release-increment per instruction, tags then only verify
    P.use_waits = c->sync == MK_SYNC_COUNTERS ? 1 : 0;
    P.use_signals = P.use_waits;
    P.pdl = 0;
    cudaError_t e = launch_step(P, p.bs, p.n_ctas, s, true, false);
    if (e != cudaSuccess) {
        int per_sm = -1;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, step_kernel_func(P), kThreads, smem_bytes(P));
        cudaFuncAttributes fa{};
        cudaFuncGetAttributes(&fa, step_kernel_func(P));
        char buf[256];
        snprintf(buf, sizeof buf, "megakernel launch: %s (occupancy %d CTA/SM at %d threads, %d B smem, %d regs, max %d threads)",
                 cudaGetErrorString(e), per_sm, kThreads, smem_bytes(P), fa.numRegs, fa.maxThreadsPerBlock);
        return fail(c, MK_ERR_CUDA, buf);
    }
    return MK_OK;
}

// The separate-kernels variants: one launch of the same interpreter per
// phase.  MK_GRAPH and MK_GRAPH_PDL wait for the whole previous kernel (its
// end, or griddepcontrol.wait); MK_GRAPH_TILESYNC lets every kernel but the
// first launch early (its CTAs trigger their dependents as they start) and
// start on the tiles it reads, like the megakernel's instructions.
static KParams phase_params(mk_ctx *c, int k, const int32_t *tok, int32_t *next, float *logits, int variant) {
    KParams P = make_params(c, tok, 1, next, logits);
    const Plan &p = c->plan;
    const int32_t *ranges = reinterpret_cast<const int32_t *>(c->ws + p.off_ranges);
    const bool tiles = variant == MK_GRAPH_TILESYNC;
    P.use_waits = tiles && c->sync == MK_SYNC_COUNTERS ? 1 : 0;
    P.use_signals = P.use_waits;
    P.cta_begin = ranges + (size_t)(2 + k) * p.n_ctas;
    P.cta_end = ranges + (size_t)(3 + k) * p.n_ctas;
    P.pdl = tiles ? 2 : ((variant == MK_GRAPH_PDL && k > 0) ? 1 : 0);
    return P;
}

static mk_status launch_phases(mk_ctx *c, const int32_t *tok, int32_t *next, float *logits, cudaStream_t s,
                               int variant, std::vector<cudaGraphNode_t> *nodes) {
    const Plan &p = c->plan;
    const bool early = variant == MK_GRAPH_PDL || variant == MK_GRAPH_TILESYNC;
    for (int k = 0; k < p.n_phases; ++k) {
        KParams P = phase_params(c, k, tok, next, logits, variant);
        CK(launch_step(P, p.bs, p.n_ctas, s, false, early && k > 0));
        if (nodes) {
            cudaStreamCaptureStatus cs;
            const cudaGraphNode_t *deps = nullptr;
            size_t nd = 0;
            CK(cudaStreamGetCaptureInfo(s, &cs, nullptr, nullptr, &deps, &nd));
            if (nd != 1) return fail(c, MK_ERR_CUDA, "unexpected capture dependencies");
            nodes->push_back(deps[0]);
        }
    }
    return MK_OK;
}

// Point the captured graph at new token / output buffers: only the phases
// that read the tokens (layer-0 QKV and O-projection) or write the outputs (LM
// head) are patched, so a new pointer costs three node updates, not a
// re-capture.
static mk_status retarget_graph(mk_ctx *c, const int32_t *tok, int32_t *next, float *logits, int variant) {
    const Plan &p = c->plan;
    for (int k : p.token_phases) {
        KParams P = phase_params(c, k, tok, next, logits, variant);
        void *args[1] = {&P};
        cudaKernelNodeParams np = {};
        np.func = const_cast<void *>(step_kernel_func(P));
        np.gridDim = dim3(p.n_ctas);
        np.blockDim = dim3(kThreads);
        np.sharedMemBytes = smem_bytes(P);
        np.kernelParams = args;
        CK(cudaGraphExecKernelNodeSetParams(c->gexec, c->gnodes[k], &np));
    }
    c->g_tok = tok;
    c->g_next = next;
    c->g_logits = logits;
    return MK_OK;
}

static mk_status decode_tensor_cores(mk_ctx *c, const int32_t *d_tokens, int32_t *d_next, float *d_logits,
                                     cudaStream_t s);

mk_status mk_decode_step(mk_ctx *c, const int32_t *d_tokens, int32_t *d_next, float *d_logits, void *stream) {
    if (!c) return MK_ERR_INVALID;
    if (!c->loaded) return fail(c, MK_ERR_STATE, "mk_decode_step before mk_load_weights");
    if (c->poisoned) return fail(c, MK_ERR_STATE, "context poisoned by a device error; call mk_reset");
    if (!d_tokens) return fail(c, MK_ERR_INVALID, "d_tokens is null");
    if (c->pos >= c->plan.cfg.max_seq) return fail(c, MK_ERR_INVALID, "position reached max_seq");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    mk_status st;
    if (c->variant == MK_MEGAKERNEL) {
        st = launch_megakernel(c, d_tokens, 1, d_next, d_logits, s);
    } else if (c->variant == MK_TENSOR_CORES) {
        st = decode_tensor_cores(c, d_tokens, d_next, d_logits, s);
    } else {
        if (!c->gexec || c->g_variant != c->variant) {
            drop_graph(c);
            cudaStream_t cap;
            CK(cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking));
            cudaError_t e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal);
            if (e != cudaSuccess) {
                cudaStreamDestroy(cap);
                return cuda_fail(c, e, "cudaStreamBeginCapture");
            }
            st = launch_phases(c, d_tokens, d_next, d_logits, cap, c->variant, &c->gnodes);
            cudaGraph_t graph = nullptr;
            e = cudaStreamEndCapture(cap, &graph);
            cudaStreamDestroy(cap);
            if (st != MK_OK) {
                if (graph) cudaGraphDestroy(graph);
                c->gnodes.clear();
                return st;
            }
            if (e != cudaSuccess) return cuda_fail(c, e, "cudaStreamEndCapture");
            c->graph = graph;
            e = cudaGraphInstantiate(&c->gexec, graph, 0);
            if (e != cudaSuccess) {
                drop_graph(c);
                return cuda_fail(c, e, "cudaGraphInstantiate");
            }
            c->g_tok = d_tokens;
            c->g_next = d_next;
            c->g_logits = d_logits;
            c->g_variant = c->variant;
        } else if (c->g_tok != d_tokens || c->g_next != d_next || c->g_logits != d_logits) {
            st = retarget_graph(c, d_tokens, d_next, d_logits, c->variant);
            if (st != MK_OK) return st;
        }
        CK(cudaGraphLaunch(c->gexec, s));
        st = MK_OK;
    }
    if (st == MK_OK) c->pos += 1;
    return st;
}

// The row passes on the tensor cores (mk_tcdec.cu) over this context's
// packed weights, cache and scratch region.
static PrefillTc tc_args(mk_ctx *c) {
    const Plan &p = c->plan;
    const mk_config &g = p.cfg;
    PrefillTc a{};
    a.L = g.n_layers; a.H = g.hidden; a.nq = g.n_heads; a.nkv = g.n_kv_heads; a.d = g.head_dim;
    a.I = g.intermediate; a.V = g.vocab; a.B = g.batch; a.max_seq = g.max_seq; a.qk_norm = g.qk_norm;
    a.eps = g.rms_eps;
    a.theta = (double)g.rope_theta;
    a.embed = c->embed;
    a.layers = c->lw.data();
    a.qkv = p.qkv;
    a.o = p.o;
    a.gu = p.gu;
    a.down = p.down;
    a.lm = p.lm;
    a.lm_w = c->ws + p.lm.offset;
    a.final_norm = c->ws + p.off_norms + (size_t)g.n_layers * (2 * g.hidden + 2 * g.head_dim) * 2;
    a.kcache = reinterpret_cast<uint16_t *>(c->kv);
    a.vcache = reinterpret_cast<uint16_t *>(c->kv + p.kv_bytes / 2);
    a.state = reinterpret_cast<State *>(c->ws + p.off_state);
    a.scratch = c->ws + p.off_prefill;
    a.scratch_bytes = p.prefill_bytes;
    return a;
}

// The prefill on the tensor cores: every position of the prompt of every
// sequence goes through the decoder in chunks of kPrefillRows positions, each
// projection one GEMM over the packed weights (mk_tcdec.cu, prefill_tc).
static mk_status prefill_tensor_cores(mk_ctx *c, const int32_t *d_tokens, int T, cudaStream_t s) {
    const Plan &p = c->plan;
    const PrefillTc a = tc_args(c);
    const std::string err = prefill_tc(a, d_tokens, T, s);
    if (!err.empty()) return fail(c, MK_ERR_CUDA, "mk_prefill_kv (tensor cores): " + err);
    CK(launch_set_position(reinterpret_cast<State *>(c->ws + p.off_state), T, s));
    return MK_OK;
}

// One decode step on the tensor cores (MK_TENSOR_CORES).  The step's launches
// read the position from the device state and the tokens from the scratch's
// token row, so the first call runs them directly (setting the kernels'
// attributes) and the next captures them once into a CUDA graph that every
// later call replays: a token copy in, the graph, the argmax copy out.  The
// logits pointer is part of the capture; a different one captures again.
static mk_status decode_tensor_cores(mk_ctx *c, const int32_t *d_tokens, int32_t *d_next, float *d_logits,
                                     cudaStream_t s) {
    const PrefillTc a = tc_args(c);
    const int B = c->plan.cfg.batch;
    int32_t *tok = decode_tc_tokens(a), *nxt = decode_tc_next(a);
    if (!tok || !nxt) return fail(c, MK_ERR_STATE, "tensor-core decode: no scratch region");
    CK(cudaMemcpyAsync(tok, d_tokens, (size_t)B * 4, cudaMemcpyDeviceToDevice, s));
    if (!c->tc_warmed || c->tc_exec == nullptr || c->tc_logits != d_logits) {
        if (c->tc_exec) {
            cudaGraphExecDestroy(c->tc_exec);
            c->tc_exec = nullptr;
        }
        if (!c->tc_warmed) {
            const std::string err = decode_tc(a, tok, nxt, d_logits, s);
            if (!err.empty()) return fail(c, MK_ERR_CUDA, "tensor-core decode: " + err);
            c->tc_warmed = true;
        } else {
            cudaStream_t cap;
            CK(cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking));
            cudaError_t e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeRelaxed);
            if (e != cudaSuccess) {
                cudaStreamDestroy(cap);
                return cuda_fail(c, e, "cudaStreamBeginCapture");
            }
            const std::string err = decode_tc(a, tok, nxt, d_logits, cap);
            cudaGraph_t graph = nullptr;
            e = cudaStreamEndCapture(cap, &graph);
            cudaStreamDestroy(cap);
            if (!err.empty() || e != cudaSuccess) {
                if (graph) cudaGraphDestroy(graph);
                return fail(c, MK_ERR_CUDA, "tensor-core decode capture: " + (err.empty() ? std::string(cudaGetErrorString(e)) : err));
            }
            e = cudaGraphInstantiate(&c->tc_exec, graph, 0);
            cudaGraphDestroy(graph);
            if (e != cudaSuccess) return cuda_fail(c, e, "cudaGraphInstantiate");
            c->tc_logits = d_logits;
            CK(cudaGraphLaunch(c->tc_exec, s));
        }
    } else {
        CK(cudaGraphLaunch(c->tc_exec, s));
    }
    if (d_next) CK(cudaMemcpyAsync(d_next, nxt, (size_t)B * 4, cudaMemcpyDeviceToDevice, s));
    return MK_OK;
}

mk_status mk_prefill_kv(mk_ctx *c, const int32_t *d_tokens, int batch, int T, void *stream) {
    if (!c) return MK_ERR_INVALID;
    if (!c->loaded) return fail(c, MK_ERR_STATE, "mk_prefill_kv before mk_load_weights");
    if (c->poisoned) return fail(c, MK_ERR_STATE, "context poisoned by a device error; call mk_reset");
    if (!d_tokens || batch != c->plan.cfg.batch || T < 1 || T > c->plan.cfg.max_seq)
        return fail(c, MK_ERR_INVALID, "mk_prefill_kv: bad tokens, batch or length");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Plan &p = c->plan;
    if (c->prefill != MK_PREFILL_STEPS && p.prefill_tc) {
        c->pos = 0;
        mk_status st = prefill_tensor_cores(c, d_tokens, T, s);
        if (st != MK_OK) return st;
        c->pos = T;
        return MK_OK;
    }
    CK(cudaMemsetAsync(c->ws + p.off_state + offsetof(State, pos), 0, 4, s));
    c->pos = 0;
    int32_t *scratch = reinterpret_cast<int32_t *>(c->ws + p.off_next_scratch);
    for (int t = 0; t < T; ++t) {
        mk_status st = launch_megakernel(c, d_tokens + t, T, scratch, nullptr, s);
        if (st != MK_OK) return st;
        c->pos += 1;
    }
    return MK_OK;
}

mk_status mk_set_prefill(mk_ctx *c, int mode) {
    if (!c) return MK_ERR_INVALID;
    if (mode != MK_PREFILL_AUTO && mode != MK_PREFILL_STEPS && mode != MK_PREFILL_TC)
        return fail(c, MK_ERR_INVALID, "unknown prefill mode");
    c->prefill = mode;
    return MK_OK;
}

mk_status mk_get_status(mk_ctx *c, void *stream) {
    if (!c) return MK_ERR_INVALID;
    if (!c->loaded) return MK_OK;
    CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    State st;
    CK(cudaMemcpy(&st, c->ws + c->plan.off_state, sizeof st, cudaMemcpyDeviceToHost));
    if (st.err) {
        c->poisoned = true;
        char buf[200];
        snprintf(buf, sizeof buf, "device wait gave up (code %u) in CTA %u, instruction %u, counter %u", st.err,
                 st.err_cta, st.err_instr, st.err_ctr);
        c->err = buf;
        return MK_ERR_TIMEOUT;
    }
    if (st.tok_err) {
        c->poisoned = true;
        char buf[200];
        snprintf(buf, sizeof buf, "token %d of sequence %u is outside [0, %d): the step decoded token 0 in its place",
                 st.tok_bad, st.tok_err - 1u, c->plan.cfg.vocab);
        c->err = buf;
        return MK_ERR_INVALID;
    }
    return MK_OK;
}

mk_status mk_reset(mk_ctx *c, void *stream) {
    if (!c) return MK_ERR_INVALID;
    if (!c->loaded) return fail(c, MK_ERR_STATE, "mk_reset before mk_load_weights");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CK(cudaStreamSynchronize(s));
    mk_status st = reset_device_state(c, s);
    if (st != MK_OK) return st;
    CK(cudaStreamSynchronize(s));
    return MK_OK;
}

mk_status mk_get_position(const mk_ctx *c, int *pos) {
    if (!c || !pos) return MK_ERR_INVALID;
    *pos = c->pos;
    return MK_OK;
}

mk_status mk_set_position(mk_ctx *c, int pos, void *stream) {
    if (!c) return MK_ERR_INVALID;
    if (!c->loaded) return fail(c, MK_ERR_STATE, "mk_set_position before mk_load_weights");
    if (pos < 0 || pos > c->plan.cfg.max_seq) return fail(c, MK_ERR_INVALID, "position out of range");
    CK(launch_set_position(reinterpret_cast<State *>(c->ws + c->plan.off_state), pos, static_cast<cudaStream_t>(stream)));
    c->pos = pos;
    return MK_OK;
}

mk_status mk_set_variant(mk_ctx *c, int variant) {
    if (!c) return MK_ERR_INVALID;
    if (variant < MK_MEGAKERNEL || variant > MK_TENSOR_CORES) return fail(c, MK_ERR_INVALID, "unknown variant");
    c->variant = variant;
    return MK_OK;
}

mk_status mk_set_prefetch(mk_ctx *c, int blocks) {
    if (!c || blocks < 0 || blocks > 64) return MK_ERR_INVALID;
    c->prefetch = blocks;
    drop_graph(c);
    return MK_OK;
}

mk_status mk_set_ring_stages(mk_ctx *c, int stages) {
    if (!c || stages < 0 || stages > kMaxStages) return MK_ERR_INVALID;
    if (stages == 1) return fail(c, MK_ERR_INVALID, "the ring needs at least 2 slots");
    c->stages = stages;
    drop_graph(c);
    return MK_OK;
}

mk_status mk_set_sync(mk_ctx *c, int mode) {
    if (!c) return MK_ERR_INVALID;
    if (mode != MK_SYNC_TAGS && mode != MK_SYNC_COUNTERS) return fail(c, MK_ERR_INVALID, "unknown sync mode");
    if (mode != c->sync) drop_graph(c);  // the tile-synchronised graph captured the old waits
    c->sync = mode;
    return MK_OK;
}

mk_status mk_set_timeout_ns(mk_ctx *c, unsigned long long ns) {
    if (!c || ns == 0) return MK_ERR_INVALID;
    c->timeout_ns = ns;
    drop_graph(c);
    return MK_OK;
}

mk_status mk_debug_drop_signal(mk_ctx *c, int instr) {
    if (!c) return MK_ERR_INVALID;
    if (instr >= (int)c->plan.instrs.size()) return fail(c, MK_ERR_INVALID, "instruction index out of range");
    c->drop_instr = instr;
    if (c->loaded) {
        drop_graph(c);
        return upload_schedule(c, nullptr);
    }
    return MK_OK;
}

mk_status mk_debug_poison_activations(mk_ctx *c, void *stream) {
    if (!c) return MK_ERR_INVALID;
    if (!c->loaded) return fail(c, MK_ERR_STATE, "mk_debug_poison_activations before mk_load_weights");
    const Plan &p = c->plan;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CK(cudaMemsetAsync(c->ws + p.off_x, 0xFF, p.off_lm_best - p.off_x, s));
    CK(cudaMemsetAsync(c->ws + p.off_lm_best, 0xFF, (size_t)p.B * p.n_ctas * sizeof(LmBest), s));
    CK(cudaStreamSynchronize(s));
    return MK_OK;
}

mk_status mk_debug_shuffle_schedule(mk_ctx *c, unsigned long long seed) {
    if (!c) return MK_ERR_INVALID;
    mk_status st = shuffle_plan(c->plan, seed, c->err);
    if (st != MK_OK) return st;
    if (c->loaded) {
        drop_graph(c);
        return upload_schedule(c, nullptr);
    }
    return MK_OK;
}

// Swap the active gate/up tiling (same layout); counters restart.
static mk_status switch_plan(mk_ctx *c, cudaStream_t s) {
    std::swap(c->plan, c->plan_alt);
    drop_graph(c);
    int pos = c->pos;
    mk_status st = upload_schedule(c, s);
    if (st != MK_OK) return st;
    const Plan &p = c->plan;
    CK(cudaMemsetAsync(c->ws + p.off_x, 0, p.off_lm_best - p.off_x, s));  // the step count restarts
    CK(cudaMemsetAsync(c->ws + p.off_state, 0, sizeof(State), s));
    CK(cudaMemsetAsync(c->ws + p.off_counters, 0, (size_t)p.n_counters * 4, s));
    CK(cudaMemcpyAsync(c->ws + p.off_state + offsetof(State, pos), &pos, 4, cudaMemcpyHostToDevice, s));
    CK(cudaStreamSynchronize(s));
    return MK_OK;
}

mk_status mk_set_swiglu_tiling(mk_ctx *c, int variant, void *stream) {
    if (!c) return MK_ERR_INVALID;
    if (variant != MK_SWIGLU_ROW && variant != MK_SWIGLU_COL)
        return fail(c, MK_ERR_INVALID, "mk_set_swiglu_tiling: MK_SWIGLU_ROW or MK_SWIGLU_COL");
    if (!c->loaded) return fail(c, MK_ERR_STATE, "mk_set_swiglu_tiling before mk_load_weights");
    if (c->poisoned) return fail(c, MK_ERR_STATE, "context poisoned by a device error; call mk_reset");
    if (c->plan.swiglu_variant == variant) return MK_OK;
    return switch_plan(c, static_cast<cudaStream_t>(stream));
}

mk_status mk_get_swiglu_tiling(const mk_ctx *c, int *variant) {
    if (!c || !variant) return MK_ERR_INVALID;
    *variant = c->plan.swiglu_variant;
    return MK_OK;
}

mk_status mk_tune(mk_ctx *c, void *stream, int *chosen) {
    if (!c) return MK_ERR_INVALID;
    if (!c->loaded) return fail(c, MK_ERR_STATE, "mk_tune before mk_load_weights");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int reps = 5;
    if (c->plan.B == 1) {  // both tilings are the same single pass at batch 1
        if (c->plan.swiglu_variant != MK_SWIGLU_COL) {
            mk_status st = switch_plan(c, s);
            if (st != MK_OK) return st;
        }
        if (chosen) *chosen = MK_SWIGLU_COL;
        return MK_OK;
    }
    if (c->pos + 2 * (reps + 1) > c->plan.cfg.max_seq) return fail(c, MK_ERR_INVALID, "mk_tune needs free KV positions");
    const int pos0 = c->pos;
    int32_t *scratch = reinterpret_cast<int32_t *>(c->ws + c->plan.off_next_scratch);
    float ms[2] = {0, 0};
    int variants[2];
    cudaEvent_t e0, e1;
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
    for (int v = 0; v < 2; ++v) {
        variants[v] = c->plan.swiglu_variant;
        // tokens: reuse the scratch (zeros or last argmax) as inputs -- values do not matter for timing
        mk_status st = launch_megakernel(c, scratch, 0, scratch, nullptr, s);
        if (st != MK_OK) return st;
        CK(cudaEventRecord(e0, s));
        for (int r = 0; r < reps; ++r) {
            st = launch_megakernel(c, scratch, 0, scratch, nullptr, s);
            if (st != MK_OK) return st;
        }
        CK(cudaEventRecord(e1, s));
        CK(cudaEventSynchronize(e1));
        CK(cudaEventElapsedTime(&ms[v], e0, e1));
        c->pos = pos0;
        st = switch_plan(c, s);  // also restores the position
        if (st != MK_OK) return st;
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    // After two switches the original plan is active again; keep the faster.
    const int best = ms[0] <= ms[1] ? variants[0] : variants[1];
    if (c->plan.swiglu_variant != best) {
        mk_status st = switch_plan(c, s);
        if (st != MK_OK) return st;
    }
    if (chosen) *chosen = best;
    return mk_get_status(c, s);
}

}  // extern "C"

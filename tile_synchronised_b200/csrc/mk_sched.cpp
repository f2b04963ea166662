// mk_sched.cpp -- host-side planner of the decode megakernel.
//
// The step is a fixed sequence of phases per layer -- QKV, attention, O-proj,
// gate/up, down -- and a final LM-head phase.  Each phase is cut into
// instructions (a GEMV row tile over a K range and a batch range, or one
// split-KV attention chunk); every instruction is handed to one CTA, and each
// CTA runs its instructions in phase order.  Instead of a kernel boundary
// between phases, a consumer instruction waits on one global counter until it
// has received the number of increments its producers make per step; the
// counters only grow (the target is (step + 1) * count), so nothing is reset
// between steps.  This is the tile-level producer/consumer synchronisation of
// "MegaOps: A Kernel Overlapping Framework ..." ("In plain words", "Keep
// kernels separate"), here inside one persistent kernel.
//
// Deadlock freedom: instructions only wait on counters fed by earlier phases
// and every CTA runs its list in phase order, so with all CTAs resident the
// earliest unfinished phase always makes progress.  validate_plan() checks
// this, and every count, by simulating the lists.
#include "mk_sched.h"

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <queue>

namespace mk {

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Tiles are `rows` x kc blocks with kc = K rounded up to 256 (one 8-column
// chunk per lane of a warp) and rows the largest power of two <= 8 that keeps
// a block within one 32 KB ring slot: K <= 2048 -> 8 rows, 4096 -> 4, 8192 -> 2,
// up to 16384 -> 1.  `ksplit` cuts K into that many blocks (activation budget).
// Gate/up tiles hold rows/2 gate rows then the matching rows/2 up rows.
static PackedMat make_mat(int n_rows, int k, bool pair = false, int ksplit = 1) {
    PackedMat m{};
    m.n_rows = n_rows;
    m.k = k;
    const int kpad = (k + 255) / 256 * 256;
    m.nkb = std::max(1, ksplit);
    m.kc = ((kpad + m.nkb - 1) / m.nkb + 255) / 256 * 256;
    m.nkb = (kpad + m.kc - 1) / m.kc;
    m.rows = kMaxTileRows;
    while (m.rows > (pair ? 2 : 1) && m.rows * m.kc * 2 > kStageBytes) m.rows /= 2;
    m.tiles = pair ? (n_rows / 2 + m.rows / 2 - 1) / (m.rows / 2) : (n_rows + m.rows - 1) / m.rows;
    return m;
}

static size_t mat_bytes(const PackedMat &m) { return (size_t)m.tiles * m.nkb * m.rows * m.kc * 2; }

mk_status build_plan(const mk_config &c, int n_ctas, int swiglu_variant, Plan &p, std::string &err) {
    p = Plan();
    p.cfg = c;
    auto bad = [&](mk_status s, const char *msg) {
        err = msg;
        return s;
    };
    if (c.n_layers < 1 || c.hidden < 8 || c.n_heads < 1 || c.n_kv_heads < 1 || c.intermediate < 4 ||
        c.vocab < 1 || c.batch < 1 || c.max_seq < 1 || n_ctas < 1)
        return bad(MK_ERR_INVALID, "mk_config: sizes must be positive");
    if (!(c.rms_eps >= 0.0f) || !(c.rope_theta > 0.0f)) return bad(MK_ERR_INVALID, "mk_config: bad eps/theta");
    if (c.dtype != MK_BF16) return bad(MK_ERR_UNSUPPORTED, "only MK_BF16 weights are supported");
    if (c.head_dim != 64 && c.head_dim != 128) return bad(MK_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (c.n_heads % c.n_kv_heads) return bad(MK_ERR_UNSUPPORTED, "n_heads must be a multiple of n_kv_heads");
    if (c.n_heads / c.n_kv_heads > kMaxGroup) return bad(MK_ERR_UNSUPPORTED, "more than 8 query heads per KV head");
    if (c.hidden % 8 || c.intermediate % 8) return bad(MK_ERR_UNSUPPORTED, "hidden and intermediate must be multiples of 8");
    if (c.hidden > 8192) return bad(MK_ERR_UNSUPPORTED, "hidden above 8192");
    if (c.batch > 64) return bad(MK_ERR_UNSUPPORTED, "batch above 64");
    if (c.max_seq > (1 << 20)) return bad(MK_ERR_UNSUPPORTED, "max_seq above 2^20");
    if (n_ctas > 1024) return bad(MK_ERR_UNSUPPORTED, "more than 1024 CTAs");
    if (c.variant < MK_MEGAKERNEL || c.variant > MK_TENSOR_CORES) return bad(MK_ERR_INVALID, "unknown variant");

    const int L = c.n_layers, H = c.hidden, nq = c.n_heads, nkv = c.n_kv_heads, d = c.head_dim;
    const int I = c.intermediate, V = c.vocab, B = c.batch;
    p.n_ctas = n_ctas;
    p.B = B;
    p.swiglu_variant = swiglu_variant;
    p.qkv_rows = (nq + 2 * nkv) * d;
    p.qkv = make_mat(p.qkv_rows, H);
    p.o = make_mat(H, nq * d);
    p.gu = make_mat(2 * I, H, true);
    p.down = make_mat(H, I);
    p.lm = make_mat(V, H);
    if (p.qkv.rows * p.qkv.kc * 2 > kStageBytes || p.gu.rows * p.gu.kc * 2 > kStageBytes)
        return bad(MK_ERR_UNSUPPORTED, "hidden too large for one ring slot per tile row");
    if ((nq * d) % p.qkv.rows || (nkv * d) % p.qkv.rows) return bad(MK_ERR_UNSUPPORTED, "q/k/v rows not tile-aligned");

    // Batch rows per instruction and the activation region.  Activations are
    // staged in shared memory as fp32 [rows][K range]; the region is capped at
    // 64 KB so at least four 32 KB ring slots remain.  A GEMV whose rows do not
    // fit carries fewer batch rows (its weights stream once per row group); the
    // down projection splits K instead (atomic residual update).
    const int kActMax = 65536;
    p.bs = std::min(B, kMaxBatchRows);
    auto fit_bs = [&](const PackedMat &m) { return std::max(1, std::min(p.bs, kActMax / (m.nkb * m.kc * 4))); };
    p.bs = std::min({fit_bs(p.qkv), fit_bs(p.gu), fit_bs(p.lm), fit_bs(p.o)});
    if ((size_t)p.bs * p.qkv.nkb * p.qkv.kc * 4 > (size_t)kActMax) return bad(MK_ERR_UNSUPPORTED, "hidden too large");
    if ((size_t)p.bs * p.o.nkb * p.o.kc * 4 > (size_t)kActMax) return bad(MK_ERR_UNSUPPORTED, "n_heads*head_dim too large");
    p.gu_bs = p.bs;
    if (swiglu_variant == MK_SWIGLU_ROW && B > 1) p.gu_bs = std::max(1, (std::min(B, p.bs) + 1) / 2);
    // the down projection's K (= intermediate) is split so bs rows x kc fit the region
    int down_split = 1;
    while ((size_t)p.bs * (((I + 255) / 256 * 256 + down_split - 1) / down_split) * 4 > (size_t)kActMax) ++down_split;
    p.down = make_mat(H, I, false, down_split);
    p.down_ksplit = p.down.nkb;  // one K block per range: each range writes its own partial output
    p.down_per = 1;
    p.i_pad = p.down.nkb * p.down.kc;
    const int down_blocks_per_range = 1;
    int act = 0;
    act = std::max(act, p.bs * p.qkv.nkb * p.qkv.kc * 4);
    act = std::max(act, p.bs * p.o.nkb * p.o.kc * 4);
    act = std::max(act, p.bs * p.lm.nkb * p.lm.kc * 4);
    act = std::max(act, p.gu_bs * p.gu.nkb * p.gu.kc * 4);
    act = std::max(act, p.bs * down_blocks_per_range * p.down.kc * 4);
    const int G = nq / nkv;
    // Split-KV chunks: as many units as fit one per CTA (an attention phase is
    // one unit deep), at most kMaxAttnChunks per (sequence, KV head) since the
    // last unit of a (sequence, KV head) gathers every chunk's partial.
    p.chunks = std::max(1, std::min(kMaxAttnChunks, n_ctas / (B * nkv)));
    p.chunks = std::min(p.chunks, std::max(1, c.max_seq / 16));
    const int attn_scratch = G * d * 4 + 2 * d * 4 + kConsumerWarps * (d + 2) * 4 + kConsumerWarps * 64 * 4;
    act = std::max(act, attn_scratch);
    p.act_bytes = (int)align_up(act, 128);
    p.stages = kMaxStages;
    while (p.stages >= 2 && (size_t)p.stages * kStageBytes + p.act_bytes + misc_bytes(p.bs, p.stages) > (size_t)kMaxSmem)
        --p.stages;
    if (p.stages < 2) return bad(MK_ERR_UNSUPPORTED, "not enough shared memory for the ring");

    // Counters: six per layer (QKV, attention, combine, O, gate/up, down),
    // then the LM-head arrival counter.
    p.n_counters = kCountersPerLayer * L + 1;
    if (p.n_counters >= kNoCounter) return bad(MK_ERR_UNSUPPORTED, "too many counters");
    const int arr_lm = kCountersPerLayer * L;
    p.counter_count.assign(p.n_counters, 0);

    // ---------------------------------------------------------- instructions per phase
    std::vector<std::vector<Instr>> phases;
    std::vector<std::vector<double>> costs;
    // A GEMV phase is cut into runs of consecutive row tiles, about one run
    // per CTA for every (K range, batch range) combination, so each CTA streams
    // contiguous weights and pays the per-instruction cost once per run.
    auto gemv_phase = [&](uint8_t op, int l, const PackedMat &m, int bs, int ksplit, uint8_t flags, int wait,
                          int signal) {
        std::vector<Instr> v;
        std::vector<double> cost;
        const int per = (m.nkb + ksplit - 1) / ksplit;
        const int nk = (m.nkb + per - 1) / per, nbr = (B + bs - 1) / bs;
        const int combos = nk * nbr;
        const int runs = std::max(1, std::min(m.tiles, (n_ctas + combos - 1) / combos));
        for (int r = 0; r < runs; ++r) {
            const int t0 = (int)((long long)r * m.tiles / runs), t1 = (int)((long long)(r + 1) * m.tiles / runs);
            if (t1 <= t0) continue;
            for (int kb = 0; kb < m.nkb; kb += per)
                for (int b0 = 0; b0 < B; b0 += bs) {
                    Instr in{};
                    in.op = op;
                    in.flags = flags;
                    in.layer = (uint16_t)l;
                    in.tile = (uint32_t)t0;
                    in.ntiles = (uint16_t)(t1 - t0);
                    in.kb0 = (uint16_t)kb;
                    in.kb1 = (uint16_t)std::min(m.nkb, kb + per);
                    in.b0 = (uint16_t)b0;
                    in.nb = (uint16_t)std::min(bs, B - b0);
                    in.wait_ctr = wait < 0 ? kNoCounter : (uint16_t)wait;
                    in.signal_ctr = signal < 0 ? kNoCounter : (uint16_t)signal;
                    in.signal2_ctr = kNoCounter;
                    v.push_back(in);
                    cost.push_back((double)(t1 - t0) * (in.kb1 - in.kb0) * m.rows * m.kc * 2 + 4096.0);
                }
        }
        if (signal >= 0) p.counter_count[signal] += (uint32_t)v.size();
        phases.push_back(v);
        costs.push_back(cost);
    };
    const double typical_ctx = std::max(1.0, 0.75 * c.max_seq);
    for (int l = 0; l < L; ++l) {
        gemv_phase(OP_QKV, l, p.qkv, p.bs, 1, l == 0 ? F_EMBED_X : 0, l == 0 ? -1 : counter_down(l - 1),
                   counter_qkv(l));
        {
            std::vector<Instr> v;
            std::vector<double> cost;
            for (int b = 0; b < B; ++b)
                for (int g = 0; g < nkv; ++g)
                    for (int ch = 0; ch < p.chunks; ++ch) {
                        Instr in{};
                        in.op = OP_ATTN;
                        in.layer = (uint16_t)l;
                        in.tile = (uint32_t)((b * nkv + g) * p.chunks + ch);
                        in.b0 = (uint16_t)b;
                        in.nb = 1;
                        in.wait_ctr = (uint16_t)counter_qkv(l);
                        in.signal_ctr = (uint16_t)counter_att(l);
                        in.signal2_ctr = kNoCounter;
                        v.push_back(in);
                        cost.push_back(typical_ctx / p.chunks * d * 4 + 8192.0);
                    }
            p.counter_count[counter_att(l)] += (uint32_t)v.size();
            phases.push_back(v);
            costs.push_back(cost);
        }
        {  // one log-sum-exp combine per (sequence, KV head)
            std::vector<Instr> v;
            std::vector<double> cost;
            for (int b = 0; b < B; ++b)
                for (int g = 0; g < nkv; ++g) {
                    Instr in{};
                    in.op = OP_ACOMB;
                    in.layer = (uint16_t)l;
                    in.tile = (uint32_t)(b * nkv + g);
                    in.b0 = (uint16_t)b;
                    in.nb = 1;
                    in.wait_ctr = (uint16_t)counter_att(l);
                    in.signal_ctr = (uint16_t)counter_acomb(l);
                    in.signal2_ctr = kNoCounter;
                    v.push_back(in);
                    cost.push_back((double)p.chunks * G * (d + 2) * 8 + 8192.0);
                }
            p.counter_count[counter_acomb(l)] += (uint32_t)v.size();
            phases.push_back(v);
            costs.push_back(cost);
        }
        gemv_phase(OP_OPROJ, l, p.o, p.bs, 1, l == 0 ? F_EMBED_X : 0, counter_acomb(l), counter_o(l));
        gemv_phase(OP_GATEUP, l, p.gu, p.gu_bs, 1, 0, counter_o(l), counter_gu(l));
        gemv_phase(OP_DOWN, l, p.down, p.bs, p.down_ksplit, 0, counter_gu(l), counter_down(l));
    }
    gemv_phase(OP_LMHEAD, L - 1, p.lm, p.bs, 1, 0, counter_down(L - 1), -1);
    p.n_phases = (int)phases.size();
    for (int ph = 0; ph < p.n_phases; ++ph)
        if (!phases[ph].empty() && ((phases[ph][0].flags & F_EMBED_X) || phases[ph][0].op == OP_LMHEAD))
            p.token_phases.push_back(ph);

    // Fill wait counts now that every producer is known.
    for (auto &ph : phases)
        for (auto &in : ph)
            if (in.wait_ctr != kNoCounter) in.wait_count = p.counter_count[in.wait_ctr];

    // ---------------------------------------------------------- assignment to CTAs
    // Greedy least-loaded by cumulative streamed bytes, with at most
    // ceil(n / n_ctas) instructions of one phase per CTA: every SM's total
    // bytes per step stay within one instruction of the mean, and no phase
    // (attention in particular, whose units are cheap) piles several of its
    // instructions onto the same few CTAs and lengthens its critical path.
    std::vector<std::vector<std::vector<Instr>>> per(n_ctas, std::vector<std::vector<Instr>>(p.n_phases));
    std::vector<double> load(n_ctas, 0.0);
    using Item = std::pair<double, int>;
    for (int ph = 0; ph < p.n_phases; ++ph) {
        const size_t n = phases[ph].size();
        const size_t cap = (n + n_ctas - 1) / n_ctas;
        std::priority_queue<Item, std::vector<Item>, std::greater<Item>> heap;
        for (int i = 0; i < n_ctas; ++i) heap.push({load[i], i});
        std::vector<size_t> taken(n_ctas, 0);
        for (size_t j = 0; j < n; ++j) {
            Item it = heap.top();
            heap.pop();
            per[it.second][ph].push_back(phases[ph][j]);
            load[it.second] += costs[ph][j];
            if (++taken[it.second] < cap) heap.push({load[it.second], it.second});
        }
    }
    // LM-head arrivals: one per CTA that has LM work; its last LM instruction publishes.
    int lm_ctas = 0;
    const int lm_phase = p.n_phases - 1;
    for (int i = 0; i < n_ctas; ++i)
        if (!per[i][lm_phase].empty()) {
            ++lm_ctas;
            per[i][lm_phase].back().flags |= F_LAST_LM;
        }
    for (int i = 0; i < n_ctas; ++i)
        for (auto &in : per[i][lm_phase]) {
            in.signal_ctr = (uint16_t)arr_lm;
            in.arrive_count = (uint32_t)lm_ctas;
        }

    // Flatten.
    p.cta_base.assign(n_ctas + 1, 0);
    p.phase_begin.assign((size_t)(p.n_phases + 1) * n_ctas, 0);
    for (int i = 0; i < n_ctas; ++i) {
        p.cta_base[i] = (int32_t)p.instrs.size();
        for (int ph = 0; ph < p.n_phases; ++ph) {
            p.phase_begin[(size_t)ph * n_ctas + i] = (int32_t)p.instrs.size();
            for (auto &in : per[i][ph]) p.instrs.push_back(in);
        }
        p.phase_begin[(size_t)p.n_phases * n_ctas + i] = (int32_t)p.instrs.size();
    }
    p.cta_base[n_ctas] = (int32_t)p.instrs.size();

    // ---------------------------------------------------------- workspace layout
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = align_up(o, 256);
        o = at + bytes;
        return at;
    };
    p.off_state = take(sizeof(State));
    p.off_counters = take((size_t)p.n_counters * 4);
    p.off_instrs = take(p.instrs.size() * sizeof(Instr));
    p.off_ranges = take((size_t)(p.n_phases + 2) * 2 * n_ctas * 4);
    p.off_layers = take((size_t)L * sizeof(LayerW));
    p.off_rope = take((size_t)(d / 2) * 8);
    p.off_x = take((size_t)B * H * 8);  // tagged words from here to off_lm_best
    p.off_xe = take((size_t)B * H * 8);
    p.off_dpart = take((size_t)(p.down_ksplit - 1) * B * H * 8);
    p.off_qkv = take((size_t)B * p.qkv_rows * 8);
    p.off_attn = take((size_t)B * nq * d * 8);
    p.off_act_a = take((size_t)B * I * 8);
    p.off_partials = take((size_t)B * nq * p.chunks * partial_stride(d) * 8);
    p.off_lm_best = take((size_t)B * n_ctas * sizeof(LmBest));
    p.off_next_scratch = take((size_t)B * 4);
    p.off_norms = take((size_t)(L * (2 * H + 2 * d) + H) * 2);
    p.layer_weight_bytes = align_up(mat_bytes(p.qkv), 256) + align_up(mat_bytes(p.o), 256) +
                           align_up(mat_bytes(p.gu), 256) + align_up(mat_bytes(p.down), 256);
    p.off_weights = take((size_t)L * p.layer_weight_bytes);
    p.off_lm = take(mat_bytes(p.lm));
    p.prefill_tc = true;  // the tensor cores read every packed matrix (4-D tensor map over its tiles)
    if (p.prefill_tc) {
        // (also the buffers of the decode step on the tensor cores, whose LM
        // head is the widest GEMM output)
        const int kmax = std::max({p.qkv.nkb * p.qkv.kc, p.o.nkb * p.o.kc, p.gu.nkb * p.gu.kc, p.down.nkb * p.down.kc,
                                   p.lm.nkb * p.lm.kc});
        const int mmax = std::max({p.qkv.tiles * p.qkv.rows, p.o.tiles * p.o.rows, p.gu.tiles * p.gu.rows,
                                   p.down.tiles * p.down.rows, p.lm.tiles * p.lm.rows});
        p.prefill_bytes = prefill_scratch_bytes(H, nq, d, kmax, mmax);
        p.off_prefill = take(p.prefill_bytes);
    }
    p.qkv.offset = 0;
    p.o.offset = align_up(mat_bytes(p.qkv), 256);
    p.gu.offset = p.o.offset + align_up(mat_bytes(p.o), 256);
    p.down.offset = p.gu.offset + align_up(mat_bytes(p.gu), 256);
    p.lm.offset = p.off_lm;
    p.workspace_bytes = align_up(o, 256);
    p.kv_bytes = (size_t)2 * L * B * nkv * (size_t)c.max_seq * d * 2;
    return MK_OK;
}

mk_status validate_plan(const Plan &p, std::string &err) {
    const mk_config &c = p.cfg;
    char buf[256];
    auto fail = [&](const char *msg) {
        err = msg;
        return MK_ERR_STATE;
    };
    // Shared memory: ring + activations + misc (sized for the kernel instance).
    if ((size_t)p.stages * kStageBytes + p.act_bytes + misc_bytes(p.bs, p.stages) > (size_t)kMaxSmem)
        return fail("shared-memory layout exceeds the per-CTA limit");
    // Index ranges.
    for (size_t i = 0; i < p.instrs.size(); ++i) {
        const Instr &in = p.instrs[i];
        const PackedMat *m = nullptr;
        switch (in.op) {
            case OP_QKV: m = &p.qkv; break;
            case OP_OPROJ: m = &p.o; break;
            case OP_GATEUP: m = &p.gu; break;
            case OP_DOWN: m = &p.down; break;
            case OP_LMHEAD: m = &p.lm; break;
            case OP_ATTN:
            case OP_ACOMB: break;
            default:
                snprintf(buf, sizeof buf, "instruction %zu: bad opcode %d", i, in.op);
                return fail(buf);
        }
        if (in.layer >= c.n_layers) return fail("instruction layer out of range");
        if (in.b0 + in.nb > p.B || in.nb < 1) return fail("instruction batch range out of range");
        if (m) {
            if (in.ntiles < 1 || in.tile + in.ntiles > (uint32_t)m->tiles || in.kb0 >= in.kb1 || in.kb1 > m->nkb)
                return fail("GEMV instruction tile/K range out of range");
            if (in.nb > kMaxBatchRows) return fail("GEMV instruction carries too many batch rows");
            if ((size_t)in.nb * (in.kb1 - in.kb0) * m->kc * 4 > (size_t)p.act_bytes)
                return fail("GEMV activation range does not fit the shared-memory region");
        } else if (in.op == OP_ATTN) {
            if (in.tile >= (uint32_t)(p.B * c.n_kv_heads * p.chunks)) return fail("attention unit out of range");
        } else {
            if (in.tile >= (uint32_t)(p.B * c.n_kv_heads) || in.b0 != in.tile / c.n_kv_heads)
                return fail("combine unit out of range");
        }
        if (in.wait_ctr != kNoCounter && in.wait_ctr >= p.n_counters) return fail("wait counter out of range");
        if (in.signal_ctr != kNoCounter && in.signal_ctr >= p.n_counters) return fail("signal counter out of range");
        if (in.signal2_ctr != kNoCounter && in.signal2_ctr >= p.n_counters) return fail("signal2 out of range");
    }
    // Simulate one step: every CTA executes its list in order.
    std::vector<uint32_t> ctr(p.n_counters, 0);
    std::vector<int32_t> ptr(p.n_ctas);
    for (int i = 0; i < p.n_ctas; ++i) ptr[i] = p.cta_base[i];
    bool progress = true;
    size_t done = 0;
    while (progress) {
        progress = false;
        for (int i = 0; i < p.n_ctas; ++i) {
            while (ptr[i] < p.cta_base[i + 1]) {
                const Instr &in = p.instrs[ptr[i]];
                if (in.wait_ctr != kNoCounter && ctr[in.wait_ctr] < in.wait_count) break;
                if (in.op == OP_LMHEAD) {
                    if (in.flags & F_LAST_LM) {
                        const uint32_t a = ++ctr[in.signal_ctr];
                        if (a > in.arrive_count) return fail("more arrivals than expected");
                    }
                } else if (in.signal_ctr != kNoCounter) {
                    ++ctr[in.signal_ctr];
                }
                ++ptr[i];
                ++done;
                progress = true;
            }
        }
    }
    if (done != p.instrs.size()) {
        for (int i = 0; i < p.n_ctas; ++i)
            if (ptr[i] < p.cta_base[i + 1]) {
                const Instr &in = p.instrs[ptr[i]];
                snprintf(buf, sizeof buf, "deadlock: CTA %d stuck at instruction %d (op %d layer %d) waiting on counter %d (%u of %u)",
                         i, ptr[i], in.op, in.layer, in.wait_ctr, ctr[in.wait_ctr], in.wait_count);
                return fail(buf);
            }
    }
    for (size_t i = 0; i < p.instrs.size(); ++i) {
        const Instr &in = p.instrs[i];
        if (in.wait_ctr != kNoCounter && ctr[in.wait_ctr] != in.wait_count) {
            snprintf(buf, sizeof buf, "counter %d receives %u increments per step but instruction %zu expects %u",
                     in.wait_ctr, ctr[in.wait_ctr], i, in.wait_count);
            return fail(buf);
        }
        if (in.op == OP_LMHEAD && (in.flags & F_LAST_LM) && ctr[in.signal_ctr] != in.arrive_count) {
            snprintf(buf, sizeof buf, "arrival counter %d gets %u arrivals, expected %u", in.signal_ctr,
                     ctr[in.signal_ctr], in.arrive_count);
            return fail(buf);
        }
    }
    return MK_OK;
}

// A randomised schedule that keeps every dependency: for each phase, the
// groups of instructions the CTAs hold are dealt out to the CTAs in a random
// order, and each group is shuffled.  A CTA's list stays in phase order, so
// the schedule stays deadlock-free; each instruction computes the same values
// wherever it runs (a GEMV tile is one warp's fixed-order dot products, the
// K ranges of the down projection are added in a fixed order, and the argmax
// keys are order-free), so the results must be bit-identical.  A dependency
// the plan forgot to express -- a consumer that reads data its wait does not
// cover -- would show up here as a different result or a timeout.  The LM
// head's "last instruction of the CTA" flag moves with the shuffle.
mk_status shuffle_plan(Plan &p, uint64_t seed, std::string &err) {
    uint64_t st = seed * 0x9E3779B97F4A7C15ull + 0x632BE59BD9B4E019ull;
    auto next = [&]() {  // splitmix64
        uint64_t z = (st += 0x9E3779B97F4A7C15ull);
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    };
    auto shuffle = [&](auto &v) {
        for (size_t i = v.size(); i > 1; --i) std::swap(v[i - 1], v[next() % i]);
    };
    const int n = p.n_ctas, np = p.n_phases;
    std::vector<std::vector<std::vector<Instr>>> per(n, std::vector<std::vector<Instr>>(np));
    for (int ph = 0; ph < np; ++ph)
        for (int i = 0; i < n; ++i)
            for (int32_t k = p.phase_begin[(size_t)ph * n + i]; k < p.phase_begin[(size_t)(ph + 1) * n + i]; ++k)
                per[i][ph].push_back(p.instrs[k]);
    std::vector<std::vector<std::vector<Instr>>> out(n, std::vector<std::vector<Instr>>(np));
    std::vector<int> to(n);
    for (int ph = 0; ph < np; ++ph) {
        for (int i = 0; i < n; ++i) to[i] = i;
        shuffle(to);
        for (int i = 0; i < n; ++i) {
            out[to[i]][ph] = per[i][ph];
            shuffle(out[to[i]][ph]);
        }
    }
    const int lm = np - 1;
    for (int i = 0; i < n; ++i) {
        for (auto &in : out[i][lm]) in.flags &= (uint8_t)~F_LAST_LM;
        if (!out[i][lm].empty()) out[i][lm].back().flags |= F_LAST_LM;
    }
    p.instrs.clear();
    for (int i = 0; i < n; ++i) {
        p.cta_base[i] = (int32_t)p.instrs.size();
        for (int ph = 0; ph < np; ++ph) {
            p.phase_begin[(size_t)ph * n + i] = (int32_t)p.instrs.size();
            for (auto &in : out[i][ph]) p.instrs.push_back(in);
        }
        p.phase_begin[(size_t)np * n + i] = (int32_t)p.instrs.size();
    }
    p.cta_base[n] = (int32_t)p.instrs.size();
    return validate_plan(p, err);
}

}  // namespace mk

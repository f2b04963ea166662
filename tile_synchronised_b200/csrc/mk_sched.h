// mk_sched.h -- host-side planner of the decode megakernel: tile shapes,
// workspace layout, counters and the per-CTA instruction lists.
#pragma once
#include <stddef.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"

namespace mk {

struct Plan {
    mk_config cfg{};
    int n_ctas = 0;
    int B = 0;
    int bs = 0;              // batch rows per GEMV instruction (column-tiled)
    int gu_bs = 0;           // batch rows per gate/up instruction (row-tiled form may use fewer)
    int swiglu_variant = MK_SWIGLU_COL;
    int chunks = 0;          // split-KV chunks per (sequence, KV head)
    int stages = 0;          // ring slots
    int act_bytes = 0;       // shared-memory activation region
    int down_ksplit = 1;     // K ranges of the down projection (each writes its own partial output)
    int down_per = 1;        // K blocks per down-projection range
    std::vector<int> token_phases;  // phases that read the tokens or write the step's outputs
    int qkv_rows = 0, i_pad = 0;
    PackedMat qkv{}, o{}, gu{}, down{}, lm{};

    // workspace layout (byte offsets)
    size_t off_state = 0, off_counters = 0, off_instrs = 0, off_ranges = 0, off_layers = 0, off_rope = 0;
    size_t off_x = 0, off_xe = 0, off_dpart = 0, off_qkv = 0, off_attn = 0, off_act_a = 0, off_partials = 0, off_lm_best = 0;
    size_t off_next_scratch = 0, off_weights = 0, layer_weight_bytes = 0, off_lm = 0, off_norms = 0;
    // tensor-core prefill: possible when every packed layer matrix is one K
    // block (then a plain row-major [rows, kc] matrix); its scratch region
    bool prefill_tc = false;
    size_t off_prefill = 0, prefill_bytes = 0;
    size_t workspace_bytes = 0, kv_bytes = 0;

    // schedule
    int n_counters = 0;
    int n_phases = 0;
    std::vector<Instr> instrs;           // CTA-major, phase order within a CTA
    std::vector<int32_t> cta_base;       // [n_ctas + 1]
    std::vector<int32_t> phase_begin;    // [(n_phases + 1) * n_ctas], absolute instruction index
    std::vector<uint32_t> counter_count; // increments each counter receives per step (0 = arrival counter)
};

// Bytes of the tensor-core prefill's scratch (mk_tcdec.cu).
size_t prefill_scratch_bytes(int H, int nq, int d, int kmax, int mmax);
// Build a plan; returns MK_OK or an error code with a reason in `err`.
mk_status build_plan(const mk_config &cfg, int n_ctas, int swiglu_variant, Plan &plan, std::string &err);
// Simulate the schedule on the host; MK_OK or MK_ERR_STATE with a reason.
mk_status validate_plan(const Plan &plan, std::string &err);
// Reorder the schedule without changing what any instruction computes (a
// test of the dependency edges); then validate it.
mk_status shuffle_plan(Plan &plan, uint64_t seed, std::string &err);

// Tile-ready counters, six per layer, then the LM-head arrival counter.
constexpr int kCountersPerLayer = 6;
inline int counter_qkv(int l) { return kCountersPerLayer * l + 0; }
inline int counter_att(int l) { return kCountersPerLayer * l + 1; }
inline int counter_acomb(int l) { return kCountersPerLayer * l + 2; }
inline int counter_o(int l) { return kCountersPerLayer * l + 3; }
inline int counter_gu(int l) { return kCountersPerLayer * l + 4; }
inline int counter_down(int l) { return kCountersPerLayer * l + 5; }

}  // namespace mk

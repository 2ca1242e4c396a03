// mk_plan.h -- host-side schedule planning (no CUDA dependency).
#pragma once
#include <cstdint>
#include <vector>

#include "mk_internal.h"

namespace mk {

struct Planned {
    int n_sm = 0;
    int max_instr = 0;
    int kv_splits = 1;
    int n_lm = 0;                  // LM-head instructions (partial argmax slots)
    bool fused_ffn = true;         // one OP_FFN / OP_MOE_FFN per layer instead of up/gate + down
    int nb = 1;                    // sequences per step (batched decode)
    int merge_once = 0;            // W_MERGE on every ATTN and OPROJ instruction
    int ffn_gate = 0;              // W_GATE on every dense fused FFN instruction
    std::vector<int32_t> words;    // [n_sm][max_instr][W_NWORDS]
    std::vector<int32_t> n_instr;  // [n_sm]
    std::vector<uint32_t> ctr_inc; // per-step increment of every counter
};

int check_config(const mk_config& c);
int check_options(const mk_config& c, const mk_options& o);
void fill_defaults(const mk_config& c, mk_options* o);
int default_kv_splits(const mk_config& c, int n_sm, int nb = 1);
// Largest options.batch the kernels support for this shape (1: no batched decode).
int max_batch(const mk_config& c);
// Whether the schedule fuses each layer's FFN into one instruction per block:
// asked for (split_ffn == 0), the up/gate rows need no column parts, and one
// transposed down-projection row (hidden bf16 values) fits a ring stage.
bool ffn_fused(const mk_config& c, const mk_options& o);
int plan_schedule(const mk_config& c, const mk_options& o, int n_sm, Planned* out);
int validate(const mk_config& c, const Planned& p);
int simulate(const int32_t* words, int n_sm, int max_instr, const int32_t* n_instr, const uint32_t* ctr_inc,
             int nctr, int steps, uint64_t seed, long long* executed);

}  // namespace mk

// mk_internal.h -- instruction format, counter layout and the device parameter
// block shared by the host scheduler, the persistent kernel and the baseline.
#pragma once
#include <stddef.h>
#include <stdint.h>

#include <vector_types.h>
#include <cuda.h>  // CUtensorMap (the KV-cache tensor maps travel in the kernel parameters)

#include "../../include/mk.h"

#if defined(__CUDACC__)
#define MK_HD __host__ __device__
#else
#define MK_HD
#endif

namespace mk {

// Opcodes: each op that would otherwise be its own kernel launch is an opcode
// dispatched inside the persistent interpreter (Kittens VM summary page,
// "Method").  The set is the batch-1
// Llama/Mixtral decode step (epic-kernel README, "3B model support", "Mixtral
// 8x7B MoE for batch-1 inference").
enum Opcode : int32_t {
    OP_NOP = 0,
    OP_RMS_QKV = 1,          // xn = rmsnorm(x) * w_attn; rows of [Wq; Wk; Wv] xn (raw, pre-RoPE)
    OP_ATTN = 2,             // RoPE + KV append + one split of GQA decode attention (partial o, m, l)
    OP_OPROJ_RES = 3,        // x[rows] = x[rows] + Wo[rows] attn   (layer 0: embed row + ...)
    OP_RMS_UPGATE_SILU = 4,  // h[rows] = silu(Wg[rows] xn) * (Wu[rows] xn), xn = rmsnorm(x) * w_ffn
    OP_DOWN_RES = 5,         // x[rows] += Wd[rows] h
    OP_LMHEAD_ARGMAX = 6,    // logits[rows] = Wlm[rows] rmsnorm(x) * w_final; last instruction reduces argmax
    OP_MOE_UPGATE = 7,       // router + top-k in prologue; h_slot[rows] for the selected expert of `slot`
    OP_MOE_DOWN2_RES = 8,    // x[rows] += sum_slot w_slot * Wd_{e_slot}[rows] h_slot  (all slots, one instr)
    OP_FFN = 9,              // fused FFN slice: h[rows] as OP_RMS_UPGATE_SILU, then x2 += Wd[:, rows] h[rows]
                             //   (streamed as rows of the transposed down-projection, added with atomics)
    OP_MOE_FFN = 10,         // the same for one routed expert slot, scaled by its router weight
    OP_COUNT = 11
};

// Instruction words (int32 each, MK_INSTR_WORDS per instruction).
enum Word : int {
    W_OP = 0,
    W_LAYER = 1,
    W_SUB = 2,        // QKV: 0 q / 1 k / 2 v; ATTN: kv head; MOE_UPGATE: expert slot
    W_BEGIN = 3,      // first row (GEMV) or split index (ATTN)
    W_END = 4,        // one past the last row (GEMV) or number of splits (ATTN)
    W_WAIT_CTR = 5,   // counter waited on before reading activations (-1: none)
    W_WAIT_INC = 6,   // its per-step increment (target = epoch * inc)
    W_SIGNAL_CTR = 7, // counter incremented once when the instruction's outputs are visible (-1: none)
    W_AUX_CTR = 8,    // ATTN: per-head-group arrival counter; LMHEAD: arrival counter
    W_AUX_INC = 9,    // its per-step increment
    W_SEQ = 10,       // LMHEAD: slot of this instruction's partial argmax; ATTN: sequence of the batch
    W_SPEC = 11,      // speculative expert prediction.  QKV: 1 = after it, this block predicts the layer's
                      //   experts (its last QKV instruction of the layer), 2 = the same and it publishes the
                      //   prediction; MOE_FFN: 1 = the block's loader streams the predicted expert's first
                      //   stages before the routing is known (the block predicted this layer).  0: none
    W_MERGE = 12,     // ATTN: 1 = the kv head's last split to arrive merges the S splits of its query heads
                      //   into DevParams.attn before it signals; OPROJ: 1 = the input is that merged
                      //   output.  0 (both): every O-projection block merges the splits itself
    W_GATE = 13,      // FFN (dense, fused): > 0 = the loader issues the slice's stages from this index on only
                      //   once the FFN's dependency is met (the earlier ones stream during the small ops
                      //   before it); 0: no gate
    W_NWORDS = MK_INSTR_WORDS
};

constexpr int kMaxRows = 1024;       // rows per GEMV instruction
constexpr int kRowSlots = 1024;      // rows x accumulator sets held in shared memory per instruction
constexpr int kMaxPartK = 8192;      // widest row part reduced in one phase (4 chunks of 8 per thread)
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;  // + one loader warp
constexpr int kMaxGroup = 4;         // query heads per kv head
constexpr int kMaxHeadDim = 128;
constexpr int kMaxTopK = 2;
constexpr int kMaxBatch = 8;         // sequences of one batched decode step
constexpr int kMiscBytes = 1024;     // shared-memory budget of the kernel's per-block bookkeeping
constexpr int kMaxMergeSlots = 2048;  // query heads x kv splits merged in the O-projection prologue
// Above this many bytes of split partials (n_q_heads x kv_splits x head_dim fp32), which every
// O-projection block would read from L2 to merge, one split per kv head merges them instead (W_MERGE).
constexpr long long kMergeOnceBytes = 96 * 1024;
constexpr int kDefaultL2HeadStart = 0;  // ring stages of an FFN / LM-head stream prefetched into L2 past the ring

// Counter ids: per layer [QKV, ATTN (one signal per split), OPROJ, FFN1, FFN2], then the LM head's
// arrival counter.
enum CtrSlot : int { C_QKV = 0, C_ATTN = 1, C_OPROJ = 2, C_FFN1 = 3, C_FFN2 = 4, kCountersPerLayer = 5 };
MK_HD inline int ctr_id(int layer, int slot) { return layer * kCountersPerLayer + slot; }
MK_HD inline int ctr_lm(int n_layers) { return n_layers * kCountersPerLayer; }
MK_HD inline int n_counters(int n_layers) { return n_layers * kCountersPerLayer + 1; }

// Trace record of one instruction (options.trace): globaltimer stamps in ns,
// zero where not reached.  Consumer side: reached, dependency satisfied,
// input vector ready, first stage full, main stages consumed, signalled.
// Loader side: first and last stage issued.  Then, for the instruction's
// first kTraceStages ring stages: consumer thread 0's full-barrier wait
// returned (T_SREADY + s), its share of the stage consumed (T_SDONE + s), and
// the loader's issue (T_SISSUE + s).
constexpr int kTraceStages = 8;
enum TraceStamp : int {
    T_START = 0, T_DEP, T_READY, T_FIRST, T_MAIN, T_END, T_LD_FIRST, T_LD_LAST,
    T_SREADY = 8, T_SDONE = T_SREADY + kTraceStages, T_SISSUE = T_SDONE + kTraceStages,
    kTraceWords = T_SISSUE + kTraceStages
};

// Weight pointer table: per layer kLayerFixed entries, then gate/up/down per expert.
// Slot wt_down_t holds the library's transposed copy [ffn][hidden] of w_down
// (null unless the fused FFN is used).
enum WSlot : int { WT_ATTN_NORM = 0, WT_Q, WT_K, WT_V, WT_O, WT_FFN_NORM, WT_ROUTER, kLayerFixed };
MK_HD inline int wt_stride(int n_experts) { return kLayerFixed + 4 * (n_experts > 0 ? n_experts : 1); }
MK_HD inline int wt_gate(int e) { return kLayerFixed + e; }
MK_HD inline int wt_up(int e, int n_experts) { return kLayerFixed + (n_experts > 0 ? n_experts : 1) + e; }
MK_HD inline int wt_down(int e, int n_experts) { return kLayerFixed + 2 * (n_experts > 0 ? n_experts : 1) + e; }
MK_HD inline int wt_down_t(int e, int n_experts) { return kLayerFixed + 3 * (n_experts > 0 ? n_experts : 1) + e; }

// Column parts of a row of width K, and the accumulator sets an op keeps per
// row (spans x expert slots x column parts); rows per instruction are capped at
// kRowSlots / sets so that every (set, row) has a slot per consumer warp.
MK_HD inline int kparts_of(int K) { return (K + kMaxPartK - 1) / kMaxPartK; }
// Accumulator slots (rows x sets x sequences) an instruction of `rows` rows keeps in shared
// memory.  A batched LM-head instruction goes through its rows in chunks (lm_chunk_rows), so
// only one chunk's slots count.
// (rps <= kRowSlots / nb: the stage plan caps a batched LM head's rows per stage.)
MK_HD inline int lm_chunk_rows(int nb, int rps) {
    const int c = kRowSlots / (nb > 0 ? nb : 1) / rps * rps;  // whole ring stages of rps rows
    return c > rps ? c : rps;
}

// Batched decode: the one-chunk kernel with 8 sequence slots runs its GEMVs on the tensor cores
// (stages of padded rows); the other batched kernels keep the CUDA-core form, which measured
// faster there (the tensor-core form's per-instruction prologues cost more than it saves).
MK_HD constexpr bool batch_on_tensor_cores(int J, int NB) { return J == 1 && NB == 8; }

MK_HD inline int row_slots(int op, int rows, int sets, int nb) {
    return op == OP_LMHEAD_ARGMAX && nb > 1 ? 0 : rows * sets * nb;
}

MK_HD inline int acc_sets(int op, int H, int qd, int F, int topk) {
    switch (op) {
        case OP_OPROJ_RES: return kparts_of(qd);
        case OP_RMS_UPGATE_SILU:
        case OP_MOE_UPGATE:
        case OP_FFN:
        case OP_MOE_FFN: return 2 * kparts_of(H);
        case OP_DOWN_RES: return kparts_of(F);
        case OP_MOE_DOWN2_RES: return (topk > 0 ? topk : 1) * kparts_of(F);
        default: return kparts_of(H);
    }
}

struct DevStatus {
    int code, sm, instr, opcode, counter;
    unsigned int observed, expected;
    int cuda_error;
    int stop;        // stop word: nonzero makes every block leave at its next wait
    int next_token;  // argmax of the last completed step
    int pad[6];
};

// Launch-once serving (mk_serve_*): mailbox in pinned, mapped host memory.
struct ServeBox {
    int32_t req_seq;    // host -> device: number of the request (1, 2, ...), written last
    int32_t token;      // < 0: the previous step's argmax
    int32_t pos;
    int32_t stop;       // 1: leave the grid instead of stepping
    int32_t resp_seq;   // device -> host: number of the last finished request, written last
    int32_t next_token;
    int32_t code;       // device status code after the step (MK_OK or MK_ERR_*)
    int32_t pad;
};
// The step a serving grid runs next, published in device memory by block 0.
struct ServeStep {
    int32_t token, pos, stop, pad;
};

// Rows of one attention ring stage: K and V of `rows` positions, 4 * d bytes
// per position, at most 256, whole boxes of kAttnBoxRows rows (the tensor
// maps' box height: a split loads only the boxes that hold its rows).
constexpr int kAttnBoxRows = 64;
MK_HD inline int attn_stage_rows(int stage_bytes, int d) {
    int r = stage_bytes / (4 * d);
    r = r >= kAttnBoxRows ? (r & ~(kAttnBoxRows - 1)) : (r & ~15);  // whole boxes, or whole 16-row tiles
    return r < 256 ? r : 256;
}
// Box height of the tensor maps (at most one stage).
MK_HD inline int attn_box_rows(int stage_bytes, int d) {
    const int r = attn_stage_rows(stage_bytes, d);
    return r < kAttnBoxRows ? r : kAttnBoxRows;
}

// Everything the kernels read that stays fixed for a handle (device memory).
struct DevParams {
    // 2-D tensor maps over the K and V caches, viewed as [n_layers * n_kv * max_seq][d] bf16
    // rows, boxes of 64 columns x attn_box_rows rows, 128-byte swizzle (the attention
    // stage's bank-conflict-free layout for ldmatrix)
    CUtensorMap kmap;
    CUtensorMap vmap;
    // model
    int L, H, nq, nkv, d, F, V, E, topk, max_seq;
    float eps;
    int kv_splits;
    // schedule
    const int32_t* instr;    // [n_sm][max_instr][W_NWORDS]
    const int32_t* n_instr;  // [n_sm]
    int max_instr;
    int n_ctr;
    uint32_t* counters;
    DevStatus* status;
    // weights (bf16 as raw uint16)
    const uint16_t* embed;
    const uint16_t* lm_head;
    const uint16_t* final_norm;
    const uint16_t* const* wt;  // [L][wt_stride]
    uint16_t* kcache;
    uint16_t* vcache;
    const float2* rope;      // [max_seq][d/2] (cos, sin)
    // batched decode: nb sequences per step; every activation below, the logits, the snapshots and
    // the KV caches hold nb per-sequence copies one after the other (strides in elements below)
    int nb;
    int row_pad;            // bytes between weight rows in a stage beyond the row (tensor-core batched kernel: 16)
    size_t kv_seq_stride;   // L * nkv * max_seq * d
    int32_t* next_tok;      // [kMaxBatch] each sequence's argmax of the last step
    // activations (fp32)
    float* x;          // [H] residual stream read by the FFN (written by O-proj)
    float* x2;         // [H] residual stream after the FFN (O-proj writes it too; the FFN adds into it)
    float* qkv;        // [(nq + 2 nkv) d]  raw projections, pre-RoPE
    float* attn;       // [nb][nq d] attention output, merged once per kv head (W_MERGE)
    uint32_t* attn_arrive;  // [nb][L][nkv] arrivals of the kv splits (W_MERGE), epoch x kv_splits after a step
    float* part_o;     // [nq][kv_splits][d]
    float* part_ml;    // [nq][kv_splits][2]
    float* hbuf;       // [max(topk,1)][F]
    float* logits;     // [V] (internal; a caller buffer overrides per step)
    float* lm_part;    // [n_lm][2] (value, index bits)
    float* snap;       // [(L+1)][H] or null
    int32_t* router_idx;  // [L][kMaxTopK]
    float* router_w;      // [L][kMaxTopK]
    int32_t* pred_idx;    // [L][kMaxTopK] predicted experts (spec_experts)
    unsigned long long* trace;  // [n_sm][max_instr][kTraceWords] or null
    // kernel knobs
    int ring_stages;
    int stage_bytes;
    int l2_prefetch;
    int l2_head_start;
    int prefetch_ahead;
    int prefetch_max_bytes;
    int spec_experts;  // MoE: speculative expert prediction (see mk_options)
    unsigned long long spin_limit_ns;
    // serving (only read when the launch's StepArgs.serve is set)
    ServeBox* serve_box;     // device view of the pinned host mailbox
    ServeStep* serve_step;   // [1]
    uint32_t* serve_ctr;     // number of requests published so far in this launch
    unsigned long long serve_idle_ns;  // block 0 leaves after this long without a request
};

// Per-launch arguments (passed by value).
struct StepArgs {
    int token;        // < 0: use *next_token from the previous step
    int pos;
    uint32_t epoch;   // 1-based step count since the last reset
    float* logits;    // output logits (device)
    int serve = 0;    // 1: launch-once serving; the step fields come from the mailbox, epoch is the
                      // base (request k, counted from 1, runs epoch + k)
    int seq = 0;      // serving: number of this step's request
    // batched decode (DevParams.nb > 1): token (< 0: the sequence's previous argmax) and position of
    // every sequence; sequence 0 is also in token / pos
    int btok[kMaxBatch] = {0, 0, 0, 0, 0, 0, 0, 0};
    int bpos[kMaxBatch] = {0, 0, 0, 0, 0, 0, 0, 0};
};

}  // namespace mk

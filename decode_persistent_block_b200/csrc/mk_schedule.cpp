// mk_schedule.cpp -- host scheduler: splits every op of one decode step into
// instructions, assigns them to per-SM queues, sets the dependency counters,
// validates the result and can execute it on the host under random
// interleavings.
//
// The pages list what makes a megakernel schedule hard: grid-wide waits must
// never deadlock, every SM must stay busy although the ops differ in shape,
// and the result must be checkable (Hyperkernel teardown, "What a megakernel
// buys").  Here:
//  - every SM queue is sorted by global op index and every wait targets a
//    counter signalled only by strictly earlier ops, so some instruction is
//    always runnable (checked by validate() and exercised by simulate());
//  - every GEMV op is split into one contiguous row range per SM of equal
//    bytes (+-1 row), so each op spans all SMs whatever its shape;
//  - attention is split along the sequence (split-KV) into kv_heads * splits
//    instructions so that attention, which on its own would occupy few SMs,
//    still covers ~all of them (epic-kernel README, "Speculative expert
//    prediction", which notes the idle SMs during attention).
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <random>
#include <vector>

#include "mk_internal.h"
#include "mk_plan.h"

namespace mk {

namespace {

using Instr = std::array<int32_t, W_NWORDS>;

Instr blank() {
    Instr w;
    w.fill(0);
    w[W_WAIT_CTR] = -1;
    w[W_SIGNAL_CTR] = -1;
    w[W_AUX_CTR] = -1;
    return w;
}

struct Segment {
    int sub;   // tensor / slot selector stored in W_SUB
    int rows;
};

// Split the rows of `segs` (e.g. the q, k and v row blocks) over n_sm blocks
// so that every block gets rows of ONE segment only: blocks are given to the
// segments in proportion to their rows (largest remainder, at least one each
// when there are enough blocks), then each segment's rows are split evenly
// over its blocks and cut at `cap` rows.  A block holding rows of two segments
// would run two instructions back to back and finish last, delaying every
// block that waits for the op.  With fewer blocks than segments the virtual
// concatenation is split instead.  Calls emit(sm, sub, begin, end).
// `weight` (optional, one entry per block, single-segment ops only) scales a
// block's share of the rows.
template <class F>
void split_rows(const std::vector<Segment>& segs, int n_sm, int cap, F emit,
                const std::vector<double>* weight = nullptr) {
    long long total = 0;
    for (auto& s : segs) total += s.rows;
    const int ns = (int)segs.size();
    std::vector<long long> cut(n_sm + 1);
    if (weight && ns == 1) {
        double sum = 0.0, acc = 0.0;
        for (int sm = 0; sm < n_sm; ++sm) sum += (*weight)[sm];
        for (int sm = 0; sm <= n_sm; ++sm) {
            cut[sm] = sm == n_sm ? total : std::min(total, (long long)std::llround(total * acc / sum));
            if (sm < n_sm) acc += (*weight)[sm];
        }
    } else {
        for (int sm = 0; sm <= n_sm; ++sm) cut[sm] = total * sm / n_sm;
    }
    if (n_sm < ns || ns == 1) {
        for (int sm = 0; sm < n_sm; ++sm) {
            long long a = cut[sm], b = cut[sm + 1];
            long long base = 0;
            for (auto& s : segs) {
                long long lo = std::max(a, base), hi = std::min(b, base + s.rows);
                for (long long r = lo; r < hi; r += cap) emit(sm, s.sub, (int)(r - base), (int)(std::min(hi, r + cap) - base));
                base += s.rows;
            }
        }
        return;
    }
    std::vector<int> blocks(ns, 1);
    int left = n_sm - ns;
    std::vector<std::pair<double, int>> rem;
    for (int i = 0; i < ns; ++i) {
        const double share = (double)segs[i].rows * n_sm / (double)total - 1.0;
        const int extra = std::max(0, std::min(left, (int)share));
        blocks[i] += extra;
        left -= extra;
        rem.push_back({share - extra, i});
    }
    std::sort(rem.begin(), rem.end(), [](auto& x, auto& y) { return x.first > y.first || (x.first == y.first && x.second < y.second); });
    for (int k = 0; left > 0; k = (k + 1) % ns, --left) blocks[rem[k].second]++;
    int sm = 0;
    for (int i = 0; i < ns; ++i) {
        const long long R = segs[i].rows;
        for (int k = 0; k < blocks[i]; ++k, ++sm) {
            const long long a = R * k / blocks[i], b = R * (k + 1) / blocks[i];
            for (long long r = a; r < b; r += cap) emit(sm, segs[i].sub, (int)r, (int)std::min(b, r + cap));
        }
    }
}

}  // namespace

// Splits per kv head: at most one split per SM per kv head, and few enough
// that the O-projection's prologue can merge every head's splits
// (kMaxMergeSlots).  Within that:
//  - head_dim 64 (tensor-core attention): the count that minimises a model of
//    one layer's attention plus merge time at the longest context,
//      t(S) = t_row * max_seq / S + t_split * S + t_trip * ceil(S / 8),
//    with t_row = 10 ns per cached row of a split, t_split = 0.3 us for each
//    split's partials that every O-projection block reads, and t_trip = 1 us
//    per merge round trip (8 splits each).  The constants come from per-op
//    device traces of the Llama-1B shape.  The model orders its measured split
//    sweep (4 to 16 splits at 1152 positions) almost exactly.
//  - head_dim 128 (CUDA-core attention, about 5x the per-row cost): about one
//    split per 128 positions.
int default_kv_splits(const mk_config& c, int n_sm, int nb) {
    // at most one split per block across the batch's sequences and kv heads
    const int per_sm = std::max(1, n_sm / std::max(1, c.n_kv_heads * std::max(1, nb)));
    const int by_merge = std::max(1, kMaxMergeSlots / std::max(1, c.n_q_heads));
    const int cap = std::min(per_sm, by_merge);
    if (c.head_dim != 64) return std::min(cap, std::max(1, (c.max_seq + 127) / 128));
    int best = 1;
    double best_t = 0;
    for (int s = 1; s <= cap; ++s) {
        const double t = 10.0 * c.max_seq / s + 300.0 * s + 1000.0 * ((s + 7) / 8);
        if (s == 1 || t < best_t) best = s, best_t = t;
    }
    return best;
}

int check_config(const mk_config& c) {
    if (c.n_layers < 0 || c.hidden <= 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 || c.head_dim <= 0 ||
        c.ffn <= 0 || c.vocab <= 0 || c.max_seq <= 0 || c.n_experts < 0)
        return MK_ERR_INVALID_ARG;
    if (!(c.rms_eps >= 0.f) || !(c.rope_theta > 0.f)) return MK_ERR_INVALID_ARG;
    if (c.head_dim != 64 && c.head_dim != 128) return MK_ERR_UNSUPPORTED;
    if (c.n_q_heads % c.n_kv_heads) return MK_ERR_UNSUPPORTED;
    {
        const int g = c.n_q_heads / c.n_kv_heads;  // query heads per kv head (attention kernel instances)
        if (g < 1 || g > 4) return MK_ERR_UNSUPPORTED;  // attention kernel instances
    }
    const int qd = c.n_q_heads * c.head_dim;
    for (int k : {c.hidden, c.ffn, qd}) {
        if (k % 8 || k > 16384) return MK_ERR_UNSUPPORTED;
        // rows wider than 8192 columns are reduced in equal column parts of whole 8-element chunks
        const int parts = (k + 8191) / 8192;
        if (k % (8 * parts)) return MK_ERR_UNSUPPORTED;
    }
    if (c.hidden > 8192) return MK_ERR_UNSUPPORTED;  // RMSNorm inputs are never split
    if (c.n_experts > 0 && (c.top_k < 1 || c.top_k > kMaxTopK || c.top_k > c.n_experts || c.n_experts > 64))
        return MK_ERR_UNSUPPORTED;
    return MK_OK;
}

void fill_defaults(const mk_config& c, mk_options* o) {
    // The ring's shape: 3 stages of 64 KB, or 2 stages of 96 KB for dense head_dim-128 models
    // (the two-chunk kernels: each block's slices of their 3072-wide rows are larger) and for
    // batched decode (each stage carries more work per byte).  Measured: 3-4% faster on the
    // Llama-3B shape, 1-5% on the Llama-1B shape at 2 to 8 sequences; slower at batch 1 on the
    // Llama-1B and Mixtral shapes.
    const bool big = c.n_experts == 0 && (c.head_dim == 128 || o->batch >= 2);
    if (o->ring_stages <= 0 && o->stage_bytes <= 0 && big) {
        o->ring_stages = 2;
        o->stage_bytes = 98304;
    }
    if (o->ring_stages <= 0) o->ring_stages = 3;
    if (o->stage_bytes <= 0) o->stage_bytes = 65536;
    if (o->rows_per_instr <= 0 || o->rows_per_instr > kMaxRows) o->rows_per_instr = kMaxRows;
    if (o->l2_prefetch < 0) o->l2_prefetch = 0;
    if (o->prefetch_ahead < 0) o->prefetch_ahead = 0;
    if (o->l2_head_start < 0) o->l2_head_start = kDefaultL2HeadStart;
    if (o->prefetch_max_bytes <= 0) o->prefetch_max_bytes = 1 << 20;
    if (o->attn_sm_ffn_permille <= 0) o->attn_sm_ffn_permille = 1000;
    if (o->spin_limit_ns == 0) o->spin_limit_ns = 2000000000ull;
    if (o->serve_idle_ns == 0) o->serve_idle_ns = 60000000000ull;
    if (o->batch == 0) o->batch = 1;
}

// Chunks of 8 elements per consumer thread for a GEMV over k columns (per column part).
static int chunks_per_thread(int k) {
    const int parts = (k + 8191) / 8192;
    return ((k / parts) / 8 + kConsumerThreads - 1) / kConsumerThreads;
}

int max_batch(const mk_config& c) {
    // the 8-sequence kernel's tensor-core GEMVs split every row into 8 warp ranges of whole
    // 16-column k-steps (rows a multiple of 128 columns)
    const int qd = c.n_q_heads * c.head_dim;
    if (c.n_experts != 0) return 1;
    const int jh = chunks_per_thread(c.hidden), jo = chunks_per_thread(qd);
    if (jh == 1 && jo == 1 && c.head_dim == 64) return c.hidden % 128 == 0 && qd % 128 == 0 ? kMaxBatch : kMaxBatch / 2;
    if (jh == 2 && jo == 2 && c.head_dim == 128) return kMaxBatch / 2;
    return 1;
}

int check_options(const mk_config& c, const mk_options& o) {
    if (o.stage_bytes % 1024 || o.stage_bytes < 4096 || o.ring_stages < 2 || o.ring_stages > 32)
        return MK_ERR_INVALID_ARG;
    // one GEMV stage holds at least one row of every span: up/gate pairs of
    // hidden-wide rows, and one ffn-wide (down) or heads*dim-wide (o) row.
    const long long sb = o.stage_bytes;
    auto part_bytes = [](long long k) { return 2LL * (k / ((k + 8191) / 8192)); };
    if (2LL * 2 * c.hidden > sb || part_bytes(c.ffn) > sb || part_bytes((long long)c.n_q_heads * c.head_dim) > sb)
        return MK_ERR_UNSUPPORTED;
    if (2LL * 2 * c.head_dim > sb) return MK_ERR_UNSUPPORTED;
    if (attn_stage_rows(o.stage_bytes, c.head_dim) < 16) return MK_ERR_UNSUPPORTED;  // 16-row attention tiles
    if (o.kv_splits < 0 || (long long)o.kv_splits * c.n_q_heads > kMaxMergeSlots) return MK_ERR_INVALID_ARG;
    if (o.attn_sm_ffn_permille < 0 || o.attn_sm_ffn_permille > 4000) return MK_ERR_INVALID_ARG;
    if (o.l2_head_start < 0 || o.l2_head_start > 64) return MK_ERR_INVALID_ARG;
    if (o.sm_speed) {
        if (o.n_sm_speed <= 0) return MK_ERR_INVALID_ARG;
        for (int i = 0; i < o.n_sm_speed; ++i)
            if (!(o.sm_speed[i] > 0.f) || !std::isfinite(o.sm_speed[i])) return MK_ERR_INVALID_ARG;
    }
    if (o.mode < MK_MODE_MEGAKERNEL || o.mode > MK_MODE_MULTI_KERNEL_GRAPH) return MK_ERR_INVALID_ARG;
    if (o.spec_experts < 0 || o.spec_experts > 2) return MK_ERR_INVALID_ARG;
    if (o.batch < 1 || o.batch > kMaxBatch) return MK_ERR_INVALID_ARG;
    if (o.attn_merge < 0 || o.attn_merge > 2) return MK_ERR_INVALID_ARG;
    if (o.attn_merge == 2 && o.batch > 1) return MK_ERR_UNSUPPORTED;
    if (o.ffn_early_stages < -1 || o.ffn_early_stages > 64) return MK_ERR_INVALID_ARG;
    if (o.batch > 1) {  // batched decode: the specialised dense kernels with the fused FFN only
        if (o.batch > max_batch(c) || o.mode != MK_MODE_MEGAKERNEL || !ffn_fused(c, o) || o.spec_experts ||
            o.general_kernel || o.l2_prefetch > 0 || o.prefetch_ahead > 0)
            return MK_ERR_UNSUPPORTED;
    }
    // ring + barriers + partial-sum slots + misc must fit the 227 KB per-block opt-in limit
    if ((long long)o.ring_stages * o.stage_bytes + 16LL * o.ring_stages + 128 + 4LL * kRowSlots * 8 + kMiscBytes > 232448)
        return MK_ERR_INVALID_ARG;
    return MK_OK;
}

bool ffn_fused(const mk_config& c, const mk_options& o_in) {
    mk_options o = o_in;
    fill_defaults(c, &o);
    return o.split_ffn == 0 && c.hidden <= kMaxPartK && 2LL * c.hidden <= (long long)o.stage_bytes;
}

int plan_schedule(const mk_config& c, const mk_options& o_in, int n_sm, Planned* out) {
    int rc = check_config(c);
    if (rc) return rc;
    if (n_sm <= 0) return MK_ERR_INVALID_ARG;
    mk_options o = o_in;
    fill_defaults(c, &o);
    if (o.sm_speed && o.n_sm_speed != n_sm) return MK_ERR_INVALID_ARG;
    // relative streaming speed of every block: the dense FFN and LM head rows follow it
    std::vector<double> speed(n_sm, 1.0);
    if (o.sm_speed)
        for (int i = 0; i < n_sm; ++i) speed[i] = o.sm_speed[i];
    const int L = c.n_layers, nkv = c.n_kv_heads, d = c.head_dim, H = c.hidden, F = c.ffn;
    const int S = o.kv_splits > 0 ? o.kv_splits : default_kv_splits(c, n_sm, o.batch);
    const int cap = o.rows_per_instr;
    const bool moe = c.n_experts > 0;
    const bool fused = ffn_fused(c, o);

    std::vector<std::vector<Instr>> q(n_sm);
    std::vector<uint32_t> inc(n_counters(L), 0);

    auto add = [&](int sm, Instr w) {
        q[sm].push_back(w);
        if (w[W_SIGNAL_CTR] >= 0) inc[w[W_SIGNAL_CTR]]++;
        if (w[W_AUX_CTR] >= 0) inc[w[W_AUX_CTR]]++;
    };
    const int qd = c.n_q_heads * d;
    const int nb = o.batch;  // every GEMV row keeps nb accumulator sets (one per sequence)
    // Merge the attention splits once per kv head (the last split to arrive) instead of in every
    // O-projection block, when the partials that each of those blocks would read from L2 are large.
    const int merge_once = o.attn_merge == 2 ||
                           (o.attn_merge == 0 && nb == 1 && 4LL * qd * S > kMergeOnceBytes);
    // The loader streams a dense fused FFN's first stage during the small ops before it and the rest
    // only once the FFN's dependency is met, so that the weight stream leaves HBM and L2 quiet for
    // those ops' latency chain.  Default: on for one-chunk models (hidden <= 2048) at batch 1 or 2
    // whose FFN slice spans at least 4 ring stages (measured faster there; slower for a 2-stage slice,
    // for hidden 3072 at batch 4 and for hidden 2048 at batch 8).
    int ffn_gate = 0;
    if (fused && !moe) {
        const long long slice = 3LL * F * H * 2 / n_sm;
        if (o.ffn_early_stages > 0) ffn_gate = o.ffn_early_stages;
        else if (o.ffn_early_stages == 0 && nb <= 2 && H <= 2048 && slice >= 4LL * o.stage_bytes) ffn_gate = 1;
    }
    auto op_cap = [&](int op) {
        const int need = row_slots(op, 1, acc_sets(op, H, qd, F, c.top_k), nb);  // slots per row
        return need > 0 ? std::min(cap, kRowSlots / need) : cap;
    };
    auto gemv_op = [&](int op, int layer, const std::vector<Segment>& segs, int wait, int signal,
                       const std::vector<double>* weight = nullptr) {
        split_rows(segs, n_sm, op_cap(op), [&](int sm, int sub, int b, int e) {
            Instr w = blank();
            w[W_OP] = op;
            w[W_LAYER] = layer;
            w[W_SUB] = sub;
            w[W_BEGIN] = b;
            w[W_END] = e;
            w[W_WAIT_CTR] = wait;
            w[W_SIGNAL_CTR] = signal;
            add(sm, w);
        }, weight);
    };

    for (int l = 0; l < L; ++l) {
        const int prev_down = l > 0 ? ctr_id(l - 1, C_FFN2) : -1;
        gemv_op(OP_RMS_QKV, l, {{0, c.n_q_heads * d}, {1, nkv * d}, {2, nkv * d}}, prev_down,
                ctr_id(l, C_QKV));
        // attention: sequence q, kv head g, split s -> instruction k = (q * nkv + g) * S + s, rotated per layer
        const int total = nb * nkv * S;
        std::vector<double> ffn_weight = speed;  // blocks with an attention split may take fewer FFN rows
        for (int k = 0; k < total; ++k) {
            Instr w = blank();
            w[W_OP] = OP_ATTN;
            w[W_LAYER] = l;
            w[W_SUB] = (k / S) % nkv;
            w[W_BEGIN] = k % S;
            w[W_END] = S;
            w[W_SEQ] = k / (S * nkv);
            w[W_WAIT_CTR] = ctr_id(l, C_QKV);
            w[W_SIGNAL_CTR] = ctr_id(l, C_ATTN);
            w[W_MERGE] = merge_once;
            int sm = (int)(((long long)k + (long long)l * total) % n_sm);
            add(sm, w);
            ffn_weight[sm] = speed[sm] * (o.attn_sm_ffn_permille / 1000.0);
        }
        gemv_op(OP_OPROJ_RES, l, {{0, H}}, ctr_id(l, C_ATTN), ctr_id(l, C_OPROJ));
        if (merge_once)
            for (auto& qs : q)
                for (auto& w : qs)
                    if (w[W_OP] == OP_OPROJ_RES && w[W_LAYER] == l) w[W_MERGE] = 1;
        std::vector<Segment> slots;
        for (int s = 0; s < (moe ? c.top_k : 1); ++s) slots.push_back({s, F});
        if (fused) {
            // one instruction per block: its up/gate rows, then the matching down-projection columns
            gemv_op(moe ? OP_MOE_FFN : OP_FFN, l, slots, ctr_id(l, C_OPROJ), ctr_id(l, C_FFN2), &ffn_weight);
            if (ffn_gate)
                for (auto& qs : q)
                    for (auto& w : qs)
                        if (w[W_OP] == OP_FFN && w[W_LAYER] == l) w[W_GATE] = ffn_gate;
        } else if (!moe) {
            gemv_op(OP_RMS_UPGATE_SILU, l, slots, ctr_id(l, C_OPROJ), ctr_id(l, C_FFN1));
            gemv_op(OP_DOWN_RES, l, {{0, H}}, ctr_id(l, C_FFN1), ctr_id(l, C_FFN2));
        } else {
            gemv_op(OP_MOE_UPGATE, l, slots, ctr_id(l, C_OPROJ), ctr_id(l, C_FFN1));
            gemv_op(OP_MOE_DOWN2_RES, l, {{0, H}}, ctr_id(l, C_FFN1), ctr_id(l, C_FFN2));
        }
    }
    // Speculative expert prediction: in every block that runs both a QKV instruction and a slice of
    // the fused MoE FFN of a layer, the last QKV instruction of the layer predicts the experts and
    // the FFN slices stream the predicted expert's first stages early; the first such block (lowest
    // index) publishes the layer's prediction.
    if (moe && fused && o.spec_experts > 0) {
        std::vector<int> publisher(L, -1);
        for (int sm = 0; sm < n_sm; ++sm) {
            auto& qs = q[sm];
            std::vector<int> last_qkv(L, -1);
            for (size_t i = 0; i < qs.size(); ++i)
                if (qs[i][W_OP] == OP_RMS_QKV) last_qkv[qs[i][W_LAYER]] = (int)i;
            for (size_t i = 0; i < qs.size(); ++i) {
                const int l = qs[i][W_LAYER];
                if (qs[i][W_OP] != OP_MOE_FFN || last_qkv[l] < 0) continue;
                qs[i][W_SPEC] = 1;
                if (qs[last_qkv[l]][W_SPEC] == 0) qs[last_qkv[l]][W_SPEC] = 1;
                if (publisher[l] < 0) {
                    publisher[l] = sm;
                    qs[last_qkv[l]][W_SPEC] = 2;
                }
            }
        }
    }
    // LM head + argmax: partial slots numbered in emission order
    {
        int seq = 0;
        const int wait = L > 0 ? ctr_id(L - 1, C_FFN2) : -1;
        split_rows({{0, c.vocab}}, n_sm, op_cap(OP_LMHEAD_ARGMAX), [&](int sm, int, int b, int e) {
            Instr w = blank();
            w[W_OP] = OP_LMHEAD_ARGMAX;
            w[W_LAYER] = L;
            w[W_BEGIN] = b;
            w[W_END] = e;
            w[W_WAIT_CTR] = wait;
            w[W_AUX_CTR] = ctr_lm(L);
            w[W_SEQ] = seq++;
            add(sm, w);
        }, o.sm_speed ? &speed : nullptr);
    }
    // fill wait increments and aux increments
    for (auto& qs : q)
        for (auto& w : qs) {
            w[W_WAIT_INC] = w[W_WAIT_CTR] >= 0 ? (int32_t)inc[w[W_WAIT_CTR]] : 0;
            w[W_AUX_INC] = w[W_AUX_CTR] >= 0 ? (int32_t)inc[w[W_AUX_CTR]] : 0;
        }

    int max_instr = 1;
    for (auto& qs : q) max_instr = std::max<int>(max_instr, (int)qs.size());
    out->n_sm = n_sm;
    out->max_instr = max_instr;
    out->kv_splits = S;
    out->n_lm = (int)inc[ctr_lm(L)];
    out->fused_ffn = fused;
    out->nb = nb;
    out->merge_once = merge_once;
    out->ffn_gate = ffn_gate;
    out->words.assign((size_t)n_sm * max_instr * W_NWORDS, 0);
    out->n_instr.assign(n_sm, 0);
    for (int sm = 0; sm < n_sm; ++sm) {
        out->n_instr[sm] = (int32_t)q[sm].size();
        for (size_t i = 0; i < q[sm].size(); ++i)
            std::memcpy(&out->words[((size_t)sm * max_instr + i) * W_NWORDS], q[sm][i].data(),
                        sizeof(int32_t) * W_NWORDS);
    }
    out->ctr_inc = inc;
    return validate(c, *out);
}

// Global op index of an instruction: 5 ops per layer, LM head last.
static int op_index(const int32_t* w) {
    int slot = 0;
    switch (w[W_OP]) {
        case OP_RMS_QKV: slot = 0; break;
        case OP_ATTN: slot = 1; break;
        case OP_OPROJ_RES: slot = 2; break;
        case OP_RMS_UPGATE_SILU:
        case OP_MOE_UPGATE:
        case OP_FFN:
        case OP_MOE_FFN: slot = 3; break;
        case OP_DOWN_RES:
        case OP_MOE_DOWN2_RES: slot = 4; break;
        case OP_LMHEAD_ARGMAX: slot = 0; break;
        default: return -1;
    }
    return w[W_LAYER] * 5 + slot;
}

// Op index of the op that signals counter `ctr` (LM arrival counter: n_layers*5).
static int producer_op(int ctr, int L) {
    if (ctr == ctr_lm(L)) return L * 5;
    const int l = ctr / kCountersPerLayer, slot = ctr % kCountersPerLayer;
    switch (slot) {
        case C_QKV: return l * 5 + 0;
        case C_ATTN: return l * 5 + 1;
        case C_OPROJ: return l * 5 + 2;
        case C_FFN1: return l * 5 + 3;
        case C_FFN2: return l * 5 + 4;
        default: return -1;
    }
}

int validate(const mk_config& c, const Planned& p) {
    const int L = c.n_layers, nkv = c.n_kv_heads, d = c.head_dim;
    const int nctr = n_counters(L);
    if ((int)p.ctr_inc.size() != nctr) return MK_ERR_SCHEDULE;
    const bool moe = c.n_experts > 0;
    // coverage bitmaps: per (layer, op, sub) rows covered exactly once
    std::vector<std::vector<uint8_t>> cov;
    auto cov_key = [&](int l, int op, int sub) { return ((size_t)l * OP_COUNT + op) * 4 + sub; };
    cov.resize((size_t)(L + 1) * OP_COUNT * 4);
    auto rows_of = [&](int op, int sub) -> int {
        switch (op) {
            case OP_RMS_QKV: return sub == 0 ? c.n_q_heads * d : nkv * d;
            case OP_OPROJ_RES: case OP_DOWN_RES: case OP_MOE_DOWN2_RES: return c.hidden;
            case OP_RMS_UPGATE_SILU: case OP_MOE_UPGATE: case OP_FFN: case OP_MOE_FFN: return c.ffn;
            case OP_LMHEAD_ARGMAX: return c.vocab;
        }
        return -1;
    };
    std::vector<uint32_t> signals(nctr, 0);
    const int nb = p.nb;
    if (nb < 1 || nb > kMaxBatch || (nb > 1 && (moe || !p.fused_ffn))) return MK_ERR_SCHEDULE;
    if (p.merge_once != 0 && (p.merge_once != 1 || nb > 1)) return MK_ERR_SCHEDULE;
    if (p.ffn_gate < 0 || p.ffn_gate > 64 || (p.ffn_gate && (moe || !p.fused_ffn))) return MK_ERR_SCHEDULE;
    std::vector<std::vector<uint8_t>> attn_seen((size_t)std::max(L, 1) * nb * nkv,
                                                std::vector<uint8_t>(p.kv_splits, 0));
    std::vector<uint8_t> lm_seq(std::max(p.n_lm, 1), 0);
    std::vector<int> spec_publishers(std::max(L, 1), 0), spec_predictors(std::max(L, 1), 0);
    for (int sm = 0; sm < p.n_sm; ++sm) {
        int last_op = -1;
        int predicted_layer = -1;  // layer predicted by this block's last QKV instruction with W_SPEC
        std::vector<uint8_t> had_moe_ug(std::max(L, 1), 0);
        if (p.n_instr[sm] < 0 || p.n_instr[sm] > p.max_instr) return MK_ERR_SCHEDULE;
        for (int i = 0; i < p.n_instr[sm]; ++i) {
            const int32_t* w = &p.words[((size_t)sm * p.max_instr + i) * W_NWORDS];
            const int op = w[W_OP], l = w[W_LAYER];
            if (op <= OP_NOP || op >= OP_COUNT) return MK_ERR_SCHEDULE;
            const bool moe_op = op == OP_MOE_UPGATE || op == OP_MOE_DOWN2_RES || op == OP_MOE_FFN;
            const bool ffn_op = moe_op || op == OP_RMS_UPGATE_SILU || op == OP_DOWN_RES || op == OP_FFN;
            if (ffn_op && moe != moe_op) return MK_ERR_SCHEDULE;
            if (ffn_op && p.fused_ffn != (op == OP_FFN || op == OP_MOE_FFN)) return MK_ERR_SCHEDULE;
            if (op == OP_LMHEAD_ARGMAX ? l != L : (l < 0 || l >= L)) return MK_ERR_SCHEDULE;
            const int oi = op_index(w);
            if (oi < last_op) return MK_ERR_SCHEDULE;  // queue sorted by global op order
            last_op = oi;
            // waits only on counters produced by strictly earlier ops, with the planned increment
            if (w[W_WAIT_CTR] >= 0) {
                if (w[W_WAIT_CTR] >= nctr) return MK_ERR_SCHEDULE;
                const int po = producer_op(w[W_WAIT_CTR], L);
                if (po < 0 || po >= oi) return MK_ERR_SCHEDULE;
                if ((uint32_t)w[W_WAIT_INC] != p.ctr_inc[w[W_WAIT_CTR]] || w[W_WAIT_INC] <= 0) return MK_ERR_SCHEDULE;
            } else if (!(op == OP_RMS_QKV && l == 0) && !(op == OP_LMHEAD_ARGMAX && L == 0)) {
                return MK_ERR_SCHEDULE;  // everything but the first op depends on something
            }
            if (w[W_SIGNAL_CTR] >= nctr || w[W_AUX_CTR] >= nctr) return MK_ERR_SCHEDULE;
            // the merge of the attention splits: once per kv head (ATTN and OPROJ agree) or in every block
            if (w[W_MERGE] != ((op == OP_ATTN || op == OP_OPROJ_RES) ? p.merge_once : 0)) return MK_ERR_SCHEDULE;
            if (w[W_GATE] != (op == OP_FFN ? p.ffn_gate : 0)) return MK_ERR_SCHEDULE;
            // speculative expert prediction: a predicting QKV instruction is the block's last QKV of
            // its layer, and an FFN slice streams predicted stages only after its block predicted
            if (w[W_SPEC] != 0) {
                const bool qkv = op == OP_RMS_QKV && (w[W_SPEC] == 1 || w[W_SPEC] == 2);
                const bool ffn = op == OP_MOE_FFN && w[W_SPEC] == 1;
                if (!(moe && p.fused_ffn) || !(qkv || ffn)) return MK_ERR_SCHEDULE;
                if (qkv) {
                    if (predicted_layer == l) return MK_ERR_SCHEDULE;  // one predicting QKV per layer
                    predicted_layer = l;
                    spec_predictors[l]++;
                    if (w[W_SPEC] == 2) spec_publishers[l]++;
                }
                if (ffn && predicted_layer != l) return MK_ERR_SCHEDULE;
            } else if (op == OP_RMS_QKV && predicted_layer == l) {
                return MK_ERR_SCHEDULE;  // a QKV instruction after the predicting one
            }
            if (w[W_AUX_CTR] >= 0 && (uint32_t)w[W_AUX_INC] != p.ctr_inc[w[W_AUX_CTR]]) return MK_ERR_SCHEDULE;
            if (op == OP_ATTN) {
                const int g = w[W_SUB], s = w[W_BEGIN], sq = w[W_SEQ];
                if (g < 0 || g >= nkv || s < 0 || s >= p.kv_splits || w[W_END] != p.kv_splits) return MK_ERR_SCHEDULE;
                if (sq < 0 || sq >= nb) return MK_ERR_SCHEDULE;
                if (w[W_AUX_CTR] != -1 || w[W_SIGNAL_CTR] != ctr_id(l, C_ATTN)) return MK_ERR_SCHEDULE;
                if (attn_seen[((size_t)l * nb + sq) * nkv + g][s]++) return MK_ERR_SCHEDULE;
                signals[w[W_SIGNAL_CTR]]++;
                continue;
            }
            if (op == OP_MOE_UPGATE) had_moe_ug[l] = 1;
            if (op == OP_MOE_DOWN2_RES && !had_moe_ug[l]) return MK_ERR_SCHEDULE;  // routing known on this SM
            const int sub = w[W_SUB];
            const int R = rows_of(op, op == OP_RMS_QKV ? sub : 0);
            if (op == OP_RMS_QKV && (sub < 0 || sub > 2)) return MK_ERR_SCHEDULE;
            if ((op == OP_MOE_UPGATE || op == OP_MOE_FFN) && (sub < 0 || sub >= c.top_k)) return MK_ERR_SCHEDULE;
            if (op != OP_RMS_QKV && op != OP_MOE_UPGATE && op != OP_MOE_FFN && sub != 0) return MK_ERR_SCHEDULE;
            const int b = w[W_BEGIN], e = w[W_END];
            const int sets = acc_sets(op, c.hidden, c.n_q_heads * d, c.ffn, c.top_k);
            if (b < 0 || e > R || b >= e || e - b > kMaxRows || row_slots(op, e - b, sets, nb) > kRowSlots)
                return MK_ERR_SCHEDULE;
            auto& hits = cov[cov_key(l, op, sub)];
            if (hits.empty()) hits.assign(R, 0);
            for (int r = b; r < e; ++r)
                if (hits[r]++) return MK_ERR_SCHEDULE;
            if (op == OP_LMHEAD_ARGMAX) {
                if (w[W_AUX_CTR] != ctr_lm(L) || w[W_SEQ] < 0 || w[W_SEQ] >= p.n_lm || lm_seq[w[W_SEQ]]++)
                    return MK_ERR_SCHEDULE;
                signals[w[W_AUX_CTR]]++;
            } else {
                if (w[W_SIGNAL_CTR] < 0) return MK_ERR_SCHEDULE;
                signals[w[W_SIGNAL_CTR]]++;
            }
        }
    }
    // every op fully covered
    for (int l = 0; l <= L; ++l)
        for (int op = 1; op < OP_COUNT; ++op)
            for (int sub = 0; sub < 4; ++sub) {
                auto& hits = cov[cov_key(l, op, sub)];
                for (auto h : hits)
                    if (h != 1) return MK_ERR_SCHEDULE;
            }
    for (int l = 0; l < L; ++l) {
        for (int g = 0; g < nb * nkv; ++g)
            for (int s = 0; s < p.kv_splits; ++s)
                if (attn_seen[(size_t)l * nb * nkv + g][s] != 1) return MK_ERR_SCHEDULE;
        const std::vector<int> need = p.fused_ffn
            ? std::vector<int>{OP_RMS_QKV, OP_OPROJ_RES, moe ? OP_MOE_FFN : OP_FFN}
            : std::vector<int>{OP_RMS_QKV, OP_OPROJ_RES, moe ? OP_MOE_UPGATE : OP_RMS_UPGATE_SILU,
                               moe ? OP_MOE_DOWN2_RES : OP_DOWN_RES};
        for (int op : need)
            if (cov[cov_key(l, op, 0)].empty()) return MK_ERR_SCHEDULE;
        if (moe)  // every routed slot's rows are covered
            for (int sl = 1; sl < c.top_k; ++sl)
                if (cov[cov_key(l, p.fused_ffn ? OP_MOE_FFN : OP_MOE_UPGATE, sl)].empty()) return MK_ERR_SCHEDULE;
    }
    if (cov[cov_key(L, OP_LMHEAD_ARGMAX, 0)].empty()) return MK_ERR_SCHEDULE;
    for (int l = 0; l < L; ++l)  // a predicted layer has exactly one publisher
        if (spec_publishers[l] != (spec_predictors[l] > 0 ? 1 : 0)) return MK_ERR_SCHEDULE;
    for (int i = 0; i < nctr; ++i)
        if (signals[i] != p.ctr_inc[i]) return MK_ERR_SCHEDULE;
    return MK_OK;
}

int simulate(const int32_t* words, int n_sm, int max_instr, const int32_t* n_instr, const uint32_t* ctr_inc,
             int nctr, int steps, uint64_t seed, long long* executed) {
    std::vector<uint64_t> ctr(nctr, 0);
    std::mt19937_64 rng(seed);
    long long done = 0;
    for (int e = 1; e <= steps; ++e) {
        std::vector<int> pc(n_sm, 0);
        long long remaining = 0;
        for (int sm = 0; sm < n_sm; ++sm) remaining += n_instr[sm];
        std::vector<int> ready;
        while (remaining > 0) {
            ready.clear();
            for (int sm = 0; sm < n_sm; ++sm) {
                if (pc[sm] >= n_instr[sm]) continue;
                const int32_t* w = words + ((size_t)sm * max_instr + pc[sm]) * W_NWORDS;
                const int wc = w[W_WAIT_CTR];
                if (wc < 0 || ctr[wc] >= (uint64_t)e * (uint32_t)w[W_WAIT_INC]) ready.push_back(sm);
            }
            if (ready.empty()) {
                if (executed) *executed = done;
                return MK_ERR_SCHEDULE;  // deadlock
            }
            const int sm = ready[rng() % ready.size()];
            const int32_t* w = words + ((size_t)sm * max_instr + pc[sm]) * W_NWORDS;
            if (w[W_AUX_CTR] >= 0) ctr[w[W_AUX_CTR]]++;
            if (w[W_SIGNAL_CTR] >= 0) ctr[w[W_SIGNAL_CTR]]++;
            pc[sm]++;
            remaining--;
            done++;
        }
    }
    if (executed) *executed = done;
    for (int i = 0; i < nctr; ++i)
        if (ctr[i] != (uint64_t)steps * ctr_inc[i]) return MK_ERR_SCHEDULE;
    return MK_OK;
}

}  // namespace mk

extern "C" int mk_plan(const mk_config* cfg, const mk_options* opt, int n_sm, int32_t* buf, size_t cap,
                       int* max_instr, int32_t* n_instr, uint32_t* ctr_inc, size_t ctr_cap, int* n_ctr) {
    if (!cfg || n_sm <= 0) return MK_ERR_INVALID_ARG;
    mk_options o;
    if (opt) o = *opt; else mk_default_options(&o);
    mk::fill_defaults(*cfg, &o);
    int rc = mk::check_config(*cfg);
    if (rc) return rc;
    rc = mk::check_options(*cfg, o);
    if (rc) return rc;
    mk::Planned p;
    rc = mk::plan_schedule(*cfg, o, n_sm, &p);
    if (rc) return rc;
    if (max_instr) *max_instr = p.max_instr;
    if (n_ctr) *n_ctr = (int)p.ctr_inc.size();
    if (!buf || cap < p.words.size() || !n_instr || (ctr_inc && ctr_cap < p.ctr_inc.size())) return MK_ERR_CAPACITY;
    std::memcpy(buf, p.words.data(), p.words.size() * sizeof(int32_t));
    std::memcpy(n_instr, p.n_instr.data(), sizeof(int32_t) * n_sm);
    if (ctr_inc) std::memcpy(ctr_inc, p.ctr_inc.data(), p.ctr_inc.size() * sizeof(uint32_t));
    return MK_OK;
}

extern "C" int mk_simulate(const int32_t* buf, int n_sm, int max_instr, const int32_t* n_instr,
                           const uint32_t* ctr_inc, int n_counters, int steps, uint64_t seed, long long* executed) {
    if (!buf || !n_instr || !ctr_inc || n_sm <= 0 || max_instr <= 0 || n_counters <= 0 || steps < 0)
        return MK_ERR_INVALID_ARG;
    // reject out-of-range counter ids before touching them
    for (int sm = 0; sm < n_sm; ++sm) {
        if (n_instr[sm] < 0 || n_instr[sm] > max_instr) return MK_ERR_INVALID_ARG;
        for (int i = 0; i < n_instr[sm]; ++i) {
            const int32_t* w = buf + ((size_t)sm * max_instr + i) * mk::W_NWORDS;
            for (int k : {mk::W_WAIT_CTR, mk::W_SIGNAL_CTR, mk::W_AUX_CTR})
                if (w[k] >= n_counters || w[k] < -1) return MK_ERR_INVALID_ARG;
        }
    }
    return mk::simulate(buf, n_sm, max_instr, n_instr, ctr_inc, n_counters, steps, seed, executed);
}

// mk_megakernel.cu -- the persistent batch-1 decode kernel for sm_100a.
//
// One block per SM, launched cooperatively so that every block is resident;
// each block interprets its queue of the host-built instruction tensor and
// never returns to the host inside a step.  This is the megakernel shape the
// pages describe: one resident kernel that owns every SM and learns its work
// from a tensor read at run time, with the blocks synchronising among
// themselves on the device instead of through kernel boundaries (Kittens VM
// summary page, "Method"; Hyperkernel teardown, "What a megakernel buys").
//
// Block = 8 consumer warps + 1 loader warp (warp-specialised roles: epic-kernel
// README, "Fence removal and barrier reduction"):
//  * the loader (one elected lane) walks the block's queue and streams every
//    instruction's bf16 weight rows (or KV-cache rows) into a ring of
//    shared-memory stages with TMA bulk copies completed on mbarriers.  Weight
//    loads do not depend on activations, so the loader runs ahead across the
//    consumers' dependency waits, overlapping the next op's weight traffic
//    with the current op's compute (Hyperkernel teardown, "What a megakernel
//    buys").  After each stage it keeps a configurable
//    number of bytes of the following stages, across instruction boundaries,
//    prefetched into L2 (epic-kernel README, "L2 prefetching overlapped with
//    prior instructions").
//  * the consumers wait on the instruction's global dependency counter (one
//    acquiring lane, bounded), build the fp32 input vector in registers, run
//    the fp32-accumulate dot products from the ring, reduce across the warp
//    with shuffles and across warps with shared-memory atomics, and in the
//    epilogue act as the storer: write outputs, then release-increment the
//    signal counter.
// Every wait is bounded by a spin limit; on expiry the block records where it
// gave up in the status block, sets the stop word (every other block leaves at
// its next wait), drains its in-flight copies and returns (Hyperkernel
// teardown, "Hardware fault detection and replanning": watchdog word, stop
// word, bounds flags).
#include <cuda_runtime.h>
#include <math_constants.h>

#include "mk_device.cuh"
#include "mk_internal.h"
#include "mk_kernels.h"

namespace mk {

// ---------------------------------------------------------------------------
// shared memory layout
// ---------------------------------------------------------------------------
constexpr int kScratchBytes = 4 * kRowSlots * kConsumerWarps;  // partial row sums; attention merge and router reuse it

__device__ void serve_respond(const DevParams& p, const StepArgs& a, int next_token);

// Key of one layer's routing in one step (steps share a launch when serving).
__device__ __forceinline__ int route_key(uint32_t epoch, int layer, int n_layers) {
    return (int)((epoch * (uint32_t)(n_layers + 1) + (uint32_t)layer) & 0x7FFFFFFFu);
}

struct Misc {
    float red[kConsumerWarps * 2];
    int redi[kConsumerWarps];
    int abort_flag;
    int router_layer;  // route_key(epoch, layer) of the routing in eidx/ew (-1: none)
    int eidx[kMaxTopK];
    float ew[kMaxTopK];
    int pred_layer;    // route_key(epoch, layer) of the predicted experts in pred_eidx (-1: none)
    int pred_eidx[kMaxTopK];
    int is_last;
    int ffn_go;        // route_key(epoch, layer) of the last dense FFN whose dependency the consumers passed
    int pad[2];
    // batched decode: every sequence's position and token of this step (token resolved: < 0 read
    // from the previous step's argmax)
    int bpos[kMaxBatch];
    int btok[kMaxBatch];
    float bred[kMaxBatch * kConsumerWarps];  // per-sequence, per-warp argmax partials
    int bredi[kMaxBatch * kConsumerWarps];
    // serving: the step block 0 published, as taken by this block's consumer thread 0
    int s_go, s_token, s_pos, s_seq;
    uint32_t s_epoch;
};

static_assert(sizeof(Misc) <= kMiscBytes, "per-block bookkeeping outgrew its shared-memory budget");

__host__ __device__ inline size_t smem_bars_off(int ns, int sb) { return (size_t)ns * sb; }
__host__ __device__ inline size_t smem_scratch_off(int ns, int sb) {
    return (smem_bars_off(ns, sb) + 16 * (size_t)ns + 127) & ~(size_t)127;
}
__host__ __device__ inline size_t smem_misc_off(int ns, int sb) { return smem_scratch_off(ns, sb) + kScratchBytes; }
size_t megakernel_smem_bytes(int ns, int sb) { return smem_misc_off(ns, sb) + sizeof(Misc); }

__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Per-stage trace stamp (stage index s of the instruction; only the first kTraceStages are kept).
__device__ __forceinline__ void stage_stamp(unsigned long long* tr, int base, int s) {
    if (tr && s < kTraceStages) tr[base + s] = globaltimer_ns();
}

__device__ __forceinline__ int vload(const int* p) { return *(volatile const int*)p; }
__device__ __forceinline__ void vstore(int* p, int v) { *(volatile int*)p = v; }

// ---------------------------------------------------------------------------
// bounded waits
// ---------------------------------------------------------------------------
// The stop word and the block's abort flag are only polled once a wait has
// lasted kStopPollNs: a global load inside every spin iteration would put an
// L2 round trip between a barrier completing and the waiter noticing it.
constexpr uint64_t kStopPollNs = 20000;

__device__ bool wait_counter(const DevParams& p, Misc& m, int ctr, uint32_t target, int ii, int op) {
    const uint32_t* addr = p.counters + ctr;
    uint32_t v = ld_acquire_u32(addr);
    if ((int32_t)(v - target) >= 0) return true;
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + kStopPollNs;
    for (;;) {
        v = ld_acquire_u32(addr);
        if ((int32_t)(v - target) >= 0) return true;
        const uint64_t now = globaltimer_ns();
        if (now >= next) {
            if (ld_relaxed_s32(&p.status->stop) || vload(&m.abort_flag)) return false;
            if (now - t0 > p.spin_limit_ns) {
                record_error(p.status, MK_ERR_TIMEOUT, blockIdx.x, ii, op, ctr, v, target);
                return false;
            }
            next = now + kStopPollNs;
        }
    }
}

constexpr uint32_t kSuspendHintNs = 20000;

__device__ bool wait_mbar(uint64_t* bar, uint32_t parity, const DevParams& p, Misc& m, int ii, int op) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + kStopPollNs;
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, kSuspendHintNs)) return true;
        const uint64_t now = globaltimer_ns();
        if (now >= next) {
            if (ld_relaxed_s32(&p.status->stop) || vload(&m.abort_flag)) return false;
            if (now - t0 > p.spin_limit_ns) {
                record_error(p.status, MK_ERR_TIMEOUT, blockIdx.x, ii, op, -1, parity, 0);
                return false;
            }
            next = now + kStopPollNs;
        }
    }
}

// Warp-uniform wait for a full ring stage: lane 0 waits (bounded), the result
// is broadcast, then every lane takes its own acquire of the completed phase.
__device__ bool warp_wait_full(uint64_t* bar, uint32_t parity, const DevParams& p, Misc& m, int ii, int op) {
    const int lane = threadIdx.x & 31;
    int ok = 1;
    if (lane == 0) ok = wait_mbar(bar, parity, p, m, ii, op) ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (ok) {
        for (int k = 0; k < 64 && !mbar_try_wait(bar, parity); ++k) {
        }
    }
    return ok != 0;
}

// ---------------------------------------------------------------------------
// instruction checks and the stage plan shared by loader and consumers
// ---------------------------------------------------------------------------
__device__ __forceinline__ int op_rows(const DevParams& p, int op, int sub) {
    switch (op) {
        case OP_RMS_QKV: return sub == 0 ? p.nq * p.d : p.nkv * p.d;
        case OP_OPROJ_RES:
        case OP_DOWN_RES:
        case OP_MOE_DOWN2_RES: return p.H;
        case OP_RMS_UPGATE_SILU:
        case OP_MOE_UPGATE:
        case OP_FFN:
        case OP_MOE_FFN: return p.F;
        case OP_LMHEAD_ARGMAX: return p.V;
    }
    return 0;
}

// Bounds flags: every index an instruction carries is checked before use.
__device__ bool instr_ok(const DevParams& p, const int32_t* w) {
    const int op = w[W_OP], l = w[W_LAYER], sub = w[W_SUB], b = w[W_BEGIN], e = w[W_END];
    if (op <= OP_NOP || op >= OP_COUNT) return false;
    const bool moe_op = op == OP_MOE_UPGATE || op == OP_MOE_DOWN2_RES || op == OP_MOE_FFN;
    if ((p.E > 0) != moe_op && (moe_op || op == OP_RMS_UPGATE_SILU || op == OP_DOWN_RES || op == OP_FFN))
        return false;
    if (op == OP_LMHEAD_ARGMAX ? l != p.L : (l < 0 || l >= p.L)) return false;
    if (w[W_WAIT_CTR] < -1 || w[W_WAIT_CTR] >= p.n_ctr || w[W_SIGNAL_CTR] < -1 || w[W_SIGNAL_CTR] >= p.n_ctr ||
        w[W_AUX_CTR] < -1 || w[W_AUX_CTR] >= p.n_ctr)
        return false;
    if (w[W_WAIT_CTR] >= 0 && w[W_WAIT_INC] <= 0) return false;
    if (w[W_MERGE] != 0 && (w[W_MERGE] != 1 || (op != OP_ATTN && op != OP_OPROJ_RES) || p.nb > 1)) return false;
    if (w[W_GATE] < 0 || (w[W_GATE] != 0 && op != OP_FFN)) return false;
    if (op == OP_ATTN) {
        if (sub < 0 || sub >= p.nkv || e != p.kv_splits || b < 0 || b >= e) return false;
        if (w[W_SEQ] < 0 || w[W_SEQ] >= p.nb) return false;
        return w[W_SIGNAL_CTR] >= 0;
    }
    if (op == OP_RMS_QKV && (sub < 0 || sub > 2)) return false;
    if ((op == OP_MOE_UPGATE || op == OP_MOE_FFN) && (sub < 0 || sub >= p.topk)) return false;
    if (op == OP_FFN && sub != 0) return false;
    if ((op == OP_FFN || op == OP_MOE_FFN) && (p.H > kMaxPartK || 2 * p.H > p.stage_bytes)) return false;
    if (b < 0 || b >= e || e > op_rows(p, op, sub) || e - b > kMaxRows) return false;
    if (row_slots(op, e - b, acc_sets(op, p.H, p.nq * p.d, p.F, p.topk), p.nb) > kRowSlots) return false;
    if (op == OP_LMHEAD_ARGMAX) return w[W_AUX_CTR] >= 0 && w[W_AUX_INC] > 0 && w[W_SEQ] >= 0 && w[W_SEQ] < w[W_AUX_INC];
    return w[W_SIGNAL_CTR] >= 0;
}

// Column parts: rows wider than kMaxPartK columns are streamed and reduced in
// column parts (one phase per part) so that each thread's slice of the input
// vector stays within 4 chunks of 8 in registers.
static_assert(kMaxPartK == 8 * kConsumerThreads * 4, "a column part is 4 chunks of 8 per consumer thread");

struct Plan {
    int n_stages;   // stages of the whole instruction
    int nphase;     // slots * kparts (slots: top_k for the fused expert down-projection, else 1)
    int kparts;     // column parts per row
    int nspan;      // spans per stage (gate+up, K+V: 2)
    int rows;       // rows of the instruction
    int rps;        // rows per stage
    int spp;        // stages per phase
    uint32_t row_bytes;   // bytes of one row part in shared memory
    uint32_t pitch;       // bytes between consecutive rows in the stage (batched decode: row_bytes + 16,
                          // so that the 8 rows of an ldmatrix tile fall in different banks)
    uint32_t src_stride;  // bytes between consecutive rows in global memory
    const unsigned char* src[kMaxTopK][2];  // [slot][span]: row 0 of the instruction, column 0
    // fused FFN: after the main stages, `tail_spp` stages of the transposed
    // down-projection rows (one span, whole rows of tail_row_bytes)
    int main_stages;
    int tail_rps, tail_spp;
    uint32_t tail_row_bytes, tail_pitch;
    const unsigned char* tail_src;
    int tma_row0;  // attention: first cache row of the split in the tensor maps' row space (-1: not attention)
};

struct AttnRange {
    int jb, je, ncached;
    bool has_new;
};
__device__ __forceinline__ AttnRange attn_range(int pos, int split, int S) {
    const long long npos = (long long)pos + 1;
    AttnRange r;
    r.jb = (int)(npos * split / S);
    r.je = (int)(npos * (split + 1) / S);
    const int jce = r.je < pos ? r.je : pos;
    r.ncached = jce > r.jb ? jce - r.jb : 0;
    r.has_new = (r.je == npos);
    return r;
}

// Slot k of a fused MoE FFN instruction takes the k-th smallest of the top-k
// experts in e (the layer's output sums over the routed experts, so the order
// does not change it).  A prediction of the routed set in another order then
// still names every slot's expert.  Returns the index into e.
__device__ __forceinline__ int ffn_slot(const int* e, int topk, int sub) {
    return (topk == 2 && e[1] < e[0]) ? 1 - sub : sub;
}

// eidx: the routed (or predicted) experts of the instruction's layer (MoE ops only).
__device__ void make_plan(const DevParams& p, int pos, const int32_t* w, const int* eidx, Plan& pl) {
    const int op = w[W_OP], l = w[W_LAYER], sub = w[W_SUB], b = w[W_BEGIN], e = w[W_END];
    const uint16_t* const* wt = p.wt + (size_t)(l < p.L ? l : 0) * wt_stride(p.E);
    const uint32_t SB = (uint32_t)p.stage_bytes;
    int nslot = 1;
    pl.nspan = 1;
    pl.kparts = 1;
    pl.src[0][1] = pl.src[1][0] = pl.src[1][1] = nullptr;
    pl.tail_rps = pl.tail_spp = 0;
    pl.tail_row_bytes = pl.tail_pitch = 0;
    pl.tail_src = nullptr;
    pl.tma_row0 = -1;
    const uint16_t* tail = nullptr;  // transposed down-projection rows of a fused FFN
    int K = p.H;
    const uint16_t* s0 = nullptr;
    const uint16_t* s1 = nullptr;
    const uint16_t* s2 = nullptr;  // second slot's matrix (fused expert down-projection)
    switch (op) {
        case OP_ATTN: {
            // K and V rows of the split, as tensor-map boxes (row coordinate tma_row0 + stage row)
            const AttnRange r = attn_range(pos, b, e);
            pl.nphase = 1;
            pl.nspan = 2;
            pl.rows = r.ncached;
            pl.row_bytes = pl.src_stride = pl.pitch = (uint32_t)p.d * 2u;
            pl.rps = attn_stage_rows((int)SB, p.d);
            pl.spp = (pl.rows + pl.rps - 1) / pl.rps;
            pl.n_stages = pl.main_stages = pl.spp;
            // (batched decode: the sequence's cache follows the previous sequences' caches)
            pl.tma_row0 = (int)((((size_t)w[W_SEQ] * p.L + l) * p.nkv + sub) * (size_t)p.max_seq + (size_t)r.jb);
            pl.src[0][0] = (const unsigned char*)(p.kcache + (size_t)pl.tma_row0 * p.d);
            pl.src[0][1] = (const unsigned char*)(p.vcache + (size_t)pl.tma_row0 * p.d);
            return;
        }
        case OP_RMS_QKV: s0 = wt[WT_Q + sub]; break;
        case OP_OPROJ_RES: K = p.nq * p.d; s0 = wt[WT_O]; break;
        case OP_RMS_UPGATE_SILU: pl.nspan = 2; s0 = wt[wt_gate(0)]; s1 = wt[wt_up(0, p.E)]; break;
        case OP_DOWN_RES: K = p.F; s0 = wt[wt_down(0, p.E)]; break;
        case OP_LMHEAD_ARGMAX: s0 = p.lm_head; break;
        case OP_MOE_UPGATE:
            pl.nspan = 2;
            s0 = wt[wt_gate(eidx[sub])];
            s1 = wt[wt_up(eidx[sub], p.E)];
            break;
        case OP_MOE_DOWN2_RES:
            K = p.F;
            nslot = p.topk;
            s0 = wt[wt_down(eidx[0], p.E)];
            if (p.topk > 1) s2 = wt[wt_down(eidx[1], p.E)];
            break;
        case OP_FFN:
            pl.nspan = 2;
            s0 = wt[wt_gate(0)];
            s1 = wt[wt_up(0, p.E)];
            tail = wt[wt_down_t(0, p.E)];
            break;
        case OP_MOE_FFN: {
            const int x = eidx[ffn_slot(eidx, p.topk, sub)];
            pl.nspan = 2;
            s0 = wt[wt_gate(x)];
            s1 = wt[wt_up(x, p.E)];
            tail = wt[wt_down_t(x, p.E)];
            break;
        }
    }
    pl.kparts = kparts_of(K);
    pl.nphase = nslot * pl.kparts;
    pl.rows = e - b;
    pl.src_stride = (uint32_t)K * 2u;
    pl.row_bytes = pl.src_stride / (uint32_t)pl.kparts;
    const uint32_t pad = (uint32_t)p.row_pad;  // tensor-core batched kernel: padded rows
    pl.pitch = pl.row_bytes + pad;
    int rps = (int)(SB / ((uint32_t)pl.nspan * pl.pitch));
    // a batched LM head keeps every sequence's sums of a stage's rows at once (lm_chunk_rows)
    if (p.nb > 1 && op == OP_LMHEAD_ARGMAX && rps > kRowSlots / p.nb) rps = kRowSlots / p.nb;
    pl.rps = rps < pl.rows ? rps : pl.rows;
    pl.spp = (pl.rows + pl.rps - 1) / pl.rps;
    pl.n_stages = pl.main_stages = pl.spp * pl.nphase;
    if (tail) {
        pl.tail_row_bytes = (uint32_t)p.H * 2u;
        pl.tail_pitch = pl.tail_row_bytes + pad;
        const int trps = (int)(SB / pl.tail_pitch);
        pl.tail_rps = trps < pl.rows ? trps : pl.rows;
        pl.tail_spp = (pl.rows + pl.tail_rps - 1) / pl.tail_rps;
        pl.tail_src = (const unsigned char*)(tail + (size_t)b * p.H);
        pl.n_stages += pl.tail_spp;
    }
    pl.src[0][0] = (const unsigned char*)(s0 + (size_t)b * K);
    if (s1) pl.src[0][1] = (const unsigned char*)(s1 + (size_t)b * K);
    if (s2) pl.src[1][0] = (const unsigned char*)(s2 + (size_t)b * K);
}

// Pull this instruction's row of the weight-pointer table into L1 (one line
// per thread of the first warp), so that make_plan's loads hit.
__device__ __forceinline__ void prefetch_plan_l1(const DevParams& p, const int32_t* w) {
    const int l = w[W_LAYER];
    if (threadIdx.x >= 32 || l >= p.L) return;
    const int stride = wt_stride(p.E);
    const char* row = reinterpret_cast<const char*>(p.wt + (size_t)l * stride);
    const int bytes = stride * (int)sizeof(void*);
    const int lines = (bytes + 127) / 128 + 1;  // the row may start mid-line
    const int off = 128 * (int)threadIdx.x < bytes ? 128 * (int)threadIdx.x : bytes - 1;
    if ((int)threadIdx.x < lines) asm volatile("prefetch.global.L1 [%0];" ::"l"(row + off));
}

__device__ __forceinline__ bool needs_routing(int op) {
    return op == OP_MOE_UPGATE || op == OP_MOE_DOWN2_RES || op == OP_MOE_FFN;
}

// ---------------------------------------------------------------------------
// loader warp (one lane)
// ---------------------------------------------------------------------------
// TC: attention stages are tensor-map boxes (for attn_tc); otherwise contiguous
// K and V spans (for attn_cc).
template <bool TC, int NB = 1>
__device__ void issue_stage(const DevParams& p, const Plan& pl, int st, unsigned char* dst_stage, uint64_t* bar) {
    if (TC && pl.tma_row0 >= 0) {  // attention: K and V in boxes of attn_box_rows rows (past the split: masked)
        const int halves = p.d / 64, y = pl.tma_row0 + st * pl.rps;
        const int nr = (pl.rows - st * pl.rps) < pl.rps ? (pl.rows - st * pl.rps) : pl.rps;
        const int br = attn_box_rows(p.stage_bytes, p.d);  // divides pl.rps
        const int nb = (nr + br - 1) / br;
        const uint32_t half = (uint32_t)pl.rps * 128u, box = (uint32_t)br * 128u;
        mbar_arrive_expect_tx(bar, 2u * (uint32_t)halves * (uint32_t)nb * box);
        unsigned char* vdst = dst_stage + (size_t)pl.rps * p.d * 2;
        for (int h = 0; h < halves; ++h)
            for (int b = 0; b < nb; ++b) {
                tma_load_2d(dst_stage + (size_t)h * half + (size_t)b * box, &p.kmap, 64 * h, y + b * br, bar);
                tma_load_2d(vdst + (size_t)h * half + (size_t)b * box, &p.vmap, 64 * h, y + b * br, bar);
            }
        return;
    }
    // Weight rows are read once per step: they are loaded with the evict-first L2 policy, which
    // leaves L2 to what is reused across steps (the KV cache, whose rows up to the position are
    // read again by the next step, the activations and the counters).  K/V rows keep the normal
    // policy.
    const uint64_t pol = make_evict_first_policy();
    if (st >= pl.main_stages) {  // fused FFN: transposed down-projection rows
        const int r0 = (st - pl.main_stages) * pl.tail_rps;
        const int nr = (pl.rows - r0) < pl.tail_rps ? (pl.rows - r0) : pl.tail_rps;
        const uint32_t bytes = (uint32_t)nr * pl.tail_row_bytes;
        mbar_arrive_expect_tx(bar, bytes);
        if (NB > 1 && pl.tail_pitch != pl.tail_row_bytes) {  // padded rows
            for (int r = 0; r < nr; ++r)
                bulk_g2s_hint(dst_stage + (size_t)r * pl.tail_pitch, pl.tail_src + (size_t)(r0 + r) * pl.tail_row_bytes,
                              pl.tail_row_bytes, bar, pol);
        } else {
            bulk_g2s_hint(dst_stage, pl.tail_src + (size_t)r0 * pl.tail_row_bytes, bytes, bar, pol);
        }
        return;
    }
    const int ph = st / pl.spp, sst = st % pl.spp;
    const int slot = ph / pl.kparts, part = ph % pl.kparts;
    const int r0 = sst * pl.rps;
    const int nr = (pl.rows - r0) < pl.rps ? (pl.rows - r0) : pl.rps;
    const uint32_t bytes = (uint32_t)nr * pl.row_bytes;
    mbar_arrive_expect_tx(bar, bytes * (uint32_t)pl.nspan);
    for (int s = 0; s < pl.nspan; ++s) {
        const unsigned char* src = pl.src[slot][s] + (size_t)r0 * pl.src_stride + (size_t)part * pl.row_bytes;
        unsigned char* dst = dst_stage + (size_t)s * pl.rps * pl.pitch;
        const bool kv = pl.tma_row0 >= 0;  // K/V rows of an attention split (contiguous-copy path)
        if (NB > 1 && !kv && pl.pitch != pl.row_bytes) {  // tensor-core batched kernel: padded rows
            for (int r = 0; r < nr; ++r)
                bulk_g2s_hint(dst + (size_t)r * pl.pitch, src + (size_t)r * pl.src_stride, pl.row_bytes, bar, pol);
        } else if (pl.kparts == 1) {
            if (kv) bulk_g2s(dst, src, bytes, bar);
            else bulk_g2s_hint(dst, src, bytes, bar, pol);
        } else {
            for (int r = 0; r < nr; ++r)
                bulk_g2s_hint(dst + (size_t)r * pl.row_bytes, src + (size_t)r * pl.src_stride, pl.row_bytes, bar, pol);
        }
    }
}

__device__ void prefetch_stage(const Plan& pl, int st) {
    if (st >= pl.main_stages) {
        const int r0 = (st - pl.main_stages) * pl.tail_rps;
        const int nr = (pl.rows - r0) < pl.tail_rps ? (pl.rows - r0) : pl.tail_rps;
        prefetch_l2(pl.tail_src + (size_t)r0 * pl.tail_row_bytes, (uint32_t)nr * pl.tail_row_bytes);
        return;
    }
    const int ph = st / pl.spp, sst = st % pl.spp;
    const int slot = ph / pl.kparts, part = ph % pl.kparts;
    const int r0 = sst * pl.rps;
    const int nr = (pl.rows - r0) < pl.rps ? (pl.rows - r0) : pl.rps;
    for (int s = 0; s < pl.nspan; ++s) {
        const unsigned char* src = pl.src[slot][s] + (size_t)r0 * pl.src_stride + (size_t)part * pl.row_bytes;
        if (pl.kparts == 1) {
            prefetch_l2(src, (uint32_t)nr * pl.row_bytes);
        } else {
            for (int r = 0; r < nr; ++r) prefetch_l2(src + (size_t)r * pl.src_stride, pl.row_bytes);
        }
    }
}

// Loader: wait (bounded) until the consumers have set *field to key (a
// route_key of the routing or of the prediction); false on stop, abort or
// timeout (recorded).
__device__ bool wait_misc_key(const DevParams& p, Misc& m, const int* field, int key, int ii, int op) {
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + kStopPollNs;
    while (vload(field) != key) {
        const uint64_t now = globaltimer_ns();
        if (now >= next) {
            if (ld_relaxed_s32(&p.status->stop) || vload(&m.abort_flag)) return false;
            if (now - t0 > p.spin_limit_ns) {
                record_error(p.status, MK_ERR_TIMEOUT, blockIdx.x, ii, op, -1, 0, 0);
                return false;
            }
            next = now + kStopPollNs;
        }
    }
    return true;
}

// Loader side of the FFN stage gate: wait (bounded) until this block's
// consumers have passed the dense FFN's dependency and published its key.  The
// loader polls shared memory, with a short sleep, instead of the global
// counter: a second poller per block on the counter's line slowed the
// consumers' own dependency polls on the neighbouring counters.
__device__ bool wait_ffn_go(const DevParams& p, Misc& m, int key, int ii, int op) {
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + kStopPollNs;
    while (vload(&m.ffn_go) != key) {
        __nanosleep(64);
        const uint64_t now = globaltimer_ns();
        if (now >= next) {
            if (ld_relaxed_s32(&p.status->stop) || vload(&m.abort_flag)) return false;
            if (now - t0 > p.spin_limit_ns) {
                record_error(p.status, MK_ERR_TIMEOUT, blockIdx.x, ii, op, -1, 0, 0);
                return false;
            }
            next = now + kStopPollNs;
        }
    }
    return true;
}

// A fused MoE FFN slice's speculative stages hold the routed expert's rows:
// the predicted and the routed experts of its slot are the same (both known).
__device__ __forceinline__ bool spec_hit(const DevParams& p, const Misc& m, int sub) {
    int e[kMaxTopK], q[kMaxTopK];
    for (int k = 0; k < kMaxTopK; ++k) {
        e[k] = vload(&m.eidx[k]);
        q[k] = vload(&m.pred_eidx[k]);
    }
    return e[ffn_slot(e, p.topk, sub)] == q[ffn_slot(q, p.topk, sub)];
}

// Plan instruction i for the loader; for MoE ops wait (bounded) until the
// consumers have routed the layer, unless `block` is false.  MOE: the
// instantiation runs MoE schedules (dense ones carry no routing code).
template <bool MOE, int NB>
__device__ bool loader_plan(const DevParams& p, const StepArgs& a, const int32_t* w, Misc& m, Plan& pl, bool block,
                            int ii) {
    if (!instr_ok(p, w)) {
        pl.n_stages = 0;
        return true;
    }
    if (MOE && needs_routing(w[W_OP])) {
        const int key = route_key(a.epoch, w[W_LAYER], p.L);
        if (vload(&m.router_layer) != key) {
            if (!block) return false;
            if (!wait_misc_key(p, m, &m.router_layer, key, ii, w[W_OP])) return false;
        }
        __threadfence_block();
        int eidx[kMaxTopK];
        for (int k = 0; k < kMaxTopK; ++k) eidx[k] = vload(&m.eidx[k]);
        make_plan(p, a.pos, w, eidx, pl);
        return true;
    }
    make_plan(p, NB > 1 && w[W_OP] == OP_ATTN ? m.bpos[w[W_SEQ]] : a.pos, w, nullptr, pl);
    return true;
}

// PF: the L2 prefetch cursor (options.l2_prefetch) is compiled in.
// Ring position of the loader, kept across the steps of a serving launch.
struct LoaderRing {
    int slot = 0;
    uint32_t phase = 0;
    uint32_t used = 0, last_parity = 0;  // slots ever filled, parity of their last fill
};

// One step's queue; false if a wait gave up (the block is leaving).
template <bool PF, bool TC, bool MOE, int NB>
__device__ bool loader(const DevParams& p, const StepArgs& a, const int32_t* q, int n, unsigned char* ring,
                       uint64_t* full, uint64_t* empty, Misc& m, LoaderRing& lr) {
    const int NS = p.ring_stages;
    const uint32_t SB = (uint32_t)p.stage_bytes;
    const int pf_stages = PF && p.l2_prefetch > 0 ? (int)((uint32_t)p.l2_prefetch / SB) : 0;
    int& slot = lr.slot;
    uint32_t& phase = lr.phase;
    uint32_t& used = lr.used;
    uint32_t& last_parity = lr.last_parity;
    // L2 prefetch cursor: next (instruction, stage) to prefetch and its global stage index
    int pf_i = 0, pf_st = 0;
    long long pf_g = 0, g = 0;
    Plan pf_plan;
    pf_plan.n_stages = 0;
    bool pf_stalled = false;

    for (int i = 0; i < n; ++i) {
        const int32_t* w = q + (size_t)i * W_NWORDS;
        Plan pl;
        int st0 = 0;  // first stage of pl issued below
        if constexpr (MOE && !PF) {
            // Speculative expert prediction: the slice's first ring stages come from the expert that
            // this block predicted after its QKV instruction, issued before the routing is known.
            // Once it is: on a hit the stream goes on from there, on a miss it restarts with the
            // routed expert and the consumers drop the speculative stages.
            if (w[W_OP] == OP_MOE_FFN && w[W_SPEC] != 0 && p.spec_experts) {
                if (!wait_misc_key(p, m, &m.pred_layer, route_key(a.epoch, w[W_LAYER], p.L), i, w[W_OP])) break;
                __threadfence_block();
                int pe[kMaxTopK];
                for (int k = 0; k < kMaxTopK; ++k) pe[k] = vload(&m.pred_eidx[k]);
                Plan sp;
                make_plan(p, a.pos, w, pe, sp);
                const int ns = sp.n_stages < NS ? sp.n_stages : NS;
                bool sok = true;
                for (int st = 0; st < ns; ++st) {
                    if (!wait_mbar(&empty[slot], phase ^ 1u, p, m, i, w[W_OP])) {
                        sok = false;
                        break;
                    }
                    if (st == 0 && p.trace)  // stamped before the copy is issued: it cannot land earlier
                        p.trace[((size_t)blockIdx.x * p.max_instr + i) * kTraceWords + T_LD_FIRST] = globaltimer_ns();
                    issue_stage<TC, NB>(p, sp, st, ring + (size_t)slot * SB, &full[slot]);
                    used |= 1u << slot;
                    last_parity = (last_parity & ~(1u << slot)) | (phase << slot);
                    if (++slot == NS) {
                        slot = 0;
                        phase ^= 1u;
                    }
                }
                if (!sok) return false;
                if (!loader_plan<MOE, NB>(p, a, w, m, pl, true, i)) break;
                if (spec_hit(p, m, w[W_SUB])) st0 = ns;
            } else if (!loader_plan<MOE, NB>(p, a, w, m, pl, true, i)) {
                break;
            }
        } else {
            if (!loader_plan<MOE, NB>(p, a, w, m, pl, true, i)) break;
        }
        bool ok = true;
        unsigned long long* tr = p.trace ? p.trace + ((size_t)blockIdx.x * p.max_instr + i) * kTraceWords : nullptr;
        for (int st = st0; st < pl.n_stages; ++st, ++g) {
            // gated FFN slice: the stages from W_GATE on wait until the consumers pass the FFN's dependency
            if (st == w[W_GATE] && st > 0 && !wait_ffn_go(p, m, route_key(a.epoch, w[W_LAYER], p.L), i, w[W_OP])) {
                ok = false;
                break;
            }
            if (!wait_mbar(&empty[slot], phase ^ 1u, p, m, i, w[W_OP])) {
                ok = false;
                break;
            }
            // issue stamps are taken before the copy is issued, so a copy never lands before its stamp
            if (tr && st == 0) tr[T_LD_FIRST] = globaltimer_ns();
            stage_stamp(tr, T_SISSUE, st);
            if (tr && st == pl.n_stages - 1) tr[T_LD_LAST] = globaltimer_ns();
            issue_stage<TC, NB>(p, pl, st, ring + (size_t)slot * SB, &full[slot]);
            // Head start of a long stream: the loader reaches the first stage of the
            // dense FFN (or the LM head) while the consumers still wait on the small
            // ops before it and HBM is mostly idle.  The stages that follow the
            // ring's worth are prefetched into L2 now, so they are close when the
            // consumers free the ring's slots.
            if (st == 0 && p.l2_head_start > 0 && (w[W_OP] == OP_FFN || w[W_OP] == OP_LMHEAD_ARGMAX)) {
                const int e = pl.n_stages < NS + p.l2_head_start ? pl.n_stages : NS + p.l2_head_start;
                for (int s2 = NS; s2 < e; ++s2) prefetch_stage(pl, s2);
            }
            used |= 1u << slot;
            last_parity = (last_parity & ~(1u << slot)) | (phase << slot);
            if (++slot == NS) {
                slot = 0;
                phase ^= 1u;
            }
            if (PF && pf_stages > 0) {
                if (pf_g <= g) {  // cursor caught up: restart right after this stage
                    pf_i = i;
                    pf_st = st + 1;
                    pf_g = g + 1;
                    pf_plan = pl;
                    pf_stalled = false;
                }
                while (pf_g <= g + pf_stages && !pf_stalled) {
                    if (pf_st >= pf_plan.n_stages) {
                        if (pf_i + 1 >= n) {
                            pf_stalled = true;
                            break;
                        }
                        Plan np;
                        if (!loader_plan<MOE, NB>(p, a, q + (size_t)(pf_i + 1) * W_NWORDS, m, np, false, pf_i + 1)) break;
                        pf_i++;
                        pf_plan = np;
                        pf_st = 0;
                        continue;
                    }
                    prefetch_stage(pf_plan, pf_st);
                    pf_st++;
                    pf_g++;
                }
            }
        }
        if (!ok) return false;
    }
    return true;
}

// Before the block leaves: wait (bounded) for the last copy issued into every
// used slot.  A copy that does not land within the spin limit is an error of
// the step: it is recorded (MK_ERR_TIMEOUT, counter -1, observed = the slot)
// and the stop word is set, so the host voids the step instead of returning
// its result.
__device__ void loader_drain(const DevParams& p, uint64_t* full, const LoaderRing& lr) {
    for (int s = 0; s < p.ring_stages; ++s) {
        if (!((lr.used >> s) & 1u)) continue;
        const uint32_t par = (lr.last_parity >> s) & 1u;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[s], par)) {
            if (globaltimer_ns() - t0 > p.spin_limit_ns) {
                record_error(p.status, MK_ERR_TIMEOUT, blockIdx.x, -1, 0, -1, (uint32_t)s, par);
                return;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// consumers: GEMV-type instructions
// ---------------------------------------------------------------------------
enum VecKind { VK_RMS, VK_ATTN, VK_H };

// Fill v[j][0..8) with the input vector slice of this thread (chunks
// c = tid + 256 j of 8 elements; zero outside [0, K)).
template <int J>
__device__ __forceinline__ void load_vec(const float* __restrict__ src, int K, float (&v)[J][8]) {
    const int tid = threadIdx.x, nch = K >> 3;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int c = tid + kConsumerThreads * j;
        if (c < nch) {
            const float4 a0 = __ldcg(reinterpret_cast<const float4*>(src) + 2 * c);
            const float4 a1 = __ldcg(reinterpret_cast<const float4*>(src) + 2 * c + 1);
            v[j][0] = a0.x; v[j][1] = a0.y; v[j][2] = a0.z; v[j][3] = a0.w;
            v[j][4] = a1.x; v[j][5] = a1.y; v[j][6] = a1.z; v[j][7] = a1.w;
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[j][k] = 0.f;
        }
    }
}

// Input of the O-projection, columns [col0, col0 + K): the attention output of
// every query head, merged here from its kv splits' partials (unnormalised
// o_s, running max m_s in the log2 domain, sum l_s):
//   attn = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s,
// taken B splits per round trip with an online rescale, in split order.
// sq: the sequence of a batched decode step.
template <int J, int B>
__device__ __forceinline__ void load_attn_merged(const DevParams& p, int col0, int K, float (&v)[J][8], int sq = 0) {
    const int tid = threadIdx.x, nch = K >> 3, S = p.kv_splits, D = p.d;
    const float* part_ml = p.part_ml + (size_t)sq * p.nq * S * 2;
    const float* part_o = p.part_o + (size_t)sq * p.nq * S * D;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int c = tid + kConsumerThreads * j;
        if (c >= nch) {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[j][k] = 0.f;
            continue;
        }
        const int col = col0 + 8 * c, h = col / D, dc = col - h * D;
        const float2* ml = reinterpret_cast<const float2*>(part_ml) + (size_t)h * S;
        const float4* po = reinterpret_cast<const float4*>(part_o + (size_t)h * S * D + dc);
        const int D4 = D >> 2;
        float M = -CUDART_INF_F, den = 0.f, acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
        for (int s0 = 0; s0 < S; s0 += B) {
            float2 t[B];
            float4 o0[B], o1[B];
#pragma unroll
            for (int k = 0; k < B; ++k) {
                if (s0 + k < S) {
                    t[k] = __ldcg(ml + s0 + k);
                    o0[k] = __ldcg(po + (size_t)(s0 + k) * D4);
                    o1[k] = __ldcg(po + (size_t)(s0 + k) * D4 + 1);
                } else {
                    t[k] = make_float2(-CUDART_INF_F, 0.f);
                    o0[k] = o1[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            float bm = M;
#pragma unroll
            for (int k = 0; k < B; ++k) bm = fmaxf(bm, t[k].x);
            if (bm == -CUDART_INF_F) continue;  // no position in these splits yet
            const float r = exp2f(M - bm);
            den *= r;
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] *= r;
#pragma unroll
            for (int k = 0; k < B; ++k) {
                const float f = exp2f(t[k].x - bm);
                den = fmaf(f, t[k].y, den);
                acc[0] = fmaf(f, o0[k].x, acc[0]);
                acc[1] = fmaf(f, o0[k].y, acc[1]);
                acc[2] = fmaf(f, o0[k].z, acc[2]);
                acc[3] = fmaf(f, o0[k].w, acc[3]);
                acc[4] = fmaf(f, o1[k].x, acc[4]);
                acc[5] = fmaf(f, o1[k].y, acc[5]);
                acc[6] = fmaf(f, o1[k].z, acc[6]);
                acc[7] = fmaf(f, o1[k].w, acc[7]);
            }
            M = bm;
        }
        const float inv = 1.0f / den;
#pragma unroll
        for (int k = 0; k < 8; ++k) v[j][k] = acc[k] * inv;
    }
}

// v = rmsnorm(x) * w for x fp32 (or the bf16 embedding row), all threads.
// The norm weights are loaded together with x so both round trips overlap.
template <int J>
__device__ void load_rms(const DevParams& p, Misc& m, const float* x32, const uint16_t* x16, const uint16_t* nw,
                         float (&v)[J][8], float* snap = nullptr) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, K = p.H, nch = K >> 3;
    uint4 wraw[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int c = tid + kConsumerThreads * j;
        wraw[j] = c < nch ? __ldg(reinterpret_cast<const uint4*>(nw) + c) : make_uint4(0u, 0u, 0u, 0u);
        if (c < nch) {
            if (x16) {
                unpack8(__ldg(reinterpret_cast<const uint4*>(x16) + c), v[j]);
            } else {
                const float4 a0 = __ldcg(reinterpret_cast<const float4*>(x32) + 2 * c);
                const float4 a1 = __ldcg(reinterpret_cast<const float4*>(x32) + 2 * c + 1);
                v[j][0] = a0.x; v[j][1] = a0.y; v[j][2] = a0.z; v[j][3] = a0.w;
                v[j][4] = a1.x; v[j][5] = a1.y; v[j][6] = a1.z; v[j][7] = a1.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[j][k] = 0.f;
        }
    }
    if (snap) {  // record the residual stream the op reads (hidden-state snapshot)
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int c = tid + kConsumerThreads * j;
            if (c < nch) {
                reinterpret_cast<float4*>(snap)[2 * c] = make_float4(v[j][0], v[j][1], v[j][2], v[j][3]);
                reinterpret_cast<float4*>(snap)[2 * c + 1] = make_float4(v[j][4], v[j][5], v[j][6], v[j][7]);
            }
        }
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
        for (int k = 0; k < 8; ++k) ss = fmaf(v[j][k], v[j][k], ss);
    ss = warp_sum(ss);
    if (lane == 0) m.red[warp] = ss;
    cbar();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += m.red[w];
    const float rs = 1.0f / sqrtf(tot / (float)K + p.eps);
#pragma unroll
    for (int j = 0; j < J; ++j) {
        float wf[8];
        unpack8(wraw[j], wf);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[j][k] = v[j][k] * rs * wf[k];
    }
    cbar();  // m.red free again
}

// Two interleaved fp32 chains over the 8 bf16 of w (even / odd elements).
__device__ __forceinline__ void dot8x2(const uint4 w, const float* v, float& a0, float& a1) {
    a0 = fmaf(bf_lo(w.x), v[0], a0);
    a1 = fmaf(bf_hi(w.x), v[1], a1);
    a0 = fmaf(bf_lo(w.y), v[2], a0);
    a1 = fmaf(bf_hi(w.y), v[3], a1);
    a0 = fmaf(bf_lo(w.z), v[4], a0);
    a1 = fmaf(bf_hi(w.z), v[5], a1);
    a0 = fmaf(bf_lo(w.w), v[6], a0);
    a1 = fmaf(bf_hi(w.w), v[7], a1);
}

// Router of a MoE layer from xn (this thread's slice in v): logits of all
// experts, top-k (ties to the lower index), softmax over the selected.
// PRED: the speculative prediction (into pred_eidx / pred_idx / pred_layer)
// instead of the routing.  The expert rows are read in batches of RB whose
// loads are all issued before their FMAs (one L2 round trip per batch), each
// batch's dot products are reduced across the warp together, and warp 0 adds
// the 8 warps' partials (in warp order) and selects the top k by shuffles.
template <int J, bool PRED = false>
__device__ void route(const DevParams& p, Misc& m, float* scratch, const uint16_t* wr, int layer, bool publish,
                      float (&v)[J][8], uint32_t epoch) {
    constexpr int RB = J <= 2 ? 8 : 2;  // expert rows per batch: RB * J live 128-bit loads
    constexpr int LPR = 32 / RB;        // lanes that hold each row's sum after the reduction
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, K = p.H, nch = K >> 3, E = p.E;
    for (int e0 = 0; e0 < E; e0 += RB) {
        uint4 wv[RB][J];
#pragma unroll
        for (int k = 0; k < RB; ++k)
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int c = tid + kConsumerThreads * j;
                wv[k][j] = (e0 + k < E && c < nch) ? __ldg(reinterpret_cast<const uint4*>(wr + (size_t)(e0 + k) * K) + c)
                                                   : make_uint4(0u, 0u, 0u, 0u);
            }
        float a[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int j = 0; j < J; ++j)
                if (tid + kConsumerThreads * j < nch) dot8x2(wv[k][j], v[j], a0, a1);
            a[k] = a0 + a1;
        }
        const float s_e = reduce_rows<RB>(a, lane);
        const int e = e0 + lane / LPR;
        if (lane % LPR == 0 && e < E) scratch[warp * 64 + e] = s_e;
    }
    cbar();
    if (warp == 0) {
        // lane holds experts lane and lane + 32; the prediction's check mode (spec_experts == 2)
        // takes the lowest scores instead
        const float sgn = PRED && p.spec_experts == 2 ? -1.0f : 1.0f;
        float lg[2] = {0.f, 0.f};
        bool open[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = lane + 32 * h;
            open[h] = e < E;
            if (open[h])
                for (int w = 0; w < kConsumerWarps; ++w) lg[h] += scratch[w * 64 + e];
        }
        int idx[kMaxTopK];
        float sel[kMaxTopK];
        for (int k = 0; k < p.topk; ++k) {
            float bv = -CUDART_INF_F;
            int bi = 0x7FFFFFFF;
            if (open[0]) { bv = sgn * lg[0]; bi = lane; }
            if (open[1] && (bi == 0x7FFFFFFF || sgn * lg[1] > bv)) { bv = sgn * lg[1]; bi = lane + 32; }
            warp_argmax(bv, bi);
            idx[k] = bi;
            sel[k] = sgn * bv;
            if (bi == lane) open[0] = false;
            if (bi == lane + 32) open[1] = false;
        }
        if (lane == 0) {
            if constexpr (PRED) {
                for (int k = 0; k < p.topk; ++k) {
                    m.pred_eidx[k] = idx[k];
                    if (publish) p.pred_idx[layer * kMaxTopK + k] = idx[k];
                }
                __threadfence_block();
                vstore(&m.pred_layer, route_key(epoch, layer, p.L));
            } else {
                float z = 0.f, ex[kMaxTopK];
                for (int k = 0; k < p.topk; ++k) {
                    ex[k] = expf(sel[k] - sel[0]);
                    z += ex[k];
                }
                for (int k = 0; k < p.topk; ++k) {
                    m.eidx[k] = idx[k];
                    m.ew[k] = ex[k] / z;
                    if (publish) {
                        p.router_idx[layer * kMaxTopK + k] = idx[k];
                        p.router_w[layer * kMaxTopK + k] = ex[k] / z;
                    }
                }
                __threadfence_block();
                vstore(&m.router_layer, route_key(epoch, layer, p.L));
            }
        }
    }
    cbar();
}


// RG full rows [rg, rg + RG) of a stage span: every chunk this thread owns is
// loaded before any FMA, then each row sum is reduced across the warp and
// stored in this warp's slot A[row * 8 + warp] (shared memory; the epilogue
// adds the 8 warps' slots in a fixed order, so results are bitwise
// reproducible).  jv[j]: chunk j of this thread exists.
template <int J, int RG>
__device__ __forceinline__ void rows_block(const uint4* __restrict__ Ws, int row16, int rg, const bool (&jv)[J],
                                           const float (&v)[J][8], float* A, int lane) {
    const int tid = threadIdx.x;
    uint4 wv[RG][J];
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
        for (int j = 0; j < J; ++j)
            wv[r][j] = jv[j] ? Ws[(rg + r) * row16 + tid + kConsumerThreads * j] : make_uint4(0u, 0u, 0u, 0u);
    float part[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int j = 0; j < J; ++j) dot8x2(wv[r][j], v[j], a0, a1);
        part[r] = a0 + a1;
    }
    const float s_row = reduce_rows<RG>(part, lane);
    if (reduce_rows_writer<RG>(lane)) A[(rg + reduce_rows_lane_row<RG>(lane)) * kConsumerWarps + (tid >> 5)] = s_row;
}

// rows_block for rows [rg, rg + RG) of which those at or past nr read as zero
// and are not stored: one copy of the block code covers every row count (a
// smaller kernel; the stages of one-chunk-per-thread ops hold 8 or 16 rows, so
// little work is spent on the padding).
template <int J, int RG>
__device__ __forceinline__ void rows_block_pred(const uint4* __restrict__ Ws, int row16, int rg, int nr,
                                                const bool (&jv)[J], const float (&v)[J][8], float* A, int lane) {
    const int tid = threadIdx.x;
    uint4 wv[RG][J];
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
        for (int j = 0; j < J; ++j)
            wv[r][j] = (jv[j] && rg + r < nr) ? Ws[(rg + r) * row16 + tid + kConsumerThreads * j]
                                              : make_uint4(0u, 0u, 0u, 0u);
    float part[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int j = 0; j < J; ++j) dot8x2(wv[r][j], v[j], a0, a1);
        part[r] = a0 + a1;
    }
    const float s_row = reduce_rows<RG>(part, lane);
    const int row = rg + reduce_rows_lane_row<RG>(lane);
    if (reduce_rows_writer<RG>(lane) && row < nr) A[row * kConsumerWarps + (tid >> 5)] = s_row;
}

// This thread's column slice of rows [0, nr) of one span of a ring stage (Ws:
// the span in shared memory, row16 16-byte chunks per row) dotted with its
// slice v of the input vector, into the warp slots of rows [0, nr) of A.  Rows go in blocks of
// RG, then RG/2, ... 1, so no row needs a guard; a chunk that lies outside
// the row (widths that are not a multiple of 2048) is a per-thread predicate,
// uniform across each warp for widths that are multiples of 256.
template <int J, int RG>
__device__ __forceinline__ void stage_rows(const uint4* __restrict__ Ws, int row16, int nr, int nch,
                                           const float (&v)[J][8], float* A, int lane) {
    bool jv[J];
#pragma unroll
    for (int j = 0; j < J; ++j) jv[j] = (int)threadIdx.x + kConsumerThreads * j < nch;
    int rg = 0;
    if constexpr (J == 1) {  // one chunk per thread: 8-row blocks, the last one predicated
        for (; rg < nr; rg += RG) rows_block_pred<J, RG>(Ws, row16, rg, nr, jv, v, A, lane);
        return;
    }
    for (; rg + RG <= nr; rg += RG) rows_block<J, RG>(Ws, row16, rg, jv, v, A, lane);
    if constexpr (RG >= 8) {
        if (rg + 4 <= nr) { rows_block<J, 4>(Ws, row16, rg, jv, v, A, lane); rg += 4; }
    }
    if constexpr (RG >= 4) {
        if (rg + 2 <= nr) { rows_block<J, 2>(Ws, row16, rg, jv, v, A, lane); rg += 2; }
    }
    if constexpr (RG >= 2) {
        if (rg < nr) rows_block<J, 1>(Ws, row16, rg, jv, v, A, lane);
    }
}

// HOIST: dense instructions make their stage plan before the dependency wait
// (costs registers across the wait; used by the specialised kernels).
// SPEC: a QKV instruction marked for it predicts the layer's experts after it
// signals (MoE instantiations).
template <int J, bool HOIST, bool SPEC = false>
__device__ bool gemv_instr(const DevParams& p, const StepArgs& a, const int32_t* w, int ii, unsigned char* ring,
                           uint64_t* full, uint64_t* empty, float* scratch, Misc& m, int& slot, uint32_t& phase,
                           int token) {
    // rows reduced together: keeps the live 128-bit weight loads at RG * J <= 8 (4 for J = 4)
    constexpr int RG = J == 1 ? 8 : J == 2 ? 4 : J == 3 ? 2 : 1;
    const int tid = threadIdx.x, lane = tid & 31;
    const int op = w[W_OP], l = w[W_LAYER], sub = w[W_SUB], b = w[W_BEGIN], rows = w[W_END] - b;
    const uint32_t SB = (uint32_t)p.stage_bytes;
    float* part_sums = scratch;  // [set * rows + row][8 warps]
    unsigned long long* tr = p.trace ? p.trace + ((size_t)blockIdx.x * p.max_instr + ii) * kTraceWords : nullptr;

    // 1. dependency (the weight-pointer table entries of the plan are fetched meanwhile, or the
    // plan of a dense op is made before the wait)
    Plan pl;
    const bool early = HOIST && !needs_routing(op);
    if (early) make_plan(p, a.pos, w, nullptr, pl);
    else prefetch_plan_l1(p, w);
    if (tid == 0) {
        if (w[W_WAIT_CTR] >= 0 &&
            !wait_counter(p, m, w[W_WAIT_CTR], a.epoch * (uint32_t)w[W_WAIT_INC], ii, op))
            vstore(&m.abort_flag, 1);
        if (tr) tr[T_DEP] = globaltimer_ns();
    }
    cbar();
    if (vload(&m.abort_flag)) return false;

    // 2. input vector (first column part)
    float v[J][8];
    const uint16_t* const* wt = p.wt + (size_t)(l < p.L ? l : 0) * wt_stride(p.E);
    int K = p.H;
    const float* vsrc = nullptr;  // fp32 input for OPROJ / DOWN (all column parts)
    switch (op) {
        case OP_RMS_QKV:
            // the residual after layer l-1 (x2); one block records it as snapshot l
            load_rms<J>(p, m, p.x2, l == 0 ? p.embed + (size_t)token * p.H : nullptr, wt[WT_ATTN_NORM], v,
                        (p.snap && l > 0 && sub == 0 && b == 0) ? p.snap + (size_t)l * p.H : nullptr);
            break;
        case OP_RMS_UPGATE_SILU:
        case OP_MOE_UPGATE:
            if constexpr (!HOIST) load_rms<J>(p, m, p.x, nullptr, wt[WT_FFN_NORM], v);
            break;
        case OP_LMHEAD_ARGMAX:
            // the residual after the last layer (or the embedding row without layers): snapshot L
            load_rms<J>(p, m, p.x2, p.L == 0 ? p.embed + (size_t)token * p.H : nullptr, p.final_norm, v,
                        (p.snap && w[W_SEQ] == 0) ? p.snap + (size_t)p.L * p.H : nullptr);
            break;
        case OP_OPROJ_RES:
            K = p.nq * p.d;  // input: the attention output, merged once (W_MERGE) or from the kv splits below
            if (w[W_MERGE]) vsrc = p.attn;
            break;
        case OP_DOWN_RES:
        case OP_MOE_DOWN2_RES:
            K = p.F;
            vsrc = p.hbuf;
            break;
    }
    const int kp = K / kparts_of(K);  // columns per part
    if (op == OP_OPROJ_RES && !vsrc) load_attn_merged<J, HOIST ? 8 : 4>(p, 0, kp, v);
    if (vsrc) load_vec<J>(vsrc, kp, v);
    // 3. routing (once per layer per block; the loader waits for it)
    if constexpr (!HOIST) {
        if (op == OP_MOE_UPGATE && vload(&m.router_layer) != route_key(a.epoch, l, p.L))
            route<J>(p, m, scratch, wt[WT_ROUTER], l, sub == 0 && b == 0, v, a.epoch);
    }
    if (tr && tid == 0) tr[T_READY] = globaltimer_ns();
    if (!early) {
        int eidx[kMaxTopK];
        for (int k = 0; k < kMaxTopK; ++k) eidx[k] = m.eidx[k];
        make_plan(p, a.pos, w, eidx, pl);
    }

    // 4. stages: every warp covers its column slice of every row of the stage
    const int nch = kp >> 3;
    for (int ph = 0; ph < pl.nphase; ++ph) {
        const int vslot = ph / pl.kparts, part = ph % pl.kparts;
        if (ph > 0 && op == OP_OPROJ_RES && !vsrc) load_attn_merged<J, HOIST ? 8 : 4>(p, part * kp, kp, v);
        else if (ph > 0) load_vec<J>(vsrc + (size_t)vslot * p.F + (size_t)part * kp, kp, v);
        for (int sst = 0; sst < pl.spp; ++sst) {
            const int r0 = sst * pl.rps;
            const int nr = (rows - r0) < pl.rps ? (rows - r0) : pl.rps;
            const bool ok = warp_wait_full(&full[slot], phase, p, m, ii, op);
            if (tr && tid == 0 && ph == 0 && sst == 0) tr[T_FIRST] = globaltimer_ns();
            if (tid == 0) stage_stamp(tr, T_SREADY, ph * pl.spp + sst);
            if (ok) {
                const unsigned char* stage = ring + (size_t)slot * SB;
                for (int s = 0; s < pl.nspan; ++s) {
                    const uint4* Ws = reinterpret_cast<const uint4*>(stage + (size_t)s * pl.rps * pl.row_bytes);
                    const int set = (vslot * pl.nspan + s) * pl.kparts + part;
                    stage_rows<J, RG>(Ws, (int)(pl.row_bytes >> 4), nr, nch, v,
                                      part_sums + ((size_t)set * rows + r0) * kConsumerWarps, lane);
                }
                __syncwarp();
                if (tid == 0) stage_stamp(tr, T_SDONE, ph * pl.spp + sst);
                if (lane == 0) mbar_arrive(&empty[slot]);
            } else if (tid == 0) {
                vstore(&m.abort_flag, 1);
            }
            if (++slot == p.ring_stages) {
                slot = 0;
                phase ^= 1u;
            }
        }
    }
    cbar();
    if (vload(&m.abort_flag)) return false;
    if (tr && tid == 0) tr[T_MAIN] = globaltimer_ns();

    // 5. epilogue (storer role): row value of accumulator set k (spans x
    // slots) = the 8 warps' partial sums of every column part, in fixed order
    auto acc = [&](int k, int r) {
        float t = 0.f;
        for (int q2 = 0; q2 < pl.kparts; ++q2) {
            const float4* ps = reinterpret_cast<const float4*>(
                part_sums + ((size_t)(k * pl.kparts + q2) * rows + r) * kConsumerWarps);
            const float4 x0 = ps[0], x1 = ps[1];
            t += ((x0.x + x0.y) + (x0.z + x0.w)) + ((x1.x + x1.y) + (x1.z + x1.w));
        }
        return t;
    };
    switch (op) {
        case OP_RMS_QKV: {
            const int off = sub == 0 ? 0 : (sub == 1 ? p.nq * p.d : (p.nq + p.nkv) * p.d);
            for (int r = tid; r < rows; r += kConsumerThreads) p.qkv[off + b + r] = acc(0, r);
            break;
        }
        case OP_OPROJ_RES:
            for (int r = tid; r < rows; r += kConsumerThreads) {
                float base;
                if (l == 0) {
                    const uint16_t e = p.embed[(size_t)token * p.H + b + r];
                    base = __uint_as_float((uint32_t)e << 16);
                    if (p.snap) p.snap[b + r] = base;
                } else {
                    base = __ldcg(p.x2 + b + r);
                }
                const float nx = base + acc(0, r);
                p.x[b + r] = nx;   // read by the FFN's RMSNorm
                p.x2[b + r] = nx;  // the FFN adds its output here
            }
            break;
        case OP_RMS_UPGATE_SILU:
        case OP_MOE_UPGATE:
            if constexpr (!HOIST) {  // split-FFN ops run in the general instantiation only
                float* h = p.hbuf + (op == OP_MOE_UPGATE ? (size_t)sub * p.F : 0);
                for (int r = tid; r < rows; r += kConsumerThreads) {
                    const float g = acc(0, r), u = acc(1, r);
                    h[b + r] = g / (1.0f + expf(-g)) * u;
                }
            }
            break;
        case OP_DOWN_RES:
        case OP_MOE_DOWN2_RES:
            if constexpr (!HOIST) {
                for (int r = tid; r < rows; r += kConsumerThreads) {
                    float add = acc(0, r);
                    if (op == OP_MOE_DOWN2_RES) {
                        add = m.ew[0] * add;
                        if (p.topk > 1) add += m.ew[1] * acc(1, r);
                    }
                    p.x2[b + r] = __ldcg(p.x2 + b + r) + add;
                }
            }
            break;
        case OP_LMHEAD_ARGMAX: {
            float bv = -CUDART_INF_F;
            int bi = 0x7FFFFFFF;
            for (int r = tid; r < rows; r += kConsumerThreads) {
                const float val = acc(0, r);
                a.logits[b + r] = val;
                if (val > bv || (val == bv && b + r < bi)) {
                    bv = val;
                    bi = b + r;
                }
            }
            warp_argmax(bv, bi);
            const int warp = tid >> 5;
            if (lane == 0) {
                m.red[warp] = bv;
                m.redi[warp] = bi;
            }
            cbar();
            if (tid == 0) {
                for (int k = 1; k < kConsumerWarps; ++k)
                    if (m.red[k] > bv || (m.red[k] == bv && m.redi[k] < bi)) {
                        bv = m.red[k];
                        bi = m.redi[k];
                    }
                // lanes other than 0 of warp 0 keep their own partial; only tid 0 writes
                p.lm_part[2 * w[W_SEQ]] = bv;
                p.lm_part[2 * w[W_SEQ] + 1] = __int_as_float(bi);
                const uint32_t old = arrive_release(p.counters + w[W_AUX_CTR]);
                m.is_last = (old + 1u == a.epoch * (uint32_t)w[W_AUX_INC]) ? 1 : 0;
            }
            cbar();
            if (m.is_last) {
                const int n_lm = w[W_AUX_INC];
                float cv = -CUDART_INF_F;
                int ci = 0x7FFFFFFF;
                for (int k = tid; k < n_lm; k += kConsumerThreads) {
                    const float val = __ldcg(p.lm_part + 2 * k);
                    const int idx = __float_as_int(__ldcg(p.lm_part + 2 * k + 1));
                    if (val > cv || (val == cv && idx < ci)) {
                        cv = val;
                        ci = idx;
                    }
                }
                warp_argmax(cv, ci);
                cbar();
                if (lane == 0) {
                    m.red[warp] = cv;
                    m.redi[warp] = ci;
                }
                cbar();
                if (tid == 0) {
                    for (int k = 1; k < kConsumerWarps; ++k)
                        if (m.red[k] > cv || (m.red[k] == cv && m.redi[k] < ci)) {
                            cv = m.red[k];
                            ci = m.redi[k];
                        }
                    p.status->next_token = ci;
                    if (a.serve) serve_respond(p, a, ci);
                }
            }
            break;
        }
    }
    cbar();
    if (tid == 0 && w[W_SIGNAL_CTR] >= 0 && op != OP_LMHEAD_ARGMAX) signal_release(p.counters + w[W_SIGNAL_CTR]);
    if constexpr (SPEC) {
        // Speculative expert prediction: the router applied to this instruction's input (the
        // attention input of the layer), off the critical path: the QKV outputs are already
        // signalled, and the loader streams the predicted experts' first FFN stages meanwhile.
        if (op == OP_RMS_QKV && w[W_SPEC] != 0 && p.spec_experts)
            route<J, true>(p, m, scratch, wt[WT_ROUTER], l, w[W_SPEC] == 2, v, a.epoch);
    }
    return true;
}

// Fused FFN slice (OP_FFN / OP_MOE_FFN).  Rows [b, e) of the up/gate
// projections give h = silu(Wg xn) * (Wu xn) for this block's rows (MoE: of
// its routed expert, scaled by the router weight); the block then streams the
// same rows of the transposed down-projection, Wd^T[b..e) = Wd[:, b..e)^T, and
// accumulates its column chunks of Wd[:, b..e) h[b..e) in registers, which are
// added into the post-FFN residual x2 with float4 atomics.  One instruction,
// one continuous weight stream per block: the up/gate -> down dependency stays
// inside the block.
template <int J, bool HOIST, bool MOE>
__device__ bool ffn_instr(const DevParams& p, const StepArgs& a, const int32_t* w, int ii, unsigned char* ring,
                          uint64_t* full, uint64_t* empty, float* scratch, Misc& m, int& slot, uint32_t& phase) {
    constexpr int RG = J == 1 ? 8 : J == 2 ? 4 : J == 3 ? 2 : 1;
    const int tid = threadIdx.x, lane = tid & 31;
    const int op = w[W_OP], l = w[W_LAYER], sub = w[W_SUB], b = w[W_BEGIN], rows = w[W_END] - b;
    const uint32_t SB = (uint32_t)p.stage_bytes;
    float* part_sums = scratch;  // [2 * rows][8 warps] gate / up row sums, then h[rows]
    unsigned long long* tr = p.trace ? p.trace + ((size_t)blockIdx.x * p.max_instr + ii) * kTraceWords : nullptr;
    Plan pl;
    const bool early = HOIST && (!MOE || op == OP_FFN);  // dense: planned before the wait
    if (early) make_plan(p, a.pos, w, nullptr, pl);
    else prefetch_plan_l1(p, w);  // weight-pointer table entries, while the dependency is pending

    if (tid == 0) {
        if (!wait_counter(p, m, w[W_WAIT_CTR], a.epoch * (uint32_t)w[W_WAIT_INC], ii, op)) vstore(&m.abort_flag, 1);
        else if (op == OP_FFN) vstore(&m.ffn_go, route_key(a.epoch, l, p.L));  // the loader's gate
        if (tr) tr[T_DEP] = globaltimer_ns();
    }
    cbar();
    if (vload(&m.abort_flag)) return false;

    float v[J][8];
    const uint16_t* const* wt = p.wt + (size_t)l * wt_stride(p.E);
    load_rms<J>(p, m, p.x, nullptr, wt[WT_FFN_NORM], v);
    if constexpr (MOE) {
        if (op == OP_MOE_FFN && vload(&m.router_layer) != route_key(a.epoch, l, p.L))
            route<J>(p, m, scratch, wt[WT_ROUTER], l, sub == 0 && b == 0, v, a.epoch);
    }
    if (tr && tid == 0) tr[T_READY] = globaltimer_ns();
    if (!early) {
        int eidx[kMaxTopK];
        for (int k = 0; k < kMaxTopK; ++k) eidx[k] = m.eidx[k];
        make_plan(p, a.pos, w, eidx, pl);
    }
    if constexpr (MOE) {
        // speculative stages of a mispredicted expert: released unread (the loader streams the
        // routed expert's rows after them)
        if (op == OP_MOE_FFN && w[W_SPEC] != 0 && p.spec_experts && !spec_hit(p, m, sub)) {
            const int ns = pl.n_stages < p.ring_stages ? pl.n_stages : p.ring_stages;
            for (int st = 0; st < ns; ++st) {
                if (warp_wait_full(&full[slot], phase, p, m, ii, op)) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[slot]);
                } else if (tid == 0) {
                    vstore(&m.abort_flag, 1);
                }
                if (++slot == p.ring_stages) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
        }
    }
    const int nch = p.H >> 3;

    // up/gate rows
    for (int sst = 0; sst < pl.spp; ++sst) {
        const int r0 = sst * pl.rps;
        const int nr = (rows - r0) < pl.rps ? (rows - r0) : pl.rps;
        const bool ok = warp_wait_full(&full[slot], phase, p, m, ii, op);
        if (tr && tid == 0 && sst == 0) tr[T_FIRST] = globaltimer_ns();
        if (tid == 0) stage_stamp(tr, T_SREADY, sst);
        if (ok) {
            const unsigned char* stage = ring + (size_t)slot * SB;
            for (int s = 0; s < 2; ++s) {
                const uint4* Ws = reinterpret_cast<const uint4*>(stage + (size_t)s * pl.rps * pl.row_bytes);
                stage_rows<J, RG>(Ws, (int)(pl.row_bytes >> 4), nr, nch, v,
                                  part_sums + ((size_t)s * rows + r0) * kConsumerWarps, lane);
            }
            __syncwarp();
            if (tid == 0) stage_stamp(tr, T_SDONE, sst);
            if (lane == 0) mbar_arrive(&empty[slot]);
        } else if (tid == 0) {
            vstore(&m.abort_flag, 1);
        }
        if (++slot == p.ring_stages) {
            slot = 0;
            phase ^= 1u;
        }
    }
    cbar();
    if (vload(&m.abort_flag)) return false;
    if (tr && tid == 0) tr[T_MAIN] = globaltimer_ns();

    // h = silu(g) * u (times the router weight), then kept at the start of the scratch
    const float wgt = MOE && op == OP_MOE_FFN ? m.ew[ffn_slot(m.eidx, p.topk, sub)] : 1.0f;
    float hv[2] = {0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int r = tid + kConsumerThreads * k;
        if (r < rows) {
            const float4* pg = reinterpret_cast<const float4*>(part_sums + (size_t)r * kConsumerWarps);
            const float4* pu = reinterpret_cast<const float4*>(part_sums + ((size_t)rows + r) * kConsumerWarps);
            const float4 g0 = pg[0], g1 = pg[1], u0 = pu[0], u1 = pu[1];
            const float g = ((g0.x + g0.y) + (g0.z + g0.w)) + ((g1.x + g1.y) + (g1.z + g1.w));
            const float u = ((u0.x + u0.y) + (u0.z + u0.w)) + ((u1.x + u1.y) + (u1.z + u1.w));
            hv[k] = wgt * (g / (1.0f + expf(-g)) * u);
        }
    }
    cbar();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int r = tid + kConsumerThreads * k;
        if (r < rows) scratch[r] = hv[k];
    }
    cbar();

    // transposed down-projection rows: this thread's column chunks of Wd[:, rows] h
    float y[J][8];
    bool jv[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
        jv[j] = tid + kConsumerThreads * j < nch;
#pragma unroll
        for (int k = 0; k < 8; ++k) y[j][k] = 0.f;
    }
    for (int tst = 0; tst < pl.tail_spp; ++tst) {
        const int r0 = tst * pl.tail_rps;
        const int nr = (rows - r0) < pl.tail_rps ? (rows - r0) : pl.tail_rps;
        const bool ok = warp_wait_full(&full[slot], phase, p, m, ii, op);
        if (tid == 0) stage_stamp(tr, T_SREADY, pl.spp + tst);
        if (ok) {
            const uint4* Ws = reinterpret_cast<const uint4*>(ring + (size_t)slot * SB);
            constexpr int RQ = J <= 2 ? 4 : 2;  // rows in flight per thread
            int r = 0;
            for (; r + RQ <= nr; r += RQ) {
                uint4 wv[RQ][J];
#pragma unroll
                for (int q = 0; q < RQ; ++q)
#pragma unroll
                    for (int j = 0; j < J; ++j)
                        wv[q][j] = jv[j] ? Ws[(r + q) * nch + tid + kConsumerThreads * j] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int q = 0; q < RQ; ++q) {
                    const float hk = scratch[r0 + r + q];
#pragma unroll
                    for (int j = 0; j < J; ++j) {
                        float f[8];
                        unpack8(wv[q][j], f);
#pragma unroll
                        for (int k = 0; k < 8; ++k) y[j][k] = fmaf(f[k], hk, y[j][k]);
                    }
                }
            }
            for (; r < nr; ++r) {
                const float hk = scratch[r0 + r];
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    if (!jv[j]) continue;
                    float f[8];
                    unpack8(Ws[r * nch + tid + kConsumerThreads * j], f);
#pragma unroll
                    for (int k = 0; k < 8; ++k) y[j][k] = fmaf(f[k], hk, y[j][k]);
                }
            }
            __syncwarp();
            if (tid == 0) stage_stamp(tr, T_SDONE, pl.spp + tst);
            if (lane == 0) mbar_arrive(&empty[slot]);
        } else if (tid == 0) {
            vstore(&m.abort_flag, 1);
        }
        if (++slot == p.ring_stages) {
            slot = 0;
            phase ^= 1u;
        }
    }
    cbar();
    if (vload(&m.abort_flag)) return false;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        if (!jv[j]) continue;
        float4* dst = reinterpret_cast<float4*>(p.x2) + 2 * (tid + kConsumerThreads * j);
        atomicAdd(dst, make_float4(y[j][0], y[j][1], y[j][2], y[j][3]));
        atomicAdd(dst + 1, make_float4(y[j][4], y[j][5], y[j][6], y[j][7]));
    }
    cbar();
    if (tid == 0) signal_release(p.counters + w[W_SIGNAL_CTR]);
    return true;
}

// ---------------------------------------------------------------------------
// consumers: batched decode (NB > 1 sequences per step, nb of them in use)
// ---------------------------------------------------------------------------
// A batched GEMV is a skinny GEMM, y[row][q] = sum_k W[row][k] x_q[k].  The
// one-chunk kernel with 8 sequence slots (batch_on_tensor_cores) runs it on the
// tensor cores; the other batched kernels use the CUDA-core form further down.
// On the tensor cores each ring stage's rows (stored at a pitch of
// row_bytes + 16, so the 8 rows of an ldmatrix tile fall in different banks)
// are the A operand of m16n8k16 bf16 MMAs whose N dimension is the 8 sequence
// slots (unused slots hold zeros).  Warp w takes columns [w K/8, (w + 1) K/8)
// of every row.  The fp32 activations enter as bf16 high and low parts (x = hi
// + lo to about 16 mantissa bits), two MMAs per k-step, fp32 accumulation.

// x0, x1 as bf16x2 high parts (rounded to nearest) and the bf16x2 of what the
// high parts leave (x0 in the low half of each word).
__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16x2(x0, x1);
    lo = pack_bf16x2(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xFFFF0000u));
}

// B fragments of one warp's k-range for the 8 sequence slots: lane (g, t) =
// (lane / 4, lane % 4) holds sequence g's columns kb + 2t, 2t + 1 (word 0) and
// kb + 2t + 8, 2t + 9 (word 1) of every k-step of 16 columns, high and low parts.
template <int KS>
struct BFrag {
    uint32_t hi[KS][2], lo[KS][2];
};

// The sequences' input vectors, held in the CUDA-core layout (thread tid: the
// 8-column chunks tid + 256 j), rearranged into B fragments through the
// scratch, as many sequences per pass as fit.
template <int J, int NB, int KS>
__device__ __forceinline__ void to_bfrag(const float (&v)[NB][J][8], int K, float* scratch, BFrag<KS>& bf, int lane,
                                         int warp) {
    const int tid = threadIdx.x, g = lane >> 2, t = lane & 3, nch = K >> 3;
    const int SP = kRowSlots * kConsumerWarps / K;  // sequences per pass
    const int kw = K / kConsumerWarps, ksr = kw / 16;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) bf.hi[ks][0] = bf.hi[ks][1] = bf.lo[ks][0] = bf.lo[ks][1] = 0u;
    for (int p0 = 0; p0 < NB; p0 += SP) {
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            if (q < p0 || q >= p0 + SP) continue;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int c = tid + kConsumerThreads * j;
                if (c < nch) {
                    float4* dst = reinterpret_cast<float4*>(scratch + (size_t)(q - p0) * K) + 2 * c;
                    dst[0] = make_float4(v[q][j][0], v[q][j][1], v[q][j][2], v[q][j][3]);
                    dst[1] = make_float4(v[q][j][4], v[q][j][5], v[q][j][6], v[q][j][7]);
                }
            }
        }
        cbar();
        if (g >= p0 && g < p0 + SP) {
            const float* src = scratch + (size_t)(g - p0) * K + warp * kw + 2 * t;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                if (ks >= ksr) continue;  // (not break: the unrolled loop keeps static indices)
                const float2 x = *reinterpret_cast<const float2*>(src + 16 * ks);
                const float2 y = *reinterpret_cast<const float2*>(src + 16 * ks + 8);
                split_pack(x.x, x.y, bf.hi[ks][0], bf.lo[ks][0]);
                split_pack(y.x, y.y, bf.hi[ks][1], bf.lo[ks][1]);
            }
        }
        cbar();
    }
}

// The nb sequences' RMSNorm-ed inputs straight into B fragments (no detour
// through the CUDA-core layout): lane (g, t) of warp w loads sequence g's
// columns of its k-steps (x fp32 at x32 + g H, or the bf16 embedding row of
// the sequence's token when from_embed) and the norm weights there; the
// sums of squares of each sequence meet in one block reduction; the scaled
// values are split into bf16 high and low parts.  snap (optional): sequence
// g's un-normalised input is stored at snap + g * snap_stride.
template <int KS>
__device__ __forceinline__ void rms_bfrag(const DevParams& p, Misc& m, const float* x32, bool from_embed,
                                          const uint16_t* nw, BFrag<KS>& bf, float* snap, size_t snap_stride,
                                          int lane, int warp) {
    const int K = p.H, g = lane >> 2, t = lane & 3, ksr = K / (16 * kConsumerWarps);
    const int c0 = warp * (K / kConsumerWarps) + 2 * t;
    const bool live = g < p.nb;
    float x[KS][4];
    uint32_t wn[KS][2];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        x[ks][0] = x[ks][1] = x[ks][2] = x[ks][3] = 0.f;
        wn[ks][0] = wn[ks][1] = 0u;
        if (ks >= ksr) continue;
        const int c = c0 + 16 * ks;
        wn[ks][0] = __ldg(reinterpret_cast<const uint32_t*>(nw + c));
        wn[ks][1] = __ldg(reinterpret_cast<const uint32_t*>(nw + c + 8));
        if (!live) continue;
        if (from_embed) {
            const uint16_t* e = p.embed + (size_t)m.btok[g] * K + c;
            const uint32_t e0 = __ldg(reinterpret_cast<const uint32_t*>(e));
            const uint32_t e1 = __ldg(reinterpret_cast<const uint32_t*>(e + 8));
            x[ks][0] = __uint_as_float(e0 << 16);
            x[ks][1] = __uint_as_float(e0 & 0xFFFF0000u);
            x[ks][2] = __uint_as_float(e1 << 16);
            x[ks][3] = __uint_as_float(e1 & 0xFFFF0000u);
        } else {
            const float* src = x32 + (size_t)g * K + c;
            const float2 a = __ldcg(reinterpret_cast<const float2*>(src));
            const float2 b = __ldcg(reinterpret_cast<const float2*>(src + 8));
            x[ks][0] = a.x;
            x[ks][1] = a.y;
            x[ks][2] = b.x;
            x[ks][3] = b.y;
        }
    }
    if (snap && live) {
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            if (ks >= ksr) continue;
            float* dst = snap + (size_t)g * snap_stride + c0 + 16 * ks;
            *reinterpret_cast<float2*>(dst) = make_float2(x[ks][0], x[ks][1]);
            *reinterpret_cast<float2*>(dst + 8) = make_float2(x[ks][2], x[ks][3]);
        }
    }
    float ss = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(x[ks][e], x[ks][e], ss);
    ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 1);  // the 4 lanes of sequence g in this warp
    ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 2);
    if (t == 0) m.bred[g * kConsumerWarps + warp] = ss;
    cbar();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += m.bred[g * kConsumerWarps + w];
    const float rs = live ? 1.0f / sqrtf(tot / (float)K + p.eps) : 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        const float w0 = __uint_as_float(wn[ks][0] << 16), w1 = __uint_as_float(wn[ks][0] & 0xFFFF0000u);
        const float w2 = __uint_as_float(wn[ks][1] << 16), w3 = __uint_as_float(wn[ks][1] & 0xFFFF0000u);
        split_pack(x[ks][0] * rs * w0, x[ks][1] * rs * w1, bf.hi[ks][0], bf.lo[ks][0]);
        split_pack(x[ks][2] * rs * w2, x[ks][3] * rs * w3, bf.hi[ks][1], bf.lo[ks][1]);
    }
    cbar();  // m.bred free again
}

// Rows [0, nr) of one span of a stage (pitch bytes apart) against the 8
// sequence slots, 16 rows per MMA tile: this warp's k-range in k-steps of two
// MMAs (high and low activation parts).  The warp's row sums land in each
// sequence's accumulator set, A + q * aset at [row][warp], as the CUDA-core
// consumers' do (the epilogue adds the 8 warps in order).
template <int KS>
__device__ __forceinline__ void stage_rows_tc(const unsigned char* Ws, uint32_t pitch, int nr, int K,
                                              const BFrag<KS>& bf, float* A, int aset, int nb, int lane, int warp) {
    const int g = lane >> 2, t = lane & 3, ksr = K / (16 * kConsumerWarps);
    const uint32_t col = (uint32_t)(warp * (K / kConsumerWarps) + (lane >> 4) * 8) * 2u;
    for (int m0 = 0; m0 < nr; m0 += 16) {
        // ldmatrix x4: matrices (rows m0..m0+7 | m0+8..m0+15) x (k 0..7 | 8..15); lane l gives row l % 16
        // (rows past nr read the last row; their sums are dropped)
        const int ar = m0 + (lane & 15) < nr ? m0 + (lane & 15) : nr - 1;
        const uint32_t base = smem_u32(Ws) + (uint32_t)ar * pitch + col;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            if (ks >= ksr) continue;  // (not break: the unrolled loop keeps static indices)
            uint32_t a0, a1, a2, a3;
            ldsm_x4(base + 32u * ks, a0, a1, a2, a3);
            mma_bf16(c, a0, a1, a2, a3, bf.hi[ks][0], bf.hi[ks][1]);
            mma_bf16(c, a0, a1, a2, a3, bf.lo[ks][0], bf.lo[ks][1]);
        }
        // c0, c1: row m0 + g, sequences 2t, 2t + 1; c2, c3: row m0 + g + 8
        const int q = 2 * t, w = warp;
        if (m0 + g < nr) {
            if (q < nb) A[(size_t)q * aset + (m0 + g) * kConsumerWarps + w] = c[0];
            if (q + 1 < nb) A[(size_t)(q + 1) * aset + (m0 + g) * kConsumerWarps + w] = c[1];
        }
        if (m0 + g + 8 < nr) {
            if (q < nb) A[(size_t)q * aset + (m0 + g + 8) * kConsumerWarps + w] = c[2];
            if (q + 1 < nb) A[(size_t)(q + 1) * aset + (m0 + g + 8) * kConsumerWarps + w] = c[3];
        }
    }
}

// Transposed down-projection rows [0, nr) of one stage (pitch bytes apart)
// into this warp's output columns: y[col][q] += sum_r Wt[r][col] h[r][q] for
// the warp's H/8 columns in MT tiles of 16 (A = Wt^T through ldmatrix.trans,
// B = h of 16 rows for the 8 sequence slots, high and low parts).  h holds the
// stage's rows at h[r * hstride + q], zero for unused sequences.
template <int MT>
__device__ __forceinline__ void down_rows_tc(const unsigned char* Ws, uint32_t pitch, int nr, int H, const float* h,
                                             int hstride, int nb, float (&y)[MT][4], int lane, int warp) {
    const int g = lane >> 2, t = lane & 3, mtr = H / (16 * kConsumerWarps);
    const uint32_t col = (uint32_t)(warp * (H / kConsumerWarps) + 8 * ((lane >> 3) & 1)) * 2u;
    for (int k0 = 0; k0 < nr; k0 += 16) {
        auto hv = [&](int r) { return (k0 + r < nr && g < nb) ? h[(size_t)(k0 + r) * hstride + g] : 0.f; };
        uint32_t bh0, bl0, bh1, bl1;
        split_pack(hv(2 * t), hv(2 * t + 1), bh0, bl0);
        split_pack(hv(2 * t + 8), hv(2 * t + 9), bh1, bl1);
        // ldmatrix.trans x4: matrices (cols 0..7 | 8..15) x (rows k0..k0+7 | k0+8..k0+15) of the stage;
        // lane l gives stage row k0 + l % 8 + 8 (l / 16) at column block 8 ((l / 8) % 2)
        const int r = k0 + (lane & 7) + 8 * (lane >> 4);
        const uint32_t base = smem_u32(Ws) + (uint32_t)(r < nr ? r : nr - 1) * pitch + col;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            if (mt >= mtr) continue;  // (not break: the unrolled loop keeps static indices)
            uint32_t a0, a1, a2, a3;
            ldsm_x4_trans(base + 32u * mt, a0, a1, a2, a3);
            mma_bf16(y[mt], a0, a1, a2, a3, bh0, bh1);
            mma_bf16(y[mt], a0, a1, a2, a3, bl0, bl1);
        }
    }
}

// Row sum r of accumulator set k (one per sequence and span): the 8 warps'
// partial sums in fixed order.
__device__ __forceinline__ float acc_row(const float* part_sums, int aset, int k, int r) {
    const float4* ps = reinterpret_cast<const float4*>(part_sums + (size_t)k * aset + (size_t)r * kConsumerWarps);
    const float4 x0 = ps[0], x1 = ps[1];
    return ((x0.x + x0.y) + (x0.z + x0.w)) + ((x1.x + x1.y) + (x1.z + x1.w));
}

// CUDA-core form of the batched GEMV (small batches, and the two-chunk kernels):
// RG rows [rg, rg + RG) of a stage against the sequences' input vectors: the
// rows' weights are loaded and widened to fp32 once, then every sequence's dot
// products reuse them (all NB, the unused ones against zero vectors, so the
// chains interleave); the NB x RG row sums are reduced across the warp in one
// transpose-reduce and stored in each sequence's accumulator set (A + q *
// aset, one slot per row and warp, added in warp order by the epilogue).  Rows
// at or past nr are predicated off.
template <int J, int RG, int NB>
__device__ __forceinline__ void rows_block_b(const uint4* __restrict__ Ws, int row16, int rg, int nr,
                                             const bool (&jv)[J], const float (&v)[NB][J][8], float* A, int aset,
                                             int nb, int lane) {
    const int tid = threadIdx.x;
    float wf[RG][J][8];
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
        for (int j = 0; j < J; ++j)
            unpack8((jv[j] && rg + r < nr) ? Ws[(rg + r) * row16 + tid + kConsumerThreads * j]
                                           : make_uint4(0u, 0u, 0u, 0u),
                    wf[r][j]);
    constexpr int N = NB * RG;  // index q * RG + r
    float part[N];
#pragma unroll
    for (int q = 0; q < NB; ++q)
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            float2 a = make_float2(0.f, 0.f);  // even / odd elements, two FMAs per instruction
#pragma unroll
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int k = 0; k < 8; k += 2)
                    a = fma2(make_float2(wf[r][j][k], wf[r][j][k + 1]), make_float2(v[q][j][k], v[q][j][k + 1]), a);
            part[q * RG + r] = a.x + a.y;
        }
    const float s = reduce_rows<N>(part, lane);
    const int idx = reduce_rows_lane_row<N>(lane), q = idx / RG, row = rg + idx % RG;
    if (reduce_rows_writer<N>(lane) && q < nb && row < nr)
        A[(size_t)q * aset + row * kConsumerWarps + (tid >> 5)] = s;
}

template <int J, int RG, int NB>
__device__ __forceinline__ void stage_rows_b(const uint4* __restrict__ Ws, int row16, int nr, int nch,
                                             const float (&v)[NB][J][8], float* A, int aset, int nb, int lane) {
    bool jv[J];
#pragma unroll
    for (int j = 0; j < J; ++j) jv[j] = (int)threadIdx.x + kConsumerThreads * j < nch;
    for (int rg = 0; rg < nr; rg += RG) rows_block_b<J, RG, NB>(Ws, row16, rg, nr, jv, v, A, aset, nb, lane);
}

// v[q] = rmsnorm(x_q) * w for the nb sequences of a batched step (x_q fp32 at
// x32 + q * H, or the bf16 embedding row of the sequence's token when
// from_embed): every sequence's slice and the norm weights are loaded before
// any is used, and the sequences' sums of squares share one block reduction.
// snap (optional): sequence q's un-normalised input is stored at snap + q * snap_stride.
template <int J, int NB>
__device__ void load_rms_b(const DevParams& p, Misc& m, const float* x32, bool from_embed, const uint16_t* nw,
                           float (&v)[NB][J][8], float* snap = nullptr, size_t snap_stride = 0) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, K = p.H, nch = K >> 3, nb = p.nb;
    uint4 wraw[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int c = tid + kConsumerThreads * j;
        wraw[j] = c < nch ? __ldg(reinterpret_cast<const uint4*>(nw) + c) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < NB; ++q)
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int c = tid + kConsumerThreads * j;
            if (q < nb && c < nch) {
                if (from_embed) {
                    unpack8(__ldg(reinterpret_cast<const uint4*>(p.embed + (size_t)m.btok[q] * K) + c), v[q][j]);
                } else {
                    const float4* src = reinterpret_cast<const float4*>(x32 + (size_t)q * K);
                    const float4 a0 = __ldcg(src + 2 * c), a1 = __ldcg(src + 2 * c + 1);
                    v[q][j][0] = a0.x; v[q][j][1] = a0.y; v[q][j][2] = a0.z; v[q][j][3] = a0.w;
                    v[q][j][4] = a1.x; v[q][j][5] = a1.y; v[q][j][6] = a1.z; v[q][j][7] = a1.w;
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[q][j][k] = 0.f;
            }
        }
    if (snap) {
#pragma unroll
        for (int q = 0; q < NB; ++q)
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int c = tid + kConsumerThreads * j;
                if (q < nb && c < nch) {
                    float4* dst = reinterpret_cast<float4*>(snap + (size_t)q * snap_stride);
                    dst[2 * c] = make_float4(v[q][j][0], v[q][j][1], v[q][j][2], v[q][j][3]);
                    dst[2 * c + 1] = make_float4(v[q][j][4], v[q][j][5], v[q][j][6], v[q][j][7]);
                }
            }
    }
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < J; ++j)
#pragma unroll
            for (int k = 0; k < 8; ++k) ss = fmaf(v[q][j][k], v[q][j][k], ss);
        ss = warp_sum(ss);
        if (lane == 0) m.bred[q * kConsumerWarps + warp] = ss;
    }
    cbar();
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) tot += m.bred[q * kConsumerWarps + w];
        const float rs = 1.0f / sqrtf(tot / (float)K + p.eps);
#pragma unroll
        for (int j = 0; j < J; ++j) {
            float wf[8];
            unpack8(wraw[j], wf);
#pragma unroll
            for (int k = 0; k < 8; ++k) v[q][j][k] = v[q][j][k] * rs * wf[k];
        }
    }
    cbar();  // m.bred free again
}

// The O-projection's input for the nb sequences of a batched step: the
// attention output of every query head, merged from its kv splits as in
// load_attn_merged, with the loads of QG sequences x SG splits issued together
// per round trip.
template <int J, int NB>
__device__ void load_attn_merged_b(const DevParams& p, int K, float (&v)[NB][J][8]) {
    constexpr int QG = NB < 4 ? NB : 4;        // sequences per round
    constexpr int SG = NB >= 8 ? 1 : 8 / QG;   // splits per round (QG x SG x 10 live floats)
    const int tid = threadIdx.x, nch = K >> 3, S = p.kv_splits, D = p.d, nb = p.nb;
    const size_t seq_ml = (size_t)p.nq * S * 2, seq_o = (size_t)p.nq * S * D;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int c = tid + kConsumerThreads * j;
        const int col = 8 * c, h = col / D, dc = col - h * D;
#pragma unroll
        for (int q0 = 0; q0 < NB; q0 += QG) {
            float M[QG], den[QG], acc[QG][8];
#pragma unroll
            for (int g = 0; g < QG; ++g) {
                M[g] = -CUDART_INF_F;
                den[g] = 0.f;
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[g][k] = 0.f;
            }
            const bool live = c < nch && q0 < nb;
            for (int s0 = 0; live && s0 < S; s0 += SG) {
                float2 t[QG][SG];
                float4 o0[QG][SG], o1[QG][SG];
#pragma unroll
                for (int g = 0; g < QG; ++g)
#pragma unroll
                    for (int k = 0; k < SG; ++k) {
                        if (q0 + g < nb && s0 + k < S) {
                            const float2* ml = reinterpret_cast<const float2*>(p.part_ml + (q0 + g) * seq_ml) +
                                               (size_t)h * S + s0 + k;
                            const float4* po = reinterpret_cast<const float4*>(
                                p.part_o + (q0 + g) * seq_o + ((size_t)h * S + s0 + k) * D + dc);
                            t[g][k] = __ldcg(ml);
                            o0[g][k] = __ldcg(po);
                            o1[g][k] = __ldcg(po + 1);
                        } else {
                            t[g][k] = make_float2(-CUDART_INF_F, 0.f);
                            o0[g][k] = o1[g][k] = make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                    }
#pragma unroll
                for (int g = 0; g < QG; ++g) {
                    float bm = M[g];
#pragma unroll
                    for (int k = 0; k < SG; ++k) bm = fmaxf(bm, t[g][k].x);
                    if (bm == -CUDART_INF_F) continue;  // no position in these splits yet
                    const float r = exp2f(M[g] - bm);
                    den[g] *= r;
#pragma unroll
                    for (int k = 0; k < 8; ++k) acc[g][k] *= r;
#pragma unroll
                    for (int k = 0; k < SG; ++k) {
                        const float f = exp2f(t[g][k].x - bm);
                        den[g] = fmaf(f, t[g][k].y, den[g]);
                        acc[g][0] = fmaf(f, o0[g][k].x, acc[g][0]);
                        acc[g][1] = fmaf(f, o0[g][k].y, acc[g][1]);
                        acc[g][2] = fmaf(f, o0[g][k].z, acc[g][2]);
                        acc[g][3] = fmaf(f, o0[g][k].w, acc[g][3]);
                        acc[g][4] = fmaf(f, o1[g][k].x, acc[g][4]);
                        acc[g][5] = fmaf(f, o1[g][k].y, acc[g][5]);
                        acc[g][6] = fmaf(f, o1[g][k].z, acc[g][6]);
                        acc[g][7] = fmaf(f, o1[g][k].w, acc[g][7]);
                    }
                    M[g] = bm;
                }
            }
#pragma unroll
            for (int g = 0; g < QG; ++g) {
                const bool ok = live && q0 + g < nb;
                const float inv = ok ? 1.0f / den[g] : 0.f;
#pragma unroll
                for (int k = 0; k < 8; ++k) v[q0 + g][j][k] = ok ? acc[g][k] * inv : 0.f;
            }
        }
    }
}

// Batched QKV, O-projection and LM head (one column part, one span): each
// stage of weights is applied to the nb sequences' input vectors before its
// slot is freed, and the epilogue writes every sequence's outputs.
template <int J, int NB>
__device__ bool gemv_instr_b(const DevParams& p, const StepArgs& a, const int32_t* w, int ii, unsigned char* ring,
                             uint64_t* full, uint64_t* empty, float* scratch, Misc& m, int& slot, uint32_t& phase) {
    constexpr int KS = J == 1 ? 16 : 24;  // k-steps of 16 columns per warp at the widest row (2048 or 3072)
    constexpr bool TCP = batch_on_tensor_cores(J, NB);
    constexpr int RG = J == 1 ? 4 : 2;    // CUDA-core form: rows per block
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nb = p.nb;
    const int op = w[W_OP], l = w[W_LAYER], sub = w[W_SUB], b = w[W_BEGIN], rows = w[W_END] - b;
    const uint32_t SB = (uint32_t)p.stage_bytes;
    const size_t H = (size_t)p.H;
    float* part_sums = scratch;  // [sequence][row of the chunk][8 warps]
    unsigned long long* tr = p.trace ? p.trace + ((size_t)blockIdx.x * p.max_instr + ii) * kTraceWords : nullptr;
    Plan pl;
    make_plan(p, a.pos, w, nullptr, pl);
    // The LM head's rows go through in chunks of whole stages whose partial sums fit the scratch
    // (its logits and argmax need no other rows); the other ops' rows fit in one chunk.
    const bool lm = op == OP_LMHEAD_ARGMAX;
    const int chunk = lm ? lm_chunk_rows(nb, pl.rps) : rows;
    const int aset = chunk * kConsumerWarps;
    float bv[NB];  // LM head: each sequence's best logit and its row over the chunks so far
    int bi[NB];
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        bv[q] = -CUDART_INF_F;
        bi[q] = 0x7FFFFFFF;
    }
    if (tid == 0 && w[W_WAIT_CTR] >= 0 &&
        !wait_counter(p, m, w[W_WAIT_CTR], a.epoch * (uint32_t)w[W_WAIT_INC], ii, op))
        vstore(&m.abort_flag, 1);
    if (tr && tid == 0) tr[T_DEP] = globaltimer_ns();
    cbar();
    if (vload(&m.abort_flag)) return false;

    // input vectors of the sequences: as the MMAs' B operand (tensor cores), or per thread chunk
    BFrag<KS> bf;
    float v[NB][J][8];
    const uint16_t* const* wt = p.wt + (size_t)(l < p.L ? l : 0) * wt_stride(p.E);
    const int K = op == OP_OPROJ_RES ? p.nq * p.d : p.H;
    const size_t snap_stride = (size_t)(p.L + 1) * H;
    if constexpr (!TCP) {
        if (op == OP_RMS_QKV)
            load_rms_b<J, NB>(p, m, p.x2, l == 0, wt[WT_ATTN_NORM], v,
                              (p.snap && l > 0 && sub == 0 && b == 0) ? p.snap + (size_t)l * H : nullptr,
                              snap_stride);
        else if (op == OP_LMHEAD_ARGMAX)
            load_rms_b<J, NB>(p, m, p.x2, p.L == 0, p.final_norm, v,
                              (p.snap && w[W_SEQ] == 0) ? p.snap + (size_t)p.L * H : nullptr, snap_stride);
        else
            load_attn_merged_b<J, NB>(p, K, v);
    } else if (op == OP_RMS_QKV) {
        rms_bfrag<KS>(p, m, p.x2, l == 0, wt[WT_ATTN_NORM], bf,
                      (p.snap && l > 0 && sub == 0 && b == 0) ? p.snap + (size_t)l * H : nullptr, snap_stride, lane,
                      warp);
    } else if (op == OP_LMHEAD_ARGMAX) {
        rms_bfrag<KS>(p, m, p.x2, p.L == 0, p.final_norm, bf,
                      (p.snap && w[W_SEQ] == 0) ? p.snap + (size_t)p.L * H : nullptr, snap_stride, lane, warp);
    } else {  // the merged attention output, through the CUDA-core layout
        load_attn_merged_b<J, NB>(p, K, v);
        to_bfrag<J, NB, KS>(v, K, scratch, bf, lane, warp);
    }
    if (tr && tid == 0) tr[T_READY] = globaltimer_ns();

    // stages
    for (int sst = 0; sst < pl.spp; ++sst) {
        const int r0 = sst * pl.rps;
        const int nr = (rows - r0) < pl.rps ? (rows - r0) : pl.rps;
        if (warp_wait_full(&full[slot], phase, p, m, ii, op)) {
            if (tid == 0) {
                if (tr && sst == 0) tr[T_FIRST] = globaltimer_ns();
                stage_stamp(tr, T_SREADY, sst);
            }
            if constexpr (TCP)
                stage_rows_tc<KS>(ring + (size_t)slot * SB, pl.pitch, nr, K, bf,
                                  part_sums + (size_t)(r0 % chunk) * kConsumerWarps, aset, nb, lane, warp);
            else
                stage_rows_b<J, RG, NB>(reinterpret_cast<const uint4*>(ring + (size_t)slot * SB), (int)(pl.pitch >> 4),
                                        nr, K >> 3, v, part_sums + (size_t)(r0 % chunk) * kConsumerWarps, aset, nb,
                                        lane);
            __syncwarp();
            if (tid == 0) stage_stamp(tr, T_SDONE, sst);
            if (lane == 0) mbar_arrive(&empty[slot]);
        } else if (tid == 0) {
            vstore(&m.abort_flag, 1);
        }
        if (++slot == p.ring_stages) {
            slot = 0;
            phase ^= 1u;
        }
        const int done = r0 + nr;
        if (lm && (done == rows || done % chunk == 0)) {  // a chunk of the LM head is complete
            const int c0 = (done - 1) / chunk * chunk, cn = done - c0;
            cbar();
            if (vload(&m.abort_flag)) return false;
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                if (q >= nb) continue;  // (not break: the unrolled loop keeps static indices)
                for (int r = tid; r < cn; r += kConsumerThreads) {
                    const float val = acc_row(part_sums, aset, q, r);
                    const int row = b + c0 + r;
                    a.logits[(size_t)q * p.V + row] = val;
                    if (val > bv[q]) {  // rows ascend for every thread: ties keep the lower row
                        bv[q] = val;
                        bi[q] = row;
                    }
                }
            }
            cbar();  // the scratch takes the next chunk
        }
    }
    cbar();
    if (vload(&m.abort_flag)) return false;
    if (tr && tid == 0) tr[T_MAIN] = globaltimer_ns();

    // epilogue
    if (op == OP_RMS_QKV) {
        const int qkvn = (p.nq + 2 * p.nkv) * p.d;
        const int off = sub == 0 ? 0 : (sub == 1 ? p.nq * p.d : (p.nq + p.nkv) * p.d);
        for (int q = 0; q < nb; ++q)
            for (int r = tid; r < rows; r += kConsumerThreads)
                p.qkv[(size_t)q * qkvn + off + b + r] = acc_row(part_sums, aset, q, r);
    } else if (op == OP_OPROJ_RES) {
        for (int r = tid; r < rows; r += kConsumerThreads) {
            float base[NB];
#pragma unroll
            for (int q = 0; q < NB; ++q) {  // every sequence's residual load first (one round trip)
                base[q] = 0.f;
                if (q < nb) {
                    if (l == 0)
                        base[q] = __uint_as_float((uint32_t)p.embed[(size_t)m.btok[q] * H + b + r] << 16);
                    else
                        base[q] = __ldcg(p.x2 + q * H + b + r);
                }
            }
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                if (q >= nb) continue;  // (not break: the unrolled loop keeps static indices)
                const size_t i = q * H + b + r;
                if (l == 0 && p.snap) p.snap[(size_t)q * (p.L + 1) * H + b + r] = base[q];
                const float nx = base[q] + acc_row(part_sums, aset, q, r);
                p.x[i] = nx;
                p.x2[i] = nx;
            }
        }
    } else {  // LM head: each sequence's argmax over this instruction's rows (logits written per chunk)
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            if (q >= nb) continue;
            warp_argmax(bv[q], bi[q]);
            if (lane == 0) {
                m.bred[q * kConsumerWarps + warp] = bv[q];
                m.bredi[q * kConsumerWarps + warp] = bi[q];
            }
        }
        cbar();
        if (tid == 0) {
            for (int q = 0; q < nb; ++q) {
                float cv = m.bred[q * kConsumerWarps];
                int ci = m.bredi[q * kConsumerWarps];
                for (int k = 1; k < kConsumerWarps; ++k) {
                    const float ov = m.bred[q * kConsumerWarps + k];
                    const int oi = m.bredi[q * kConsumerWarps + k];
                    if (ov > cv || (ov == cv && oi < ci)) {
                        cv = ov;
                        ci = oi;
                    }
                }
                const size_t slot_q = ((size_t)w[W_SEQ] * nb + q) * 2;
                p.lm_part[slot_q] = cv;
                p.lm_part[slot_q + 1] = __int_as_float(ci);
            }
            const uint32_t old = arrive_release(p.counters + w[W_AUX_CTR]);
            m.is_last = (old + 1u == a.epoch * (uint32_t)w[W_AUX_INC]) ? 1 : 0;
        }
        cbar();
        if (m.is_last) {  // the last LM-head instruction to finish picks every sequence's token
            const int n_lm = w[W_AUX_INC];
            for (int q = 0; q < nb; ++q) {
                float cv = -CUDART_INF_F;
                int ci = 0x7FFFFFFF;
                for (int k = tid; k < n_lm; k += kConsumerThreads) {
                    const float val = __ldcg(p.lm_part + ((size_t)k * nb + q) * 2);
                    const int idx = __float_as_int(__ldcg(p.lm_part + ((size_t)k * nb + q) * 2 + 1));
                    if (val > cv || (val == cv && idx < ci)) {
                        cv = val;
                        ci = idx;
                    }
                }
                warp_argmax(cv, ci);
                if (lane == 0) {
                    m.bred[q * kConsumerWarps + warp] = cv;
                    m.bredi[q * kConsumerWarps + warp] = ci;
                }
            }
            cbar();
            if (tid == 0) {
                for (int q = 0; q < nb; ++q) {
                    float cv = m.bred[q * kConsumerWarps];
                    int ci = m.bredi[q * kConsumerWarps];
                    for (int k = 1; k < kConsumerWarps; ++k) {
                        const float ov = m.bred[q * kConsumerWarps + k];
                        const int oi = m.bredi[q * kConsumerWarps + k];
                        if (ov > cv || (ov == cv && oi < ci)) {
                            cv = ov;
                            ci = oi;
                        }
                    }
                    p.next_tok[q] = ci;
                    if (q == 0) p.status->next_token = ci;
                }
            }
        }
    }
    cbar();
    if (tid == 0 && w[W_SIGNAL_CTR] >= 0 && op != OP_LMHEAD_ARGMAX) signal_release(p.counters + w[W_SIGNAL_CTR]);
    return true;
}

// Batched fused FFN slice (OP_FFN): rows [b, e) of the up/gate projections for
// every sequence (each stage applied to the nb input vectors), h per sequence
// and row, then the same rows of the transposed down-projection: each weight
// chunk is widened once and accumulated into every sequence's column chunks,
// which are added into the sequences' residuals with float4 atomics.
template <int J, int NB>
__device__ bool ffn_instr_b(const DevParams& p, const StepArgs& a, const int32_t* w, int ii, unsigned char* ring,
                            uint64_t* full, uint64_t* empty, float* scratch, Misc& m, int& slot, uint32_t& phase) {
    constexpr int KS = J == 1 ? 16 : 24;  // k-steps per warp (up/gate) and column tiles per warp (down) at the widest row
    constexpr bool TCP = batch_on_tensor_cores(J, NB);
    constexpr int RG = J == 1 ? 4 : 2;    // CUDA-core form: rows per block
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nb = p.nb;
    const int op = w[W_OP], l = w[W_LAYER], b = w[W_BEGIN], rows = w[W_END] - b;
    const uint32_t SB = (uint32_t)p.stage_bytes;
    const size_t H = (size_t)p.H;
    float* part_sums = scratch;  // [span][sequence < nb][row][8 warps]
    const int aset = rows * kConsumerWarps;
    unsigned long long* tr = p.trace ? p.trace + ((size_t)blockIdx.x * p.max_instr + ii) * kTraceWords : nullptr;
    Plan pl;
    make_plan(p, a.pos, w, nullptr, pl);
    if (tid == 0) {
        if (!wait_counter(p, m, w[W_WAIT_CTR], a.epoch * (uint32_t)w[W_WAIT_INC], ii, op)) vstore(&m.abort_flag, 1);
        else vstore(&m.ffn_go, route_key(a.epoch, l, p.L));  // the loader's gate
    }
    if (tr && tid == 0) tr[T_DEP] = globaltimer_ns();
    cbar();
    if (vload(&m.abort_flag)) return false;

    const uint16_t* const* wt = p.wt + (size_t)l * wt_stride(p.E);
    BFrag<KS> bf;
    float v[NB][J][8];
    if constexpr (TCP)
        rms_bfrag<KS>(p, m, p.x, false, wt[WT_FFN_NORM], bf, nullptr, 0, lane, warp);
    else
        load_rms_b<J, NB>(p, m, p.x, false, wt[WT_FFN_NORM], v);
    const int nch = p.H >> 3;
    if (tr && tid == 0) tr[T_READY] = globaltimer_ns();

    // up/gate rows (gate span, then up span, of each stage)
    for (int sst = 0; sst < pl.spp; ++sst) {
        const int r0 = sst * pl.rps;
        const int nr = (rows - r0) < pl.rps ? (rows - r0) : pl.rps;
        if (warp_wait_full(&full[slot], phase, p, m, ii, op)) {
            if (tid == 0) {
                if (tr && sst == 0) tr[T_FIRST] = globaltimer_ns();
                stage_stamp(tr, T_SREADY, sst);
            }
            const unsigned char* stage = ring + (size_t)slot * SB;
            for (int s = 0; s < 2; ++s) {
                float* A = part_sums + ((size_t)s * nb * rows + r0) * kConsumerWarps;
                if constexpr (TCP)
                    stage_rows_tc<KS>(stage + (size_t)s * pl.rps * pl.pitch, pl.pitch, nr, p.H, bf, A, aset, nb, lane,
                                      warp);
                else
                    stage_rows_b<J, RG, NB>(reinterpret_cast<const uint4*>(stage + (size_t)s * pl.rps * pl.pitch),
                                            (int)(pl.pitch >> 4), nr, nch, v, A, aset, nb, lane);
            }
            __syncwarp();
            if (tid == 0) stage_stamp(tr, T_SDONE, sst);
            if (lane == 0) mbar_arrive(&empty[slot]);
        } else if (tid == 0) {
            vstore(&m.abort_flag, 1);
        }
        if (++slot == p.ring_stages) {
            slot = 0;
            phase ^= 1u;
        }
    }
    cbar();
    if (vload(&m.abort_flag)) return false;
    if (tr && tid == 0) tr[T_MAIN] = globaltimer_ns();

    // h[q][r] = silu(g) * u, kept at the start of the scratch (after every thread read its sums)
    constexpr int HR = 2;  // rows per thread (rows <= 512)
    float hv[NB][HR];
#pragma unroll
    for (int q = 0; q < NB; ++q)
#pragma unroll
        for (int k = 0; k < HR; ++k) {
            const int r = tid + kConsumerThreads * k;
            hv[q][k] = 0.f;
            if (q < nb && r < rows) {
                const float g = acc_row(part_sums, aset, q, r);
                const float u = acc_row(part_sums, aset, nb + q, r);
                hv[q][k] = g / (1.0f + expf(-g)) * u;
            }
        }
    cbar();
#pragma unroll
    for (int q = 0; q < NB; ++q)
#pragma unroll
        for (int k = 0; k < HR; ++k) {
            const int r = tid + kConsumerThreads * k;
            if (r < rows) scratch[(size_t)r * NB + q] = hv[q][k];  // 0 for unused sequences
        }
    cbar();

    if constexpr (TCP) {
        // transposed down-projection rows on the tensor cores: this warp's columns of Wd[:, rows] h_q
        float y[KS][4];
    #pragma unroll
        for (int mt = 0; mt < KS; ++mt) y[mt][0] = y[mt][1] = y[mt][2] = y[mt][3] = 0.f;
        for (int tst = 0; tst < pl.tail_spp; ++tst) {
            const int r0 = tst * pl.tail_rps;
            const int nr = (rows - r0) < pl.tail_rps ? (rows - r0) : pl.tail_rps;
            if (warp_wait_full(&full[slot], phase, p, m, ii, op)) {
                if (tid == 0) stage_stamp(tr, T_SREADY, pl.spp + tst);
                down_rows_tc<KS>(ring + (size_t)slot * SB, pl.tail_pitch, nr, p.H, scratch + (size_t)r0 * NB, NB, nb, y,
                                 lane, warp);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
            } else if (tid == 0) {
                vstore(&m.abort_flag, 1);
            }
            if (++slot == p.ring_stages) {
                slot = 0;
                phase ^= 1u;
            }
        }
        cbar();
        if (vload(&m.abort_flag)) return false;
        // Into the residuals: the warps' tiles go through the scratch, as many sequences per pass as
        // fit, and leave as float4 atomics over contiguous columns.  Lane (g, t) holds, per tile mt,
        // columns c = 16 mt + g and c + 8 for sequences 2t and 2t + 1.
        {
            const int g = lane >> 2, t = lane & 3, mtr = p.H / (16 * kConsumerWarps);
            const int SP = kRowSlots * kConsumerWarps / p.H, H4 = p.H / 4;
            for (int p0 = 0; p0 < nb; p0 += SP) {
    #pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    if (mt >= mtr) continue;  // (not break: the unrolled loop keeps static indices)
                    const int c = warp * (p.H / kConsumerWarps) + 16 * mt + g;
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int q = 2 * t + (e & 1) - p0;
                        if (q >= 0 && q < SP) scratch[(size_t)q * H + c + 8 * (e >> 1)] = y[mt][e];
                    }
                }
                cbar();
                const int n4 = (nb - p0 < SP ? nb - p0 : SP) * H4;
                for (int i = tid; i < n4; i += kConsumerThreads) {
                    const int q = i / H4;
                    atomicAdd(reinterpret_cast<float4*>(p.x2 + (p0 + q) * H) + (i - q * H4),
                              reinterpret_cast<const float4*>(scratch)[i]);
                }
                cbar();
            }
        }
    } else {
        // transposed down-projection rows: this thread's column chunks of Wd[:, rows] h_q, every q
        float y[NB][J][8];
        bool jv[J];
    #pragma unroll
        for (int j = 0; j < J; ++j) jv[j] = tid + kConsumerThreads * j < nch;
    #pragma unroll
        for (int q = 0; q < NB; ++q)
    #pragma unroll
            for (int j = 0; j < J; ++j)
    #pragma unroll
                for (int k = 0; k < 8; ++k) y[q][j][k] = 0.f;
        for (int tst = 0; tst < pl.tail_spp; ++tst) {
            const int r0 = tst * pl.tail_rps;
            const int nr = (rows - r0) < pl.tail_rps ? (rows - r0) : pl.tail_rps;
            if (warp_wait_full(&full[slot], phase, p, m, ii, op)) {
                if (tid == 0) stage_stamp(tr, T_SREADY, pl.spp + tst);
                const uint4* Ws = reinterpret_cast<const uint4*>(ring + (size_t)slot * SB);
                const int tpitch16 = (int)(pl.tail_pitch >> 4);
                // two rows per iteration (the unused sequences' h are zero)
                for (int r = 0; r < nr; r += 2) {
                    float f[2][J][8], hk[2][NB];
    #pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const bool live = r + u < nr;
    #pragma unroll
                        for (int j = 0; j < J; ++j)
                            unpack8((live && jv[j]) ? Ws[(r + u) * tpitch16 + tid + kConsumerThreads * j]
                                                    : make_uint4(0u, 0u, 0u, 0u),
                                    f[u][j]);
    #pragma unroll
                        for (int q = 0; q < NB; ++q) hk[u][q] = live ? scratch[(size_t)(r0 + r + u) * NB + q] : 0.f;
                    }
    #pragma unroll
                    for (int u = 0; u < 2; ++u)
    #pragma unroll
                        for (int q = 0; q < NB; ++q)
    #pragma unroll
                            for (int j = 0; j < J; ++j)
    #pragma unroll
                                for (int k = 0; k < 8; k += 2) {
                                    const float2 t = fma2(make_float2(f[u][j][k], f[u][j][k + 1]),
                                                          make_float2(hk[u][q], hk[u][q]),
                                                          make_float2(y[q][j][k], y[q][j][k + 1]));
                                    y[q][j][k] = t.x;
                                    y[q][j][k + 1] = t.y;
                                }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
            } else if (tid == 0) {
                vstore(&m.abort_flag, 1);
            }
            if (++slot == p.ring_stages) {
                slot = 0;
                phase ^= 1u;
            }
        }
        cbar();
        if (vload(&m.abort_flag)) return false;
    #pragma unroll
        for (int q = 0; q < NB; ++q) {
            if (q >= nb) continue;
    #pragma unroll
            for (int j = 0; j < J; ++j) {
                if (!jv[j]) continue;
                float4* dst = reinterpret_cast<float4*>(p.x2 + q * H) + 2 * (tid + kConsumerThreads * j);
                atomicAdd(dst, make_float4(y[q][j][0], y[q][j][1], y[q][j][2], y[q][j][3]));
                atomicAdd(dst + 1, make_float4(y[q][j][4], y[q][j][5], y[q][j][6], y[q][j][7]));
            }
        }
    }
    cbar();
    if (tid == 0) signal_release(p.counters + w[W_SIGNAL_CTR]);
    return true;
}

// ---------------------------------------------------------------------------
// consumers: attention (RoPE + append + one split of GQA decode attention)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ml_combine(float& m, float& l, float* o, float m2, float l2, const float* o2) {
    const float M = fmaxf(m, m2);
    if (M == -CUDART_INF_F) return;
    const float a = exp2f(m - M), b = exp2f(m2 - M);
    l = a * l + b * l2;
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = a * o[k] + b * o2[k];
    m = M;
}

// End of an attention split whose partials are written: signal the attention
// counter.  With W_MERGE the split also counts itself on its kv head's arrival
// counter; the last of the S splits to arrive merges the S partials of each of
// the kv head's G query heads (the rescaled combination that load_attn_merged
// computes in the O-projection otherwise) and writes the attention output to
// p.attn before it signals.  The other splits signal at once, so the counter
// still completes only once every head's output is final.  One thread per two
// adjacent columns (G * head_dim / 2 <= 256), 16 splits per round trip.
__device__ void attn_finish(const DevParams& p, const StepArgs& a, const int32_t* w, Misc& m, int sq, int l,
                            int g, int G, int S, int D) {
    const int tid = threadIdx.x;
    uint32_t* ctr = p.counters + w[W_SIGNAL_CTR];
    cbar();
    if (!w[W_MERGE]) {
        if (tid == 0) signal_release(ctr);
        return;
    }
    if (tid == 0) {
        const uint32_t old = arrive_release(p.attn_arrive + ((size_t)sq * p.L + l) * p.nkv + g);
        const int last = old + 1u == a.epoch * (uint32_t)S;
        if (!last) signal_release(ctr);
        m.is_last = last;
    }
    cbar();
    if (!m.is_last) return;
    constexpr int B = 16;
    if (tid < G * D / 2) {
        const int h = (2 * tid) / D, col = 2 * tid - h * D;
        const size_t base = (size_t)sq * p.nq * S + (size_t)(g * G + h) * S;  // partial slot of split 0
        const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + base;
        const float2* po = reinterpret_cast<const float2*>(p.part_o + base * D + col);
        const int D2 = D >> 1;
        float M = -CUDART_INF_F, den = 0.f, acc0 = 0.f, acc1 = 0.f;
        for (int s0 = 0; s0 < S; s0 += B) {
            float2 t[B], o[B];
#pragma unroll
            for (int k = 0; k < B; ++k) {
                if (s0 + k < S) {
                    t[k] = __ldcg(ml + s0 + k);
                    o[k] = __ldcg(po + (size_t)(s0 + k) * D2);
                } else {
                    t[k] = make_float2(-CUDART_INF_F, 0.f);
                    o[k] = make_float2(0.f, 0.f);
                }
            }
            float bm = M;
#pragma unroll
            for (int k = 0; k < B; ++k) bm = fmaxf(bm, t[k].x);
            if (bm == -CUDART_INF_F) continue;  // no position in these splits
            const float r = exp2f(M - bm);
            den *= r;
            acc0 *= r;
            acc1 *= r;
#pragma unroll
            for (int k = 0; k < B; ++k) {
                const float f = exp2f(t[k].x - bm);
                den = fmaf(f, t[k].y, den);
                acc0 = fmaf(f, o[k].x, acc0);
                acc1 = fmaf(f, o[k].y, acc1);
            }
            M = bm;
        }
        const float inv = 1.0f / den;
        *reinterpret_cast<float2*>(p.attn + (size_t)sq * p.nq * D + (size_t)(g * G + h) * D + col) =
            make_float2(acc0 * inv, acc1 * inv);
    }
    cbar();
    if (tid == 0) signal_release(ctr);
}

// CUDA-core split attention (the general and head_dim-128 kernels): query
// heads are split between the two halves of the consumer warps (each half owns
// at most 2 of the kv head's query heads and streams every K/V row of the stage
// for them), which keeps the per-thread q and output accumulators to 2 x 8 +
// 2 x 8 registers.  The stage holds K then V rows, contiguous (bulk copies).
template <int NB>
__device__ bool attn_cc(const DevParams& p, const StepArgs& a, const int32_t* w, int ii, unsigned char* ring,
                           uint64_t* full, uint64_t* empty, float* scratch, Misc& m, int& slot, uint32_t& phase) {
    const int D = p.d;                                  // head_dim, 64 or 128
    const int LPR = D / 8;                              // lanes per K/V row, 8 columns each
    constexpr int GW = 2;                               // head slots per set
    constexpr int AR = 4;                               // K/V rows per lane group per pass
    constexpr int SET_THREADS = kConsumerThreads / 2;
    constexpr int SET_WARPS = kConsumerWarps / 2;
    const int RGN = SET_THREADS / LPR;                  // rows per pass of a set
    const int G = p.nq / p.nkv;                         // query heads per kv head (1..4)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int set = warp / SET_WARPS;
    const int stid = tid - set * SET_THREADS;
    const int h0 = set * GW;                            // first query head (within the group) of this set
    const int l = w[W_LAYER], g = w[W_SUB], c = w[W_BEGIN], S = w[W_END];
    // batched decode: the instruction's sequence (its position, projections, cache and partials)
    const int sq = NB > 1 ? w[W_SEQ] : 0;
    const int pos = NB > 1 ? m.bpos[sq] : a.pos;
    const float* qkv_s = p.qkv + (size_t)sq * (p.nq + 2 * p.nkv) * p.d;
    uint16_t* kc_s = p.kcache + (size_t)sq * p.kv_seq_stride;
    uint16_t* vc_s = p.vcache + (size_t)sq * p.kv_seq_stride;
    float* part_o_s = p.part_o + (size_t)sq * p.nq * p.kv_splits * p.d;
    float* part_ml_s = p.part_ml + (size_t)sq * p.nq * p.kv_splits * 2;
    const uint32_t SB = (uint32_t)p.stage_bytes;
    const AttnRange rg = attn_range(pos, c, S);
    unsigned long long* tr = p.trace ? p.trace + ((size_t)blockIdx.x * p.max_instr + ii) * kTraceWords : nullptr;
    Plan pl;  // stage plan (weights only: computed while the dependency is still pending)
    make_plan(p, pos, w, nullptr, pl);

    if (tid == 0) {
        if (!wait_counter(p, m, w[W_WAIT_CTR], a.epoch * (uint32_t)w[W_WAIT_INC], ii, OP_ATTN))
            vstore(&m.abort_flag, 1);
        if (tr) tr[T_DEP] = globaltimer_ns();
    }
    cbar();
    if (vload(&m.abort_flag)) return false;

    // Prologue loads, all issued before any is used (one round trip): this
    // thread's 8 columns (and their rotate-half partners) of q for the set's
    // heads, of the new k and v, and the RoPE cos/sin of this position.
    const int col0 = (stid % LPR) * 8;
    const int pcol = col0 ^ (D / 2);
    const bool first_half = col0 < D / 2;
    const float qscale = 1.4426950408889634f / sqrtf((float)D);
    const float4* rp4 = reinterpret_cast<const float4*>(p.rope + (size_t)pos * (D / 2) + (col0 & (D / 2 - 1)));
    const float* ks = qkv_s + (size_t)p.nq * D + (size_t)g * D;
    const float* vs = qkv_s + (size_t)(p.nq + p.nkv) * D + (size_t)g * D;
    float4 qx[GW][2], qy[GW][2], rc[4], kx[2], ky[2], vx[2];
#pragma unroll
    for (int hh = 0; hh < GW; ++hh) {
        const int h = h0 + hh < G ? h0 + hh : G - 1;  // spare head slots compute a copy that is never stored
        const float4* src = reinterpret_cast<const float4*>(qkv_s + (size_t)(g * G + h) * D);
        qx[hh][0] = __ldcg(src + col0 / 4);
        qx[hh][1] = __ldcg(src + col0 / 4 + 1);
        qy[hh][0] = __ldcg(src + pcol / 4);
        qy[hh][1] = __ldcg(src + pcol / 4 + 1);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) rc[k] = __ldg(rp4 + k);
    kx[0] = __ldcg(reinterpret_cast<const float4*>(ks + col0));
    kx[1] = __ldcg(reinterpret_cast<const float4*>(ks + col0) + 1);
    ky[0] = __ldcg(reinterpret_cast<const float4*>(ks + pcol));
    ky[1] = __ldcg(reinterpret_cast<const float4*>(ks + pcol) + 1);
    vx[0] = __ldcg(reinterpret_cast<const float4*>(vs + col0));
    vx[1] = __ldcg(reinterpret_cast<const float4*>(vs + col0) + 1);
    float cs[8], sn[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        cs[2 * k] = rc[k].x;
        sn[2 * k] = rc[k].y;
        cs[2 * k + 1] = rc[k].z;
        sn[2 * k + 1] = rc[k].w;
    }
    // rotate-half RoPE of one 8-column slice: x' = x cos - y sin (first half), x cos + y sin (second)
    auto rope8 = [&](const float4 (&x)[2], const float4 (&y)[2], float scale, float* out) {
        const float xv[8] = {x[0].x, x[0].y, x[0].z, x[0].w, x[1].x, x[1].y, x[1].z, x[1].w};
        const float yv[8] = {y[0].x, y[0].y, y[0].z, y[0].w, y[1].x, y[1].y, y[1].z, y[1].w};
#pragma unroll
        for (int k = 0; k < 8; ++k)
            out[k] = (first_half ? xv[k] * cs[k] - yv[k] * sn[k] : xv[k] * cs[k] + yv[k] * sn[k]) * scale;
    };
    float q[GW][8];
#pragma unroll
    for (int hh = 0; hh < GW; ++hh) rope8(qx[hh], qy[hh], qscale, q[hh]);

    // the new position: rotated k and v rounded to bf16 (the cache format); the
    // first row group of each set holds it, set 0 appends it to the cache
    float kn[8], vn[8];
    const bool new_rows = rg.has_new && stid < 32;  // first warp of each set
    {
        float kr[8];
        rope8(kx, ky, 1.0f, kr);
        const float vv[8] = {vx[0].x, vx[0].y, vx[0].z, vx[0].w, vx[1].x, vx[1].y, vx[1].z, vx[1].w};
        uint32_t kb[8], vb[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            kb[k] = f2bf(kr[k]);
            vb[k] = f2bf(vv[k]);
            kn[k] = __uint_as_float(kb[k] << 16);
            vn[k] = __uint_as_float(vb[k] << 16);
        }
        if (new_rows && set == 0 && stid < LPR) {
            const size_t off = (((size_t)l * p.nkv + g) * (size_t)p.max_seq + (size_t)pos) * D + col0;
            uint4 ku, vu;
            ku.x = kb[0] | (kb[1] << 16); ku.y = kb[2] | (kb[3] << 16); ku.z = kb[4] | (kb[5] << 16); ku.w = kb[6] | (kb[7] << 16);
            vu.x = vb[0] | (vb[1] << 16); vu.y = vb[2] | (vb[3] << 16); vu.z = vb[4] | (vb[5] << 16); vu.w = vb[6] | (vb[7] << 16);
            *reinterpret_cast<uint4*>(kc_s + off) = ku;
            *reinterpret_cast<uint4*>(vc_s + off) = vu;
        }
    }

    if (tr && tid == 0) tr[T_READY] = globaltimer_ns();

    // online softmax over the cached positions streamed through the ring
    float mx[GW], ls[GW], o[GW][8];
#pragma unroll
    for (int hh = 0; hh < GW; ++hh) {
        mx[hh] = -CUDART_INF_F;
        ls[hh] = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) o[hh][k] = 0.f;
    }
    auto row_update = [&](const float* kf, const float* vf, bool valid) {
        float sc[GW];
#pragma unroll
        for (int hh = 0; hh < GW; ++hh) {
            float t0 = 0.f, t1 = 0.f;
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
                t0 = fmaf(q[hh][k], kf[k], t0);
                t1 = fmaf(q[hh][k + 1], kf[k + 1], t1);
            }
            sc[hh] = t0 + t1;
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1)
#pragma unroll
            for (int hh = 0; hh < GW; ++hh) sc[hh] += __shfl_xor_sync(0xFFFFFFFFu, sc[hh], off);
        if (valid) {
#pragma unroll
            for (int hh = 0; hh < GW; ++hh) {
                const float mn = fmaxf(mx[hh], sc[hh]);
                const float al = exp2f(mx[hh] - mn), pr = exp2f(sc[hh] - mn);
                ls[hh] = ls[hh] * al + pr;
#pragma unroll
                for (int k = 0; k < 8; ++k) o[hh][k] = fmaf(pr, vf[k], o[hh][k] * al);
                mx[hh] = mn;
            }
        }
    };

    for (int st = 0; st < pl.n_stages; ++st) {
        const int r0 = st * pl.rps;
        const int nr = (pl.rows - r0) < pl.rps ? (pl.rows - r0) : pl.rps;
        const bool ok = warp_wait_full(&full[slot], phase, p, m, ii, OP_ATTN);
        if (tr && tid == 0 && st == 0) tr[T_FIRST] = globaltimer_ns();
        if (tid == 0) stage_stamp(tr, T_SREADY, st);
        if (ok) {
            const uint4* Ks = reinterpret_cast<const uint4*>(ring + (size_t)slot * SB);
            const uint4* Vs = Ks + (size_t)pl.rps * (D / 8);
            // AR rows per lane group per pass: their scores are independent, and
            // the running max / rescale is taken once per pass instead of per row
            for (int base = 0; base < nr; base += RGN * AR) {
                uint4 kw[AR], vw[AR];
                bool valid[AR];
#pragma unroll
                for (int i = 0; i < AR; ++i) {
                    const int r = base + i * RGN + stid / LPR;
                    valid[i] = r < nr;
                    const int rr = valid[i] ? r : 0;
                    kw[i] = Ks[rr * (D / 8) + col0 / 8];
                    vw[i] = Vs[rr * (D / 8) + col0 / 8];
                }
                float sc[AR][GW];
#pragma unroll
                for (int i = 0; i < AR; ++i) {
                    float kf[8];
                    unpack8(kw[i], kf);
#pragma unroll
                    for (int hh = 0; hh < GW; ++hh) {
                        float t0 = 0.f, t1 = 0.f;
#pragma unroll
                        for (int k = 0; k < 8; k += 2) {
                            t0 = fmaf(q[hh][k], kf[k], t0);
                            t1 = fmaf(q[hh][k + 1], kf[k + 1], t1);
                        }
                        sc[i][hh] = t0 + t1;
                    }
                }
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1)
#pragma unroll
                    for (int i = 0; i < AR; ++i)
#pragma unroll
                        for (int hh = 0; hh < GW; ++hh) sc[i][hh] += __shfl_xor_sync(0xFFFFFFFFu, sc[i][hh], off);
#pragma unroll
                for (int hh = 0; hh < GW; ++hh) {
                    float mn = mx[hh];
#pragma unroll
                    for (int i = 0; i < AR; ++i)
                        if (valid[i]) mn = fmaxf(mn, sc[i][hh]);
                    if (mn == -CUDART_INF_F) continue;  // no valid row in this pass
                    const float al = exp2f(mx[hh] - mn);
                    float pr[AR];
                    float psum = 0.f;
#pragma unroll
                    for (int i = 0; i < AR; ++i) {
                        pr[i] = valid[i] ? exp2f(sc[i][hh] - mn) : 0.f;
                        psum += pr[i];
                    }
                    ls[hh] = fmaf(ls[hh], al, psum);
#pragma unroll
                    for (int k = 0; k < 8; ++k) o[hh][k] *= al;
#pragma unroll
                    for (int i = 0; i < AR; ++i) {
                        float vf[8];
                        unpack8(vw[i], vf);
#pragma unroll
                        for (int k = 0; k < 8; ++k) o[hh][k] = fmaf(pr[i], vf[k], o[hh][k]);
                    }
                    mx[hh] = mn;
                }
            }
            __syncwarp();
            if (tid == 0) stage_stamp(tr, T_SDONE, st);
            if (lane == 0) mbar_arrive(&empty[slot]);
        } else if (tid == 0) {
            vstore(&m.abort_flag, 1);
        }
        if (++slot == p.ring_stages) {
            slot = 0;
            phase ^= 1u;
        }
    }
    if (new_rows) row_update(kn, vn, lane < LPR);
    if (tr && tid == 0) tr[T_MAIN] = globaltimer_ns();

    // merge row groups within the warp, then the set's warps through shared memory
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
        for (int hh = 0; hh < GW; ++hh) {
            const float m2 = __shfl_xor_sync(0xFFFFFFFFu, mx[hh], off);
            const float l2 = __shfl_xor_sync(0xFFFFFFFFu, ls[hh], off);
            float o2[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) o2[k] = __shfl_xor_sync(0xFFFFFFFFu, o[hh][k], off);
            ml_combine(mx[hh], ls[hh], o[hh], m2, l2, o2);
        }
    }
    float* sm_o = scratch;                          // [8 warps][GW][D]
    float* sm_ml = scratch + kConsumerWarps * 512;  // [8 warps][GW][2]
    cbar();
    if (lane < LPR) {
#pragma unroll
        for (int hh = 0; hh < GW; ++hh) {
#pragma unroll
            for (int k = 0; k < 8; ++k) sm_o[(warp * GW + hh) * D + col0 + k] = o[hh][k];
            if (lane == 0) {
                sm_ml[(warp * GW + hh) * 2] = mx[hh];
                sm_ml[(warp * GW + hh) * 2 + 1] = ls[hh];
            }
        }
    }
    cbar();
    if (vload(&m.abort_flag)) return false;
    for (int idx = tid; idx < G * D; idx += kConsumerThreads) {
        const int h = idx / D, col = idx % D;
        const int hs = h / GW, hh = h % GW;  // owning set and head slot
        float M = -CUDART_INF_F;
        for (int wv = hs * SET_WARPS; wv < (hs + 1) * SET_WARPS; ++wv) M = fmaxf(M, sm_ml[(wv * GW + hh) * 2]);
        float O = 0.f, Ls = 0.f;
        if (M != -CUDART_INF_F) {
            for (int wv = hs * SET_WARPS; wv < (hs + 1) * SET_WARPS; ++wv) {
                const float f = exp2f(sm_ml[(wv * GW + hh) * 2] - M);
                O += f * sm_o[(wv * GW + hh) * D + col];
                Ls += f * sm_ml[(wv * GW + hh) * 2 + 1];
            }
        }
        const size_t part = (size_t)(g * G + h) * S + c;
        part_o_s[part * D + col] = O;
        if (col == 0) {
            part_ml_s[part * 2] = M;
            part_ml_s[part * 2 + 1] = Ls;
        }
    }
    attn_finish(p, a, w, m, sq, l, g, G, S, D);
    return true;
}

// Tensor-core split attention (the head_dim-64 kernel).  DH: head_dim fixed at
// compile time.  The stage holds K then V rows in 128-byte-swizzled tensor-map
// boxes.
template <int DH, int NB>
__device__ bool attn_tc(const DevParams& p, const StepArgs& a, const int32_t* w, int ii, unsigned char* ring,
                           uint64_t* full, uint64_t* empty, float* scratch, Misc& m, int& slot, uint32_t& phase) {
    constexpr int DMAX = DH > 0 ? DH : kMaxHeadDim;
    const int D = DH > 0 ? DH : p.d;                    // head_dim, 64 or 128
    const int LPR = D / 8;                              // lanes per K/V row, 8 columns each
    constexpr int GW = 2;                               // head slots per set
    constexpr int SET_THREADS = kConsumerThreads / 2;
    constexpr int SET_WARPS = kConsumerWarps / 2;
    const int G = p.nq / p.nkv;                         // query heads per kv head (1..4)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int set = warp / SET_WARPS;
    const int stid = tid - set * SET_THREADS;
    const int h0 = set * GW;                            // first query head (within the group) of this set
    const int l = w[W_LAYER], g = w[W_SUB], c = w[W_BEGIN], S = w[W_END];
    // batched decode: the instruction's sequence (its position, projections, cache and partials)
    const int sq = NB > 1 ? w[W_SEQ] : 0;
    const int pos = NB > 1 ? m.bpos[sq] : a.pos;
    const float* qkv_s = p.qkv + (size_t)sq * (p.nq + 2 * p.nkv) * p.d;
    uint16_t* kc_s = p.kcache + (size_t)sq * p.kv_seq_stride;
    uint16_t* vc_s = p.vcache + (size_t)sq * p.kv_seq_stride;
    float* part_o_s = p.part_o + (size_t)sq * p.nq * p.kv_splits * p.d;
    float* part_ml_s = p.part_ml + (size_t)sq * p.nq * p.kv_splits * 2;
    const uint32_t SB = (uint32_t)p.stage_bytes;
    const AttnRange rg = attn_range(pos, c, S);
    unsigned long long* tr = p.trace ? p.trace + ((size_t)blockIdx.x * p.max_instr + ii) * kTraceWords : nullptr;
    Plan pl;  // stage plan (weights only: computed while the dependency is still pending)
    make_plan(p, pos, w, nullptr, pl);

    if (tid == 0) {
        if (!wait_counter(p, m, w[W_WAIT_CTR], a.epoch * (uint32_t)w[W_WAIT_INC], ii, OP_ATTN))
            vstore(&m.abort_flag, 1);
        if (tr) tr[T_DEP] = globaltimer_ns();
    }
    cbar();
    if (vload(&m.abort_flag)) return false;

    // Prologue loads, all issued before any is used (one round trip): this
    // thread's 8 columns (and their rotate-half partners) of q for the set's
    // heads, of the new k and v, and the RoPE cos/sin of this position.
    const int col0 = (stid % LPR) * 8;
    const int pcol = col0 ^ (D / 2);
    const bool first_half = col0 < D / 2;
    const float qscale = 1.4426950408889634f / sqrtf((float)D);
    const float4* rp4 = reinterpret_cast<const float4*>(p.rope + (size_t)pos * (D / 2) + (col0 & (D / 2 - 1)));
    const float* ks = qkv_s + (size_t)p.nq * D + (size_t)g * D;
    const float* vs = qkv_s + (size_t)(p.nq + p.nkv) * D + (size_t)g * D;
    float4 qx[GW][2], qy[GW][2], rc[4], kx[2], ky[2], vx[2];
#pragma unroll
    for (int hh = 0; hh < GW; ++hh) {
        const int h = h0 + hh < G ? h0 + hh : G - 1;  // spare head slots compute a copy that is never stored
        const float4* src = reinterpret_cast<const float4*>(qkv_s + (size_t)(g * G + h) * D);
        qx[hh][0] = __ldcg(src + col0 / 4);
        qx[hh][1] = __ldcg(src + col0 / 4 + 1);
        qy[hh][0] = __ldcg(src + pcol / 4);
        qy[hh][1] = __ldcg(src + pcol / 4 + 1);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) rc[k] = __ldg(rp4 + k);
    kx[0] = __ldcg(reinterpret_cast<const float4*>(ks + col0));
    kx[1] = __ldcg(reinterpret_cast<const float4*>(ks + col0) + 1);
    ky[0] = __ldcg(reinterpret_cast<const float4*>(ks + pcol));
    ky[1] = __ldcg(reinterpret_cast<const float4*>(ks + pcol) + 1);
    vx[0] = __ldcg(reinterpret_cast<const float4*>(vs + col0));
    vx[1] = __ldcg(reinterpret_cast<const float4*>(vs + col0) + 1);
    float cs[8], sn[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        cs[2 * k] = rc[k].x;
        sn[2 * k] = rc[k].y;
        cs[2 * k + 1] = rc[k].z;
        sn[2 * k + 1] = rc[k].w;
    }
    // rotate-half RoPE of one 8-column slice: x' = x cos - y sin (first half), x cos + y sin (second)
    auto rope8 = [&](const float4 (&x)[2], const float4 (&y)[2], float scale, float* out) {
        const float xv[8] = {x[0].x, x[0].y, x[0].z, x[0].w, x[1].x, x[1].y, x[1].z, x[1].w};
        const float yv[8] = {y[0].x, y[0].y, y[0].z, y[0].w, y[1].x, y[1].y, y[1].z, y[1].w};
#pragma unroll
        for (int k = 0; k < 8; ++k)
            out[k] = (first_half ? xv[k] * cs[k] - yv[k] * sn[k] : xv[k] * cs[k] + yv[k] * sn[k]) * scale;
    };
    float q[GW][8];
#pragma unroll
    for (int hh = 0; hh < GW; ++hh) rope8(qx[hh], qy[hh], qscale, q[hh]);

    // the new position: rotated k and v rounded to bf16 (the cache format); the
    // first row group of each set holds it, set 0 appends it to the cache
    float kn[8], vn[8];
    const bool new_rows = rg.has_new && stid < 32;  // first warp of each set
    {
        float kr[8];
        rope8(kx, ky, 1.0f, kr);
        const float vv[8] = {vx[0].x, vx[0].y, vx[0].z, vx[0].w, vx[1].x, vx[1].y, vx[1].z, vx[1].w};
        uint32_t kb[8], vb[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            kb[k] = f2bf(kr[k]);
            vb[k] = f2bf(vv[k]);
            kn[k] = __uint_as_float(kb[k] << 16);
            vn[k] = __uint_as_float(vb[k] << 16);
        }
        if (new_rows && set == 0 && stid < LPR) {
            const size_t off = (((size_t)l * p.nkv + g) * (size_t)p.max_seq + (size_t)pos) * D + col0;
            uint4 ku, vu;
            ku.x = kb[0] | (kb[1] << 16); ku.y = kb[2] | (kb[3] << 16); ku.z = kb[4] | (kb[5] << 16); ku.w = kb[6] | (kb[7] << 16);
            vu.x = vb[0] | (vb[1] << 16); vu.y = vb[2] | (vb[3] << 16); vu.z = vb[4] | (vb[5] << 16); vu.w = vb[6] | (vb[7] << 16);
            *reinterpret_cast<uint4*>(kc_s + off) = ku;
            *reinterpret_cast<uint4*>(vc_s + off) = vu;
        }
    }

    // q (rotated, scaled) of every head of the group and the new k, v to shared
    // memory: the tensor-core loop below takes its fragments from there
    float* sm_o = scratch;                           // [8 warps][4][D]  per-warp outputs
    float* sm_ml = scratch + kConsumerWarps * 512;   // [8 warps][4][2]  per-warp (max, sum)
    float* sm_q = scratch + kConsumerWarps * 512 + 256;  // [4][D]
    float* sm_kv = sm_q + 4 * kMaxHeadDim;               // [2][D] new k, v (bf16 values)
    if (stid < LPR) {
#pragma unroll
        for (int hh = 0; hh < GW; ++hh)
            if (h0 + hh < G)
#pragma unroll
                for (int k = 0; k < 8; ++k) sm_q[(h0 + hh) * D + col0 + k] = q[hh][k];
        if (set == 0)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                sm_kv[col0 + k] = kn[k];
                sm_kv[D + col0 + k] = vn[k];
            }
    }
    cbar();
    if (tr && tid == 0) tr[T_READY] = globaltimer_ns();

    // Tensor-core split attention (mma m16n8k16, bf16 operands, fp32 accumulate).
    // Row r = lane/4 of the 16-row operand is head r & 3, the high (r < 4) or low
    // (r >= 4) bf16 part of q or of the probabilities, so hi + lo keeps fp32
    // accuracy; rows 8..15 are zero.  Each warp takes 16-position tiles w, w+8, ...
    // of every stage with its own online softmax (log2 domain); warps merge at the end.
    const int g4 = lane >> 2, t4 = lane & 3;
    const int hrow = g4 & 3;
    const bool lo_row = g4 >= 4, real = hrow < G;
    const int KS = D / 16, NT = D / 8;
    uint32_t qa[DMAX / 16][2];
#pragma unroll
    for (int kk = 0; kk < DMAX / 16; ++kk) {
        qa[kk][0] = qa[kk][1] = 0u;
        if (kk < KS && real) {
            float x[4];
            const float* qr = sm_q + hrow * D + kk * 16 + 2 * t4;
            x[0] = qr[0]; x[1] = qr[1]; x[2] = qr[8]; x[3] = qr[9];
            uint32_t h16[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t hi = f2bf(x[k]);
                h16[k] = lo_row ? f2bf(x[k] - __uint_as_float(hi << 16)) : hi;
            }
            qa[kk][0] = h16[0] | (h16[1] << 16);
            qa[kk][1] = h16[2] | (h16[3] << 16);
        }
    }
    float m_run = -CUDART_INF_F, l_run = 0.f;
    float oacc[DMAX / 8][2];  // rows 0..7 of each 8-column output tile (this lane: row g4, 2 columns)
#pragma unroll
    for (int nt = 0; nt < DMAX / 8; ++nt) oacc[nt][0] = oacc[nt][1] = 0.f;

    const int lm_i = lane >> 3, lm_j = lane & 7;  // ldmatrix: matrix index, row within it
    for (int st = 0; st < pl.n_stages; ++st) {
        const int r0 = st * pl.rps;
        const int nr = (pl.rows - r0) < pl.rps ? (pl.rows - r0) : pl.rps;
        const bool ok = warp_wait_full(&full[slot], phase, p, m, ii, OP_ATTN);
        if (tr && tid == 0 && st == 0) tr[T_FIRST] = globaltimer_ns();
        if (tid == 0) stage_stamp(tr, T_SREADY, st);
        if (ok) {
            const uint32_t kbase = smem_u32(ring + (size_t)slot * SB);
            const uint32_t vbase = kbase + (uint32_t)pl.rps * D * 2;
            const uint32_t half_bytes = (uint32_t)pl.rps * 128u;
            // byte offset of (row, column) in a 128-byte-swizzled stage: 16-byte chunk c of row r sits at c ^ (r & 7)
            auto swz = [&](int row, int col) -> uint32_t {
                return (uint32_t)(col >> 6) * half_bytes + (uint32_t)row * 128u +
                       ((((uint32_t)(col & 63) >> 3) ^ ((uint32_t)row & 7u)) << 4);
            };
            const int ntiles = (nr + 15) >> 4;
            for (int tile = warp; tile < ntiles; tile += kConsumerWarps) {
                const int tb = tile * 16;
                // scores: S[16 x 16 positions] = Q . K^T, two n-halves of 8 positions
                float sc0[2] = {0.f, 0.f}, sc1[2] = {0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < DMAX / 16; ++kk) {
                    if (kk >= KS) break;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kbase + swz(tb + ((lm_i >> 1) << 3) + lm_j, kk * 16 + ((lm_i & 1) << 3)), b0, b1, b2, b3);
                    mma_bf16_top(sc0[0], sc0[1], qa[kk][0], qa[kk][1], b0, b1);
                    mma_bf16_top(sc1[0], sc1[1], qa[kk][0], qa[kk][1], b2, b3);
                }
                // this lane's 4 positions of row g4: tb + 2t4, +1, tb + 8 + 2t4, +1; hi + lo rows
                float sv[4] = {sc0[0], sc0[1], sc1[0], sc1[1]};
                const int pp[4] = {tb + 2 * t4, tb + 2 * t4 + 1, tb + 8 + 2 * t4, tb + 9 + 2 * t4};
                float tmax = -CUDART_INF_F;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    sv[k] += __shfl_xor_sync(0xFFFFFFFFu, sv[k], 16);
                    if (pp[k] >= nr) sv[k] = -CUDART_INF_F;
                    tmax = fmaxf(tmax, sv[k]);
                }
                tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, 1));
                tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, 2));
                const float mn = fmaxf(m_run, tmax);  // finite: every tile has a valid position
                const float al = exp2f(m_run - mn);
                float pv[4], psum = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    pv[k] = pp[k] < nr ? exp2f(sv[k] - mn) : 0.f;
                    psum += pv[k];
                }
                psum += __shfl_xor_sync(0xFFFFFFFFu, psum, 1);
                psum += __shfl_xor_sync(0xFFFFFFFFu, psum, 2);
                l_run = fmaf(l_run, al, psum);
                m_run = mn;
                uint32_t ph[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t hi = f2bf(pv[k]);
                    ph[k] = lo_row ? f2bf(pv[k] - __uint_as_float(hi << 16)) : hi;
                }
                const uint32_t pa0 = ph[0] | (ph[1] << 16), pa2 = ph[2] | (ph[3] << 16);
#pragma unroll
                for (int nt = 0; nt < DMAX / 8; ++nt) {
                    oacc[nt][0] *= al;
                    oacc[nt][1] *= al;
                }
                // O += P . V, two 8-column tiles per ldmatrix
#pragma unroll
                for (int n2 = 0; n2 < DMAX / 16; ++n2) {
                    if (n2 >= KS) break;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(vbase + swz(tb + ((lm_i & 1) << 3) + lm_j, (2 * n2 + (lm_i >> 1)) * 8), b0, b1, b2, b3);
                    mma_bf16_top(oacc[2 * n2][0], oacc[2 * n2][1], pa0, pa2, b0, b1);
                    mma_bf16_top(oacc[2 * n2 + 1][0], oacc[2 * n2 + 1][1], pa0, pa2, b2, b3);
                }
            }
            __syncwarp();
            if (tid == 0) stage_stamp(tr, T_SDONE, st);
            if (lane == 0) mbar_arrive(&empty[slot]);
        } else if (tid == 0) {
            vstore(&m.abort_flag, 1);
        }
        if (++slot == p.ring_stages) {
            slot = 0;
            phase ^= 1u;
        }
    }
    // the new position (its k, v are not in the cache stream): warp 0 adds it
    if (warp == 0 && rg.has_new) {
        float part = 0.f;
        const int dq = D / 4;
        for (int k = t4 * dq; k < (t4 + 1) * dq; ++k) part = fmaf(sm_q[(real ? hrow : 0) * D + k], sm_kv[k], part);
        part += __shfl_xor_sync(0xFFFFFFFFu, part, 1);
        part += __shfl_xor_sync(0xFFFFFFFFu, part, 2);
        const float mn = fmaxf(m_run, part);
        const float al = exp2f(m_run - mn), pr = exp2f(part - mn);
        l_run = fmaf(l_run, al, pr);
        m_run = mn;
#pragma unroll
        for (int nt = 0; nt < DMAX / 8; ++nt) {
            if (nt >= NT) break;
            const int col = nt * 8 + 2 * t4;
            const float add0 = lo_row ? 0.f : pr * sm_kv[D + col], add1 = lo_row ? 0.f : pr * sm_kv[D + col + 1];
            oacc[nt][0] = fmaf(oacc[nt][0], al, add0);
            oacc[nt][1] = fmaf(oacc[nt][1], al, add1);
        }
    }
    if (tr && tid == 0) tr[T_MAIN] = globaltimer_ns();

    // hi + lo rows, then each warp's (max, sum, output) of every head to shared memory
#pragma unroll
    for (int nt = 0; nt < DMAX / 8; ++nt) {
        oacc[nt][0] += __shfl_xor_sync(0xFFFFFFFFu, oacc[nt][0], 16);
        oacc[nt][1] += __shfl_xor_sync(0xFFFFFFFFu, oacc[nt][1], 16);
    }
    cbar();  // the scratch held q and the new k, v until every warp was done with them
    if (lane < 16 && real) {
#pragma unroll
        for (int nt = 0; nt < DMAX / 8; ++nt) {
            if (nt >= NT) break;
            sm_o[(warp * 4 + hrow) * D + nt * 8 + 2 * t4] = oacc[nt][0];
            sm_o[(warp * 4 + hrow) * D + nt * 8 + 2 * t4 + 1] = oacc[nt][1];
        }
        if (t4 == 0) {
            sm_ml[(warp * 4 + hrow) * 2] = m_run;
            sm_ml[(warp * 4 + hrow) * 2 + 1] = l_run;
        }
    }
    cbar();
    if (vload(&m.abort_flag)) return false;
    for (int idx = tid; idx < G * D; idx += kConsumerThreads) {
        const int h = idx / D, col = idx % D;
        float M = -CUDART_INF_F;
        for (int wv = 0; wv < kConsumerWarps; ++wv) M = fmaxf(M, sm_ml[(wv * 4 + h) * 2]);
        float O = 0.f, Ls = 0.f;
        if (M != -CUDART_INF_F) {
            for (int wv = 0; wv < kConsumerWarps; ++wv) {
                const float f = exp2f(sm_ml[(wv * 4 + h) * 2] - M);
                O += f * sm_o[(wv * 4 + h) * D + col];
                Ls += f * sm_ml[(wv * 4 + h) * 2 + 1];
            }
        }
        const size_t part = (size_t)(g * G + h) * S + c;
        part_o_s[part * D + col] = O;
        if (col == 0) {
            part_ml_s[part * 2] = M;
            part_ml_s[part * 2 + 1] = Ls;
        }
    }
    attn_finish(p, a, w, m, sq, l, g, G, S, D);
    return true;
}

__device__ __forceinline__ int gemv_k(const DevParams& p, int op) {
    switch (op) {
        case OP_OPROJ_RES: return p.nq * p.d;
        case OP_DOWN_RES:
        case OP_MOE_DOWN2_RES: return p.F;
    }
    return p.H;
}

// JF > 0: every GEMV-type instruction of the schedule has J == JF (checked on
// the host), so only that instantiation is compiled into the kernel; JF == 0:
// dispatch on the instruction's J at run time.
template <int JF, bool MOE>
__device__ bool gemv_dispatch(const DevParams& p, const StepArgs& a, const int32_t* w, int ii, unsigned char* ring,
                              uint64_t* full, uint64_t* empty, float* scratch, Misc& m, int& slot, uint32_t& phase,
                              int token) {
    if constexpr (JF > 0) {
        // the specialised instantiations run fused-FFN schedules only (chosen on the host)
        if (w[W_OP] == OP_FFN || (MOE && w[W_OP] == OP_MOE_FFN))
            return ffn_instr<JF, true, MOE>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase);
        if (w[W_OP] == OP_RMS_QKV || w[W_OP] == OP_OPROJ_RES || w[W_OP] == OP_LMHEAD_ARGMAX)
            return gemv_instr<JF, true, MOE>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase, token);
        if (threadIdx.x == 0) {
            record_error(p.status, MK_ERR_BAD_INSTR, blockIdx.x, ii, w[W_OP], -1, 0, 0);
            vstore(&m.abort_flag, 1);
        }
        return false;
    }
    const int K = gemv_k(p, w[W_OP]);
    const int kp = K / kparts_of(K);
    const int J = ((kp >> 3) + kConsumerThreads - 1) / kConsumerThreads;
    if (w[W_OP] == OP_FFN || w[W_OP] == OP_MOE_FFN) {
        switch (J) {
            case 1: return ffn_instr<1, false, true>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase);
            case 2: return ffn_instr<2, false, true>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase);
            case 3: return ffn_instr<3, false, true>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase);
            case 4: return ffn_instr<4, false, true>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase);
        }
        return false;
    }
    switch (J) {
        case 1: return gemv_instr<1, false>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase, token);
        case 2: return gemv_instr<2, false>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase, token);
        case 3: return gemv_instr<3, false>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase, token);
        case 4: return gemv_instr<4, false>(p, a, w, ii, ring, full, empty, scratch, m, slot, phase, token);
    }
    return false;
}

// Consumers prefetch, into L2, the weight (or KV-cache) rows of the
// instruction `ahead` places further in their block's queue, spread over the
// 256 consumer threads one 128-byte line each.  Issued before the dependency
// wait of the current instruction, so the HBM keeps streaming while the block
// waits; each instruction is prefetched once.  MoE instructions whose routing
// is not known yet are skipped.
__device__ void prefetch_instr(const DevParams& p, const StepArgs& a, const int32_t* w, const Misc& m) {
    if (!instr_ok(p, w)) return;
    int eidx[kMaxTopK] = {0, 0};
    if (needs_routing(w[W_OP])) {
        if (m.router_layer != route_key(a.epoch, w[W_LAYER], p.L)) return;
        eidx[0] = m.eidx[0];
        eidx[1] = m.eidx[1];
    }
    Plan pl;
    make_plan(p, a.pos, w, eidx, pl);
    const size_t cap = (size_t)p.prefetch_max_bytes;
    size_t done = 0;
    const int nslot = pl.nphase / pl.kparts;
    for (int sl = 0; sl < nslot; ++sl)
        for (int s = 0; s < pl.nspan; ++s) {
            const unsigned char* base = pl.src[sl][s];
            size_t bytes = (size_t)pl.rows * pl.src_stride;
            if (done + bytes > cap) bytes = cap > done ? cap - done : 0;
            for (size_t off = (size_t)threadIdx.x * 128; off < bytes; off += (size_t)kConsumerThreads * 128)
                prefetch_line_l2(base + off);
            done += bytes;
        }
    if (pl.tail_src) {
        size_t bytes = (size_t)pl.rows * pl.tail_row_bytes;
        if (done + bytes > cap) bytes = cap > done ? cap - done : 0;
        for (size_t off = (size_t)threadIdx.x * 128; off < bytes; off += (size_t)kConsumerThreads * 128)
            prefetch_line_l2(pl.tail_src + off);
    }
}

// ---------------------------------------------------------------------------
// launch-once serving: the step hand-off
// ---------------------------------------------------------------------------
__device__ __forceinline__ int ld_sys_acquire(const int32_t* ptr) {
    int v;
    asm volatile("ld.acquire.sys.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

// Block 0's consumer thread 0: take request k + 1 from the host mailbox
// (bounded by serve_idle_ns; past it the grid leaves as if stopped) and
// publish it to every block.
__device__ void serve_publish(const DevParams& p, Misc& m, uint32_t k) {
    const ServeBox* box = p.serve_box;
    int stop = 1, token = -1, pos = 0;
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + kStopPollNs;
    for (;;) {
        if (ld_sys_acquire(&box->req_seq) == (int)(k + 1)) {
            token = *(volatile const int32_t*)&box->token;
            pos = *(volatile const int32_t*)&box->pos;
            stop = *(volatile const int32_t*)&box->stop;
            break;
        }
        const uint64_t now = globaltimer_ns();
        if (now >= next) {
            if (ld_relaxed_s32(&p.status->stop) || vload(&m.abort_flag)) break;
            if (now - t0 > p.serve_idle_ns) break;  // idle: leave (stop = 1)
            next = now + kStopPollNs;
        }
    }
    p.serve_step->token = token;
    p.serve_step->pos = pos;
    p.serve_step->stop = stop;
    signal_release(p.serve_ctr);
}

// Every block's consumer thread 0 and loader lane: wait (bounded) for request
// k + 1 and fill the step's arguments; false when the grid is to leave.
__device__ bool serve_take(const DevParams& p, Misc& m, uint32_t k, const StepArgs& a0, StepArgs& a) {
    const uint32_t* ctr = p.serve_ctr;
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + kStopPollNs;
    const unsigned long long limit = p.serve_idle_ns + p.spin_limit_ns;
    while ((int32_t)(ld_acquire_u32(ctr) - (k + 1)) < 0) {
        const uint64_t now = globaltimer_ns();
        if (now >= next) {
            if (ld_relaxed_s32(&p.status->stop) || vload(&m.abort_flag)) return false;
            if (now - t0 > limit) {
                record_error(p.status, MK_ERR_TIMEOUT, blockIdx.x, -1, 0, -1, 0, k + 1);
                return false;
            }
            next = now + kStopPollNs;
        }
    }
    if (__ldcg(&p.serve_step->stop)) return false;
    a = a0;
    a.token = __ldcg(&p.serve_step->token);
    a.pos = __ldcg(&p.serve_step->pos);
    a.epoch = a0.epoch + k + 1;
    a.seq = (int)(k + 1);
    return a.pos >= 0 && a.pos < p.max_seq && a.token < p.V;
}

// The last LM-head arrival of a served step hands the result to the host.
__device__ void serve_respond(const DevParams& p, const StepArgs& a, int next_token) {
    ServeBox* box = p.serve_box;
    *(volatile int32_t*)&box->next_token = next_token;
    *(volatile int32_t*)&box->code = *(volatile int*)&p.status->code;
    __threadfence_system();
    *(volatile int32_t*)&box->resp_seq = a.seq;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// One instantiation per JF (see gemv_dispatch).  PF: the loader's L2-prefetch
// cursor (options.l2_prefetch) is compiled in; the specialised instantiations
// exist with and without it, so the default ones carry no prefetch code.  The
// consumers' per-instruction prefetch (prefetch_ahead) is in the general one only.
// MOE: MoE routing is compiled in (dense models run instantiations without it).
// NB > 1: batched decode of up to NB sequences per step (p.nb of them).
template <int JF, int DH, bool PF, bool MOE, int NB = 1>
__global__ void __launch_bounds__(kThreads, 1) megakernel(const __grid_constant__ DevParams p, const StepArgs a) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int NS = p.ring_stages, SB = p.stage_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + smem_bars_off(NS, SB));
    uint64_t* empty = full + NS;
    float* scratch = reinterpret_cast<float*>(smem + smem_scratch_off(NS, SB));
    Misc& m = *reinterpret_cast<Misc*>(smem + smem_misc_off(NS, SB));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        m.router_layer = -1;
        m.pred_layer = -1;
        m.is_last = 0;
        m.ffn_go = -1;
        m.abort_flag = ld_relaxed_s32(&p.status->stop) ? 1 : 0;
        if (m.abort_flag && atomicCAS(&p.status->code, 0, MK_ERR_STOPPED) == 0) p.status->sm = blockIdx.x;
        if constexpr (NB > 1) {  // every sequence's position and token (< 0: its previous argmax)
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                m.bpos[q] = a.bpos[q];
                m.btok[q] = q < p.nb ? (a.btok[q] >= 0 ? a.btok[q] : __ldcg(p.next_tok + q)) : 0;
            }
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (m.abort_flag) return;

    const int n = p.n_instr[blockIdx.x];
    const int32_t* q = p.instr + (size_t)blockIdx.x * p.max_instr * W_NWORDS;
    if (warp == kConsumerWarps) {
        if (lane == 0) {
            LoaderRing lr;
            for (uint32_t k = 0;; ++k) {
                StepArgs sa = a;
                if (a.serve && !serve_take(p, m, k, a, sa)) break;
                if (!loader<PF, DH == 64, MOE, NB>(p, sa, q, n, smem, full, empty, m, lr) || !a.serve) break;
            }
            loader_drain(p, full, lr);
        }
        return;
    }

    int slot = 0;
    uint32_t phase = 0;
    for (uint32_t k = 0;; ++k) {
        StepArgs sa = a;
        if (a.serve) {  // launch-once serving: one request per iteration
            if (tid == 0) {
                if (blockIdx.x == 0) serve_publish(p, m, k);
                StepArgs t = a;
                const bool go = serve_take(p, m, k, a, t);
                m.s_go = go ? 1 : 0;
                m.s_token = t.token;
                m.s_pos = t.pos;
                m.s_seq = t.seq;
                m.s_epoch = t.epoch;
            }
            cbar();
            if (!m.s_go) break;
            sa.token = m.s_token;
            sa.pos = m.s_pos;
            sa.seq = m.s_seq;
            sa.epoch = m.s_epoch;
        }
        int token = sa.token >= 0 ? sa.token : __ldcg(&p.status->next_token);
        if constexpr (NB > 1) {  // any sequence's token out of range fails the step
            for (int q = 0; q < p.nb; ++q)
                if (m.btok[q] < 0 || m.btok[q] >= p.V) token = -1;
        }
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            const int32_t* w = q + (size_t)i * W_NWORDS;
            if (p.trace && tid == 0) p.trace[((size_t)blockIdx.x * p.max_instr + i) * kTraceWords + T_START] = globaltimer_ns();
            if (JF == 0 && p.prefetch_ahead > 0 && i + p.prefetch_ahead < n)
                prefetch_instr(p, sa, q + (size_t)(i + p.prefetch_ahead) * W_NWORDS, m);
            if (!instr_ok(p, w) || token < 0 || token >= p.V) {
                if (tid == 0) {
                    record_error(p.status, MK_ERR_BAD_INSTR, blockIdx.x, i, w[W_OP], -1, (uint32_t)token, 0);
                    vstore(&m.abort_flag, 1);
                }
                ok = false;
            } else if (w[W_OP] == OP_ATTN) {
                if constexpr (DH == 64)
                    ok = attn_tc<64, NB>(p, sa, w, i, smem, full, empty, scratch, m, slot, phase);
                else
                    ok = attn_cc<NB>(p, sa, w, i, smem, full, empty, scratch, m, slot, phase);
            } else if constexpr (NB > 1) {
                if (w[W_OP] == OP_FFN) {
                    ok = ffn_instr_b<JF, NB>(p, sa, w, i, smem, full, empty, scratch, m, slot, phase);
                } else if (w[W_OP] == OP_RMS_QKV || w[W_OP] == OP_OPROJ_RES || w[W_OP] == OP_LMHEAD_ARGMAX) {
                    ok = gemv_instr_b<JF, NB>(p, sa, w, i, smem, full, empty, scratch, m, slot, phase);
                } else {
                    if (tid == 0) {
                        record_error(p.status, MK_ERR_BAD_INSTR, blockIdx.x, i, w[W_OP], -1, 0, 0);
                        vstore(&m.abort_flag, 1);
                    }
                    ok = false;
                }
            } else {
                ok = gemv_dispatch<JF, MOE>(p, sa, w, i, smem, full, empty, scratch, m, slot, phase, token);
            }
            if (p.trace && tid == 0) p.trace[((size_t)blockIdx.x * p.max_instr + i) * kTraceWords + T_END] = globaltimer_ns();
            if (!ok) break;
        }
        if (!ok || !a.serve) break;
        cbar();  // every thread has read this request's fields before thread 0 takes the next
    }
    if (tid == 0) vstore(&m.abort_flag, 1);  // lets the loader stop early if it is still waiting
}

namespace {
using KernelFn = void (*)(DevParams, StepArgs);
KernelFn kernel_of(int variant) {
    switch (variant) {
        case 1: return megakernel<1, 64, false, false>;
        case 2: return megakernel<2, 128, false, false>;
        case 3: return megakernel<1, 64, true, false>;
        case 4: return megakernel<2, 128, true, false>;
        case 5: return megakernel<1, 64, false, true>;
        case 6: return megakernel<2, 128, false, true>;
        case 7: return megakernel<1, 64, false, false, 2>;
        case 8: return megakernel<1, 64, false, false, 4>;
        case 9: return megakernel<1, 64, false, false, 8>;
        case 10: return megakernel<2, 128, false, false, 2>;
        case 11: return megakernel<2, 128, false, false, 4>;
    }
    return megakernel<0, 0, true, true>;
}
// J of a GEMV over K columns (chunks of 8 per consumer thread, per column part)
int j_of(int K) {
    const int kp = K / kparts_of(K);
    return ((kp >> 3) + kConsumerThreads - 1) / kConsumerThreads;
}
}  // namespace

// 0: general; 1 / 2: dense, specialised for one chunk (head_dim 64) / two chunks (head_dim 128)
// per thread; 3 / 4: the same with the loader's L2-prefetch cursor (options.l2_prefetch > 0);
// 5 / 6: MoE, specialised (without the prefetch cursor; MoE with it runs the general kernel);
// 7 / 8 / 9: batched decode of up to 2 / 4 / 8 sequences, one chunk per thread (head_dim 64);
// 10 / 11: up to 2 / 4 sequences, two chunks (head_dim 128).  -1: no kernel for the batch.
int megakernel_variant(const DevParams& p, bool fused_ffn) {
    const int jh = j_of(p.H), jo = j_of(p.nq * p.d);
    const int base = (jh == 1 && jo == 1 && p.d == 64) ? 1 : (jh == 2 && jo == 2 && p.d == 128) ? 2 : 0;
    if (p.nb > 1) {
        if (!fused_ffn || p.E > 0 || p.prefetch_ahead > 0 || p.l2_prefetch > 0) return -1;
        if (base == 1) return p.nb <= 2 ? 7 : p.nb <= 4 ? 8 : p.nb <= 8 ? 9 : -1;
        if (base == 2) return p.nb <= 2 ? 10 : p.nb <= 4 ? 11 : -1;
        return -1;
    }
    if (!fused_ffn || p.prefetch_ahead > 0) return 0;
    if (base == 0) return 0;
    if (p.E > 0) return p.l2_prefetch > 0 ? 0 : base + 4;
    return p.l2_prefetch > 0 ? base + 2 : base;
}

// Bytes between the weight rows of a stage beyond the row itself, for an instantiation (its
// tensor-core batched GEMVs read the stage with ldmatrix: 16 keeps each 8-row tile in distinct banks).
int megakernel_row_pad(int variant) { return variant == 9 ? 16 : 0; }

cudaError_t launch_megakernel(const DevParams& p, const StepArgs& a, int n_sm, int variant, cudaStream_t stream) {
    const size_t smem = megakernel_smem_bytes(p.ring_stages, p.stage_bytes);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_sm);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel_of(variant), p, a);
}

cudaError_t prepare_megakernel(int ring_stages, int stage_bytes, int* max_blocks_per_sm) {
    const size_t smem = megakernel_smem_bytes(ring_stages, stage_bytes);
    *max_blocks_per_sm = 1 << 30;
    for (int v = 0; v <= 11; ++v) {
        cudaError_t e = cudaFuncSetAttribute(kernel_of(v), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel_of(v), kThreads, smem);
        if (e != cudaSuccess) return e;
        if (per_sm < *max_blocks_per_sm) *max_blocks_per_sm = per_sm;
    }
    return cudaSuccess;
}

}  // namespace mk

// mk_api.cu -- the C ABI (include/mk.h): handle lifetime, device buffers,
// schedule upload, the step launch with a host-side watchdog, fault injection
// and the debug getters.
#include <cuda_runtime.h>

#include <atomic>
#include <chrono>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include <cudaTypedefs.h>  // PFN_cuTensorMapEncodeTiled

#include "mk_internal.h"
#include "mk_kernels.h"
#include "mk_plan.h"

struct mk_handle {
    mk_config cfg;
    mk_options opt;
    cudaStream_t stream = nullptr;
    int device = 0;
    int n_sm = 0;
    mk::DevParams p;
    std::vector<const uint16_t*> wt_host;
    std::vector<void*> allocs;
    mk::Planned plan;
    bool scheduled = false;
    uint32_t epoch = 0;
    mk::StepBuf* stepbuf = nullptr;
    mk::DevStatus* status_pinned = nullptr;
    cudaEvent_t ev0 = nullptr, ev1 = nullptr, ev_done = nullptr;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t graph_exec = nullptr;
    int lm_slots = 0;
    int variant = 0;  // megakernel instantiation for the built schedule
    // launch-once serving
    mk::ServeBox* box_host = nullptr;  // pinned, mapped
    mk::ServeBox* box_dev = nullptr;
    mk::ServeStep* serve_step = nullptr;
    uint32_t* serve_ctr = nullptr;
    cudaEvent_t ev_serve = nullptr;
    bool serving = false;
    int32_t serve_seq = 0;  // requests answered since mk_serve_start
    bool down_t = false;  // transposed down-projection copies exist (fused FFN schedules)
    int last_cuda = 0;
    int last_error = MK_OK;
    std::vector<float> sm_speed;  // copy of options.sm_speed (opt.sm_speed points here)
};

namespace {

int cuda_fail(mk_handle* h, cudaError_t e) {
    if (h) h->last_cuda = (int)e;
    return MK_ERR_CUDA;
}

#define CK(expr)                                   \
    do {                                           \
        cudaError_t e_ = (expr);                   \
        if (e_ != cudaSuccess) return cuda_fail(h, e_); \
    } while (0)

template <class T>
int dalloc(mk_handle* h, T** out, size_t count) {
    void* ptr = nullptr;
    const size_t bytes = count * sizeof(T) > 0 ? count * sizeof(T) : 16;
    cudaError_t e = cudaMalloc(&ptr, bytes);
    if (e != cudaSuccess) return cuda_fail(h, e);
    e = cudaMemset(ptr, 0, bytes);
    if (e != cudaSuccess) {
        cudaFree(ptr);
        return cuda_fail(h, e);
    }
    h->allocs.push_back(ptr);
    *out = static_cast<T*>(ptr);
    return MK_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_weights(const mk_config& c, const mk_weights* w) {
    if (!w || !w->embed || !w->lm_head || !w->final_norm) return MK_ERR_INVALID_ARG;
    if (c.n_layers > 0 && (!w->k_cache || !w->v_cache)) return MK_ERR_INVALID_ARG;  // no cache without layers
    if (!aligned16(w->embed) || !aligned16(w->lm_head) || !aligned16(w->final_norm) || !aligned16(w->k_cache) ||
        !aligned16(w->v_cache))
        return MK_ERR_INVALID_ARG;
    const int L = c.n_layers;
    const int ne = c.n_experts > 0 ? L * c.n_experts : L;
    const void* const* per_layer[] = {w->attn_norm, w->wq, w->wk, w->wv, w->wo, w->ffn_norm};
    for (auto arr : per_layer) {
        if (L > 0 && !arr) return MK_ERR_INVALID_ARG;
        for (int l = 0; l < L; ++l)
            if (!arr[l] || !aligned16(arr[l])) return MK_ERR_INVALID_ARG;
    }
    const void* const* per_expert[] = {w->w_gate, w->w_up, w->w_down};
    for (auto arr : per_expert) {
        if (ne > 0 && !arr) return MK_ERR_INVALID_ARG;
        for (int i = 0; i < ne; ++i)
            if (!arr[i] || !aligned16(arr[i])) return MK_ERR_INVALID_ARG;
    }
    if (c.n_experts > 0) {
        if (L > 0 && !w->router) return MK_ERR_INVALID_ARG;
        for (int l = 0; l < L; ++l)
            if (!w->router[l] || !aligned16(w->router[l])) return MK_ERR_INVALID_ARG;
    }
    return MK_OK;
}

// Tensor maps over the K and V caches for the attention stages: rows of d bf16,
// [n_layers * n_kv * max_seq] rows, boxes of 64 columns x attn_box_rows rows,
// 128-byte swizzle.  The driver entry point is looked up through the runtime.
int make_kv_maps(mk_handle* h, const mk_config& c, const mk_options& o, void* kcache, void* vcache) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cuda_fail(h, e != cudaSuccess ? e : cudaErrorNotSupported);
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const int d = c.head_dim;
    const cuuint64_t rows = (cuuint64_t)std::max(o.batch, 1) * std::max(c.n_layers, 1) * c.n_kv_heads * c.max_seq;
    const cuuint64_t dims[2] = {(cuuint64_t)d, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)mk::attn_box_rows(o.stage_bytes, d)};
    const cuuint32_t estr[2] = {1u, 1u};
    CUtensorMap* maps[2] = {&h->p.kmap, &h->p.vmap};
    void* bases[2] = {kcache, vcache};
    for (int i = 0; i < 2; ++i) {
        CUresult r = encode(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, bases[i], dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return MK_ERR_UNSUPPORTED;
    }
    return MK_OK;
}

int upload_schedule(mk_handle* h) {
    CK(cudaMemcpy(const_cast<int32_t*>(h->p.instr), h->plan.words.data(), h->plan.words.size() * sizeof(int32_t),
                  cudaMemcpyHostToDevice));
    CK(cudaMemcpy(const_cast<int32_t*>(h->p.n_instr), h->plan.n_instr.data(), h->plan.n_instr.size() * sizeof(int32_t),
                  cudaMemcpyHostToDevice));
    return MK_OK;
}

// Wait for the step's completion event with a deadline (host-side watchdog,
// the backstop behind the kernel's own bounded waits).
int wait_event(mk_handle* h, cudaEvent_t ev) {
    const double limit_s = std::max(10.0, 4.0 * (double)h->opt.spin_limit_ns * 1e-9);
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t e = cudaEventQuery(ev);
        if (e == cudaSuccess) return MK_OK;
        if (e != cudaErrorNotReady) return cuda_fail(h, e);
        if (std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count() > limit_s)
            return MK_ERR_TIMEOUT;
        std::this_thread::yield();
    }
}

int read_status(mk_handle* h, mk::DevStatus* out) {
    CK(cudaMemcpyAsync(h->status_pinned, h->p.status, sizeof(mk::DevStatus), cudaMemcpyDeviceToHost, h->stream));
    CK(cudaEventRecord(h->ev_done, h->stream));
    int rc = wait_event(h, h->ev_done);
    if (rc) return rc;
    *out = *h->status_pinned;
    return MK_OK;
}

}  // namespace

extern "C" {

void mk_default_options(mk_options* o) {
    if (!o) return;
    std::memset(o, 0, sizeof(*o));
    o->l2_prefetch = -1;
    o->prefetch_ahead = -1;
    o->l2_head_start = -1;
    o->mode = MK_MODE_MEGAKERNEL;
}

const char* mk_strerror(int code) {
    switch (code) {
        case MK_OK: return "ok";
        case MK_ERR_INVALID_ARG: return "invalid argument";
        case MK_ERR_CUDA: return "CUDA runtime error";
        case MK_ERR_NOT_RESIDENT: return "persistent grid cannot be co-resident";
        case MK_ERR_TIMEOUT: return "bounded device wait timed out";
        case MK_ERR_BAD_INSTR: return "bad instruction or index";
        case MK_ERR_SCHEDULE: return "schedule rejected by the validator";
        case MK_ERR_STOPPED: return "stop word set";
        case MK_ERR_NO_SCHEDULE: return "no schedule built";
        case MK_ERR_CAPACITY: return "buffer too small";
        case MK_ERR_UNSUPPORTED: return "unsupported shape";
    }
    return "unknown error";
}

int mk_create(const mk_config* cfg, const mk_weights* w, const mk_options* opt, void* cuda_stream, mk_handle** out) {
    if (!cfg || !out) return MK_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = mk::check_config(*cfg);
    if (rc) return rc;
    rc = check_weights(*cfg, w);
    if (rc) return rc;
    mk_options o;
    if (opt) o = *opt; else mk_default_options(&o);
    mk::fill_defaults(*cfg, &o);
    rc = mk::check_options(*cfg, o);
    if (rc) return rc;
    if (o.mode != MK_MODE_MEGAKERNEL) o.split_ffn = 1;  // the schedule of the plain launches is never fused

    mk_handle* h = new mk_handle();
    h->cfg = *cfg;
    h->opt = o;
    h->stream = static_cast<cudaStream_t>(cuda_stream);
    auto fail = [&](int code) {
        mk_destroy(h);
        return code;
    };
    cudaError_t e = cudaGetDevice(&h->device);
    if (e != cudaSuccess) { h->last_cuda = e; return fail(MK_ERR_CUDA); }
    int dev_sms = 0, coop = 0;
    cudaDeviceGetAttribute(&dev_sms, cudaDevAttrMultiProcessorCount, h->device);
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, h->device);
    if (dev_sms <= 0) return fail(MK_ERR_CUDA);
    h->n_sm = (o.n_sm > 0 && o.n_sm < dev_sms) ? o.n_sm : dev_sms;
    if (o.sm_speed) {
        if (o.n_sm_speed != h->n_sm) return fail(MK_ERR_INVALID_ARG);
        h->sm_speed.assign(o.sm_speed, o.sm_speed + o.n_sm_speed);
        h->opt.sm_speed = h->sm_speed.data();
    }

    const mk_config& c = *cfg;
    const int L = c.n_layers, H = c.hidden, d = c.head_dim, nq = c.n_q_heads, nkv = c.n_kv_heads;
    const int NB = o.batch;
    const int S = o.kv_splits > 0 ? o.kv_splits : mk::default_kv_splits(c, h->n_sm, NB);
    const int E = c.n_experts, topk = E > 0 ? c.top_k : 1;
    mk::DevParams& p = h->p;
    std::memset(&p, 0, sizeof(p));
    p.L = L; p.H = H; p.nq = nq; p.nkv = nkv; p.d = d; p.F = c.ffn; p.V = c.vocab; p.E = E;
    p.topk = E > 0 ? c.top_k : 0; p.max_seq = c.max_seq; p.eps = c.rms_eps; p.kv_splits = S;
    p.n_ctr = mk::n_counters(L);
    p.nb = NB;
    p.kv_seq_stride = (size_t)L * nkv * c.max_seq * d;
    p.embed = static_cast<const uint16_t*>(w->embed);
    p.lm_head = static_cast<const uint16_t*>(w->lm_head);
    p.final_norm = static_cast<const uint16_t*>(w->final_norm);
    p.kcache = static_cast<uint16_t*>(w->k_cache);
    p.vcache = static_cast<uint16_t*>(w->v_cache);
    p.ring_stages = o.ring_stages;
    p.stage_bytes = o.stage_bytes;
    p.l2_prefetch = o.l2_prefetch;
    p.l2_head_start = o.l2_head_start;
    p.prefetch_ahead = o.prefetch_ahead;
    p.prefetch_max_bytes = o.prefetch_max_bytes;
    p.spin_limit_ns = o.spin_limit_ns;

    // weight pointer table
    const int stride = mk::wt_stride(E);
    h->wt_host.assign((size_t)std::max(L, 1) * stride, nullptr);
    for (int l = 0; l < L; ++l) {
        const uint16_t** t = &h->wt_host[(size_t)l * stride];
        t[mk::WT_ATTN_NORM] = static_cast<const uint16_t*>(w->attn_norm[l]);
        t[mk::WT_Q] = static_cast<const uint16_t*>(w->wq[l]);
        t[mk::WT_K] = static_cast<const uint16_t*>(w->wk[l]);
        t[mk::WT_V] = static_cast<const uint16_t*>(w->wv[l]);
        t[mk::WT_O] = static_cast<const uint16_t*>(w->wo[l]);
        t[mk::WT_FFN_NORM] = static_cast<const uint16_t*>(w->ffn_norm[l]);
        t[mk::WT_ROUTER] = E > 0 ? static_cast<const uint16_t*>(w->router[l]) : nullptr;
        const int ne = E > 0 ? E : 1;
        for (int x = 0; x < ne; ++x) {
            const size_t src = E > 0 ? (size_t)l * E + x : (size_t)l;
            t[mk::wt_gate(x)] = static_cast<const uint16_t*>(w->w_gate[src]);
            t[mk::wt_up(x, E)] = static_cast<const uint16_t*>(w->w_up[src]);
            t[mk::wt_down(x, E)] = static_cast<const uint16_t*>(w->w_down[src]);
        }
    }
    const uint16_t** wt_dev = nullptr;
    const int lm_rows = std::min(o.rows_per_instr, mk::kRowSlots / NB);  // LM-head rows per instruction, at most
    const int lm_slots = std::max(h->n_sm + c.vocab / lm_rows + 1, mk::baseline_lm_blocks(p, h->n_sm));
    h->lm_slots = lm_slots;
    if ((rc = dalloc(h, &wt_dev, h->wt_host.size()))) return fail(rc);
    if ((rc = dalloc(h, &p.counters, (size_t)p.n_ctr))) return fail(rc);
    if ((rc = dalloc(h, &p.status, 1))) return fail(rc);
    // per-sequence activations: NB copies one after the other
    if ((rc = dalloc(h, &p.x, (size_t)NB * H))) return fail(rc);
    if ((rc = dalloc(h, &p.x2, (size_t)NB * H))) return fail(rc);
    if ((rc = dalloc(h, &p.qkv, (size_t)NB * (nq + 2 * nkv) * d))) return fail(rc);
    if ((rc = dalloc(h, &p.attn, (size_t)NB * nq * d))) return fail(rc);
    if ((rc = dalloc(h, &p.attn_arrive, (size_t)NB * std::max(L, 1) * nkv))) return fail(rc);
    if ((rc = dalloc(h, &p.part_o, (size_t)NB * nq * S * d))) return fail(rc);
    if ((rc = dalloc(h, &p.part_ml, (size_t)NB * nq * S * 2))) return fail(rc);
    if ((rc = dalloc(h, &p.hbuf, (size_t)topk * c.ffn))) return fail(rc);
    if ((rc = dalloc(h, &p.logits, (size_t)NB * c.vocab))) return fail(rc);
    if ((rc = dalloc(h, &p.lm_part, (size_t)lm_slots * NB * 2))) return fail(rc);
    if ((rc = dalloc(h, &p.next_tok, (size_t)mk::kMaxBatch))) return fail(rc);
    if ((rc = dalloc(h, &p.router_idx, (size_t)std::max(L, 1) * mk::kMaxTopK))) return fail(rc);
    if ((rc = dalloc(h, &p.router_w, (size_t)std::max(L, 1) * mk::kMaxTopK))) return fail(rc);
    if ((rc = dalloc(h, &p.pred_idx, (size_t)std::max(L, 1) * mk::kMaxTopK))) return fail(rc);
    e = cudaMemset(p.pred_idx, 0xFF, sizeof(int32_t) * (size_t)std::max(L, 1) * mk::kMaxTopK);  // -1: none
    if (e != cudaSuccess) { h->last_cuda = e; return fail(MK_ERR_CUDA); }
    p.spec_experts = E > 0 ? o.spec_experts : 0;
    if (o.snapshots && (rc = dalloc(h, &p.snap, (size_t)NB * (L + 1) * H))) return fail(rc);
    float2* rope = nullptr;
    if ((rc = dalloc(h, &rope, (size_t)c.max_seq * (d / 2)))) return fail(rc);
    if ((rc = dalloc(h, &h->stepbuf, 1))) return fail(rc);
    if ((rc = dalloc(h, &h->serve_step, 1))) return fail(rc);
    if ((rc = dalloc(h, &h->serve_ctr, 1))) return fail(rc);
    // The fused FFN streams the down-projection by its input index: keep a
    // transposed copy [ffn][hidden] of every w_down (library-owned).
    if (o.mode == MK_MODE_MEGAKERNEL && mk::ffn_fused(c, o)) {
        const int ne = E > 0 ? E : 1;
        for (int l = 0; l < L; ++l)
            for (int x = 0; x < ne; ++x) {
                const uint16_t** t = &h->wt_host[(size_t)l * stride];
                uint16_t* dt = nullptr;
                if ((rc = dalloc(h, &dt, (size_t)c.ffn * H))) return fail(rc);
                e = mk::launch_transpose_bf16(t[mk::wt_down(x, E)], dt, H, c.ffn, nullptr);
                if (e != cudaSuccess) { h->last_cuda = e; return fail(MK_ERR_CUDA); }
                t[mk::wt_down_t(x, E)] = dt;
            }
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) { h->last_cuda = e; return fail(MK_ERR_CUDA); }
        h->down_t = true;
    }
    p.wt = wt_dev;
    p.rope = rope;
    e = cudaMemcpy(wt_dev, h->wt_host.data(), h->wt_host.size() * sizeof(void*), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { h->last_cuda = e; return fail(MK_ERR_CUDA); }

    // RoPE table: angle = pos * theta^(-2i/d), evaluated in double
    {
        std::vector<float2> tab((size_t)c.max_seq * (d / 2));
        for (int pos = 0; pos < c.max_seq; ++pos)
            for (int i = 0; i < d / 2; ++i) {
                const double a = (double)pos * std::pow((double)c.rope_theta, -2.0 * i / d);
                tab[(size_t)pos * (d / 2) + i] = make_float2((float)std::cos(a), (float)std::sin(a));
            }
        e = cudaMemcpy(rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) { h->last_cuda = e; return fail(MK_ERR_CUDA); }
    }

    e = cudaMallocHost(&h->status_pinned, sizeof(mk::DevStatus));
    if (e != cudaSuccess) { h->last_cuda = e; h->status_pinned = nullptr; return fail(MK_ERR_CUDA); }
    if (cudaEventCreate(&h->ev0) || cudaEventCreate(&h->ev1) ||
        cudaEventCreateWithFlags(&h->ev_done, cudaEventDisableTiming) ||
        cudaEventCreateWithFlags(&h->ev_serve, cudaEventDisableTiming))
        return fail(MK_ERR_CUDA);

    if (o.mode == MK_MODE_MEGAKERNEL && L > 0 && (rc = make_kv_maps(h, c, o, w->k_cache, w->v_cache)))
        return fail(rc);
    if (o.mode == MK_MODE_MEGAKERNEL) {
        int per_sm = 0;
        e = mk::prepare_megakernel(o.ring_stages, o.stage_bytes, &per_sm);
        if (e != cudaSuccess) { h->last_cuda = e; return fail(MK_ERR_CUDA); }
        if (!coop || per_sm < 1) return fail(MK_ERR_NOT_RESIDENT);
    } else {
        e = mk::prepare_baseline();
        if (e != cudaSuccess) { h->last_cuda = e; return fail(MK_ERR_CUDA); }
    }
    *out = h;
    return MK_OK;
}

int mk_build_schedule(mk_handle* h) {
    if (!h || h->serving) return MK_ERR_INVALID_ARG;
    mk::Planned plan;
    int rc = mk::plan_schedule(h->cfg, h->opt, h->n_sm, &plan);
    if (rc) return rc;
    if (plan.kv_splits != h->p.kv_splits) return MK_ERR_SCHEDULE;
    if (plan.n_lm > h->lm_slots) return MK_ERR_SCHEDULE;
    if (plan.fused_ffn && h->cfg.n_layers > 0 && !h->down_t) return MK_ERR_SCHEDULE;
    h->plan = plan;
    h->variant = h->opt.general_kernel ? 0 : mk::megakernel_variant(h->p, plan.fused_ffn);
    if (h->variant < 0) return MK_ERR_UNSUPPORTED;  // no kernel instantiation for this batch
    h->p.row_pad = mk::megakernel_row_pad(h->variant);
    // the prediction runs in the specialised MoE kernels (the general one keeps the prefetch cursor)
    h->p.spec_experts = h->variant != 0 && plan.fused_ffn && h->cfg.n_experts > 0 ? h->opt.spec_experts : 0;
    int32_t* words = nullptr;
    int32_t* n_instr = nullptr;
    if ((rc = dalloc(h, &words, plan.words.size()))) return rc;
    if ((rc = dalloc(h, &n_instr, (size_t)plan.n_sm))) return rc;
    h->p.instr = words;
    h->p.n_instr = n_instr;
    h->p.max_instr = plan.max_instr;
    if (h->opt.trace) {
        unsigned long long* tr = nullptr;
        if ((rc = dalloc(h, &tr, (size_t)plan.n_sm * plan.max_instr * mk::kTraceWords))) return rc;
        h->p.trace = tr;
    }
    if ((rc = upload_schedule(h))) return rc;
    h->scheduled = true;
    return MK_OK;
}

int mk_get_schedule(mk_handle* h, int32_t* buf, size_t cap, size_t* n_words, int* n_sm, int* max_instr) {
    if (!h) return MK_ERR_INVALID_ARG;
    if (!h->scheduled) return MK_ERR_NO_SCHEDULE;
    if (n_words) *n_words = h->plan.words.size();
    if (n_sm) *n_sm = h->plan.n_sm;
    if (max_instr) *max_instr = h->plan.max_instr;
    if (!buf) return MK_OK;
    if (cap < h->plan.words.size()) return MK_ERR_CAPACITY;
    std::memcpy(buf, h->plan.words.data(), h->plan.words.size() * sizeof(int32_t));
    return MK_OK;
}

int mk_decode_step(mk_handle* h, int32_t token, int32_t pos, float* logits_dev, int32_t* next_token_host) {
    if (!h || h->serving || h->p.nb > 1) return MK_ERR_INVALID_ARG;  // batched handles: mk_decode_step_batch
    if (token >= h->cfg.vocab || pos < 0 || pos >= h->cfg.max_seq) return MK_ERR_INVALID_ARG;
    if (!h->scheduled) return MK_ERR_NO_SCHEDULE;
    if (token < 0) token = -1;
    h->epoch++;
    mk::DevParams& p = h->p;
    if (h->opt.mode == MK_MODE_MEGAKERNEL) {
        mk::StepArgs a;
        a.token = token;
        a.pos = pos;
        a.epoch = h->epoch;
        a.logits = logits_dev ? logits_dev : p.logits;
        CK(cudaEventRecord(h->ev0, h->stream));
        CK(mk::launch_megakernel(p, a, h->n_sm, h->variant, h->stream));
        CK(cudaEventRecord(h->ev1, h->stream));
    } else {
        mk::BaselineShape bs{h->n_sm, mk::baseline_lm_blocks(p, h->n_sm)};
        CK(mk::launch_baseline_set_step(p, h->stepbuf, token, pos, h->stream));
        CK(cudaEventRecord(h->ev0, h->stream));
        if (h->opt.mode == MK_MODE_MULTI_KERNEL_GRAPH) {
            if (!h->graph_exec) {
                cudaStream_t cap = nullptr;
                CK(cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking));
                cudaError_t e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal);
                if (e == cudaSuccess) {
                    mk::launch_baseline_layers(p, h->wt_host.data(), h->stepbuf, bs, p.logits, cap);
                    e = cudaStreamEndCapture(cap, &h->graph);
                }
                if (e == cudaSuccess) e = cudaGraphInstantiate(&h->graph_exec, h->graph, 0);
                cudaStreamDestroy(cap);
                if (e != cudaSuccess) return cuda_fail(h, e);
            }
            CK(cudaGraphLaunch(h->graph_exec, h->stream));
        } else {
            CK(mk::launch_baseline_layers(p, h->wt_host.data(), h->stepbuf, bs, p.logits, h->stream));
        }
        CK(cudaEventRecord(h->ev1, h->stream));
        if (logits_dev)
            CK(cudaMemcpyAsync(logits_dev, p.logits, sizeof(float) * h->cfg.vocab, cudaMemcpyDeviceToDevice,
                               h->stream));
    }
    if (next_token_host) {
        mk::DevStatus st;
        int rc = read_status(h, &st);
        if (rc) return rc;
        if (st.code != MK_OK) return st.code;
        *next_token_host = st.next_token;
    }
    return MK_OK;
}

int mk_decode_step_batch(mk_handle* h, const int32_t* tokens, const int32_t* pos, float* logits_dev,
                         int32_t* next_host) {
    if (!h || h->serving || !tokens || !pos) return MK_ERR_INVALID_ARG;
    const int nb = h->p.nb;
    if (nb == 1) {
        int32_t nxt = 0;
        const int rc = mk_decode_step(h, tokens[0], pos[0], logits_dev, next_host ? &nxt : nullptr);
        if (rc == MK_OK && next_host) next_host[0] = nxt;
        return rc;
    }
    for (int b = 0; b < nb; ++b)
        if (tokens[b] >= h->cfg.vocab || pos[b] < 0 || pos[b] >= h->cfg.max_seq) return MK_ERR_INVALID_ARG;
    if (!h->scheduled) return MK_ERR_NO_SCHEDULE;
    h->epoch++;
    mk::DevParams& p = h->p;
    mk::StepArgs a;
    for (int b = 0; b < nb; ++b) {
        a.btok[b] = tokens[b] < 0 ? -1 : tokens[b];
        a.bpos[b] = pos[b];
    }
    a.token = a.btok[0];
    a.pos = a.bpos[0];
    a.epoch = h->epoch;
    a.logits = logits_dev ? logits_dev : p.logits;
    CK(cudaEventRecord(h->ev0, h->stream));
    CK(mk::launch_megakernel(p, a, h->n_sm, h->variant, h->stream));
    CK(cudaEventRecord(h->ev1, h->stream));
    if (next_host) {
        mk::DevStatus st;
        int rc = read_status(h, &st);
        if (rc) return rc;
        if (st.code != MK_OK) return st.code;
        CK(cudaMemcpy(next_host, p.next_tok, sizeof(int32_t) * nb, cudaMemcpyDeviceToHost));
    }
    return MK_OK;
}

int mk_get_hidden(mk_handle* h, int layer, float* out_host) {
    if (!h || h->serving || !out_host || layer < 0 || layer > h->cfg.n_layers || !h->p.snap) return MK_ERR_INVALID_ARG;
    CK(cudaStreamSynchronize(h->stream));
    const size_t H = (size_t)h->cfg.hidden, per_seq = (size_t)(h->cfg.n_layers + 1) * H;
    CK(cudaMemcpy2D(out_host, sizeof(float) * H, h->p.snap + (size_t)layer * H, sizeof(float) * per_seq,
                    sizeof(float) * H, (size_t)h->p.nb, cudaMemcpyDeviceToHost));
    return MK_OK;
}

int mk_get_router(mk_handle* h, int layer, int32_t* idx, float* wts) {
    if (!h || h->serving || !idx || !wts || h->cfg.n_experts <= 0 || layer < 0 || layer >= h->cfg.n_layers)
        return MK_ERR_INVALID_ARG;
    CK(cudaStreamSynchronize(h->stream));
    CK(cudaMemcpy(idx, h->p.router_idx + (size_t)layer * mk::kMaxTopK, sizeof(int32_t) * h->cfg.top_k,
                  cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(wts, h->p.router_w + (size_t)layer * mk::kMaxTopK, sizeof(float) * h->cfg.top_k,
                  cudaMemcpyDeviceToHost));
    return MK_OK;
}

int mk_get_predicted_experts(mk_handle* h, int layer, int32_t* idx) {
    if (!h || h->serving || !idx || h->cfg.n_experts <= 0 || !h->p.spec_experts || layer < 0 ||
        layer >= h->cfg.n_layers)
        return MK_ERR_INVALID_ARG;
    CK(cudaStreamSynchronize(h->stream));
    CK(cudaMemcpy(idx, h->p.pred_idx + (size_t)layer * mk::kMaxTopK, sizeof(int32_t) * h->cfg.top_k,
                  cudaMemcpyDeviceToHost));
    return MK_OK;
}

int mk_get_counters(mk_handle* h, uint32_t* out, size_t cap, size_t* n) {
    if (!h || h->serving) return MK_ERR_INVALID_ARG;
    if (n) *n = (size_t)h->p.n_ctr;
    if (!out) return MK_OK;
    if (cap < (size_t)h->p.n_ctr) return MK_ERR_CAPACITY;
    CK(cudaStreamSynchronize(h->stream));
    CK(cudaMemcpy(out, h->p.counters, sizeof(uint32_t) * h->p.n_ctr, cudaMemcpyDeviceToHost));
    return MK_OK;
}

int mk_get_counter_increments(mk_handle* h, uint32_t* out, size_t cap, size_t* n) {
    if (!h) return MK_ERR_INVALID_ARG;
    if (!h->scheduled) return MK_ERR_NO_SCHEDULE;
    if (n) *n = h->plan.ctr_inc.size();
    if (!out) return MK_OK;
    if (cap < h->plan.ctr_inc.size()) return MK_ERR_CAPACITY;
    std::memcpy(out, h->plan.ctr_inc.data(), h->plan.ctr_inc.size() * sizeof(uint32_t));
    return MK_OK;
}

int mk_get_status(mk_handle* h, mk_status* out) {
    if (!h || h->serving || !out) return MK_ERR_INVALID_ARG;
    mk::DevStatus st;
    int rc = read_status(h, &st);
    if (rc) return rc;
    out->code = st.code;
    out->sm = st.sm;
    out->instr = st.instr;
    out->opcode = st.opcode;
    out->counter = st.counter;
    out->observed = st.observed;
    out->expected = st.expected;
    out->cuda_error = h->last_cuda;
    return MK_OK;
}

int mk_get_trace(mk_handle* h, uint64_t* out, size_t cap, size_t* n) {
    if (!h || h->serving || !h->p.trace) return MK_ERR_INVALID_ARG;
    const size_t cnt = (size_t)h->plan.n_sm * h->plan.max_instr * mk::kTraceWords;
    if (n) *n = cnt;
    if (!out) return MK_OK;
    if (cap < cnt) return MK_ERR_CAPACITY;
    CK(cudaStreamSynchronize(h->stream));
    CK(cudaMemcpy(out, h->p.trace, cnt * sizeof(uint64_t), cudaMemcpyDeviceToHost));
    return MK_OK;
}

int mk_reset(mk_handle* h) {
    if (!h || h->serving) return MK_ERR_INVALID_ARG;
    CK(cudaStreamSynchronize(h->stream));
    CK(cudaMemset(h->p.counters, 0, sizeof(uint32_t) * h->p.n_ctr));
    CK(cudaMemset(h->p.attn_arrive, 0, sizeof(uint32_t) * h->p.nb * std::max(h->p.L, 1) * h->p.nkv));
    CK(cudaMemset(h->p.status, 0, sizeof(mk::DevStatus)));
    if (h->p.trace) CK(cudaMemset(h->p.trace, 0, sizeof(uint64_t) * h->plan.n_sm * h->plan.max_instr * mk::kTraceWords));
    h->epoch = 0;
    if (h->scheduled) return upload_schedule(h);
    return MK_OK;
}

int mk_inject_fault(mk_handle* h, int kind, int arg) {
    if (!h || h->serving) return MK_ERR_INVALID_ARG;
    if (kind == MK_FAULT_NONE) return mk_reset(h);
    if (kind == MK_FAULT_PRESET_STOP) {
        const int one = 1;
        CK(cudaStreamSynchronize(h->stream));
        CK(cudaMemcpy(&h->p.status->stop, &one, sizeof(int), cudaMemcpyHostToDevice));
        return MK_OK;
    }
    if (!h->scheduled) return MK_ERR_NO_SCHEDULE;
    if (kind != MK_FAULT_UNREACHABLE_WAIT && kind != MK_FAULT_BAD_OPCODE) return MK_ERR_INVALID_ARG;
    std::vector<int32_t> words = h->plan.words;
    const int sm = ((arg % h->plan.n_sm) + h->plan.n_sm) % h->plan.n_sm;
    bool done = false;
    for (int i = 0; i < h->plan.n_instr[sm] && !done; ++i) {
        int32_t* w = &words[((size_t)sm * h->plan.max_instr + i) * mk::W_NWORDS];
        if (kind == MK_FAULT_BAD_OPCODE) {
            w[mk::W_OP] = 99;
            done = true;
        } else if (w[mk::W_WAIT_CTR] >= 0) {
            w[mk::W_WAIT_INC] += 1000000;  // a target no step reaches
            done = true;
        }
    }
    if (!done) return MK_ERR_INVALID_ARG;
    CK(cudaStreamSynchronize(h->stream));
    CK(cudaMemcpy(const_cast<int32_t*>(h->p.instr), words.data(), words.size() * sizeof(int32_t),
                  cudaMemcpyHostToDevice));
    return MK_OK;
}

int mk_last_step_ns(mk_handle* h, double* ns) {
    if (!h || h->serving || !ns) return MK_ERR_INVALID_ARG;
    CK(cudaEventSynchronize(h->ev1));
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, h->ev0, h->ev1));
    *ns = (double)ms * 1e6;
    return MK_OK;
}

// ---- launch-once serving ---------------------------------------------------------------
namespace {
double host_wait_limit_s(const mk_handle* h) {
    return std::max(10.0, 4.0 * (double)h->opt.spin_limit_ns * 1e-9);
}
void post_request(mk_handle* h, int32_t token, int32_t pos, int32_t stop, int32_t seq) {
    volatile mk::ServeBox* b = h->box_host;
    b->token = token;
    b->pos = pos;
    b->stop = stop;
    std::atomic_thread_fence(std::memory_order_seq_cst);
    b->req_seq = seq;  // the grid reads the other fields after it sees this
    std::atomic_thread_fence(std::memory_order_seq_cst);
}
// The serving grid has left (launch complete): collect its status.
int serve_ended(mk_handle* h) {
    h->serving = false;
    mk::DevStatus st;
    int rc = read_status(h, &st);
    if (rc) return rc;
    return st.code != MK_OK ? st.code : MK_ERR_STOPPED;
}
}  // namespace

int mk_serve_start(mk_handle* h, float* logits_dev) {
    if (!h || h->serving || h->opt.mode != MK_MODE_MEGAKERNEL || h->p.nb > 1) return MK_ERR_INVALID_ARG;
    if (!h->scheduled) return MK_ERR_NO_SCHEDULE;
    if (!h->box_host) {
        void* ptr = nullptr;
        cudaError_t e = cudaHostAlloc(&ptr, sizeof(mk::ServeBox), cudaHostAllocMapped);
        if (e != cudaSuccess) return cuda_fail(h, e);
        h->box_host = static_cast<mk::ServeBox*>(ptr);
        void* dptr = nullptr;
        e = cudaHostGetDevicePointer(&dptr, ptr, 0);
        if (e != cudaSuccess) return cuda_fail(h, e);
        h->box_dev = static_cast<mk::ServeBox*>(dptr);
    }
    std::memset(h->box_host, 0, sizeof(mk::ServeBox));
    CK(cudaMemsetAsync(h->serve_ctr, 0, sizeof(uint32_t), h->stream));
    CK(cudaMemsetAsync(h->serve_step, 0, sizeof(mk::ServeStep), h->stream));
    mk::DevParams p = h->p;
    p.serve_box = h->box_dev;
    p.serve_step = h->serve_step;
    p.serve_ctr = h->serve_ctr;
    p.serve_idle_ns = h->opt.serve_idle_ns;
    mk::StepArgs a;
    a.token = 0;
    a.pos = 0;
    a.epoch = h->epoch;  // request k runs epoch + k
    a.logits = logits_dev ? logits_dev : h->p.logits;
    a.serve = 1;
    a.seq = 0;
    CK(mk::launch_megakernel(p, a, h->n_sm, h->variant, h->stream));
    CK(cudaEventRecord(h->ev_serve, h->stream));
    h->serving = true;
    h->serve_seq = 0;
    return MK_OK;
}

int mk_serve_step(mk_handle* h, int32_t token, int32_t pos, int32_t* next_token_host) {
    if (!h || !h->serving) return MK_ERR_INVALID_ARG;
    if (token >= h->cfg.vocab || pos < 0 || pos >= h->cfg.max_seq) return MK_ERR_INVALID_ARG;
    if (token < 0) token = -1;
    if (cudaEventQuery(h->ev_serve) != cudaErrorNotReady) return serve_ended(h);
    const int32_t seq = h->serve_seq + 1;
    post_request(h, token, pos, 0, seq);
    volatile mk::ServeBox* b = h->box_host;
    const double limit_s = host_wait_limit_s(h);
    const auto t0 = std::chrono::steady_clock::now();
    for (long it = 0;; ++it) {
        if (b->resp_seq == seq) break;
        if ((it & 1023) == 1023) {
            if (cudaEventQuery(h->ev_serve) != cudaErrorNotReady) {
                if (b->resp_seq == seq) break;
                return serve_ended(h);
            }
            if (std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count() > limit_s)
                return MK_ERR_TIMEOUT;
        }
    }
    std::atomic_thread_fence(std::memory_order_seq_cst);
    h->serve_seq = seq;
    h->epoch++;
    if (next_token_host) *next_token_host = b->next_token;
    return b->code;
}

int mk_serve_stop(mk_handle* h) {
    if (!h) return MK_ERR_INVALID_ARG;
    if (!h->serving) return MK_OK;
    post_request(h, 0, 0, 1, h->serve_seq + 1);
    int rc = wait_event(h, h->ev_serve);
    h->serving = false;
    if (rc) return rc;
    mk::DevStatus st;
    rc = read_status(h, &st);
    if (rc) return rc;
    return st.code;
}

void mk_destroy(mk_handle* h) {
    if (!h) return;
    if (h->serving) mk_serve_stop(h);
    cudaStreamSynchronize(h->stream);
    if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
    if (h->graph) cudaGraphDestroy(h->graph);
    for (void* ptr : h->allocs) cudaFree(ptr);
    if (h->status_pinned) cudaFreeHost(h->status_pinned);
    if (h->ev0) cudaEventDestroy(h->ev0);
    if (h->ev1) cudaEventDestroy(h->ev1);
    if (h->ev_done) cudaEventDestroy(h->ev_done);
    if (h->ev_serve) cudaEventDestroy(h->ev_serve);
    if (h->box_host) cudaFreeHost(h->box_host);
    delete h;
}

}  // extern "C"

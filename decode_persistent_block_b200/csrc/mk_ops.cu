// mk_ops.cu -- standalone opcode entry points (one plain launch per call),
// used for per-opcode parity tests and by callers that want a single op.
//
// mk_attention_decode: GQA decode attention of one layer over cached
// positions [0, n_pos), split along the sequence (split-KV) so that the
// low-occupancy op still spreads over many SMs, then merged by the
// log-sum-exp rule.  Query head h reads kv head floor(h / (n_q / n_kv)).
#include <cuda_runtime.h>
#include <math_constants.h>

#include <mutex>

#include "mk_device.cuh"
#include "mk_internal.h"
#include "mk_kernels.h"

namespace mk {
namespace {

constexpr int kOpThreads = 256;
constexpr int kOpWarps = kOpThreads / 32;

struct AttnOpArgs {
    const float* q;          // [nq][d], already rotated
    const uint16_t* kcache;  // [nkv][max_seq][d] bf16
    const uint16_t* vcache;
    int nq, nkv, n_pos, max_seq, splits;
    float* part_o;           // [nq][splits][d]
    float* part_ml;          // [nq][splits][2] (max score in log2 units, sum of exponentials)
    float* out;              // [nq][d]
};

// One block per (split, kv head): every query head of the group over the
// split's positions, online softmax per thread, merged across the block.
template <int D>
__global__ void __launch_bounds__(kOpThreads) attn_op_split(const AttnOpArgs a) {
    constexpr int LPR = D / 8;
    constexpr int RGN = kOpThreads / LPR;
    __shared__ float sq[kMaxGroup * D];
    __shared__ float sm_o[kOpWarps * kMaxGroup * D];
    __shared__ float sm_ml[kOpWarps * kMaxGroup * 2];
    const int G = a.nq / a.nkv;
    const int c = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int jb = (int)((long long)a.n_pos * c / a.splits), je = (int)((long long)a.n_pos * (c + 1) / a.splits);
    const float qscale = 1.4426950408889634f / sqrtf((float)D);
    for (int i = tid; i < G * D; i += kOpThreads) sq[i] = a.q[(size_t)g * G * D + i] * qscale;
    __syncthreads();
    const int col0 = (tid % LPR) * 8;
    float q[kMaxGroup][8], mx[kMaxGroup], ls[kMaxGroup], o[kMaxGroup][8];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        mx[h] = -CUDART_INF_F;
        ls[h] = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            o[h][k] = 0.f;
            q[h][k] = h < G ? sq[h * D + col0 + k] : 0.f;
        }
    }
    const uint16_t* K = a.kcache + (size_t)g * a.max_seq * D;
    const uint16_t* V = a.vcache + (size_t)g * a.max_seq * D;
    for (int base = jb; base < je; base += RGN) {
        const int j = base + tid / LPR;
        const bool valid = j < je;
        float kf[8], vf[8];
        if (valid) {
            unpack8(*reinterpret_cast<const uint4*>(K + (size_t)j * D + col0), kf);
            unpack8(*reinterpret_cast<const uint4*>(V + (size_t)j * D + col0), vf);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) kf[k] = vf[k] = 0.f;
        }
        float s[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            float t = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) t = fmaf(q[h][k], kf[k], t);
            s[h] = t;
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1)
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) s[h] += __shfl_xor_sync(0xFFFFFFFFu, s[h], off);
        if (valid) {
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) {
                if (h >= G) break;
                const float mn = fmaxf(mx[h], s[h]);
                const float al = exp2f(mx[h] - mn), pr = exp2f(s[h] - mn);
                ls[h] = ls[h] * al + pr;
#pragma unroll
                for (int k = 0; k < 8; ++k) o[h][k] = fmaf(pr, vf[k], o[h][k] * al);
                mx[h] = mn;
            }
        }
    }
    // merge the row groups of a warp, then the warps
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            const float m2 = __shfl_xor_sync(0xFFFFFFFFu, mx[h], off);
            const float l2 = __shfl_xor_sync(0xFFFFFFFFu, ls[h], off);
            float o2[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) o2[k] = __shfl_xor_sync(0xFFFFFFFFu, o[h][k], off);
            const float M = fmaxf(mx[h], m2);
            if (M != -CUDART_INF_F) {
                const float x = exp2f(mx[h] - M), y = exp2f(m2 - M);
                ls[h] = x * ls[h] + y * l2;
#pragma unroll
                for (int k = 0; k < 8; ++k) o[h][k] = x * o[h][k] + y * o2[k];
                mx[h] = M;
            }
        }
    if (lane < LPR)
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int k = 0; k < 8; ++k) sm_o[(warp * kMaxGroup + h) * D + col0 + k] = o[h][k];
            if (lane == 0) {
                sm_ml[(warp * kMaxGroup + h) * 2] = mx[h];
                sm_ml[(warp * kMaxGroup + h) * 2 + 1] = ls[h];
            }
        }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kOpThreads) {
        const int h = idx / D, col = idx % D;
        float M = -CUDART_INF_F;
        for (int w = 0; w < kOpWarps; ++w) M = fmaxf(M, sm_ml[(w * kMaxGroup + h) * 2]);
        float O = 0.f, L = 0.f;
        if (M != -CUDART_INF_F)
            for (int w = 0; w < kOpWarps; ++w) {
                const float f = exp2f(sm_ml[(w * kMaxGroup + h) * 2] - M);
                O += f * sm_o[(w * kMaxGroup + h) * D + col];
                L += f * sm_ml[(w * kMaxGroup + h) * 2 + 1];
            }
        const size_t slot = (size_t)(g * G + h) * a.splits + c;
        a.part_o[slot * D + col] = O;
        if (col == 0) {
            a.part_ml[slot * 2] = M;
            a.part_ml[slot * 2 + 1] = L;
        }
    }
}

// out[h] = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) L_c; grid nq, block d.
__global__ void attn_op_merge(const AttnOpArgs a, int D) {
    const int h = blockIdx.x, col = threadIdx.x;
    if (col >= D) return;
    float M = -CUDART_INF_F;
    for (int c = 0; c < a.splits; ++c) M = fmaxf(M, a.part_ml[((size_t)h * a.splits + c) * 2]);
    float num = 0.f, den = 0.f;
    for (int c = 0; c < a.splits; ++c) {
        const float m = a.part_ml[((size_t)h * a.splits + c) * 2];
        const float f = m == -CUDART_INF_F ? 0.f : exp2f(m - M);
        num += f * a.part_o[((size_t)h * a.splits + c) * D + col];
        den += f * a.part_ml[((size_t)h * a.splits + c) * 2 + 1];
    }
    a.out[(size_t)h * D + col] = num / den;
}

int check_attn_args(const float* q, const void* kc, const void* vc, int nq, int nkv, int d, int n_pos, int max_seq,
                    float* out, int splits) {
    if (!q || !kc || !vc || !out) return MK_ERR_INVALID_ARG;
    if (nq <= 0 || nkv <= 0 || n_pos <= 0 || max_seq < n_pos || splits <= 0) return MK_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return MK_ERR_UNSUPPORTED;
    if (nq % nkv || nq / nkv > kMaxGroup) return MK_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(kc) | reinterpret_cast<uintptr_t>(vc)) & 15u) return MK_ERR_INVALID_ARG;
    return MK_OK;
}

int launch_attn(const AttnOpArgs& a, int d, cudaStream_t s) {
    const dim3 grid(a.splits, a.nkv);
    if (d == 64) attn_op_split<64><<<grid, kOpThreads, 0, s>>>(a);
    else attn_op_split<128><<<grid, kOpThreads, 0, s>>>(a);
    attn_op_merge<<<a.nq, d, 0, s>>>(a, d);
    return cudaGetLastError() == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}

}  // namespace
}  // namespace mk

extern "C" size_t mk_attention_workspace_bytes(int n_q_heads, int head_dim, int splits) {
    if (n_q_heads <= 0 || head_dim <= 0 || splits <= 0) return 0;
    return sizeof(float) * (size_t)n_q_heads * (size_t)splits * (size_t)(head_dim + 2);
}

extern "C" int mk_attention_decode(const float* q, const void* k_cache, const void* v_cache, int n_q_heads,
                                   int n_kv_heads, int head_dim, int n_pos, int max_seq, int splits, float* out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    int rc = mk::check_attn_args(q, k_cache, v_cache, n_q_heads, n_kv_heads, head_dim, n_pos, max_seq, out, splits);
    if (rc) return rc;
    const size_t need = mk_attention_workspace_bytes(n_q_heads, head_dim, splits);
    if (!workspace || workspace_bytes < need) return MK_ERR_CAPACITY;
    mk::AttnOpArgs a;
    a.q = q;
    a.kcache = static_cast<const uint16_t*>(k_cache);
    a.vcache = static_cast<const uint16_t*>(v_cache);
    a.nq = n_q_heads;
    a.nkv = n_kv_heads;
    a.n_pos = n_pos;
    a.max_seq = max_seq;
    a.splits = splits;
    a.part_o = static_cast<float*>(workspace);
    a.part_ml = a.part_o + (size_t)n_q_heads * splits * head_dim;
    a.out = out;
    return mk::launch_attn(a, head_dim, static_cast<cudaStream_t>(stream));
}

// ---- variant without allocation -------------------------------------------------------------
//
// Scratch for mk_attention_decode_noalloc: the split partials live in this
// file-scope device array instead of a caller workspace.  Every GPU that loads
// the library holds it (MK_ATTENTION_NOALLOC_SCRATCH_BYTES) until the process
// exits.  All calls share it and it keeps the last call's contents; the split
// kernel writes every partial slot a call reads, so nothing needs clearing.
static __device__ __align__(256) float g_attn_noalloc_scratch[MK_ATTENTION_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {
constexpr int kMaxDevices = 64;
// Host-side cache of the array's device address, per device ordinal, with the
// context it was looked up in: a device reset (cudaDeviceReset) gives the
// device a new context and the module a new address, so the lookup is redone
// whenever the current context differs from the cached one.
float* g_scratch_addr[kMaxDevices];
CUcontext g_scratch_ctx[kMaxDevices];
std::mutex g_scratch_mu;

CUresult current_context(CUcontext* ctx) {
    using GetCurrent = CUresult (*)(CUcontext*);
    static GetCurrent fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p)
            return CUDA_ERROR_NOT_FOUND;
        fn = reinterpret_cast<GetCurrent>(p);
    }
    return fn(ctx);
}
}  // namespace

extern "C" int mk_attention_decode_noalloc(const float* q, const void* k_cache, const void* v_cache, int n_q_heads,
                                           int n_kv_heads, int head_dim, int n_pos, int max_seq, int splits,
                                           float* out, void* stream) {
    int rc = mk::check_attn_args(q, k_cache, v_cache, n_q_heads, n_kv_heads, head_dim, n_pos, max_seq, out, splits);
    if (rc) return rc;
    if (mk_attention_workspace_bytes(n_q_heads, head_dim, splits) > MK_ATTENTION_NOALLOC_SCRATCH_BYTES)
        return MK_ERR_CAPACITY;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MK_ERR_CUDA;
    float* scratch = nullptr;
    {
        // Set-up, once per device, with that device current: the array's name is a
        // host-side stand-in, so its device address has to be looked up.
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        CUcontext ctx = nullptr;
        if (!g_scratch_addr[dev] || current_context(&ctx) != CUDA_SUCCESS || ctx != g_scratch_ctx[dev]) {
            void* addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_attn_noalloc_scratch) != cudaSuccess || !addr) return MK_ERR_CUDA;
            if (current_context(&ctx) != CUDA_SUCCESS) ctx = nullptr;
            g_scratch_addr[dev] = static_cast<float*>(addr);
            g_scratch_ctx[dev] = ctx;
        }
        scratch = g_scratch_addr[dev];
    }
    mk::AttnOpArgs a;
    a.q = q;
    a.kcache = static_cast<const uint16_t*>(k_cache);
    a.vcache = static_cast<const uint16_t*>(v_cache);
    a.nq = n_q_heads;
    a.nkv = n_kv_heads;
    a.n_pos = n_pos;
    a.max_seq = max_seq;
    a.splits = splits;
    a.part_o = scratch;
    a.part_ml = scratch + (size_t)n_q_heads * splits * head_dim;
    a.out = out;
    return mk::launch_attn(a, head_dim, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Set-up: bf16 transpose through a 32 x 33 shared tile (coalesced on both sides).
namespace mk {
namespace {
__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int rows,
                                      int cols) {
    __shared__ uint16_t tile[32][33];
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < cols) tile[i][threadIdx.x] = src[(size_t)r * cols + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (r < rows && c < cols) dst[(size_t)c * rows + r] = tile[threadIdx.x][i];
    }
}
}  // namespace

cudaError_t launch_transpose_bf16(const uint16_t* src, uint16_t* dst, int rows, int cols, cudaStream_t stream) {
    if (rows <= 0 || cols <= 0) return cudaSuccess;
    const dim3 grid((unsigned)((cols + 31) / 32), (unsigned)((rows + 31) / 32));
    transpose_bf16_kernel<<<grid, dim3(32, 8), 0, stream>>>(src, dst, rows, cols);
    return cudaGetLastError();
}
}  // namespace mk

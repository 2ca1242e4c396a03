// mk_baseline.cu -- the plain multi-kernel baseline of the same opcodes.
//
// One ordinary launch per op and layer (about 5 per layer plus the LM head and
// the argmax), each kernel reading its weights straight from global memory
// with 128-bit loads, one warp per output row.  Between launches every kernel
// starts cold: its operands come in from memory, its result goes back out, and
// the next launch reads that result again.  That round trip is the cost the
// persistent kernel removes (Hyperkernel teardown, "What a megakernel buys").  Step parameters come from a small device buffer so the
// launch sequence can be replayed from a CUDA graph.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "mk_device.cuh"
#include "mk_internal.h"
#include "mk_kernels.h"

namespace mk {

namespace {

constexpr int kBT = 256;  // threads per block
constexpr int kBW = kBT / 32;

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Fill smem vec[0..K) with rmsnorm(x) * nw (x fp32 or a bf16 row).
__device__ void block_rmsnorm(const float* x32, const uint16_t* x16, const uint16_t* nw, int K, float eps,
                              float* vec, float* red) {
    const int tid = threadIdx.x;
    float ss = 0.f;
    for (int i = tid; i < K; i += kBT) {
        const float xv = x16 ? __uint_as_float((uint32_t)x16[i] << 16) : __ldcg(x32 + i);
        vec[i] = xv;
        ss = fmaf(xv, xv, ss);
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < kBW; ++w) tot += red[w];
    const float rs = 1.0f / sqrtf(tot / (float)K + eps);
    for (int i = tid; i < K; i += kBT) vec[i] = vec[i] * rs * __uint_as_float((uint32_t)nw[i] << 16);
    __syncthreads();
}

// One row of W (bf16, K columns) dotted with smem vec, by one warp.
__device__ __forceinline__ float warp_row_dot(const uint16_t* row, const float* vec, int K) {
    const int lane = threadIdx.x & 31;
    float acc = 0.f;
    const int nch = K >> 3;
    for (int c = lane; c < nch; c += 32) {
        const uint4 wv = ldg_stream(reinterpret_cast<const uint4*>(row) + c);
        acc = dot8(wv, vec + 8 * c, acc);
    }
    return warp_sum(acc);
}

__device__ __forceinline__ int step_token(const StepBuf* sb) { return sb->token; }

// ---- kernels ------------------------------------------------------------------------------

__global__ void bl_set_step(StepBuf* sb, DevStatus* st, int token, int pos) {
    sb->token = token >= 0 ? token : st->next_token;
    sb->pos = pos;
}

// out[r] = W[r] . rmsnorm(x) * nw, rows [0, rows), `rpb` rows per block.
// x is the embedding row of the step's token when `embed_input` is set.
__global__ void __launch_bounds__(kBT) bl_rms_matvec(const __grid_constant__ DevParams p, const StepBuf* sb,
                                                     int embed_input, const uint16_t* nw, const uint16_t* W,
                                                     int rows, int rpb, float* out) {
    extern __shared__ float vec[];
    __shared__ float red[kBW];
    const int K = p.H;
    const uint16_t* x16 = embed_input ? p.embed + (size_t)step_token(sb) * K : nullptr;
    block_rmsnorm(p.x, x16, nw, K, p.eps, vec, red);
    const int r0 = blockIdx.x * rpb, r1 = min(rows, r0 + rpb);
    for (int r = r0 + (threadIdx.x >> 5); r < r1; r += kBW) {
        const float s = warp_row_dot(W + (size_t)r * K, vec, K);
        if ((threadIdx.x & 31) == 0) out[r] = s;
    }
}

// h[r] = silu(Wg[r] . xn) * (Wu[r] . xn), xn = rmsnorm(x) * w_ffn.  For MoE
// (`slot` >= 0) the expert is the routed one of that slot.
__global__ void __launch_bounds__(kBT) bl_rms_upgate(const __grid_constant__ DevParams p, int layer, int slot,
                                                     int rpb) {
    extern __shared__ float vec[];
    __shared__ float red[kBW];
    const int K = p.H;
    const uint16_t* const* wt = p.wt + (size_t)layer * wt_stride(p.E);
    const int e = slot >= 0 ? p.router_idx[layer * kMaxTopK + slot] : 0;
    const uint16_t* Wg = wt[wt_gate(e)];
    const uint16_t* Wu = wt[wt_up(e, p.E)];
    float* h = p.hbuf + (slot > 0 ? (size_t)slot * p.F : 0);
    block_rmsnorm(p.x, nullptr, wt[WT_FFN_NORM], K, p.eps, vec, red);
    const int r0 = blockIdx.x * rpb, r1 = min(p.F, r0 + rpb);
    for (int r = r0 + (threadIdx.x >> 5); r < r1; r += kBW) {
        const float g = warp_row_dot(Wg + (size_t)r * K, vec, K);
        const float u = warp_row_dot(Wu + (size_t)r * K, vec, K);
        if ((threadIdx.x & 31) == 0) h[r] = g / (1.0f + expf(-g)) * u;
    }
}

// x[r] = base[r] + sum_s wgt_s * W_s[r] . vec_s: O-proj (vec = attn, one
// slot), dense down (vec = h) or the fused expert down-projection (vec_s = h of
// slot s, W_s the routed expert's rows, wgt_s its router weight).  base = the
// embedding row for layer 0's O-proj, else x.
__global__ void __launch_bounds__(kBT) bl_matvec_res(const __grid_constant__ DevParams p, const StepBuf* sb,
                                                     int layer, int which, int rpb) {
    extern __shared__ float vec[];
    const uint16_t* const* wt = p.wt + (size_t)layer * wt_stride(p.E);
    const bool oproj = which == 0;
    const int K = oproj ? p.nq * p.d : p.F;
    const int nslot = (!oproj && p.E > 0) ? p.topk : 1;
    for (int s = 0; s < nslot; ++s)
        for (int i = threadIdx.x; i < K; i += kBT)
            vec[(size_t)s * K + i] = __ldcg((oproj ? p.attn : p.hbuf + (size_t)s * p.F) + i);
    __syncthreads();
    const int r0 = blockIdx.x * rpb, r1 = min(p.H, r0 + rpb);
    for (int r = r0 + (threadIdx.x >> 5); r < r1; r += kBW) {
        float acc = 0.f;
        for (int s = 0; s < nslot; ++s) {
            const uint16_t* W;
            float wgt = 1.f;
            if (oproj) {
                W = wt[WT_O];
            } else if (p.E > 0) {
                W = wt[wt_down(p.router_idx[layer * kMaxTopK + s], p.E)];
                wgt = p.router_w[layer * kMaxTopK + s];
            } else {
                W = wt[wt_down(0, p.E)];
            }
            const float dsum = warp_row_dot(W + (size_t)r * K, vec + (size_t)s * K, K);
            acc = (p.E > 0 && !oproj) ? fmaf(wgt, dsum, acc) : dsum;
        }
        if ((threadIdx.x & 31) == 0) {
            float base;
            if (oproj && layer == 0) {
                base = __uint_as_float((uint32_t)p.embed[(size_t)step_token(sb) * p.H + r] << 16);
                if (p.snap) p.snap[r] = base;
            } else {
                base = __ldcg(p.x + r);
            }
            const float nx = base + acc;
            p.x[r] = nx;
            if (!oproj && p.snap) p.snap[(size_t)(layer + 1) * p.H + r] = nx;
        }
    }
}

// RoPE + append + one split of GQA attention per block: grid (splits, kv heads).
template <int D, int G>
__global__ void __launch_bounds__(kBT) bl_attn_split(const __grid_constant__ DevParams p, const StepBuf* sb,
                                                     int layer) {
    constexpr int LPR = D / 8;
    constexpr int RGN = kBT / LPR;
    __shared__ float sq[G * D];
    __shared__ float sm_o[kBW * G * D];
    __shared__ float sm_ml[kBW * G * 2];
    const int c = blockIdx.x, S = gridDim.x, g = blockIdx.y, pos = sb->pos;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long npos = (long long)pos + 1;
    const int jb = (int)(npos * c / S), je = (int)(npos * (c + 1) / S);
    const float2* rp = p.rope + (size_t)pos * (D / 2);
    const float qscale = 1.4426950408889634f / sqrtf((float)D);
    // rotated, scaled q of the group into smem
    for (int idx = tid; idx < G * D; idx += kBT) {
        const int h = idx / D, i = idx % D;
        const float* src = p.qkv + (size_t)(g * G + h) * D;
        const float2 cs = rp[i & (D / 2 - 1)];
        const float x = __ldcg(src + i), y = __ldcg(src + (i ^ (D / 2)));
        sq[idx] = (i < D / 2 ? x * cs.x - y * cs.y : x * cs.x + y * cs.y) * qscale;
    }
    // append the new position (its own split writes it; every split that covers
    // it reads the same bf16-rounded values from registers)
    const int col0 = (tid % LPR) * 8;
    float kn[8], vn[8];
    const bool has_new = (je == npos);
    if (has_new && tid < LPR) {
        const float* ks = p.qkv + (size_t)p.nq * D + (size_t)g * D;
        const float* vs = p.qkv + (size_t)(p.nq + p.nkv) * D + (size_t)g * D;
        uint32_t kb[8], vb[8];
        for (int k = 0; k < 8; ++k) {
            const int i = col0 + k;
            const float2 cs = rp[i & (D / 2 - 1)];
            const float x = __ldcg(ks + i), y = __ldcg(ks + (i ^ (D / 2)));
            kb[k] = f2bf(i < D / 2 ? x * cs.x - y * cs.y : x * cs.x + y * cs.y);
            vb[k] = f2bf(__ldcg(vs + i));
            kn[k] = __uint_as_float(kb[k] << 16);
            vn[k] = __uint_as_float(vb[k] << 16);
        }
        const size_t off = (((size_t)layer * p.nkv + g) * (size_t)p.max_seq + (size_t)pos) * D + col0;
        for (int k = 0; k < 8; ++k) {
            p.kcache[off + k] = (uint16_t)kb[k];
            p.vcache[off + k] = (uint16_t)vb[k];
        }
    }
    __syncthreads();
    float q[G][8], mx[G], ls[G], o[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        mx[h] = -CUDART_INF_F;
        ls[h] = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            o[h][k] = 0.f;
            q[h][k] = sq[h * D + col0 + k];
        }
    }
    const int jce = je < pos ? je : pos;
    const uint16_t* Kb = p.kcache + ((size_t)layer * p.nkv + g) * (size_t)p.max_seq * D;
    const uint16_t* Vb = p.vcache + ((size_t)layer * p.nkv + g) * (size_t)p.max_seq * D;
    auto update = [&](const float* kf, const float* vf, bool valid) {
        float s[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float t = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) t = fmaf(q[h][k], kf[k], t);
            s[h] = t;
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1)
#pragma unroll
            for (int h = 0; h < G; ++h) s[h] += __shfl_xor_sync(0xFFFFFFFFu, s[h], off);
        if (valid)
            for (int h = 0; h < G; ++h) {
                const float mn = fmaxf(mx[h], s[h]);
                const float al = exp2f(mx[h] - mn), pr = exp2f(s[h] - mn);
                ls[h] = ls[h] * al + pr;
                for (int k = 0; k < 8; ++k) o[h][k] = fmaf(pr, vf[k], o[h][k] * al);
                mx[h] = mn;
            }
    };
    for (int base = jb; base < jce; base += RGN) {
        const int j = base + tid / LPR;
        const bool valid = j < jce;
        float kf[8], vf[8];
        if (valid) {
            unpack8(ldg_stream(Kb + (size_t)j * D + col0), kf);
            unpack8(ldg_stream(Vb + (size_t)j * D + col0), vf);
        } else {
            for (int k = 0; k < 8; ++k) kf[k] = vf[k] = 0.f;
        }
        update(kf, vf, valid);
    }
    if (has_new && warp == 0) update(kn, vn, lane < LPR);
    for (int off = LPR; off < 32; off <<= 1)
        for (int h = 0; h < G; ++h) {
            const float m2 = __shfl_xor_sync(0xFFFFFFFFu, mx[h], off);
            const float l2 = __shfl_xor_sync(0xFFFFFFFFu, ls[h], off);
            float o2[8];
            for (int k = 0; k < 8; ++k) o2[k] = __shfl_xor_sync(0xFFFFFFFFu, o[h][k], off);
            const float M = fmaxf(mx[h], m2);
            if (M != -CUDART_INF_F) {
                const float a = exp2f(mx[h] - M), b = exp2f(m2 - M);
                ls[h] = a * ls[h] + b * l2;
                for (int k = 0; k < 8; ++k) o[h][k] = a * o[h][k] + b * o2[k];
                mx[h] = M;
            }
        }
    if (lane < LPR)
        for (int h = 0; h < G; ++h) {
            for (int k = 0; k < 8; ++k) sm_o[(warp * G + h) * D + col0 + k] = o[h][k];
            if (lane == 0) {
                sm_ml[(warp * G + h) * 2] = mx[h];
                sm_ml[(warp * G + h) * 2 + 1] = ls[h];
            }
        }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kBT) {
        const int h = idx / D, col = idx % D;
        float M = -CUDART_INF_F;
        for (int w = 0; w < kBW; ++w) M = fmaxf(M, sm_ml[(w * G + h) * 2]);
        float O = 0.f, Ls = 0.f;
        if (M != -CUDART_INF_F)
            for (int w = 0; w < kBW; ++w) {
                const float f = exp2f(sm_ml[(w * G + h) * 2] - M);
                O += f * sm_o[(w * G + h) * D + col];
                Ls += f * sm_ml[(w * G + h) * 2 + 1];
            }
        const size_t part = (size_t)(g * G + h) * S + c;
        p.part_o[part * D + col] = O;
        if (col == 0) {
            p.part_ml[part * 2] = M;
            p.part_ml[part * 2 + 1] = Ls;
        }
    }
}

// attn[h] = merge of the splits' (m, l, o) partials; grid nq, block d.
__global__ void bl_attn_merge(const __grid_constant__ DevParams p, int S) {
    const int h = blockIdx.x, col = threadIdx.x, D = p.d;
    if (col >= D) return;
    float M = -CUDART_INF_F;
    for (int s = 0; s < S; ++s) M = fmaxf(M, p.part_ml[((size_t)h * S + s) * 2]);
    float num = 0.f, den = 0.f;
    for (int s = 0; s < S; ++s) {
        const float ms = p.part_ml[((size_t)h * S + s) * 2];
        const float f = ms == -CUDART_INF_F ? 0.f : exp2f(ms - M);
        num += f * p.part_o[((size_t)h * S + s) * D + col];
        den += f * p.part_ml[((size_t)h * S + s) * 2 + 1];
    }
    p.attn[(size_t)h * D + col] = num / den;
}

// Router of a MoE layer: logits, top-k (ties to the lower index), softmax over the selected.
__global__ void __launch_bounds__(kBT) bl_router(const __grid_constant__ DevParams p, int layer) {
    extern __shared__ float vec[];
    __shared__ float red[kBW];
    __shared__ float logit[64];
    const uint16_t* const* wt = p.wt + (size_t)layer * wt_stride(p.E);
    block_rmsnorm(p.x, nullptr, wt[WT_FFN_NORM], p.H, p.eps, vec, red);
    for (int e = threadIdx.x >> 5; e < p.E; e += kBW) {
        const float s = warp_row_dot(wt[WT_ROUTER] + (size_t)e * p.H, vec, p.H);
        if ((threadIdx.x & 31) == 0) logit[e] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int idx[kMaxTopK];
        unsigned long long taken = 0;
        for (int k = 0; k < p.topk; ++k) {
            int best = -1;
            for (int e = 0; e < p.E; ++e) {
                if ((taken >> e) & 1ull) continue;
                if (best < 0 || logit[e] > logit[best]) best = e;
            }
            taken |= 1ull << best;
            idx[k] = best;
        }
        float z = 0.f, ex[kMaxTopK];
        for (int k = 0; k < p.topk; ++k) {
            ex[k] = expf(logit[idx[k]] - logit[idx[0]]);
            z += ex[k];
        }
        for (int k = 0; k < p.topk; ++k) {
            p.router_idx[layer * kMaxTopK + k] = idx[k];
            p.router_w[layer * kMaxTopK + k] = ex[k] / z;
        }
    }
}

// LM head rows of one block + the block's (max, argmax) partial.
__global__ void __launch_bounds__(kBT) bl_lm_head(const __grid_constant__ DevParams p, const StepBuf* sb, int rpb,
                                                  float* logits) {
    extern __shared__ float vec[];
    __shared__ float red[kBW];
    __shared__ int redi[kBW];
    const uint16_t* x16 = p.L == 0 ? p.embed + (size_t)step_token(sb) * p.H : nullptr;
    if (x16 && p.snap && blockIdx.x == 0)  // no layers: the residual stream is the embedding row
        for (int i = threadIdx.x; i < p.H; i += kBT) p.snap[i] = __uint_as_float((uint32_t)x16[i] << 16);
    block_rmsnorm(p.x, x16, p.final_norm, p.H, p.eps, vec, red);
    __syncthreads();
    const int r0 = blockIdx.x * rpb, r1 = min(p.V, r0 + rpb);
    float bv = -CUDART_INF_F;
    int bi = 0x7FFFFFFF;
    for (int r = r0 + (threadIdx.x >> 5); r < r1; r += kBW) {
        const float s = warp_row_dot(p.lm_head + (size_t)r * p.H, vec, p.H);
        if ((threadIdx.x & 31) == 0) logits[r] = s;
        if (s > bv || (s == bv && r < bi)) {
            bv = s;
            bi = r;
        }
    }
    warp_argmax(bv, bi);
    if ((threadIdx.x & 31) == 0) {
        red[threadIdx.x >> 5] = bv;
        redi[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kBW; ++w)
            if (red[w] > bv || (red[w] == bv && redi[w] < bi)) {
                bv = red[w];
                bi = redi[w];
            }
        p.lm_part[2 * blockIdx.x] = bv;
        p.lm_part[2 * blockIdx.x + 1] = __int_as_float(bi);
    }
}

__global__ void __launch_bounds__(kBT) bl_argmax(const __grid_constant__ DevParams p, int n) {
    __shared__ float red[kBW];
    __shared__ int redi[kBW];
    float bv = -CUDART_INF_F;
    int bi = 0x7FFFFFFF;
    for (int k = threadIdx.x; k < n; k += kBT) {
        const float v = p.lm_part[2 * k];
        const int i = __float_as_int(p.lm_part[2 * k + 1]);
        if (v > bv || (v == bv && i < bi)) {
            bv = v;
            bi = i;
        }
    }
    warp_argmax(bv, bi);
    if ((threadIdx.x & 31) == 0) {
        red[threadIdx.x >> 5] = bv;
        redi[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kBW; ++w)
            if (red[w] > bv || (red[w] == bv && redi[w] < bi)) {
                bv = red[w];
                bi = redi[w];
            }
        p.status->next_token = bi;
    }
}

int rows_per_block(int rows, int n_sm) {
    int r = (rows + n_sm * 4 - 1) / (n_sm * 4);
    r = (r + 7) / 8 * 8;
    if (r < 8) r = 8;
    if (r > 512) r = 512;
    return r;
}

template <int D>
void launch_attn_split(const DevParams& p, const StepBuf* sb, int layer, cudaStream_t s) {
    const dim3 grid(p.kv_splits, p.nkv);
    switch (p.nq / p.nkv) {
        case 1: bl_attn_split<D, 1><<<grid, kBT, 0, s>>>(p, sb, layer); break;
        case 2: bl_attn_split<D, 2><<<grid, kBT, 0, s>>>(p, sb, layer); break;
        case 3: bl_attn_split<D, 3><<<grid, kBT, 0, s>>>(p, sb, layer); break;
        case 4: bl_attn_split<D, 4><<<grid, kBT, 0, s>>>(p, sb, layer); break;
        case 8:
            if constexpr (D == 64) bl_attn_split<D, 8><<<grid, kBT, 0, s>>>(p, sb, layer);
            break;
    }
}

}  // namespace

int baseline_lm_blocks(const DevParams& p, int n_sm) {
    const int rpb = rows_per_block(p.V, n_sm);
    return (p.V + rpb - 1) / rpb;
}

cudaError_t prepare_baseline() {
    const int big = 2 * 16384 * 4;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(bl_rms_matvec, cudaFuncAttributeMaxDynamicSharedMemorySize, big))) return e;
    if ((e = cudaFuncSetAttribute(bl_rms_upgate, cudaFuncAttributeMaxDynamicSharedMemorySize, big))) return e;
    if ((e = cudaFuncSetAttribute(bl_matvec_res, cudaFuncAttributeMaxDynamicSharedMemorySize, big))) return e;
    if ((e = cudaFuncSetAttribute(bl_router, cudaFuncAttributeMaxDynamicSharedMemorySize, big))) return e;
    if ((e = cudaFuncSetAttribute(bl_lm_head, cudaFuncAttributeMaxDynamicSharedMemorySize, big))) return e;
    return cudaSuccess;
}

cudaError_t launch_baseline_set_step(const DevParams& p, StepBuf* sb, int token, int pos, cudaStream_t stream) {
    bl_set_step<<<1, 1, 0, stream>>>(sb, p.status, token, pos);
    return cudaGetLastError();
}

cudaError_t launch_baseline_layers(const DevParams& p, const uint16_t* const* wt_host, const StepBuf* sb,
                                   const BaselineShape& bs, float* logits, cudaStream_t s) {
    const int n_sm = bs.n_sm, H = p.H, d = p.d, F = p.F;
    const int stride = wt_stride(p.E);
    const size_t vH = (size_t)H * 4, vQ = (size_t)p.nq * d * 4;
    const size_t vF = (size_t)F * 4 * (p.E > 0 ? p.topk : 1);
    for (int l = 0; l < p.L; ++l) {
        const uint16_t* const* wt = wt_host + (size_t)l * stride;
        const int nqd = p.nq * d, nkd = p.nkv * d;
        const int rows[3] = {nqd, nkd, nkd}, off[3] = {0, nqd, nqd + nkd};
        for (int i = 0; i < 3; ++i) {
            const int rpb = rows_per_block(rows[i], n_sm);
            bl_rms_matvec<<<(rows[i] + rpb - 1) / rpb, kBT, vH, s>>>(p, sb, l == 0, wt[WT_ATTN_NORM], wt[WT_Q + i],
                                                                     rows[i], rpb, p.qkv + off[i]);
        }
        if (d == 64) launch_attn_split<64>(p, sb, l, s);
        else launch_attn_split<128>(p, sb, l, s);
        bl_attn_merge<<<p.nq, d, 0, s>>>(p, p.kv_splits);
        int rpb = rows_per_block(H, n_sm);
        bl_matvec_res<<<(H + rpb - 1) / rpb, kBT, vQ, s>>>(p, sb, l, 0, rpb);
        rpb = rows_per_block(F, n_sm);
        if (p.E == 0) {
            bl_rms_upgate<<<(F + rpb - 1) / rpb, kBT, vH, s>>>(p, l, -1, rpb);
        } else {
            bl_router<<<1, kBT, vH, s>>>(p, l);
            for (int slot = 0; slot < p.topk; ++slot)
                bl_rms_upgate<<<(F + rpb - 1) / rpb, kBT, vH, s>>>(p, l, slot, rpb);
        }
        rpb = rows_per_block(H, n_sm);
        bl_matvec_res<<<(H + rpb - 1) / rpb, kBT, vF, s>>>(p, sb, l, 1, rpb);
    }
    const int rpb = rows_per_block(p.V, n_sm);
    const int nb = (p.V + rpb - 1) / rpb;
    bl_lm_head<<<nb, kBT, vH, s>>>(p, sb, rpb, logits);
    bl_argmax<<<1, kBT, 0, s>>>(p, nb);
    return cudaGetLastError();
}

}  // namespace mk

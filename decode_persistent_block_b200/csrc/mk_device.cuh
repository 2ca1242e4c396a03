// mk_device.cuh -- sm_100a device helpers: mbarriers, TMA bulk copies, L2
// prefetch, acquire/release counter ops, globaltimer, bf16 unpacking and
// warp reductions.  Inline PTX written for this library.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "mk_internal.h"

namespace mk {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarriers ----------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// One probe of phase `parity`; true when that phase has completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Probe with a suspend-time hint: a thread whose phase is not complete is
// suspended (it issues nothing) until the phase completes or `hint_ns` passes,
// instead of spinning and taking issue slots from the other warps of its SM
// sub-partition.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// ---- TMA bulk copy (1D, no tensor map) and L2 prefetch --------------------------
// dst/src 16-byte aligned, bytes a multiple of 16.  Completion is reported as
// transaction bytes on `bar`.  Never the multicast form.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// The same with an L2 cache policy (make_evict_first_policy): the copy's lines are
// the first candidates for eviction, so a stream read once per step does not push
// the data that is reused across steps (KV cache, activations, counters) out of L2.
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
// L2 policy for the whole of a copy: evict first.
__device__ __forceinline__ uint64_t make_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// 2-D tensor-map box load (coordinates: x = column, y = row) into shared
// memory, completion as transaction bytes on `bar`.  x * 2 bytes is a
// multiple of 16 at every call site.  Never the multicast form.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// ldmatrix: four 8x8 b16 matrices, row addresses from lanes 8i..8i+7 for matrix i.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
// d = a * b + c, m16n8k16, bf16 operands (a row-major, b column-major), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same when rows 8..15 of a are zero: only the accumulators of rows 0..7
// (c0, c1 of each lane) are kept; the other two outputs are discarded.
__device__ __forceinline__ void mma_bf16_top(float& c0, float& c1, uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    float d2 = 0.f, d3 = 0.f;
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %10, %10};"
        : "+f"(c0), "+f"(c1), "=f"(d2), "=f"(d3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(0.f));
    asm volatile("" ::"f"(d2), "f"(d3));  // discarded outputs of rows 8..15
}

__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// L2 prefetch of one 128-byte line through the load/store path (not the TMA
// queue, which stays free for the ring's copies).
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// ---- global-memory counters -------------------------------------------------------
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Publish one arrival on a dependency counter: a release reduction, which
// orders every write this block made before the preceding block barrier
// (cumulatively, at gpu scope) ahead of the increment.  Measured a little
// faster than a separate fence.acq_rel followed by a relaxed reduction.
__device__ __forceinline__ void signal_release(uint32_t* ctr) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}
// Arrival that also returns the previous count (last-arriver detection): an
// acquire-release atomic, so the block's earlier writes (ordered by the
// preceding block barrier) are visible before the count moves, and the last
// arrival sees every other arrival's writes once the caller's next block
// barrier has passed.  Measured faster than a fence, a relaxed atomic and a
// second fence in the last arrival.
__device__ __forceinline__ uint32_t arrive_release(uint32_t* ctr) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(ctr) : "memory");
    return old;
}
__device__ __forceinline__ int ld_relaxed_s32(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- bf16 ------------------------------------------------------------------------
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ void unpack8(const uint4 w, float* f) {
    f[0] = bf_lo(w.x); f[1] = bf_hi(w.x);
    f[2] = bf_lo(w.y); f[3] = bf_hi(w.y);
    f[4] = bf_lo(w.z); f[5] = bf_hi(w.z);
    f[6] = bf_lo(w.w); f[7] = bf_hi(w.w);
}
// sum_k bf16(w)_k * v_k, fp32, ascending k
__device__ __forceinline__ float dot8(const uint4 w, const float* v, float acc) {
    acc = fmaf(bf_lo(w.x), v[0], acc);
    acc = fmaf(bf_hi(w.x), v[1], acc);
    acc = fmaf(bf_lo(w.y), v[2], acc);
    acc = fmaf(bf_hi(w.y), v[3], acc);
    acc = fmaf(bf_lo(w.z), v[4], acc);
    acc = fmaf(bf_hi(w.z), v[5], acc);
    acc = fmaf(bf_lo(w.w), v[6], acc);
    acc = fmaf(bf_hi(w.w), v[7], acc);
    return acc;
}
// Two fp32 values as bf16x2 (x0 in the low half), each rounded to nearest even: one cvt.
__device__ __forceinline__ uint32_t pack_bf16x2(float x0, float x1) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(x1), "f"(x0));
    return d;
}
// fp32 -> bf16 bits, round to nearest even
__device__ __forceinline__ uint32_t f2bf(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (u >> 16) | 0x40u;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return u >> 16;
}

// ---- warp reductions ----------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}
// (value, index) max with ties to the lower index
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, v, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, i, o);
        if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
    }
}
// Two fp32 FMAs in one instruction (sm_100 packed f32x2):
// (a.x * b.x + c.x, a.y * b.y + c.y), each rounded to nearest like fmaf.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Transpose-reduce of RG per-lane partials (one per row, RG a power of two up
// to 32) across the warp: log2(RG) halving rounds exchange half of the values,
// then 5 - log2(RG) butterfly rounds finish the sum (RG - 1 + 5 - log2(RG)
// shuffles instead of 5 * RG).  On return every lane holds the full sum of row
// lane >> (5 - log2(RG)).
template <int RG>
__device__ __forceinline__ float reduce_rows(float (&a)[RG], int lane) {
#pragma unroll
    for (int n = RG, off = 16; n > 1; n >>= 1, off >>= 1) {
        const bool up = lane & off;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = up ? a[i] : a[i + n / 2];
            const float keep = up ? a[i + n / 2] : a[i];
            a[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
        }
    }
    constexpr int first = RG == 32 ? 0 : RG == 16 ? 1 : RG == 8 ? 2 : RG == 4 ? 4 : RG == 2 ? 8 : 16;
    float e = a[0];
#pragma unroll
    for (int off = first; off > 0; off >>= 1) e += __shfl_xor_sync(0xFFFFFFFFu, e, off);
    return e;
}
template <int RG>
__device__ __forceinline__ int reduce_rows_lane_row(int lane) {
    return RG == 32 ? lane : RG == 16 ? lane >> 1 : RG == 8 ? lane >> 2 : RG == 4 ? lane >> 3 : RG == 2 ? lane >> 4 : 0;
}
template <int RG>
__device__ __forceinline__ bool reduce_rows_writer(int lane) {
    return (lane & (32 / RG - 1)) == 0;
}

// ---- status -------------------------------------------------------------------------
__device__ __forceinline__ void record_error(DevStatus* st, int code, int sm, int instr, int op, int ctr,
                                             uint32_t observed, uint32_t expected) {
    if (atomicCAS(&st->code, 0, code) == 0) {
        st->sm = sm;
        st->instr = instr;
        st->opcode = op;
        st->counter = ctr;
        st->observed = observed;
        st->expected = expected;
    }
    __threadfence();
    atomicExch(&st->stop, 1);
}

}  // namespace mk

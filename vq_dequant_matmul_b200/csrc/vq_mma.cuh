// vq_mma.cuh — building blocks of the tensor-core GEMV (dense decode and grouped MoE):
// shared-memory loads by 32-bit address, bulk copies, named barriers, the lane's codes
// of a 64-column scale group, and the four m16n8k16 MMAs of one group.
//
// Fragment mapping (mma.sync m16n8k16, fp16 x fp16 -> fp32): weights are the B operand
// (16 k x 8 n), lane (g = lane / 4, t = lane % 4) supplying weight row g; in MMA s of a
// group lane t covers columns [16t + 4s, 16t + 4s + 4), so its codes for a group are
// contiguous and its activations are the 16 values at 16t.  Activation rows (tokens)
// are the A operand's rows g and g + 8.
#pragma once

#include "vq_codebook.cuh"
#include "vq_internal.cuh"
#include "vq_sm100.cuh"

namespace vq {

constexpr int MMAV_ROWS = 8;   // weight rows per block (the MMA's n)

// Shared-memory loads in non-volatile form: the compiler may schedule them freely (overlapping
// the latency of independent loads and MMAs), so their ordering against barriers must
// come from data dependencies — addresses pass through launder() after the wait that
// publishes the data, and results pass through consume() before the arrive that frees it.
__device__ __forceinline__ uint32_t ldsn32(uint32_t a) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 ldsn64(uint32_t a) {
    uint2 v;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 ldsn128(uint32_t a) {
    uint4 v;
    asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t ldsn16(uint32_t a) {
    unsigned short v;
    asm("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void mman_f16_f32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mman_f16_f32_zero(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}
// A value the compiler must treat as produced at this point of the program.
__device__ __forceinline__ uint32_t launder(uint32_t v) {
    asm volatile("" : "+r"(v)::"memory");
    return v;
}
// A value the compiler must have computed by this point of the program.
__device__ __forceinline__ void consume(float v) { asm volatile("" ::"f"(v) : "memory"); }

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void bar_sync_named(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// The lane's codes of one scale group (64 columns) of its row, as they are needed by
// the four MMAs: code(j) for j < 64 / d / 4 (non-volatile loads, see ldsn32).
template <int D, int BITS>
struct LaneCodes {
    uint32_t w0, w1, w2;
    int sh;   // 12-bit d = 4 / d = 8: bit offset inside w0:w1
    static __device__ __forceinline__ uint32_t ld32(uint32_t a) { return ldsn32(a); }
    static __device__ __forceinline__ uint2 ld64(uint32_t a) { return ldsn64(a); }
    static __device__ __forceinline__ uint32_t ld16(uint32_t a) { return ldsn16(a); }
    __device__ __forceinline__ void load(uint32_t grp_addr, int t) {
        if constexpr (BITS == 8) {
            if constexpr (D == 2) { const uint2 v = ld64(grp_addr + 8 * t); w0 = v.x; w1 = v.y; }
            else if constexpr (D == 4) { w0 = ld32(grp_addr + 4 * t); }
            else { w0 = ld16(grp_addr + 2 * t); }
        } else {
            if constexpr (D == 2) {          // 12 bytes at 12t: codes at bits 12j
                w0 = ld32(grp_addr + 12 * t);
                w1 = ld32(grp_addr + 12 * t + 4);
                w2 = ld32(grp_addr + 12 * t + 8);
            } else if constexpr (D == 4) {   // 48 bits at bit 48t
                const int wi = (3 * t) >> 1;
                sh = 16 * (t & 1);
                w0 = ld32(grp_addr + 4 * wi);
                w1 = ld32(grp_addr + 4 * wi + 4);
            } else {                         // 24 bits at bit 24t
                const int bit = 24 * t;
                sh = bit & 31;
                w0 = ld32(grp_addr + 4 * (bit >> 5));
                w1 = ld32(grp_addr + 4 * (bit >> 5) + 4);
            }
        }
    }
    __device__ __forceinline__ uint32_t code(int j) const {
        if constexpr (BITS == 8) {
            if constexpr (D == 2) return ((j < 4 ? w0 : w1) >> (8 * (j & 3))) & 0xFFu;
            else return (w0 >> (8 * j)) & 0xFFu;
        } else {
            if constexpr (D == 2) {
                const int bit = 12 * j, wi = bit >> 5, s = bit & 31;
                const uint32_t lo = wi == 0 ? w0 : wi == 1 ? w1 : w2;
                const uint32_t hi = wi == 0 ? w1 : w2;
                return (s + 12 <= 32 ? (lo >> s) : __funnelshift_r(lo, hi, s)) & 0xFFFu;
            } else {
                const uint64_t v = ((uint64_t)w1 << 32) | w0;
                return (uint32_t)(v >> (sh + 12 * j)) & 0xFFFu;
            }
        }
    }
};

// One 64-column scale group of one 8-row block: d[0], d[1] = partial sums of rows 2t,
// 2t + 1 for the token in A row g; d[2], d[3] for A row g + 8.  `codes` is the shared
// address of this lane's row at this group, xa / xb the lane's 16 activations (8 packed
// fp16 pairs) for A rows g and g + 8.
template <int D, int BITS>
__device__ __forceinline__ void mma_group(uint32_t codes, int t, uint32_t cb_lane, const uint32_t (&xa)[8],
                                          const uint32_t (&xb)[8], float (&d)[4])
{
    // non-volatile loads and MMAs (see ldsn32): `codes` must come from a laundered stage
    // address and `cb_lane` from a laundered table address
    using CB = SmemCB<D, BITS>;
    LaneCodes<D, BITS> lc;
    lc.load(codes, t);
#pragma unroll
    for (int s = 0; s < 4; s++) {
        const uint32_t a[4] = {xa[2 * s], xb[2 * s], xa[2 * s + 1], xb[2 * s + 1]};
        uint32_t b0, b1;
        if constexpr (D == 2) {
            b0 = ldsn32(cb_lane + lc.code(2 * s) * CB::STRIDE);
            b1 = ldsn32(cb_lane + lc.code(2 * s + 1) * CB::STRIDE);
        } else if constexpr (D == 4) {
            const uint2 e = ldsn64(cb_lane + lc.code(s) * CB::STRIDE);
            b0 = e.x; b1 = e.y;
        } else {
            const uint4 e = ldsn128(cb_lane + lc.code(s >> 1) * CB::STRIDE);
            b0 = (s & 1) ? e.z : e.x;
            b1 = (s & 1) ? e.w : e.y;
        }
        if (s == 0) mman_f16_f32_zero(d, a, b0, b1);
        else mman_f16_f32(d, a, b0, b1);
    }
}

// 16 fp16 activations (8 packed pairs) from global memory.
__device__ __forceinline__ void ldg_x16(const __half *p, uint32_t (&x)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint4 b = __ldg(reinterpret_cast<const uint4 *>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void ldsn_x16(uint32_t addr, uint32_t (&x)[8]) {
    const uint4 a = ldsn128(addr);
    const uint4 b = ldsn128(addr + 16);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

}  // namespace vq

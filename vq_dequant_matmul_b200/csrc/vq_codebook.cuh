// vq_codebook.cuh — the per-tensor codebook held in shared memory.
//
// For K = 256 the [K][d] fp16 table is replicated so that each lane of a warp reads its
// own banks: a warp-wide 4-byte load is served 32 lanes at a time, an 8-byte load 16
// lanes at a time and a 16-byte load 8 lanes at a time, so d = 2, 4, 8 entries get 32,
// 16 and 8 interleaved copies (32 KB in every case) and lane L reads copy L mod NREP.
// Random codes then never collide on a bank.  K = 4096 tables (16/32/64 KB) are too
// large to replicate and are kept as a single copy.
#pragma once

#include "vq_internal.cuh"

namespace vq {

// ------------------------------------------------------------------ codebook staging

template <int D, int BITS>
struct SmemCB {
    static constexpr int K = 1 << BITS;
    static constexpr int NREP = BITS == 8 ? (D == 2 ? 32 : D == 4 ? 16 : 8) : 1;
    static constexpr int ENTRY = D * 2;           // bytes per entry
    static constexpr int STRIDE = NREP * ENTRY;   // bytes between entries
    static constexpr int BYTES = K * STRIDE;

    // Copy the global [K][D] fp16 table into shared memory, NREP copies interleaved:
    // entry e occupies bytes [e * STRIDE, (e + 1) * STRIDE), copy `rep` at rep * ENTRY.
    // Every global load is issued before the shared stores that use it, so a CTA pays
    // about one memory latency per pass instead of one per word.
    __device__ static void stage(uint8_t *smem, const __half *gcb) { stage(smem, gcb, threadIdx.x, blockDim.x); }

    // The same with an explicit thread index / count (a subset of the block stages it).
    __device__ static void stage(uint8_t *smem, const __half *gcb, int tid, int nthreads) {
        if constexpr (NREP > 1) {
            static_assert(STRIDE == 128, "replicated entries span 128 bytes");
            for (int e = tid; e < K; e += nthreads) {
                uint4 v;
                if constexpr (D == 2) {
                    const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(gcb) + e);
                    v = make_uint4(w, w, w, w);
                } else if constexpr (D == 4) {
                    const uint2 w = __ldg(reinterpret_cast<const uint2 *>(gcb) + e);
                    v = make_uint4(w.x, w.y, w.x, w.y);
                } else {
                    v = __ldg(reinterpret_cast<const uint4 *>(gcb) + e);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(smem + (size_t)e * STRIDE);
#pragma unroll
                for (int i = 0; i < 8; i++) dst[i] = v;
            }
        } else {
            constexpr int N16 = K * D * 2 / 16;
            const uint4 *g = reinterpret_cast<const uint4 *>(gcb);
            uint4 *dst = reinterpret_cast<uint4 *>(smem);
            constexpr int B = 8;   // loads in flight per thread
            for (int i0 = tid; i0 < N16; i0 += B * nthreads) {
                uint4 v[B];
#pragma unroll
                for (int j = 0; j < B; j++) {
                    const int i = i0 + j * nthreads;
                    if (i < N16) v[j] = __ldg(g + i);
                }
#pragma unroll
                for (int j = 0; j < B; j++) {
                    const int i = i0 + j * nthreads;
                    if (i < N16) dst[i] = v[j];
                }
            }
        }
    }
};

template <int D>
__device__ __forceinline__ void load_entry(const uint8_t *p, float (&v)[D]) {
    if constexpr (D == 2) {
        float2 a = __half22float2(*reinterpret_cast<const __half2 *>(p));
        v[0] = a.x; v[1] = a.y;
    } else if constexpr (D == 4) {
        uint2 u = *reinterpret_cast<const uint2 *>(p);
        float2 a = __half22float2(*reinterpret_cast<__half2 *>(&u.x));
        float2 b = __half22float2(*reinterpret_cast<__half2 *>(&u.y));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    } else {
        uint4 u = *reinterpret_cast<const uint4 *>(p);
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            float2 a = __half22float2(*reinterpret_cast<__half2 *>(&w[k]));
            v[2 * k] = a.x; v[2 * k + 1] = a.y;
        }
    }
}

}  // namespace vq

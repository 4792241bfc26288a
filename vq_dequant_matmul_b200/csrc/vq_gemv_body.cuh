// vq_gemv_body.cuh — the batch-1 GEMV inner loop shared by the dense decode GEMV and
// the grouped (per-expert) MoE decode kernels.
//
// A lane streams "chunks" of a row: 16 bytes = 16 8-bit codes, or 48 bytes = 32 12-bit
// codes, loaded with 128-bit non-allocating loads for R rows at once.  The matching
// activations (at most 64 columns at a time, one scale group) are loaded once into
// registers and used for all R rows; each code is looked up in the shared-memory
// codebook, multiplied against its d activations in fp32, and each 64-column partial is
// scaled by its (row, group) scale.
#pragma once

#include "vq_codebook.cuh"
#include "vq_internal.cuh"

namespace vq {

constexpr int GEMV_BODY_THREADS = 256;
constexpr int GEMV_BODY_WARPS = GEMV_BODY_THREADS / 32;

// N activations starting at p (16-byte aligned; N a multiple of 8) to fp32.
template <typename XT, int N>
__device__ __forceinline__ void load_x_vec(const XT *p, float (&xr)[N]) {
    if constexpr (sizeof(XT) == 4) {
#pragma unroll
        for (int k = 0; k < N / 4; k++) {
            float4 f = __ldg(reinterpret_cast<const float4 *>(p) + k);
            xr[4 * k] = f.x; xr[4 * k + 1] = f.y; xr[4 * k + 2] = f.z; xr[4 * k + 3] = f.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < N / 8; k++) {
            uint4 u = __ldg(reinterpret_cast<const uint4 *>(p) + k);
            uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                XT lo, hi;
                uint16_t l16 = (uint16_t)(w[j] & 0xffffu), h16 = (uint16_t)(w[j] >> 16);
                lo = *reinterpret_cast<XT *>(&l16);
                hi = *reinterpret_cast<XT *>(&h16);
                xr[8 * k + 2 * j] = to_f32<XT>(lo);
                xr[8 * k + 2 * j + 1] = to_f32<XT>(hi);
            }
        }
    }
}

// Code q of a lane chunk held as NV uint4 (q is a compile-time constant after unroll).
template <int BITS, int NV>
__device__ __forceinline__ uint32_t chunk_code(const uint4 (&cw)[NV], int q) {
    uint32_t w[NV * 4];
#pragma unroll
    for (int v = 0; v < NV; v++) { w[4 * v] = cw[v].x; w[4 * v + 1] = cw[v].y; w[4 * v + 2] = cw[v].z; w[4 * v + 3] = cw[v].w; }
    if constexpr (BITS == 8) {
        return (w[q >> 2] >> ((q & 3) * 8)) & 0xFFu;
    } else {
        const int bit = 12 * q, wi = bit >> 5, sh = bit & 31;
        if (sh + 12 <= 32) return (w[wi] >> sh) & 0xFFFu;
        return __funnelshift_r(w[wi], w[wi + 1], sh) & 0xFFFu;
    }
}

// ------------------------------------------------------------------ batch-1 kernel

template <int D, int BITS>
struct B1Shape {
    static constexpr int CPC = BITS == 8 ? 16 : 32;          // codes per lane chunk
    static constexpr int CHB = CPC * BITS / 8;               // chunk bytes: 16 or 48
    static constexpr int NV = CHB / 16;                      // uint4 per chunk
    static constexpr int SUB = CPC < 64 / D ? CPC : 64 / D;  // codes per sub-chunk
    static constexpr int NSUB = CPC / SUB;
    static constexpr int SUBCOLS = SUB * D;                  // <= 64, divides 64
    static constexpr int R = BITS == 8 ? 8 : 4;              // rows per lane group
};

// Activations of one token row of type XT.
template <typename XT>
struct XRow {
    const XT *p;
    template <int N>
    __device__ __forceinline__ void load(int col0, float (&xr)[N]) const { load_x_vec<XT, N>(p + col0, xr); }
};

// silu(g) * u from two fp32 rows (the down projection's input in the MoE layer).
struct XSiluMul {
    const float *g, *u;
    template <int N>
    __device__ __forceinline__ void load(int col0, float (&xr)[N]) const {
#pragma unroll
        for (int k = 0; k < N / 4; k++) {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(g + col0) + k);
            const float4 b = __ldg(reinterpret_cast<const float4 *>(u + col0) + k);
            xr[4 * k] = a.x / (1.f + expf(-a.x)) * b.x;
            xr[4 * k + 1] = a.y / (1.f + expf(-a.y)) * b.y;
            xr[4 * k + 2] = a.z / (1.f + expf(-a.z)) * b.z;
            xr[4 * k + 3] = a.w / (1.f + expf(-a.w)) * b.w;
        }
    }
};

// acc[i] += sum over chunks j = j0, j0 + jstep, ... of row (rbase + i) . x, for the
// matrix with packed codes `codes` (row stride crb bytes) and fp16 scales `scales`
// (row stride sre); rows >= `rows` contribute nothing.
template <int D, int BITS, class XS>
__device__ __forceinline__ void b1_accumulate(const uint8_t *__restrict__ codes, const __half *__restrict__ scales,
                                              int rows, int cols, int64_t crb, int64_t sre, const uint8_t *cbase,
                                              int rbase, int j0, int jstep, const XS &xs,
                                              float (&acc)[B1Shape<D, BITS>::R])
{
    using CB = SmemCB<D, BITS>;
    using S = B1Shape<D, BITS>;
    constexpr int R = S::R;
    const int nchunk = (cols / D + S::CPC - 1) / S::CPC;
    for (int j = j0; j < nchunk; j += jstep) {
        uint4 cw[R][S::NV];
#pragma unroll
        for (int i = 0; i < R; i++) {
            const int r = rbase + i;
            if (r < rows) {
                const uint8_t *p = codes + (int64_t)r * crb + (int64_t)j * S::CHB;
#pragma unroll
                for (int v = 0; v < S::NV; v++) cw[i][v] = ldg_stream_u4(p + 16 * v);
            } else {
#pragma unroll
                for (int v = 0; v < S::NV; v++) cw[i][v] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int s = 0; s < S::NSUB; s++) {
            const int col0 = j * S::CPC * D + s * S::SUBCOLS;
            if (col0 < cols) {
                float xr[S::SUBCOLS];
                xs.load(col0, xr);
                const int grp = col0 >> 6;
#pragma unroll
                for (int i = 0; i < R; i++) {
                    float part = 0.f;
#pragma unroll
                    for (int q = 0; q < S::SUB; q++) {
                        const uint32_t code = chunk_code<BITS, S::NV>(cw[i], s * S::SUB + q);
                        float e[D];
                        load_entry<D>(cbase + code * CB::STRIDE, e);
#pragma unroll
                        for (int t = 0; t < D; t++) part = fmaf(e[t], xr[q * D + t], part);
                    }
                    const int r = rbase + i;
                    const float sc = r < rows ? __half2float(scales[(int64_t)r * sre + grp]) : 0.f;
                    acc[i] = fmaf(sc, part, acc[i]);
                }
            }
        }
    }
}

}  // namespace vq

// vq_internal.cuh — definitions shared by the kernels of the VQ library (sm_100a).
//
// Format (model card "Qwen3.5-397B-A17B-VQ-2.4bpw", Methodology; paper "Data-Free
// Vector Quantization Beats Affine Quantization at Matched Bytes Below 5 Bits", §2.2
// and §2.3): W[r][c] = scale[r][c/64] * codebook[code(r, c/d)][c mod d]; codes are a
// little-endian LSB-first bitstream per row, ceil(ncodes/32)*4*bits bytes per row.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vq.h"

namespace vq {

// Kernel-side copy of vq_matrix (plain values, passed by value to kernels).
struct Mat {
    int32_t rows, cols, d, bits;
    const __half *codebook;
    const uint8_t *codes;
    const __half *scales;
    int64_t code_row_bytes, scale_row_elems;
    int64_t expert_code_stride, expert_scale_stride, expert_codebook_stride;
    int32_t num_experts;
};

inline Mat to_mat(const vq_matrix &m) {
    Mat k;
    k.rows = m.rows; k.cols = m.cols; k.d = m.d; k.bits = m.bits;
    k.codebook = static_cast<const __half *>(m.codebook);
    k.codes = static_cast<const uint8_t *>(m.codes);
    k.scales = static_cast<const __half *>(m.scales);
    k.code_row_bytes = m.code_row_bytes; k.scale_row_elems = m.scale_row_elems;
    k.expert_code_stride = m.expert_code_stride;
    k.expert_scale_stride = m.expert_scale_stride;
    k.expert_codebook_stride = m.expert_codebook_stride;
    k.num_experts = m.num_experts;
    return k;
}

// Geometry index used by the runtime dispatch of the grouped kernels.
enum Geom { G_D2_B8 = 0, G_D4_B8, G_D8_B8, G_D2_B12, G_D4_B12, G_D8_B12, G_COUNT };
__host__ __device__ inline int geom_of(int d, int bits) {
    int di = d == 2 ? 0 : d == 4 ? 1 : d == 8 ? 2 : -1;
    int bi = bits == 8 ? 0 : bits == 12 ? 3 : -1;
    return (di < 0 || bi < 0) ? -1 : di + bi;
}

// ------------------------------------------------------------------ device helpers

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }

// Programmatic dependent launch: a kernel launched with programmatic stream serialization
// may start while the previous kernel in the stream is still running; griddep_wait()
// returns once that kernel has completed and its writes are visible, so it must come
// before the first access to any input or output.  griddep_launch_dependents() lets the
// next such kernel be scheduled early (it still waits in its own griddep_wait()).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Store one output element converted to the requested type (runtime switch: the
// output type only matters in epilogues).
__device__ __forceinline__ void store_out(void *y, int64_t idx, float v, int yt) {
    if (yt == VQ_F32) static_cast<float *>(y)[idx] = v;
    else if (yt == VQ_F16) static_cast<__half *>(y)[idx] = __float2half_rn(v);
    else static_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(v);
}

// Read-only 128-bit global load that does not allocate in L1 (streamed once).
__device__ __forceinline__ uint4 ldg_stream_u4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Sum of v over the `width` lanes of each aligned lane group (width a power of 2).
__device__ __forceinline__ float group_sum(float v, int width) {
    for (int off = width >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

}  // namespace vq

// Launch with programmatic stream serialization (the kernel must call griddep_wait()
// before touching any input or output).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args)
{
    cudaLaunchConfig_t lc{};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, k, static_cast<KArgs>(args)...);
}

// Host-side launch helpers (status mapping).
#define VQ_CHECK_LAUNCH()                                              \
    do {                                                               \
        cudaError_t e_ = cudaGetLastError();                           \
        if (e_ != cudaSuccess) return VQ_ERR_CUDA;                     \
    } while (0)

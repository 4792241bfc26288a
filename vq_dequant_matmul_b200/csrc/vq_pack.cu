// vq_pack.cu — code packing, unpacking and whole-matrix dequantization.
//
// Packing follows model card "Qwen3.5-397B-A17B-VQ-2.4bpw", Methodology (Sub-byte
// bit-packing: uint32 words, row-local, 32-code blocks) and paper "Data-Free Vector
// Quantization Beats Affine Quantization at Matched Bytes Below 5 Bits", §2.3: each row
// is one LSB-first bitstream viewed as little-endian uint32 words.  Here every output
// word is assembled by one thread from the codes that overlap it, and every code is
// read back by one thread with a funnel shift across two words.
#include "vq_internal.cuh"

namespace vq {

__global__ void pack_kernel(const uint16_t *__restrict__ codes, int32_t rows, int32_t ncodes,
                            int32_t bits, uint32_t *__restrict__ packed, int64_t row_words)
{
    int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (idx >= (int64_t)rows * row_words) return;
    int64_t r = idx / row_words, w = idx - r * row_words;
    int64_t bit0 = w * 32;
    int64_t i0 = bit0 / bits, i1 = (bit0 + 31) / bits;
    uint32_t mask = (1u << bits) - 1u;
    uint32_t word = 0;
    const uint16_t *crow = codes + r * (int64_t)ncodes;
    for (int64_t i = i0; i <= i1 && i < ncodes; i++) {
        uint32_t c = crow[i] & mask;
        int64_t sh = i * bits - bit0;          // in (-bits, 32)
        word |= sh >= 0 ? (c << sh) : (c >> (-sh));
    }
    packed[idx] = word;
}

__global__ void unpack_kernel(const uint32_t *__restrict__ packed, int32_t rows, int32_t ncodes,
                              int32_t bits, int64_t row_words, uint16_t *__restrict__ codes)
{
    int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (idx >= (int64_t)rows * ncodes) return;
    int64_t r = idx / ncodes, i = idx - r * ncodes;
    const uint32_t *row = packed + r * row_words;
    int64_t bit = i * bits;
    int64_t w = bit >> 5;
    uint32_t s = (uint32_t)(bit & 31);
    uint32_t lo = row[w];
    uint32_t hi = (s + bits > 32) ? row[w + 1] : 0u;
    codes[idx] = (uint16_t)(__funnelshift_r(lo, hi, s) & ((1u << bits) - 1u));
}

// One thread per (row, code): w[r][i*d + t] = scale * codebook[code][t].
template <typename OT>
__global__ void dequant_kernel(Mat W, int32_t expert, OT *__restrict__ out)
{
    int32_t ncodes = W.cols / W.d;
    int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (idx >= (int64_t)W.rows * ncodes) return;
    int64_t r = idx / ncodes, i = idx - r * ncodes;
    const uint8_t *row = W.codes + expert * W.expert_code_stride + r * W.code_row_bytes;
    uint32_t code;
    if (W.bits == 8) {
        code = row[i];
    } else {  // 12-bit: the code lies in bytes b0, b0+1 at bit offset 0 or 4
        int64_t bit = i * 12;
        int64_t b0 = bit >> 3;
        uint32_t v = (uint32_t)row[b0] | ((uint32_t)row[b0 + 1] << 8);
        code = (v >> (bit & 7)) & 0xFFFu;
    }
    const __half *cb = W.codebook + expert * W.expert_codebook_stride + (int64_t)code * W.d;
    float s = __half2float(W.scales[expert * W.expert_scale_stride + r * W.scale_row_elems + (i * W.d) / 64]);
    OT *o = out + r * (int64_t)W.cols + i * W.d;
    for (int t = 0; t < W.d; t++) o[t] = from_f32<OT>(s * __half2float(cb[t]));
}

static inline unsigned nblocks(int64_t n, int bs) { return (unsigned)((n + bs - 1) / bs); }

vq_status launch_pack(const uint16_t *codes, int32_t rows, int32_t ncodes, int32_t bits,
                      void *packed, int64_t code_row_bytes, cudaStream_t s)
{
    int64_t row_words = code_row_bytes / 4;
    int64_t n = (int64_t)rows * row_words;
    if (n == 0) return VQ_OK;
    pack_kernel<<<nblocks(n, 256), 256, 0, s>>>(codes, rows, ncodes, bits, (uint32_t *)packed, row_words);
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

vq_status launch_unpack(const void *packed, int32_t rows, int32_t ncodes, int32_t bits,
                        int64_t code_row_bytes, uint16_t *codes, cudaStream_t s)
{
    int64_t n = (int64_t)rows * ncodes;
    if (n == 0) return VQ_OK;
    unpack_kernel<<<nblocks(n, 256), 256, 0, s>>>((const uint32_t *)packed, rows, ncodes, bits,
                                                  code_row_bytes / 4, codes);
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

vq_status launch_dequant(const Mat &W, int32_t expert, void *out, vq_dtype ot, cudaStream_t s)
{
    int64_t n = (int64_t)W.rows * (W.cols / W.d);
    unsigned g = nblocks(n, 256);
    if (ot == VQ_F32) dequant_kernel<float><<<g, 256, 0, s>>>(W, expert, (float *)out);
    else if (ot == VQ_F16) dequant_kernel<__half><<<g, 256, 0, s>>>(W, expert, (__half *)out);
    else dequant_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(W, expert, (__nv_bfloat16 *)out);
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

}  // namespace vq

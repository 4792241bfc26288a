// vq_gemv.cu — decode GEMV y[m][r] = sum_c W[r][c] x[m][c] straight from packed codes.
//
// This is the fused decode-and-matmul of paper "Data-Free Vector Quantization Beats
// Affine Quantization at Matched Bytes Below 5 Bits", §3.4 (codes and codebook read
// directly, code width extracted in the kernel), re-designed for sm_100a:
//   * the per-tensor codebook lives in shared memory.  For K = 256 it is replicated so
//     that every lane of a warp reads a different bank: 32 copies of 4-byte entries
//     (d=2), 16 of 8-byte entries (d=4, read in 16-lane phases) or 8 of 16-byte entries
//     (d=8, 8-lane phases) — 32 KB in every case.  K = 4096 tables (16-64 KB) are kept
//     as one copy.
//   * batch 1: each lane streams 16-byte chunks of a row (16 8-bit codes, or 48-byte
//     chunks = 32 12-bit codes) with 128-bit non-allocating loads, for R rows at a time,
//     and keeps the matching activations in registers, so each activation load serves R
//     rows.  Lanes of a row reduce with warp shuffles; when a row is split across warps
//     (split-K inside the CTA, for short-and-wide matrices) the warps reduce through
//     shared memory in a fixed order.
//   * batch 2..16: each lane owns one code position of a 32-code window and the
//     activations of all tokens for it; 12-bit codes are unpacked by having 12 lanes
//     load the window's 12 words and every lane fetch its two words by shuffle.
// Accumulation is fp32 throughout; no atomics, so results are deterministic.
#include <algorithm>

#include "vq_codebook.cuh"
#include "vq_gemv_body.cuh"
#include "vq_internal.cuh"

namespace vq {

// D activations at p (any alignment of D elements) to fp32.
template <typename XT, int D>
__device__ __forceinline__ void load_x_small(const XT *p, float (&xr)[D]) {
#pragma unroll
    for (int t = 0; t < D; t++) xr[t] = to_f32<XT>(p[t]);
}

constexpr int GEMV_THREADS = 256;
constexpr int GEMV_WARPS = GEMV_THREADS / 32;

template <int D, int BITS, typename XT>
__global__ void __launch_bounds__(GEMV_THREADS)
gemv_b1_kernel(Mat W, const XT *__restrict__ x, void *__restrict__ y, int yt, int lpr_log2, int ks)
{
    using CB = SmemCB<D, BITS>;
    using S = B1Shape<D, BITS>;
    constexpr int R = S::R;
    extern __shared__ __align__(16) uint8_t smem[];
    CB::stage(smem, W.codebook);
    float *red = reinterpret_cast<float *>(smem + CB::BYTES);
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int LPR = 1 << lpr_log2, G = 32 >> lpr_log2;
    const int g = lane >> lpr_log2, l = lane & (LPR - 1);
    const int tpc = GEMV_WARPS / ks;                 // row tasks a CTA runs at once
    const int slot = warp / ks, kk = warp % ks;
    const int rpt = R * G;                           // rows per task
    const int ntasks = (W.rows + rpt - 1) / rpt;
    const int nrounds = (ntasks + tpc - 1) / tpc;
    const uint8_t *cbase = smem + (lane % CB::NREP) * CB::ENTRY;

    for (int round = blockIdx.x; round < nrounds; round += gridDim.x) {
        const int task = round * tpc + slot;
        const int rbase = task * rpt + g * R;
        float acc[R];
#pragma unroll
        for (int i = 0; i < R; i++) acc[i] = 0.f;

        if (task < ntasks)
            b1_accumulate<D, BITS>(W.codes, W.scales, W.rows, W.cols, W.code_row_bytes, W.scale_row_elems,
                                   cbase, rbase, l + LPR * kk, LPR * ks, XRow<XT>{x}, acc);
#pragma unroll
        for (int i = 0; i < R; i++) acc[i] = group_sum(acc[i], LPR);

        if (ks == 1) {
            if (task < ntasks && l == 0) {
#pragma unroll
                for (int i = 0; i < R; i++)
                    if (rbase + i < W.rows) store_out(y, rbase + i, acc[i], yt);
            }
        } else {
            if (l == 0) {
#pragma unroll
                for (int i = 0; i < R; i++) red[(warp * G + g) * R + i] = acc[i];
            }
            __syncthreads();
            if (kk == 0 && task < ntasks && l == 0) {
#pragma unroll
                for (int i = 0; i < R; i++) {
                    float v = 0.f;
                    for (int k2 = 0; k2 < ks; k2++) v += red[((slot * ks + k2) * G + g) * R + i];
                    if (rbase + i < W.rows) store_out(y, rbase + i, v, yt);
                }
            }
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------------ batch 2..16 kernel

// Code of lane `lane` in the 32-code window starting at byte `wbytes` of a row.  All 32
// lanes must call it together (12-bit path shuffles).
template <int BITS>
__device__ __forceinline__ uint32_t window_code(const uint8_t *row_win, int lane, bool valid) {
    if constexpr (BITS == 8) {
        return valid ? (uint32_t)row_win[lane] : 0u;
    } else {
        uint32_t w = lane < 12 ? __ldg(reinterpret_cast<const uint32_t *>(row_win) + lane) : 0u;
        const int bit = 12 * lane, wi = bit >> 5, sh = bit & 31;
        uint32_t lo = __shfl_sync(0xffffffffu, w, wi);
        uint32_t hi = __shfl_sync(0xffffffffu, w, (wi + 1) & 31);
        return __funnelshift_r(lo, hi, sh) & 0xFFFu;
    }
}

template <int D, int BITS, int MB, int R, typename XT>
__global__ void __launch_bounds__(GEMV_THREADS)
gemv_bn_kernel(Mat W, const XT *__restrict__ x, int batch, void *__restrict__ y, int yt, int64_t y_stride)
{
    using CB = SmemCB<D, BITS>;
    extern __shared__ __align__(16) uint8_t smem[];
    CB::stage(smem, W.codebook);
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ncodes = W.cols / D;
    const int nwin = (ncodes + 31) / 32;
    const int ntasks = (W.rows + R - 1) / R;
    constexpr int WB = 32 * BITS / 8;                 // window bytes: 32 or 48
    const uint8_t *cbase = smem + (lane % CB::NREP) * CB::ENTRY;

    for (int task = blockIdx.x * GEMV_WARPS + warp; task < ntasks; task += gridDim.x * GEMV_WARPS) {
        const int r0 = task * R;
        float acc[R][MB];
#pragma unroll
        for (int i = 0; i < R; i++)
#pragma unroll
            for (int b = 0; b < MB; b++) acc[i][b] = 0.f;

        for (int win = 0; win < nwin; win++) {
            const int p = win * 32 + lane;
            const bool valid = p < ncodes;
            float xv[MB][D];
#pragma unroll
            for (int b = 0; b < MB; b++) {
                if (valid && b < batch) load_x_small<XT, D>(x + (int64_t)b * W.cols + (int64_t)p * D, xv[b]);
                else {
#pragma unroll
                    for (int t = 0; t < D; t++) xv[b][t] = 0.f;
                }
            }
            const int grp = (p * D) >> 6;
#pragma unroll
            for (int i = 0; i < R; i++) {
                const int r = r0 + i;
                if (r >= W.rows) break;                       // warp-uniform
                const uint8_t *row = W.codes + (int64_t)r * W.code_row_bytes + (int64_t)win * WB;
                const uint32_t code = window_code<BITS>(row, lane, valid);
                const float sc = valid ? __half2float(W.scales[(int64_t)r * W.scale_row_elems + grp]) : 0.f;
                float e[D];
                load_entry<D>(cbase + code * CB::STRIDE, e);
#pragma unroll
                for (int t = 0; t < D; t++) e[t] *= sc;
#pragma unroll
                for (int b = 0; b < MB; b++)
#pragma unroll
                    for (int t = 0; t < D; t++) acc[i][b] = fmaf(e[t], xv[b][t], acc[i][b]);
            }
        }
#pragma unroll
        for (int i = 0; i < R; i++)
#pragma unroll
            for (int b = 0; b < MB; b++) {
                const float v = group_sum(acc[i][b], 32);
                if (lane == ((i * MB + b) & 31) && r0 + i < W.rows && b < batch)
                    store_out(y, (int64_t)b * y_stride + r0 + i, v, yt);
            }
    }
}

// ------------------------------------------------------------------ host dispatch

static int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <typename K>
static int blocks_per_sm(K kernel, size_t smem) {
    int b = 0;
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, GEMV_THREADS, smem);
    return b > 0 ? b : 1;
}

template <int D, int BITS, typename XT>
static vq_status run_b1(const Mat &W, const void *x, void *y, int yt, cudaStream_t s)
{
    using CB = SmemCB<D, BITS>;
    using S = B1Shape<D, BITS>;
    const int ncodes = W.cols / D;
    const int nchunk = (ncodes + S::CPC - 1) / S::CPC;
    int lpr_log2 = 0;
    while ((1 << lpr_log2) < 32 && (1 << lpr_log2) < nchunk) lpr_log2++;
    const int LPR = 1 << lpr_log2, G = 32 / LPR;
    const size_t smem = CB::BYTES + (size_t)GEMV_WARPS * G * S::R * sizeof(float);
    auto kern = gemv_b1_kernel<D, BITS, XT>;
    static int bps = 0;
    if (!bps) bps = blocks_per_sm(kern, smem);
    else cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int target_warps = num_sms() * bps * GEMV_WARPS;
    const int ntasks = (W.rows + S::R * G - 1) / (S::R * G);
    const int steps = (nchunk + LPR - 1) / LPR;
    // Split a row across ks warps when there are too few row tasks to fill the GPU:
    // minimise (waves of warps) x (chunk steps per warp).
    int ks = 1;
    long best = -1;
    for (int k = 1; k <= GEMV_WARPS; k *= 2) {
        long waves = ((long)ntasks * k + target_warps - 1) / target_warps;
        long cost = waves * ((steps + k - 1) / k);
        if (best < 0 || cost < best) { best = cost; ks = k; }
    }
    const int tpc = GEMV_WARPS / ks;
    const int nrounds = (ntasks + tpc - 1) / tpc;
    const int grid = std::min(nrounds, num_sms() * bps);
    kern<<<grid, GEMV_THREADS, smem, s>>>(W, (const XT *)x, y, yt, lpr_log2, ks);
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

template <int D, int BITS, int MB, typename XT>
static vq_status run_bn(const Mat &W, const void *x, int batch, void *y, int yt, int64_t y_stride,
                        cudaStream_t s)
{
    using CB = SmemCB<D, BITS>;
    constexpr int R = 4;
    const size_t smem = CB::BYTES;
    auto kern = gemv_bn_kernel<D, BITS, MB, R, XT>;
    static int bps = 0;
    if (!bps) bps = blocks_per_sm(kern, smem);
    else cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int ntasks = (W.rows + R - 1) / R;
    const int grid = std::max(1, std::min((ntasks + GEMV_WARPS - 1) / GEMV_WARPS, num_sms() * bps));
    kern<<<grid, GEMV_THREADS, smem, s>>>(W, (const XT *)x, batch, y, yt, y_stride);
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

template <int D, int BITS, typename XT>
static vq_status run_geom(const Mat &W, const void *x, int batch, void *y, int yt, cudaStream_t s)
{
    if (batch == 1) return run_b1<D, BITS, XT>(W, x, y, yt, s);
    // Tokens are processed in groups of at most 16 (8 for d = 8: D*MB activations
    // per lane stay in registers).
    constexpr int MAXMB = D == 8 ? 8 : 16;
    const size_t yb_el = yt == VQ_F32 ? 4 : 2;
    for (int b0 = 0; b0 < batch; b0 += MAXMB) {
        const int nb = std::min(MAXMB, batch - b0);
        const XT *xb = (const XT *)x + (int64_t)b0 * W.cols;
        void *yb = (char *)y + (int64_t)b0 * W.rows * yb_el;
        vq_status st;
        if (nb <= 2) st = run_bn<D, BITS, 2, XT>(W, xb, nb, yb, yt, W.rows, s);
        else if (nb <= 4) st = run_bn<D, BITS, 4, XT>(W, xb, nb, yb, yt, W.rows, s);
        else if (nb <= 8 || D == 8) st = run_bn<D, BITS, 8, XT>(W, xb, nb, yb, yt, W.rows, s);
        else st = run_bn<D, BITS, (D == 8 ? 8 : 16), XT>(W, xb, nb, yb, yt, W.rows, s);
        if (st != VQ_OK) return st;
    }
    return VQ_OK;
}

template <typename XT>
static vq_status run_x(const Mat &W, const void *x, int batch, void *y, int yt, cudaStream_t s)
{
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: return run_geom<2, 8, XT>(W, x, batch, y, yt, s);
    case G_D4_B8: return run_geom<4, 8, XT>(W, x, batch, y, yt, s);
    case G_D8_B8: return run_geom<8, 8, XT>(W, x, batch, y, yt, s);
    case G_D2_B12: return run_geom<2, 12, XT>(W, x, batch, y, yt, s);
    case G_D4_B12: return run_geom<4, 12, XT>(W, x, batch, y, yt, s);
    case G_D8_B12: return run_geom<8, 12, XT>(W, x, batch, y, yt, s);
    default: return VQ_ERR_UNSUPPORTED;
    }
}

vq_status launch_gemv_mma(const Mat &W, const void *x, vq_dtype xt, int batch, void *y, vq_dtype yt, cudaStream_t s);

vq_status launch_gemv(const Mat &W, const void *x, vq_dtype xt, int batch, void *y, vq_dtype yt,
                      cudaStream_t s)
{
    {   // tensor-core path for fp16 activations
        const vq_status st = launch_gemv_mma(W, x, xt, batch, y, yt, s);
        if (st != VQ_ERR_UNSUPPORTED) return st;
    }
    if (xt == VQ_F16) return run_x<__half>(W, x, batch, y, (int)yt, s);
    if (xt == VQ_BF16) return run_x<__nv_bfloat16>(W, x, batch, y, (int)yt, s);
    return run_x<float>(W, x, batch, y, (int)yt, s);
}

}  // namespace vq

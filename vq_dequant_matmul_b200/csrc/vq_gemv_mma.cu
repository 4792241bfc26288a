// vq_gemv_mma.cu — decode GEMV (batch 1..16) with the multiply-adds on the tensor cores.
//
// The pages' fused decode-and-matmul (paper "Data-Free Vector Quantization Beats Affine
// Quantization at Matched Bytes Below 5 Bits", §3.4) spends, per code, one lookup and d
// multiply-adds.  Here the lookups stay on the shared-memory pipe and the multiply-adds
// move to mma.sync (m16n8k16, fp16 inputs, fp32 accumulation), so a lane spends about
// four instructions per code:
//
//   * weights are the MMA's B operand (16 k x 8 n): n = 8 rows of a row block, and lane
//     (g = lane / 4, t = lane % 4) supplies row g.  A B register holds two consecutive
//     columns of one row — exactly one d = 2 codebook entry, half of a d = 4 entry or a
//     quarter of a d = 8 entry — so looked-up entries go straight into B registers with
//     no conversion;
//   * the activations are the A operand (16 m x 16 k): token m in row m (tokens 0..15;
//     rows beyond the batch repeat a valid token and are dropped), so a batch of up to
//     16 costs the same lookups as one token;
//   * k-slots are permuted so that in MMA s (s = 0..3) of a 64-column scale group lane t
//     covers columns [16t + 4s, 16t + 4s + 4): a lane's codes for a group are contiguous
//     (8, 4 or 2 bytes of 8-bit codes; 12, 6 or 3 bytes of 12-bit codes) and its
//     activations are 16 contiguous values;
//   * the four MMAs of a group accumulate a fresh fp32 partial per row, which is scaled
//     by that row's group scale in fp32 and added to the row total — every product is
//     exact (fp16 x fp16 in fp32), nothing is rounded to 16 bits.
// Rows reach shared memory through bulk asynchronous copies (one per row, into padded
// slots so the eight rows of a block fall on different banks), driven by one producer
// thread over a ring of stages; each CTA owns a contiguous, balanced range of 8-row
// blocks and its consumer warps split each block's scale groups.  Row totals are reduced
// across warps in a fixed order (deterministic).
#include <algorithm>

#include "vq_mma.cuh"

namespace vq {

constexpr int MMAV_MAX_THREADS = 32 * 17;   // producer warp + up to 16 consumer warps

struct MmaGemvCfg {
    int NW;              // consumer warps
    int STAGES;
    int blk_base, blk_extra;   // blocks per CTA: base (+1 for the first `extra` CTAs)
    int slot_stride;     // bytes between row slots in a stage (code_row_bytes + 16)
    int stage_bytes;     // bytes of one stage (8 row slots + 8 rows of scales)
    int x_bytes;         // activations in shared memory (cols * 2, rounded to 16)
    unsigned int *err;
};

// NT = 1: tokens 0..7 (the MMA's rows g); NT = 2: tokens 0..15 (rows g and g + 8).
// XS: activations staged in shared memory (else read through L1 from global memory).
template <int D, int BITS, int NT, bool XS>
__global__ void __launch_bounds__(MMAV_MAX_THREADS, 1)
gemv_mma_kernel(Mat W, const __half *__restrict__ x, int batch, void *__restrict__ y, int yt, MmaGemvCfg cfg)
{
    using CB = SmemCB<D, BITS>;
    constexpr int GB = (64 / D) * BITS / 8;   // code bytes of one row per scale group
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *sCB = smem;
    uint8_t *sX = sCB + CB::BYTES;
    uint8_t *sStage = sX + cfg.x_bytes;
    constexpr int NTOK = 8 * NT;
    // partial sums: a ring of STAGES + 1 buffers [NW][NTOK][8] (a consumer warp is at most
    // STAGES - 1 blocks ahead of the slowest one, so a buffer is never rewritten while read)
    float *red = reinterpret_cast<float *>(sStage + (size_t)cfg.STAGES * cfg.stage_bytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(red + (cfg.STAGES + 1) * cfg.NW * NTOK * MMAV_ROWS);
    uint64_t *empty = full + cfg.STAGES;
    uint64_t *red_bar = empty + cfg.STAGES;   // [STAGES + 1]: partials of a block posted (one arrive per warp)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk_total = (W.rows + MMAV_ROWS - 1) / MMAV_ROWS;
    const int b_begin = blockIdx.x * cfg.blk_base + min((int)blockIdx.x, cfg.blk_extra);
    const int nblk = cfg.blk_base + ((int)blockIdx.x < cfg.blk_extra ? 1 : 0);
    const int G = W.cols / 64;
    const int scale_bytes = MMAV_ROWS * (int)W.scale_row_elems * 2;

    CB::stage(sCB, W.codebook);
    if constexpr (XS) {   // activations [batch][cols] -> shared memory
        const uint4 *src = reinterpret_cast<const uint4 *>(x);
        uint4 *dst = reinterpret_cast<uint4 *>(sX);
        for (int i = threadIdx.x; i < batch * W.cols / 8; i += blockDim.x) dst[i] = __ldg(src + i);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < cfg.STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], cfg.NW);
        }
        for (int s = 0; s <= cfg.STAGES; s++) mbar_init(&red_bar[s], cfg.NW);
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------- producer: one bulk copy per row (padded slots) + one for scales
        if (lane == 0) {
            for (int k = 0; k < nblk; k++) {
                const int slot = k % cfg.STAGES, round = k / cfg.STAGES;
                if (round > 0 && !mbar_wait(&empty[slot], (round - 1) & 1)) {
                    atomicExch(cfg.err, 1u);
                    break;
                }
                const int r0 = (b_begin + k) * MMAV_ROWS;
                const int nrows = min(MMAV_ROWS, W.rows - r0);
                const uint32_t base = smem_u32(sStage + (size_t)slot * cfg.stage_bytes);
                mbar_arrive_expect_tx(&full[slot], (uint32_t)(nrows * (W.code_row_bytes + W.scale_row_elems * 2)));
                for (int r = 0; r < nrows; r++)
                    bulk_copy_g2s(base + r * cfg.slot_stride, W.codes + (int64_t)(r0 + r) * W.code_row_bytes,
                                  (uint32_t)W.code_row_bytes, &full[slot]);
                bulk_copy_g2s(base + MMAV_ROWS * cfg.slot_stride, W.scales + (int64_t)r0 * W.scale_row_elems,
                              (uint32_t)(nrows * W.scale_row_elems * 2), &full[slot]);
            }
        }
        return;
    }

    // ---------------- consumers
    const int cw = warp - 1;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t cb_lane = smem_u32(sCB) + (lane % CB::NREP) * CB::ENTRY;
    // tokens of this lane's A rows (clamped: rows beyond the batch repeat a valid token
    // and their results are dropped)
    const int tok0 = min(g, batch - 1), tok1 = min(g + 8, batch - 1);
    const uint32_t xs0 = smem_u32(sX) + (uint32_t)(tok0 * W.cols + 16 * t) * 2;
    const uint32_t xs1 = smem_u32(sX) + (uint32_t)(tok1 * W.cols + 16 * t) * 2;
    const __half *xg0 = x + (int64_t)tok0 * W.cols + 16 * t;
    const __half *xg1 = x + (int64_t)tok1 * W.cols + 16 * t;
    bool dead = false;
    for (int k = 0; k < nblk; k++) {
        const int slot = k % cfg.STAGES, round = k / cfg.STAGES;
        if (!dead) {
            const bool ok = mbar_wait(&full[slot], round & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicExch(cfg.err, 1u);
                dead = true;
            }
        }
        const uint32_t stage = smem_u32(sStage + (size_t)slot * cfg.stage_bytes);
        const uint32_t row_lane = stage + g * cfg.slot_stride;
        const uint32_t sc_base = stage + MMAV_ROWS * cfg.slot_stride;
        const uint32_t sc0 = sc_base + (2 * t) * (int)W.scale_row_elems * 2;   // scales of rows 2t, 2t + 1
        const uint32_t sc1 = sc0 + (int)W.scale_row_elems * 2;
        float tot[2][2] = {{0.f, 0.f}, {0.f, 0.f}};   // [token g / g + 8][row 2t / 2t + 1]
        if (!dead) {
            for (int grp = cw; grp < G; grp += cfg.NW) {
                uint32_t x0[8], x1[8];
                if constexpr (XS) lds_x16(xs0 + grp * 128, x0);
                else ldg_x16(xg0 + grp * 64, x0);
                if constexpr (NT == 2) {
                    if constexpr (XS) lds_x16(xs1 + grp * 128, x1);
                    else ldg_x16(xg1 + grp * 64, x1);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; i++) x1[i] = x0[i];
                }
                float d[4];
                mma_group<D, BITS>(row_lane + grp * GB, t, cb_lane, x0, x1, d);
                const float s0 = __half2float(__ushort_as_half((unsigned short)lds16(sc0 + grp * 2)));
                const float s1 = __half2float(__ushort_as_half((unsigned short)lds16(sc1 + grp * 2)));
                tot[0][0] = fmaf(s0, d[0], tot[0][0]);
                tot[0][1] = fmaf(s1, d[1], tot[0][1]);
                if constexpr (NT == 2) {
                    tot[1][0] = fmaf(s0, d[2], tot[1][0]);
                    tot[1][1] = fmaf(s1, d[3], tot[1][1]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        // post partials [cw][token][row] (phase-tracked: one mbarrier per ring buffer);
        // warp 0 alone waits for all warps' partials of the block and reduces them
        const int rbi = k % (cfg.STAGES + 1);
        float *rb = red + rbi * cfg.NW * NTOK * MMAV_ROWS;
        rb[(cw * NTOK + g) * MMAV_ROWS + 2 * t] = tot[0][0];
        rb[(cw * NTOK + g) * MMAV_ROWS + 2 * t + 1] = tot[0][1];
        if constexpr (NT == 2) {
            rb[(cw * NTOK + g + 8) * MMAV_ROWS + 2 * t] = tot[1][0];
            rb[(cw * NTOK + g + 8) * MMAV_ROWS + 2 * t + 1] = tot[1][1];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_bar[rbi]);
        if (cw == 0) {
            const bool ok = mbar_wait(&red_bar[rbi], (k / (cfg.STAGES + 1)) & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicExch(cfg.err, 1u);
                dead = true;
            }
            if (!dead) {
                for (int q = lane; q < NTOK * MMAV_ROWS; q += 32) {   // (token, row) outputs
                    const int tok = q / MMAV_ROWS, rr = q % MMAV_ROWS;
                    float v = 0.f;
                    for (int w = 0; w < cfg.NW; w++) v += rb[(w * NTOK + tok) * MMAV_ROWS + rr];
                    const int r = (b_begin + k) * MMAV_ROWS + rr;
                    if (r < W.rows && tok < batch) store_out(y, (int64_t)tok * W.rows + r, v, yt);
                }
            }
        }
    }
    (void)scale_bytes;
    (void)nblk_total;
}

// ------------------------------------------------------------------ host

unsigned int *device_error_word();

static int mmav_num_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

static size_t mmav_cb_bytes(int d, int bits) {
    switch (geom_of(d, bits)) {
    case G_D2_B8: return SmemCB<2, 8>::BYTES;
    case G_D4_B8: return SmemCB<4, 8>::BYTES;
    case G_D8_B8: return SmemCB<8, 8>::BYTES;
    case G_D2_B12: return SmemCB<2, 12>::BYTES;
    case G_D4_B12: return SmemCB<4, 12>::BYTES;
    default: return SmemCB<8, 12>::BYTES;
    }
}

template <int D, int BITS, int NT, bool XS>
static vq_status mmav_launch3(const Mat &W, const void *x, int batch, void *y, int yt, const MmaGemvCfg &c,
                              size_t smem, int grid, cudaStream_t s)
{
    auto k = gemv_mma_kernel<D, BITS, NT, XS>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return VQ_ERR_CUDA;
    k<<<grid, 32 * (1 + c.NW), smem, s>>>(W, (const __half *)x, batch, y, yt, c);
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

template <int D, int BITS>
static vq_status mmav_launch(const Mat &W, const void *x, int batch, void *y, int yt, const MmaGemvCfg &c,
                             size_t smem, int grid, cudaStream_t s)
{
    const bool xs = c.x_bytes > 0;
    if (batch <= 8) return xs ? mmav_launch3<D, BITS, 1, true>(W, x, batch, y, yt, c, smem, grid, s)
                              : mmav_launch3<D, BITS, 1, false>(W, x, batch, y, yt, c, smem, grid, s);
    return xs ? mmav_launch3<D, BITS, 2, true>(W, x, batch, y, yt, c, smem, grid, s)
              : mmav_launch3<D, BITS, 2, false>(W, x, batch, y, yt, c, smem, grid, s);
}

// fp16-activation GEMV (batch 1..16) on the tensor-core path.  VQ_ERR_UNSUPPORTED
// (nothing launched) when it does not apply: other activation types, scale rows that
// are not whole 16-byte units, or rows too wide for the shared-memory budget.
vq_status launch_gemv_mma(const Mat &W, const void *x, vq_dtype xt, int batch, void *y, vq_dtype yt, cudaStream_t s)
{
    if (xt != VQ_F16 || batch < 1 || batch > 16) return VQ_ERR_UNSUPPORTED;
    const int64_t srow = W.scale_row_elems * 2;
    if (srow % 16 || ((uintptr_t)W.scales % 16)) return VQ_ERR_UNSUPPORTED;
    MmaGemvCfg c{};
    const int G = W.cols / 64;
    c.NW = std::min(16, G);
    c.slot_stride = (int)W.code_row_bytes + 16;
    c.stage_bytes = MMAV_ROWS * c.slot_stride + (int)((MMAV_ROWS * srow + 15) / 16 * 16);
    // activations in shared memory when they take at most 48 KB, else read through L1
    const size_t xb = (size_t)batch * W.cols * 2;
    c.x_bytes = xb <= 49152 ? (int)((xb + 15) / 16 * 16) : 0;
    const size_t cb = mmav_cb_bytes(W.d, W.bits);
    const int ntok = batch <= 8 ? 8 : 16;
    const size_t fixed = 128 + cb + c.x_bytes + (size_t)c.NW * ntok * MMAV_ROWS * 4 + 8;   // + one red buffer
    const size_t per_stage = (size_t)c.stage_bytes + (size_t)c.NW * ntok * MMAV_ROWS * 4 + 3 * 8;
    c.STAGES = 8;
    while (c.STAGES >= 2 && fixed + (size_t)c.STAGES * per_stage > 232448) c.STAGES--;
    if (c.STAGES < 2) return VQ_ERR_UNSUPPORTED;
    const size_t smem = fixed + (size_t)c.STAGES * per_stage;
    c.err = device_error_word();
    if (!c.err) return VQ_ERR_CUDA;
    const int nblk = (W.rows + MMAV_ROWS - 1) / MMAV_ROWS;
    const int grid = std::min(mmav_num_sms(), nblk);
    c.blk_base = nblk / grid;
    c.blk_extra = nblk % grid;
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: return mmav_launch<2, 8>(W, x, batch, y, (int)yt, c, smem, grid, s);
    case G_D4_B8: return mmav_launch<4, 8>(W, x, batch, y, (int)yt, c, smem, grid, s);
    case G_D8_B8: return mmav_launch<8, 8>(W, x, batch, y, (int)yt, c, smem, grid, s);
    case G_D2_B12: return mmav_launch<2, 12>(W, x, batch, y, (int)yt, c, smem, grid, s);
    case G_D4_B12: return mmav_launch<4, 12>(W, x, batch, y, (int)yt, c, smem, grid, s);
    case G_D8_B12: return mmav_launch<8, 12>(W, x, batch, y, (int)yt, c, smem, grid, s);
    default: return VQ_ERR_UNSUPPORTED;
    }
}

}  // namespace vq

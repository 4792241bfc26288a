// vq_moe.cu — routed MoE layer over VQ expert stacks.
//
// Layer (paper "Data-Free Vector Quantization Beats Affine Quantization at Matched Bytes
// Below 5 Bits", §2: routed experts with gate, up and down projections; model card
// "Qwen3.6-35B-A3B-MLX-VQ-2.4bpw": top-k routing, mixed tiers per tensor):
//   for token t and slot j: e = ids[t][j]; h = silu(Gate_e x_t) * (Up_e x_t);
//   y_t = sum_j w[t][j] * (Down_e h)   (slot order; SwiGLU is this library's reading).
//
// Steps, all on the device:
//   1. bucketing (one CTA): histogram of the T*k (token, slot) pairs over experts,
//      exclusive scan, stable scatter of pair indices ordered by (expert, token, slot),
//      the list of active experts and a tile list (expert, first row, rows);
//   2. gate/up: ONE grouped launch over (projection, active expert, row block) — each
//      projection with its own geometry, so mixed tiers share the launch.  Few tokens
//      per expert (decode): the tensor-core GEMV with the expert's tokens as MMA rows;
//      several per expert (prefill): the tcgen05 GEMM over a tile list;
//   3. h = silu(g) * u in fp16, then down: one grouped launch of the same kind;
//   4. combine: y_t = sum over slots (in order) of w * o, skipping invalid pairs.
// Pairs whose expert id is outside [0, E) are counted in the workspace status word and
// contribute nothing.  Float atomics are never used: results are deterministic.
#include <algorithm>
#include <type_traits>

#include "vq_codebook.cuh"
#include "vq_gemm_api.cuh"
#include "vq_mma.cuh"
#include "vq_internal.cuh"

namespace vq {

constexpr int MOE_MAX_EXPERTS = 1024;
constexpr int BUCKET_THREADS = 1024;

static inline size_t al256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace layout (byte offsets, each 256-aligned).
struct MoeLayout {
    size_t status, counts, offsets, sorted, pos, act, nact, t_exp, t_row, t_cnt, ntiles, g, u, h16, o, xg, total;
    int P, max_tiles;
};

static MoeLayout moe_layout(int T, int topk, int E, int hidden, int inter)
{
    MoeLayout L;
    L.P = T * topk;
    L.max_tiles = L.P + E;   // sum over experts of ceil(count / BT) <= P / BT + E
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += al256(bytes); return o; };
    L.status = take(16);
    L.counts = take(sizeof(int) * E);
    L.offsets = take(sizeof(int) * (E + 1));
    L.sorted = take(sizeof(int) * L.P);
    L.pos = take(sizeof(int) * L.P);
    L.act = take(sizeof(int) * E);
    L.nact = take(sizeof(int));
    L.t_exp = take(sizeof(int) * L.max_tiles);
    L.t_row = take(sizeof(int) * L.max_tiles);
    L.t_cnt = take(sizeof(int) * L.max_tiles);
    L.ntiles = take(sizeof(int));
    L.g = take(sizeof(float) * (size_t)L.P * inter);
    L.u = take(sizeof(float) * (size_t)L.P * inter);
    L.h16 = take(sizeof(__half) * (size_t)L.P * inter);
    L.o = take(sizeof(float) * (size_t)L.P * hidden);
    L.xg = take(sizeof(__half) * (size_t)L.P * hidden);
    L.total = off;
    return L;
}

vq_status moe_workspace_bytes(int32_t T, int32_t topk, int32_t E, int32_t hidden, int32_t inter, size_t *b)
{
    *b = 0;
    if (T < 1 || topk < 1 || E < 1 || topk > E || hidden < 64 || inter < 64) return VQ_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS || hidden % 64 || inter % 64) return VQ_ERR_UNSUPPORTED;
    *b = moe_layout(T, topk, E, hidden, inter).total;
    return VQ_OK;
}

// ------------------------------------------------------------------ 1. bucketing

struct BucketArgs {
    const int32_t *ids;
    int P, E, BT;
    unsigned int *status;
    int *counts, *offsets, *sorted, *pos, *act, *nact, *t_exp, *t_row, *t_cnt, *ntiles;
};

// Exclusive scan of v over the block (one value per thread, blockDim.x = 1024); returns
// the exclusive prefix and writes the block total to *total.
__device__ int block_exclusive_scan(int v, int *sh, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += n;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = sh[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        sh[lane] = w;           // inclusive prefix over warps
    }
    __syncthreads();
    const int excl = x - v + (warp > 0 ? sh[warp - 1] : 0);
    *total = sh[31];
    __syncthreads();
    return excl;
}

__global__ void __launch_bounds__(BUCKET_THREADS) moe_bucket_kernel(BucketArgs a)
{
    griddep_wait();
    __shared__ int cnt[MOE_MAX_EXPERTS], base[MOE_MAX_EXPERTS], scan_sh[32];
    __shared__ unsigned int bad;
    extern __shared__ unsigned short wcnt_flat[];      // [BUCKET_THREADS / 32][E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E;
    for (int e = tid; e < E; e += BUCKET_THREADS) cnt[e] = 0;
    if (tid == 0) bad = 0;
    __syncthreads();
    for (int p = tid; p < a.P; p += BUCKET_THREADS) {
        const int e = a.ids[p];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else atomicAdd(&bad, 1u);
    }
    __syncthreads();

    // offsets (exclusive scan of counts), active experts, tiles of BT rows
    int total, nact, ntl;
    const int c = tid < E ? cnt[tid] : 0;
    const int off = block_exclusive_scan(c, scan_sh, &total);
    const int aidx = block_exclusive_scan(c > 0 ? 1 : 0, scan_sh, &nact);
    const int nt = (c + a.BT - 1) / a.BT;
    const int toff = block_exclusive_scan(nt, scan_sh, &ntl);
    if (tid < E) {
        base[tid] = off;
        a.counts[tid] = c;
        a.offsets[tid] = off;
        if (c > 0) a.act[aidx] = tid;
        for (int k = 0; k < nt; k++) {
            a.t_exp[toff + k] = tid;
            a.t_row[toff + k] = off + k * a.BT;
            a.t_cnt[toff + k] = min(a.BT, c - k * a.BT);
        }
    }
    if (tid == 0) {
        a.offsets[E] = total;
        *a.nact = nact;
        *a.ntiles = ntl;
        *a.status = bad;
    }
    __syncthreads();

    // stable scatter, one chunk of BUCKET_THREADS pairs at a time
    for (int p0 = 0; p0 < a.P; p0 += BUCKET_THREADS) {
        for (int i = tid; i < (BUCKET_THREADS / 32) * E; i += BUCKET_THREADS)
            wcnt_flat[i] = 0;
        __syncthreads();
        const int p = p0 + tid;
        const int e = p < a.P ? a.ids[p] : -1;
        const bool valid = e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (valid && rank == 0) wcnt_flat[warp * E + e] = (unsigned short)__popc(peers);
        __syncthreads();
        if (valid) {
            int pre = 0;
            for (int w = 0; w < warp; w++) pre += wcnt_flat[w * E + e];
            const int pos = base[e] + pre + rank;
            a.sorted[pos] = p;
            a.pos[p] = pos;
        } else if (p < a.P) {
            a.pos[p] = -1;
        }
        __syncthreads();
        for (int e2 = tid; e2 < E; e2 += BUCKET_THREADS) {
            int s = 0;
            for (int w = 0; w < BUCKET_THREADS / 32; w++) s += wcnt_flat[w * E + e2];
            base[e2] += s;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ 2./3. grouped tensor-core GEMV (decode)

// Grouped decode projections on the tensor-core GEMV: persistent CTAs take balanced,
// contiguous ranges of items (projection p, active expert, 8-row block) in that order;
// an item's rows arrive by bulk copy in a ring of stages; consumer warps split the
// block's 64-column groups, with the expert's tokens (up to 16 at a time) as the MMA's A
// rows.  The codebook is restaged only when the projection (or, for per-expert
// codebooks, the expert) changes.
constexpr int MOE_MMA_MAX_THREADS = 32 * 9;   // producer warp + 8 consumer warps

struct MoeMmaArgs {
    Mat W[3];
    int nproj;
    int fused;                   // 1: items are (expert, block) of gate W[0] and up W[1]; h = silu(g) * u
    float *out[3];               // [P][W[p].rows], rows in bucket order (fused: unused)
    __half *h16;                 // fused: [P][W[0].rows] fp16
    const __half *ain[3];        // A rows: x by token (stage 1) or h by bucket position
    int a_by_token[3];
    const int *sorted, *offsets, *act, *nact;
    int topk;
    int NW, STAGES, stage_bytes;
    int rblk[3];                 // 8-row blocks per item (an item moves a few KB)
    int soff[3], coff[3];        // offsets in a stage: projection p's codes (coff) and scales (soff)
    int tbl_off[3];              // shared-memory offset of each projection's codebook table
    int tbl_bytes;
    unsigned int *err;
};

struct MoeItem {
    int p, e, blk;
};

__device__ __forceinline__ int moe_blocks(const Mat &W, int rblk) { return (W.rows + MMAV_ROWS * rblk - 1) / (MMAV_ROWS * rblk); }

__device__ __forceinline__ MoeItem moe_item(const MoeMmaArgs &a, int i, int nact) {
    MoeItem it{0, 0, 0};
    if (a.fused) {
        const int nb = moe_blocks(a.W[0], a.rblk[0]);
        it.e = a.act[i / nb];
        it.blk = i % nb;
        return it;
    }
    for (int p = 0; p < a.nproj; p++) {
        const int nb = moe_blocks(a.W[p], a.rblk[p]);
        if (i < nact * nb) {
            it.p = p;
            it.e = a.act[i / nb];
            it.blk = i % nb;
            return it;
        }
        i -= nact * nb;
    }
    return it;
}

// One 8-row block of one projection for one chunk of up to 16 of the expert's tokens (the
// MMA's A rows g and g + 8): tot[0 / 1][0 / 1] = rows 2t / 2t + 1 for token g / g + 8.
// `stage` holds the block's rows (code_row_bytes apart) and, at `sc`, their scales (both
// laundered after the stage's wait); x0p / x1p point at the lane's activations.
template <int D, int BITS>
__device__ __forceinline__ void moe_block_chunk(const Mat &W, uint32_t stage, uint32_t sc, uint32_t cb_lane, int lane,
                                                const __half *x0p, const __half *x1p, float (&tot)[2][2])
{
    constexpr int GB = (64 / D) * BITS / 8;
    const int g = lane >> 2, t = lane & 3;
    const int G = W.cols / 64;
    const uint32_t crb = (uint32_t)W.code_row_bytes, srow = (uint32_t)W.scale_row_elems * 2;
    const uint32_t row_lane = stage + (uint32_t)g * crb;
    const uint32_t sc0 = sc + (uint32_t)(2 * t) * srow, sc1 = sc0 + srow;   // scales of rows 2t, 2t + 1
    tot[0][0] = tot[0][1] = tot[1][0] = tot[1][1] = 0.f;
#pragma unroll 2
    for (int grp = 0; grp < G; grp++) {
        uint32_t xa[8], xb[8];
        ldg_x16(x0p + grp * 64, xa);
        ldg_x16(x1p + grp * 64, xb);
        float d[4];
        mma_group<D, BITS>(row_lane + (uint32_t)(grp * GB), t, cb_lane, xa, xb, d);
        const float s0 = __half2float(__ushort_as_half((unsigned short)ldsn16(sc0 + 2u * grp)));
        const float s1 = __half2float(__ushort_as_half((unsigned short)ldsn16(sc1 + 2u * grp)));
        tot[0][0] = fmaf(s0, d[0], tot[0][0]);
        tot[0][1] = fmaf(s1, d[1], tot[0][1]);
        tot[1][0] = fmaf(s0, d[2], tot[1][0]);
        tot[1][1] = fmaf(s1, d[3], tot[1][1]);
    }
}

// Dispatch on the projection's geometry (the table's lane copy depends on it).
__device__ __forceinline__ void moe_block_chunk_any(const Mat &W, uint32_t stage, uint32_t sc, uint32_t tbl, int lane,
                                                    const __half *x0p, const __half *x1p, float (&tot)[2][2])
{
    switch (geom_of(W.d, W.bits)) {
#define VQ_MOE_CASE(GG, DD, BB)                                                                                 \
    case GG:                                                                                                  \
        moe_block_chunk<DD, BB>(W, stage, sc, tbl + (uint32_t)((lane % SmemCB<DD, BB>::NREP) * SmemCB<DD, BB>::ENTRY), \
                                lane, x0p, x1p, tot);                                                         \
        break;
    VQ_MOE_CASE(G_D2_B8, 2, 8)
    VQ_MOE_CASE(G_D4_B8, 4, 8)
    VQ_MOE_CASE(G_D8_B8, 8, 8)
    VQ_MOE_CASE(G_D2_B12, 2, 12)
    VQ_MOE_CASE(G_D4_B12, 4, 12)
    VQ_MOE_CASE(G_D8_B12, 8, 12)
#undef VQ_MOE_CASE
    default: tot[0][0] = tot[0][1] = tot[1][0] = tot[1][1] = 0.f; break;
    }
}

// Grouped tensor-core GEMV over items: (projection, active expert, 8-row block), or in
// the fused gate/up form (active expert, 8-row block) of both projections, whose warp
// writes h = fp16(silu(g) * u) directly.  Each CTA takes a balanced contiguous range of
// items.  Warp 0 (one thread) streams each item's rows and scales into a ring of stages
// with one bulk copy for the codes and one for the scales of each projection (an
// expert's rows are contiguous) and writes the expert's bucket range [j0, j1) into the
// stage's header; consumer warp w takes items w, w + NW, ..., so the CTA works on NW
// items at once and no warp waits for another.  Every projection's codebook table stays
// resident (several projections may be in flight together), so experts must share
// their tensor's codebook on this path.
__global__ void __launch_bounds__(MOE_MMA_MAX_THREADS, 1) moe_mma_kernel(MoeMmaArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *sStage = smem + a.tbl_bytes;
    int2 *hdr = reinterpret_cast<int2 *>(sStage + (size_t)a.STAGES * a.stage_bytes);   // [STAGES]
    uint64_t *full = reinterpret_cast<uint64_t *>(hdr + a.STAGES);
    uint64_t *empty = full + a.STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    griddep_wait();   // the bucket lists are the previous kernel's
    const int nact = *a.nact;
    int N = 0;
    if (a.fused) N = nact * moe_blocks(a.W[0], a.rblk[0]);
    else
        for (int p = 0; p < a.nproj; p++) N += nact * moe_blocks(a.W[p], a.rblk[p]);
    const int i_begin = (int)(((int64_t)N * blockIdx.x) / gridDim.x);
    const int i_end = (int)(((int64_t)N * (blockIdx.x + 1)) / gridDim.x);
    if (i_begin >= i_end) return;                               // uniform over the CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) {
            for (int i = i_begin, k = 0; i < i_end; i++, k++) {
                const int slot = k % a.STAGES, round = k / a.STAGES;
                if (round > 0 && !mbar_wait_sleep(&empty[slot], (round - 1) & 1)) {
                    atomicExch(a.err, 1u);
                    break;
                }
                const MoeItem it = moe_item(a, i, nact);
                const int p0 = a.fused ? 0 : it.p, p1 = a.fused ? 1 : it.p;
                const int r0 = it.blk * MMAV_ROWS * a.rblk[p0];
                const int nrows = min(MMAV_ROWS * a.rblk[p0], a.W[p0].rows - r0);
                hdr[slot] = make_int2(a.offsets[it.e], a.offsets[it.e + 1]);   // published by the arrive below
                const uint32_t base = smem_u32(sStage + (size_t)slot * a.stage_bytes);
                uint32_t bytes = 0;
                for (int p = p0; p <= p1; p++)
                    bytes += (uint32_t)(nrows * (a.W[p].code_row_bytes + a.W[p].scale_row_elems * 2));
                mbar_arrive_expect_tx(&full[slot], bytes);
                for (int p = p0; p <= p1; p++) {
                    const Mat &W = a.W[p];
                    bulk_copy_g2s(base + (uint32_t)a.coff[p],
                                  W.codes + (int64_t)it.e * W.expert_code_stride + (int64_t)r0 * W.code_row_bytes,
                                  (uint32_t)(nrows * W.code_row_bytes), &full[slot]);
                    bulk_copy_g2s(base + (uint32_t)a.soff[p],
                                  W.scales + (int64_t)it.e * W.expert_scale_stride + (int64_t)r0 * W.scale_row_elems,
                                  (uint32_t)(nrows * W.scale_row_elems * 2), &full[slot]);
                }
            }
        }
        return;
    }

    // every projection's codebook table
    const int nthr = a.NW * 32, ctid = threadIdx.x - 32;
    for (int p = 0; p < a.nproj; p++) {
        uint8_t *tb = smem + a.tbl_off[p];
        const __half *cb = a.W[p].codebook;
        switch (geom_of(a.W[p].d, a.W[p].bits)) {
        case G_D2_B8: SmemCB<2, 8>::stage(tb, cb, ctid, nthr); break;
        case G_D4_B8: SmemCB<4, 8>::stage(tb, cb, ctid, nthr); break;
        case G_D8_B8: SmemCB<8, 8>::stage(tb, cb, ctid, nthr); break;
        case G_D2_B12: SmemCB<2, 12>::stage(tb, cb, ctid, nthr); break;
        case G_D4_B12: SmemCB<4, 12>::stage(tb, cb, ctid, nthr); break;
        default: SmemCB<8, 12>::stage(tb, cb, ctid, nthr); break;
        }
    }
    bar_sync_named(1, nthr);
    // (laundered: table reads must not move above the barrier)
    const uint32_t smem_base = launder(smem_u32(smem));

    const int cw = warp - 1;
    const int g = lane >> 2, t = lane & 3;
    for (int i = i_begin + cw, k = cw; i < i_end; i += a.NW, k += a.NW) {
        const int slot = k % a.STAGES, round = k / a.STAGES;
        const bool ok = mbar_wait_sleep(&full[slot], round & 1);
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) atomicExch(a.err, 1u);
            break;
        }
        const MoeItem it = moe_item(a, i, nact);
        const int2 jj = hdr[slot];
        // (laundered: the stage's loads must not move above the wait)
        const uint32_t stage = launder(smem_u32(sStage + (size_t)slot * a.stage_bytes));
        const int pi = a.fused ? 0 : it.p;
        const Mat &W = a.W[pi];
        const int nblk = a.rblk[pi];
        for (int c0 = jj.x; c0 < jj.y; c0 += 16) {
            const int pos0 = min(c0 + g, jj.y - 1), pos1 = min(c0 + g + 8, jj.y - 1);
            const __half *x0p, *x1p;
            if (a.a_by_token[pi]) {
                x0p = a.ain[pi] + (int64_t)(a.sorted[pos0] / a.topk) * W.cols;
                x1p = a.ain[pi] + (int64_t)(a.sorted[pos1] / a.topk) * W.cols;
            } else {
                x0p = a.ain[pi] + (int64_t)pos0 * W.cols;
                x1p = a.ain[pi] + (int64_t)pos1 * W.cols;
            }
            x0p += 16 * t;
            x1p += 16 * t;
            for (int bi = 0; bi < nblk; bi++) {
                const int r0 = (it.blk * nblk + bi) * MMAV_ROWS;
                if (r0 >= W.rows) break;
                const int ra = r0 + 2 * t, rb = ra + 1;
                float tot[2][2];
                moe_block_chunk_any(W, stage + (uint32_t)(a.coff[pi] + bi * MMAV_ROWS * (int)W.code_row_bytes),
                                    stage + (uint32_t)(a.soff[pi] + bi * MMAV_ROWS * (int)W.scale_row_elems * 2),
                                    smem_base + (uint32_t)a.tbl_off[pi], lane, x0p, x1p, tot);
                if (a.fused) {
                    const Mat &U = a.W[1];
                    float tu[2][2];
                    moe_block_chunk_any(U, stage + (uint32_t)(a.coff[1] + bi * MMAV_ROWS * (int)U.code_row_bytes),
                                        stage + (uint32_t)(a.soff[1] + bi * MMAV_ROWS * (int)U.scale_row_elems * 2),
                                        smem_base + (uint32_t)a.tbl_off[1], lane, x0p, x1p, tu);
                    // h = fp16(silu(g) * u), as the separate SiLU kernel writes it
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const int tok = c0 + g + 8 * h;
                        if (tok >= jj.y) continue;
                        if (ra < W.rows)
                            a.h16[(int64_t)tok * W.rows + ra] = __float2half_rn(tot[h][0] / (1.f + expf(-tot[h][0])) * tu[h][0]);
                        if (rb < W.rows)
                            a.h16[(int64_t)tok * W.rows + rb] = __float2half_rn(tot[h][1] / (1.f + expf(-tot[h][1])) * tu[h][1]);
                    }
                } else {
                    float *out = a.out[pi];
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const int tok = c0 + g + 8 * h;
                        if (tok >= jj.y) continue;
                        if (ra < W.rows) out[(int64_t)tok * W.rows + ra] = tot[h][0];
                        if (rb < W.rows) out[(int64_t)tok * W.rows + rb] = tot[h][1];
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }
}

// ------------------------------------------------------------------ prefill helpers

// xg[pos] = fp16(x[token of the pair at pos]) for every valid pair (bucket order).
template <typename XT>
__global__ void moe_gather_kernel(const XT *__restrict__ x, const int *__restrict__ sorted, const int *__restrict__ offsets,
                                  int E, int topk, int hidden, __half *__restrict__ xg)
{
    griddep_wait();
    const int q = hidden / 8;
    const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int total = offsets[E];
    if (idx >= (int64_t)total * q) return;
    const int j = (int)(idx / q), c = (int)(idx % q) * 8;
    const int t = sorted[j] / topk;
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)t * hidden + c));
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
    if constexpr (sizeof(XT) == 2 && !std::is_same<XT, __half>::value) {
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w[k]));
            __half2 h = __floats2half2_rn(f.x, f.y);
            w[k] = *reinterpret_cast<uint32_t *>(&h);
        }
    }
    *reinterpret_cast<uint4 *>(xg + (int64_t)j * hidden + c) = make_uint4(w[0], w[1], w[2], w[3]);
}

// h16 = fp16(silu(g) * u) for the valid rows.
__global__ void moe_silu_mul_kernel(const float *__restrict__ g, const float *__restrict__ u,
                                    const int *__restrict__ offsets, int E, int inter, __half *__restrict__ h)
{
    griddep_wait();
    const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t n4 = (int64_t)offsets[E] * inter / 4;
    if (idx >= n4) return;
    const float4 a = __ldg(reinterpret_cast<const float4 *>(g) + idx);
    const float4 b = __ldg(reinterpret_cast<const float4 *>(u) + idx);
    const __half2 lo = __floats2half2_rn(a.x / (1.f + expf(-a.x)) * b.x, a.y / (1.f + expf(-a.y)) * b.y);
    const __half2 hi = __floats2half2_rn(a.z / (1.f + expf(-a.z)) * b.z, a.w / (1.f + expf(-a.w)) * b.w);
    reinterpret_cast<__half2 *>(h)[2 * idx] = lo;
    reinterpret_cast<__half2 *>(h)[2 * idx + 1] = hi;
}

// ------------------------------------------------------------------ 4. combine

__global__ void moe_combine_kernel(const float *__restrict__ o, const int *__restrict__ pos,
                                   const float *__restrict__ w, int T, int topk, int hidden, void *y, int yt)
{
    griddep_wait();
    const int q = hidden / 4;
    const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (idx >= (int64_t)T * q) return;
    const int t = (int)(idx / q), c = (int)(idx % q) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < topk; j++) {
        const int p = pos[t * topk + j];
        if (p < 0) continue;
        const float wt = w[t * topk + j];
        const float4 v = __ldg(reinterpret_cast<const float4 *>(o + (int64_t)p * hidden + c));
        acc.x = fmaf(wt, v.x, acc.x);
        acc.y = fmaf(wt, v.y, acc.y);
        acc.z = fmaf(wt, v.z, acc.z);
        acc.w = fmaf(wt, v.w, acc.w);
    }
    const int64_t b = (int64_t)t * hidden + c;
    store_out(y, b, acc.x, yt);
    store_out(y, b + 1, acc.y, yt);
    store_out(y, b + 2, acc.z, yt);
    store_out(y, b + 3, acc.w, yt);
}

// ------------------------------------------------------------------ host


unsigned int *device_error_word();

static int moe_num_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

static size_t moe_table_bytes(const Mat &W) {
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: return SmemCB<2, 8>::BYTES;
    case G_D4_B8: return SmemCB<4, 8>::BYTES;
    case G_D8_B8: return SmemCB<8, 8>::BYTES;
    case G_D2_B12: return SmemCB<2, 12>::BYTES;
    case G_D4_B12: return SmemCB<4, 12>::BYTES;
    default: return SmemCB<8, 12>::BYTES;
    }
}

// Shared-memory plan of moe_mma_kernel: false when it does not apply (scale rows not
// whole 16-byte units, per-expert codebooks) or the tables and a ring of at least 4
// stages do not fit.
static bool plan_moe_mma(MoeMmaArgs &m, size_t *smem_out)
{
    size_t tb = 0;
    for (int p = 0; p < m.nproj; p++) {
        if ((m.W[p].scale_row_elems * 2) % 16 || ((uintptr_t)m.W[p].scales % 16)) return false;
        if (m.W[p].num_experts > 1 && (m.W[p].expert_scale_stride * 2) % 16) return false;
        if (m.W[p].num_experts > 1 && m.W[p].expert_codebook_stride != 0) return false;
        m.tbl_off[p] = (int)tb;
        tb += (moe_table_bytes(m.W[p]) + 127) / 128 * 128;
    }
    m.tbl_bytes = (int)tb;
    m.NW = 8;
    // a stage: the block's codes and scales of every projection it holds (fused: both);
    // otherwise one projection at a time, sized for the largest
    // blocks per item: about 4 KB of codes per item (all projections of a fused item)
    int64_t row_bytes = 0;
    for (int p = 0; p < (m.fused ? m.nproj : 1); p++) row_bytes += m.W[p].code_row_bytes;
    for (int p = 0; p < m.nproj; p++) {
        const int64_t rb = m.fused ? row_bytes : m.W[p].code_row_bytes;
        int r = 1;
        while (r < 4 && (int64_t)MMAV_ROWS * 2 * r * rb <= 4096) r *= 2;
        m.rblk[p] = r;
    }
    if (m.fused) m.rblk[1] = m.rblk[0];
    size_t off = 0, mx = 0;
    for (int p = 0; p < m.nproj; p++) {
        const size_t cb = (size_t)MMAV_ROWS * m.rblk[p] * m.W[p].code_row_bytes;
        const size_t sb = ((size_t)MMAV_ROWS * m.rblk[p] * m.W[p].scale_row_elems * 2 + 15) / 16 * 16;
        if (m.fused) {
            m.coff[p] = (int)off;
            m.soff[p] = (int)(off + cb);
            off += cb + sb;
        } else {
            m.coff[p] = 0;
            m.soff[p] = (int)cb;
            mx = std::max(mx, cb + sb);
        }
    }
    m.stage_bytes = (int)(((m.fused ? off : mx) + 127) / 128 * 128);
    const size_t fixed = 128 + tb;
    const size_t per_stage = (size_t)m.stage_bytes + sizeof(int2) + 16;
    m.STAGES = 32;   // ideally >= 2 NW (two items in flight per warp); any count is correct
    while (m.STAGES > 4 && fixed + (size_t)m.STAGES * per_stage > 232448) m.STAGES--;
    const size_t smem = fixed + (size_t)m.STAGES * per_stage;
    if (smem > 232448) return false;
    *smem_out = smem;
    return true;
}

static vq_status launch_moe_mma(MoeMmaArgs &m, size_t smem, cudaStream_t s)
{
    if (cudaFuncSetAttribute(moe_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return VQ_ERR_CUDA;
    if (launch_pdl(moe_mma_kernel, dim3(moe_num_sms()), dim3(32 * (1 + m.NW)), smem, s, m) != cudaSuccess)
        return VQ_ERR_CUDA;
    return VQ_OK;
}

vq_status launch_moe(const Mat &gate, const Mat &up, const Mat &down, const void *x, vq_dtype xt, int32_t T,
                     const int32_t *ids, const float *w, int32_t topk, void *y, vq_dtype yt, void *ws,
                     size_t ws_bytes, cudaStream_t s)
{
    (void)ws_bytes;
    const int E = gate.num_experts, hidden = gate.cols, inter = gate.rows;
    const MoeLayout L = moe_layout(T, topk, E, hidden, inter);
    uint8_t *W8 = static_cast<uint8_t *>(ws);
    auto I = [&](size_t off) { return reinterpret_cast<int *>(W8 + off); };
    auto F = [&](size_t off) { return reinterpret_cast<float *>(W8 + off); };

    // Decode route (few tokens per expert): fused gate/up GEMV, then down GEMV.  The
    // tcgen05 GEMM once experts see several tokens on average, or when the GEMV does not
    // apply (scale rows not whole 16-byte units, per-expert codebooks, or shared memory).
    const double per_expert = (double)L.P / std::min(E, L.P);
    MoeMmaArgs m{};
    m.nproj = 2;
    m.fused = 1;   // gate and up of a block together: the warp writes h = silu(g) * u
    m.W[0] = gate; m.W[1] = up;
    MoeMmaArgs md{};
    md.nproj = 1;
    md.W[0] = down;
    size_t smem1 = 0, smem2 = 0;
    const bool use_gemm = per_expert >= 4.0 || !plan_moe_mma(m, &smem1) || !plan_moe_mma(md, &smem2);
    const int BT = per_expert <= 24 ? 32 : per_expert <= 48 ? 64 : 128;

    BucketArgs b;
    b.ids = ids; b.P = L.P; b.E = E; b.BT = BT;
    b.status = reinterpret_cast<unsigned int *>(W8 + L.status);
    b.counts = I(L.counts); b.offsets = I(L.offsets); b.sorted = I(L.sorted); b.pos = I(L.pos);
    b.act = I(L.act); b.nact = I(L.nact); b.t_exp = I(L.t_exp); b.t_row = I(L.t_row); b.t_cnt = I(L.t_cnt);
    b.ntiles = I(L.ntiles);
    const size_t bsmem = sizeof(unsigned short) * (BUCKET_THREADS / 32) * E;
    if (cudaFuncSetAttribute(moe_bucket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bsmem) !=
        cudaSuccess)
        return VQ_ERR_CUDA;
    if (launch_pdl(moe_bucket_kernel, dim3(1), dim3(BUCKET_THREADS), bsmem, s, b) != cudaSuccess) return VQ_ERR_CUDA;

    const int max_active = std::min(E, L.P);
    vq_status st;
    if (use_gemm) {
        __half *xg = reinterpret_cast<__half *>(W8 + L.xg);
        __half *h16 = reinterpret_cast<__half *>(W8 + L.h16);
        const int64_t ng = (int64_t)L.P * (hidden / 8);
        if (xt == VQ_F16)
            st = launch_pdl(moe_gather_kernel<__half>, dim3((unsigned)((ng + 255) / 256)), dim3(256), 0, s,
                            (const __half *)x, (const int *)b.sorted, (const int *)b.offsets, E, topk, hidden, xg) == cudaSuccess ? VQ_OK : VQ_ERR_CUDA;
        else
            st = launch_pdl(moe_gather_kernel<__nv_bfloat16>, dim3((unsigned)((ng + 255) / 256)), dim3(256), 0, s,
                            (const __nv_bfloat16 *)x, (const int *)b.sorted, (const int *)b.offsets, E, topk, hidden, xg) == cudaSuccess ? VQ_OK : VQ_ERR_CUDA;
        if (st != VQ_OK) return st;
        const int max_tiles = std::min(L.max_tiles, (L.P + BT - 1) / BT + E);
        GemmArgs ga{};
        ga.W[0] = gate; ga.W[1] = up;
        ga.y[0] = F(L.g); ga.y[1] = F(L.u);
        ga.ldy[0] = ga.ldy[1] = inter;
        ga.yt = VQ_F32;
        ga.t_exp = b.t_exp; ga.t_row = b.t_row; ga.t_cnt = b.t_cnt; ga.ntiles = b.ntiles;
        if ((st = run_vq_gemm(ga, 2, xg, L.P, false, BT, max_tiles, s)) != VQ_OK) return st;
        const int64_t nh = (int64_t)L.P * inter / 4;
        if (launch_pdl(moe_silu_mul_kernel, dim3((unsigned)((nh + 255) / 256)), dim3(256), 0, s, (const float *)F(L.g),
                       (const float *)F(L.u), (const int *)b.offsets, E, inter, h16) != cudaSuccess)
            return VQ_ERR_CUDA;
        GemmArgs gd = ga;
        gd.W[0] = down;
        gd.y[0] = F(L.o);
        gd.ldy[0] = hidden;
        if ((st = run_vq_gemm(gd, 1, h16, L.P, false, BT, max_tiles, s)) != VQ_OK) return st;
        const int64_t n = (int64_t)T * (hidden / 4);
        if (launch_pdl(moe_combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, (const float *)F(L.o),
                   (const int *)b.pos, w, T, topk, hidden, y, (int)yt) != cudaSuccess)
        return VQ_ERR_CUDA;
        VQ_CHECK_LAUNCH();
        return VQ_OK;
    }
    // decode route: grouped tensor-core GEMV (tokens of an expert are the MMA's A rows)
    const int64_t ng = (int64_t)L.P * (hidden / 8);
    const __half *ain1 = static_cast<const __half *>(x);
    int by_token = 1;
    if (xt != VQ_F16) {   // bf16 activations: gather and convert to fp16 in bucket order
        __half *xg = reinterpret_cast<__half *>(W8 + L.xg);
        if (launch_pdl(moe_gather_kernel<__nv_bfloat16>, dim3((unsigned)((ng + 255) / 256)), dim3(256), 0, s,
                       (const __nv_bfloat16 *)x, (const int *)b.sorted, (const int *)b.offsets, E, topk, hidden, xg) != cudaSuccess)
            return VQ_ERR_CUDA;
        ain1 = xg;
        by_token = 0;
    }
    m.sorted = b.sorted; m.offsets = b.offsets; m.act = b.act; m.nact = b.nact; m.topk = topk;
    m.err = device_error_word();
    if (!m.err) return VQ_ERR_CUDA;
    __half *h16 = reinterpret_cast<__half *>(W8 + L.h16);
    m.h16 = h16;
    m.ain[0] = m.ain[1] = ain1;
    m.a_by_token[0] = m.a_by_token[1] = by_token;
    if ((st = launch_moe_mma(m, smem1, s)) != VQ_OK) return st;
    md.sorted = m.sorted; md.offsets = m.offsets; md.act = m.act; md.nact = m.nact; md.topk = topk;
    md.err = m.err;
    md.out[0] = F(L.o);
    md.ain[0] = h16;
    md.a_by_token[0] = 0;
    if ((st = launch_moe_mma(md, smem2, s)) != VQ_OK) return st;
    const int64_t n = (int64_t)T * (hidden / 4);
    if (launch_pdl(moe_combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, (const float *)F(L.o),
                   (const int *)b.pos, w, T, topk, hidden, y, (int)yt) != cudaSuccess)
        return VQ_ERR_CUDA;
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

vq_status read_moe_status(const void *ws, cudaStream_t s)
{
    unsigned int bad = 0;
    if (cudaMemcpyAsync(&bad, ws, sizeof(bad), cudaMemcpyDeviceToHost, s) != cudaSuccess) return VQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return VQ_ERR_CUDA;
    return bad ? VQ_ERR_DEVICE_FLAG : VQ_OK;
}

// ------------------------------------------------------------------ allocation-free variant

// Scratch of the allocation-free entry point (vq_moe_grouped_noalloc): a fixed array in
// the library's device image, present on every GPU that loads the library until exit.
constexpr size_t MOE_STATIC_SCRATCH_BYTES = (size_t)16 << 20;
static __device__ __align__(256) unsigned char g_moe_static_scratch[MOE_STATIC_SCRATCH_BYTES];

size_t moe_static_scratch_bytes() { return MOE_STATIC_SCRATCH_BYTES; }

// Device address of the static scratch on the current device.  Host code cannot use the
// array's name as a device address, so the address is looked up once per device (with
// that device current) and cached.  Returns nullptr if the lookup fails.
void *moe_static_scratch()
{
    static void *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_moe_static_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace vq

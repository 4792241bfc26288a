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
//      projection with its own geometry, so mixed tiers share the launch;
//   3. down: one grouped launch with input silu(g) * u formed on the fly;
//   4. combine: y_t = sum over slots (in order) of w * o, skipping invalid pairs.
// Pairs whose expert id is outside [0, E) are counted in the workspace status word and
// contribute nothing.  Float atomics are never used: results are deterministic.
#include <algorithm>
#include <type_traits>

#include "vq_codebook.cuh"
#include "vq_gemm_api.cuh"
#include "vq_gemv_body.cuh"
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

// ------------------------------------------------------------------ 2./3. grouped GEMV

struct MoeGemvArgs {
    Mat W[2];
    float *out[2];                    // [P][W.rows] fp32, rows in bucket order
    const void *x;                    // stage 1: activations [T][hidden]
    const float *g, *u;               // stage 2: [P][inter]
    const int *sorted, *offsets, *act, *nact;
    int topk;
};

template <int D, int BITS, int XMODE>
__device__ __forceinline__ void moe_gemv_body(const MoeGemvArgs &a, const Mat &W, int e, float *out, uint8_t *smem)
{
    using CB = SmemCB<D, BITS>;
    using S = B1Shape<D, BITS>;
    constexpr int R = S::R;
    const int nchunk = (W.cols / D + S::CPC - 1) / S::CPC;
    int lpr_log2 = 0;
    while ((1 << lpr_log2) < 32 && (1 << lpr_log2) < nchunk) lpr_log2++;
    const int LPR = 1 << lpr_log2, G = 32 >> lpr_log2;
    const int rows_per_cta = GEMV_BODY_WARPS * R * G;
    const int row0 = blockIdx.x * rows_per_cta;
    if (row0 >= W.rows) return;                          // uniform over the block

    CB::stage(smem, W.codebook + (int64_t)e * W.expert_codebook_stride);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> lpr_log2, l = lane & (LPR - 1);
    const int rbase = row0 + warp * R * G + g * R;
    const uint8_t *codes = W.codes + (int64_t)e * W.expert_code_stride;
    const __half *scales = W.scales + (int64_t)e * W.expert_scale_stride;
    const uint8_t *cbase = smem + (lane % CB::NREP) * CB::ENTRY;
    const int j_end = a.offsets[e + 1];
    for (int j = a.offsets[e]; j < j_end; j++) {
        float acc[R];
#pragma unroll
        for (int i = 0; i < R; i++) acc[i] = 0.f;
        if constexpr (XMODE == 2) {
            const int inter = W.cols;
            b1_accumulate<D, BITS>(codes, scales, W.rows, W.cols, W.code_row_bytes, W.scale_row_elems, cbase,
                                   rbase, l, LPR, XSiluMul{a.g + (int64_t)j * inter, a.u + (int64_t)j * inter},
                                   acc);
        } else {
            using XT = typename std::conditional<XMODE == 0, __half, __nv_bfloat16>::type;
            const int t = a.sorted[j] / a.topk;
            b1_accumulate<D, BITS>(codes, scales, W.rows, W.cols, W.code_row_bytes, W.scale_row_elems, cbase,
                                   rbase, l, LPR, XRow<XT>{(const XT *)a.x + (int64_t)t * W.cols}, acc);
        }
#pragma unroll
        for (int i = 0; i < R; i++) {
            const float v = group_sum(acc[i], LPR);
            if (l == 0 && rbase + i < W.rows) out[(int64_t)j * W.rows + rbase + i] = v;
        }
    }
}

template <int XMODE>
__global__ void __launch_bounds__(GEMV_BODY_THREADS) moe_gemv_kernel(MoeGemvArgs a)
{
    extern __shared__ __align__(16) uint8_t smem[];
    if ((int)blockIdx.y >= *a.nact) return;
    const int e = a.act[blockIdx.y];
    const Mat &W = a.W[blockIdx.z];
    float *out = a.out[blockIdx.z];
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: moe_gemv_body<2, 8, XMODE>(a, W, e, out, smem); break;
    case G_D4_B8: moe_gemv_body<4, 8, XMODE>(a, W, e, out, smem); break;
    case G_D8_B8: moe_gemv_body<8, 8, XMODE>(a, W, e, out, smem); break;
    case G_D2_B12: moe_gemv_body<2, 12, XMODE>(a, W, e, out, smem); break;
    case G_D4_B12: moe_gemv_body<4, 12, XMODE>(a, W, e, out, smem); break;
    case G_D8_B12: moe_gemv_body<8, 12, XMODE>(a, W, e, out, smem); break;
    default: break;
    }
}

// ------------------------------------------------------------------ prefill helpers

// xg[pos] = fp16(x[token of the pair at pos]) for every valid pair (bucket order).
template <typename XT>
__global__ void moe_gather_kernel(const XT *__restrict__ x, const int *__restrict__ sorted, const int *__restrict__ offsets,
                                  int E, int topk, int hidden, __half *__restrict__ xg)
{
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


static size_t cb_smem_bytes(const Mat &W) {
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: return SmemCB<2, 8>::BYTES;
    case G_D4_B8: return SmemCB<4, 8>::BYTES;
    case G_D8_B8: return SmemCB<8, 8>::BYTES;
    case G_D2_B12: return SmemCB<2, 12>::BYTES;
    case G_D4_B12: return SmemCB<4, 12>::BYTES;
    default: return SmemCB<8, 12>::BYTES;
    }
}

static int gemv_rows_per_cta(const Mat &W) {
    const int bits = W.bits, d = W.d;
    const int cpc = bits == 8 ? 16 : 32, R = bits == 8 ? 8 : 4;
    const int nchunk = (W.cols / d + cpc - 1) / cpc;
    int lpr = 1;
    while (lpr < 32 && lpr < nchunk) lpr *= 2;
    return GEMV_BODY_WARPS * R * (32 / lpr);
}

template <int XMODE>
static vq_status launch_moe_gemv(const MoeGemvArgs &a, int nproj, int max_active, cudaStream_t s)
{
    size_t smem = 0;
    int gx = 1;
    for (int z = 0; z < nproj; z++) {
        smem = std::max(smem, cb_smem_bytes(a.W[z]));
        const int rpc = gemv_rows_per_cta(a.W[z]);
        gx = std::max(gx, (a.W[z].rows + rpc - 1) / rpc);
    }
    auto kern = moe_gemv_kernel<XMODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return VQ_ERR_CUDA;
    dim3 grid(gx, max_active, nproj);
    kern<<<grid, GEMV_BODY_THREADS, smem, s>>>(a);
    VQ_CHECK_LAUNCH();
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

    // Tensor cores once experts see several tokens on average; the grouped GEMV otherwise.
    const double per_expert = (double)L.P / std::min(E, L.P);
    const bool use_gemm = per_expert >= 4.0;
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
    moe_bucket_kernel<<<1, BUCKET_THREADS, bsmem, s>>>(b);
    VQ_CHECK_LAUNCH();

    const int max_active = std::min(E, L.P);
    vq_status st;
    if (use_gemm) {
        __half *xg = reinterpret_cast<__half *>(W8 + L.xg);
        __half *h16 = reinterpret_cast<__half *>(W8 + L.h16);
        const int64_t ng = (int64_t)L.P * (hidden / 8);
        if (xt == VQ_F16)
            moe_gather_kernel<__half><<<(unsigned)((ng + 255) / 256), 256, 0, s>>>((const __half *)x, b.sorted, b.offsets, E, topk, hidden, xg);
        else
            moe_gather_kernel<__nv_bfloat16><<<(unsigned)((ng + 255) / 256), 256, 0, s>>>((const __nv_bfloat16 *)x, b.sorted, b.offsets, E, topk, hidden, xg);
        VQ_CHECK_LAUNCH();
        const int max_tiles = std::min(L.max_tiles, (L.P + BT - 1) / BT + E);
        GemmArgs ga{};
        ga.W[0] = gate; ga.W[1] = up;
        ga.y[0] = F(L.g); ga.y[1] = F(L.u);
        ga.ldy[0] = ga.ldy[1] = inter;
        ga.yt = VQ_F32;
        ga.t_exp = b.t_exp; ga.t_row = b.t_row; ga.t_cnt = b.t_cnt; ga.ntiles = b.ntiles;
        if ((st = run_vq_gemm(ga, 2, xg, L.P, false, BT, max_tiles, s)) != VQ_OK) return st;
        const int64_t nh = (int64_t)L.P * inter / 4;
        moe_silu_mul_kernel<<<(unsigned)((nh + 255) / 256), 256, 0, s>>>(F(L.g), F(L.u), b.offsets, E, inter, h16);
        VQ_CHECK_LAUNCH();
        GemmArgs gd = ga;
        gd.W[0] = down;
        gd.y[0] = F(L.o);
        gd.ldy[0] = hidden;
        if ((st = run_vq_gemm(gd, 1, h16, L.P, false, BT, max_tiles, s)) != VQ_OK) return st;
        const int64_t n = (int64_t)T * (hidden / 4);
        moe_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(F(L.o), b.pos, w, T, topk, hidden, y, (int)yt);
        VQ_CHECK_LAUNCH();
        return VQ_OK;
    }
    MoeGemvArgs a{};
    a.sorted = b.sorted; a.offsets = b.offsets; a.act = b.act; a.nact = b.nact; a.topk = topk;
    // gate and up in one grouped launch
    a.W[0] = gate; a.W[1] = up;
    a.out[0] = F(L.g); a.out[1] = F(L.u);
    a.x = x;
    st = xt == VQ_F16 ? launch_moe_gemv<0>(a, 2, max_active, s) : launch_moe_gemv<1>(a, 2, max_active, s);
    if (st != VQ_OK) return st;
    // down, input silu(g) * u
    a.W[0] = down;
    a.out[0] = F(L.o);
    a.g = F(L.g); a.u = F(L.u);
    if ((st = launch_moe_gemv<2>(a, 1, max_active, s)) != VQ_OK) return st;
    // combine
    const int64_t n = (int64_t)T * (hidden / 4);
    moe_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(F(L.o), b.pos, w, T, topk, hidden, y, (int)yt);
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

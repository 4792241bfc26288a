// vq_gemv_stream.cu — batch-1 decode GEMV that streams whole rows into shared memory
// with bulk asynchronous copies (the decode path of paper "Data-Free Vector Quantization
// Beats Affine Quantization at Matched Bytes Below 5 Bits", §3.4, re-designed for
// sm_100a: the copy engine keeps HBM busy independently of the lookup work).
//
//   * Each CTA owns a contiguous range of rows (ranges differ by at most one row, so the
//     work is balanced over the grid).  Consecutive rows of codes are contiguous in
//     memory, and so are consecutive rows of scales, so one stage of RB rows is two bulk
//     copies (cp.async.bulk) completing on one mbarrier.  Stages form a ring.
//   * Warp 0 (one thread) issues the copies.  Consumer warps are split into NG groups of
//     WPG warps; lane (warp wg, lane l) of a group owns the 64-column unit u = 32 wg + l
//     of every row (one scale group), with the unit's 64 activations in registers for the
//     whole kernel.  Group g takes rows g, g + NG, ... of each stage.
//   * Per row a lane reads its unit's codes from shared memory, looks them up in the
//     shared-memory codebook, and accumulates scale * sum(codebook * x) in fp32.  The RPG
//     row partials of a stage are reduced across the group with a transposed warp
//     reduction and a per-group named barrier, in a fixed order (deterministic).
#include <algorithm>

#include "vq_codebook.cuh"
#include "vq_internal.cuh"
#include "vq_sm100.cuh"

namespace vq {

constexpr int STREAM_MAX_THREADS = 544;     // producer warp + at most 16 consumer warps

struct StreamCfg {
    int U;        // 64-column units per row
    int WPG;      // warps per group (ceil(U / 32))
    int NG;       // groups
    int RPG;      // rows per group per stage (power of 2, <= 8)
    int STAGES;
    int rows_base, rows_extra;   // rows per CTA: base (+1 for the first `extra` CTAs)
    int stage_code_bytes, stage_scale_bytes;   // per stage (RB = NG * RPG rows)
    unsigned int *err;                          // library device error word
};

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// v[i] summed over the warp; lane l returns the total of v[l >> (5 - log2 N)].
template <int N>
__device__ __forceinline__ float transpose_reduce(float (&v)[N], int lane) {
#pragma unroll
    for (int n = N, o = 16; n > 1; n >>= 1, o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; i++) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float r = v[0];
#pragma unroll
    for (int o = 16 / N; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
    return r;
}

// acc += a.lo * b.lo + a.hi * b.hi with fp16 inputs and fp32 accumulation.
__device__ __forceinline__ void fma2_f16_f32(float &acc, uint32_t a, uint32_t b) {
    asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\t"
        "mov.b32 {a0, a1}, %1;\n\t"
        "mov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.f16 %0, a0, b0, %0;\n\t"
        "fma.rn.f32.f16 %0, a1, b1, %0;\n\t}"
        : "+f"(acc)
        : "r"(a), "r"(b));
}

// Activations of one 64-column unit held in registers: 32 packed fp16 pairs for fp16
// inputs (multiplied with mixed-precision FMA), 64 fp32 values otherwise.
template <typename XT>
struct UnitX {
    float f[64];
    __device__ __forceinline__ void load(const XT *p) {
        float t[64];
        load_x_vec64(p, t);
#pragma unroll
        for (int i = 0; i < 64; i++) f[i] = t[i];
    }
    __device__ __forceinline__ static void load_x_vec64(const XT *p, float (&xr)[64]) {
        if constexpr (sizeof(XT) == 4) {
#pragma unroll
            for (int k = 0; k < 16; k++) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(p) + k);
                xr[4 * k] = v.x; xr[4 * k + 1] = v.y; xr[4 * k + 2] = v.z; xr[4 * k + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 8; k++) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p) + k);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    uint16_t l16 = (uint16_t)(w[j] & 0xffffu), h16 = (uint16_t)(w[j] >> 16);
                    xr[8 * k + 2 * j] = to_f32<XT>(*reinterpret_cast<XT *>(&l16));
                    xr[8 * k + 2 * j + 1] = to_f32<XT>(*reinterpret_cast<XT *>(&h16));
                }
            }
        }
    }
    // sum over t < 2 of cb2[t] * x[col + t] (cb2: two fp16 codebook values)
    __device__ __forceinline__ void fma_pair(float &acc, uint32_t cb2, int col) const {
        const float2 c = __half22float2(*reinterpret_cast<const __half2 *>(&cb2));
        acc = fmaf(c.x, f[col], acc);
        acc = fmaf(c.y, f[col + 1], acc);
    }
};

template <>
struct UnitX<__nv_bfloat16> {
    uint32_t h[32];   // packed bf16 pairs; bf16 -> fp32 is a 16-bit shift
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
#pragma unroll
        for (int k = 0; k < 8; k++) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p) + k);
            h[4 * k] = u.x; h[4 * k + 1] = u.y; h[4 * k + 2] = u.z; h[4 * k + 3] = u.w;
        }
    }
    __device__ __forceinline__ void fma_pair(float &acc, uint32_t cb2, int col) const {
        const float2 c = __half22float2(*reinterpret_cast<const __half2 *>(&cb2));
        const uint32_t w = h[col >> 1];
        acc = fmaf(c.x, __uint_as_float(w << 16), acc);
        acc = fmaf(c.y, __uint_as_float(w & 0xffff0000u), acc);
    }
};

template <>
struct UnitX<__half> {
    uint32_t h[32];
    __device__ __forceinline__ void load(const __half *p) {
#pragma unroll
        for (int k = 0; k < 8; k++) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p) + k);
            h[4 * k] = u.x; h[4 * k + 1] = u.y; h[4 * k + 2] = u.z; h[4 * k + 3] = u.w;
        }
    }
    __device__ __forceinline__ void fma_pair(float &acc, uint32_t cb2, int col) const {
        fma2_f16_f32(acc, cb2, h[col >> 1]);
    }
};

// Code bytes of one 64-column unit: 64/d codes of BITS bits.
template <int D, int BITS>
struct UnitCodes {
    static constexpr int BYTES = (64 / D) * BITS / 8;   // 32 16 8 | 48 24 12
    static constexpr int WORDS = BYTES / 4;
    uint32_t w[WORDS];
    __device__ __forceinline__ void load(const uint8_t *p) {   // p: shared memory, BYTES-aligned
        if constexpr (BYTES % 16 == 0) {
#pragma unroll
            for (int v = 0; v < BYTES / 16; v++) {
                const uint4 u = *reinterpret_cast<const uint4 *>(p + 16 * v);
                w[4 * v] = u.x; w[4 * v + 1] = u.y; w[4 * v + 2] = u.z; w[4 * v + 3] = u.w;
            }
        } else if constexpr (BYTES % 8 == 0) {
#pragma unroll
            for (int v = 0; v < BYTES / 8; v++) {
                const uint2 u = *reinterpret_cast<const uint2 *>(p + 8 * v);
                w[2 * v] = u.x; w[2 * v + 1] = u.y;
            }
        } else {
#pragma unroll
            for (int v = 0; v < WORDS; v++) w[v] = *reinterpret_cast<const uint32_t *>(p + 4 * v);
        }
    }
    __device__ __forceinline__ uint32_t code(int q) const {
        if constexpr (BITS == 8) {
            return (w[q >> 2] >> ((q & 3) * 8)) & 0xFFu;
        } else {
            const int bit = 12 * q, wi = bit >> 5, sh = bit & 31;
            if (sh + 12 <= 32) return (w[wi] >> sh) & 0xFFFu;
            return __funnelshift_r(w[wi], w[wi + 1], sh) & 0xFFFu;
        }
    }
};

// One row's contribution of one unit: sum over the unit's codes of codebook . x.
template <int D, int BITS, typename XT>
__device__ __forceinline__ float unit_dot(const UnitCodes<D, BITS> &c, const uint8_t *cbl, const UnitX<XT> &x) {
    using CB = SmemCB<D, BITS>;
    constexpr int NC = 64 / D;
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int q = 0; q < NC; q++) {
        const uint8_t *e = cbl + c.code(q) * CB::STRIDE;
        float &acc = (q & 1) ? a1 : a0;
        if constexpr (D == 2) {
            x.fma_pair(acc, *reinterpret_cast<const uint32_t *>(e), q * 2);
        } else if constexpr (D == 4) {
            const uint2 v = *reinterpret_cast<const uint2 *>(e);
            x.fma_pair(acc, v.x, q * 4);
            x.fma_pair(acc, v.y, q * 4 + 2);
        } else {
            const uint4 v = *reinterpret_cast<const uint4 *>(e);
            x.fma_pair(acc, v.x, q * 8);
            x.fma_pair(acc, v.y, q * 8 + 2);
            x.fma_pair(acc, v.z, q * 8 + 4);
            x.fma_pair(acc, v.w, q * 8 + 6);
        }
    }
    return a0 + a1;
}

template <int D, int BITS, typename XT, int RPG>
__global__ void __launch_bounds__(STREAM_MAX_THREADS)
gemv_stream_kernel(Mat W, const XT *__restrict__ x, void *__restrict__ y, int yt, StreamCfg cfg)
{
    using CB = SmemCB<D, BITS>;
    using UC = UnitCodes<D, BITS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *sCB = smem;
    uint8_t *sCodes = sCB + CB::BYTES;
    uint8_t *sScales = sCodes + (size_t)cfg.STAGES * cfg.stage_code_bytes;
    float *red = reinterpret_cast<float *>(sScales + (size_t)cfg.STAGES * cfg.stage_scale_bytes);  // [2][NG][WPG][RPG]
    uint64_t *full = reinterpret_cast<uint64_t *>(red + 2 * cfg.NG * cfg.WPG * RPG);
    uint64_t *empty = full + cfg.STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int RB = cfg.NG * RPG;
    const int r_begin = blockIdx.x * cfg.rows_base + min((int)blockIdx.x, cfg.rows_extra);
    const int r_count = cfg.rows_base + ((int)blockIdx.x < cfg.rows_extra ? 1 : 0);
    const int nst = (r_count + RB - 1) / RB;
    const int consumers = cfg.NG * cfg.WPG;

    CB::stage(sCB, W.codebook);
    if (threadIdx.x == 0) {
        for (int s = 0; s < cfg.STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], consumers);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < nst; s++) {
                const int slot = s % cfg.STAGES, round = s / cfg.STAGES;
                if (round > 0 && !mbar_wait(&empty[slot], (round - 1) & 1)) {
                    atomicExch(cfg.err, 1u);
                    break;
                }
                const int r0 = r_begin + s * RB;
                const int nrows = min(RB, r_begin + r_count - r0);
                const uint32_t cb = (uint32_t)(nrows * W.code_row_bytes);
                const uint32_t sb = (uint32_t)(nrows * W.scale_row_elems * 2);
                mbar_arrive_expect_tx(&full[slot], cb + sb);
                bulk_g2s(sCodes + (size_t)slot * cfg.stage_code_bytes, W.codes + (int64_t)r0 * W.code_row_bytes, cb,
                         &full[slot]);
                bulk_g2s(sScales + (size_t)slot * cfg.stage_scale_bytes, W.scales + (int64_t)r0 * W.scale_row_elems,
                         sb, &full[slot]);
            }
        }
        return;
    }

    const int cw = warp - 1, g = cw / cfg.WPG, wg = cw % cfg.WPG;
    const int u = wg * 32 + lane;
    const bool active = u < cfg.U;
    UnitX<XT> xr;
    if (active) xr.load(x + (int64_t)u * 64);
    const uint8_t *cbl = sCB + (lane % CB::NREP) * CB::ENTRY;

    // A wait that runs out marks the warp dead: it stops waiting and computing but keeps
    // taking part in the group barriers, so no other warp is left blocked.
    bool dead = false;
    for (int s = 0; s < nst; s++) {
        const int slot = s % cfg.STAGES, round = s / cfg.STAGES;
        if (!dead) {
            const bool ok = mbar_wait(&full[slot], round & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicExch(cfg.err, 1u);
                dead = true;
            }
        }
        const int r0 = r_begin + s * RB;
        const int nrows = min(RB, r_begin + r_count - r0);
        const uint8_t *sc = sCodes + (size_t)slot * cfg.stage_code_bytes;
        const __half *ss = reinterpret_cast<const __half *>(sScales + (size_t)slot * cfg.stage_scale_bytes);
        float part[RPG];
#pragma unroll
        for (int i = 0; i < RPG; i++) {
            const int rr = g + i * cfg.NG;
            part[i] = 0.f;
            if (active && !dead && rr < nrows) {
                UC c;
                c.load(sc + (size_t)rr * W.code_row_bytes + (size_t)u * UC::BYTES);
                const float scale = __half2float(ss[(size_t)rr * W.scale_row_elems + u]);
                part[i] = scale * unit_dot<D, BITS, XT>(c, cbl, xr);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);     // this warp is done reading the stage

        const float tot = transpose_reduce<RPG>(part, lane);
        float *rb = red + (size_t)(s & 1) * cfg.NG * cfg.WPG * RPG;
        const int row_of_lane = lane >> (5 - (RPG == 1 ? 0 : RPG == 2 ? 1 : RPG == 4 ? 2 : 3));
        if ((lane & ((32 / RPG) - 1)) == 0) rb[(g * cfg.WPG + wg) * RPG + row_of_lane] = tot;
        named_barrier(1 + g, cfg.WPG * 32);
        if (wg == 0 && lane < RPG) {
            float v = 0.f;
            for (int k = 0; k < cfg.WPG; k++) v += rb[(g * cfg.WPG + k) * RPG + lane];
            const int rr = g + lane * cfg.NG;
            if (rr < nrows) store_out(y, r0 + rr, v, yt);
        }
    }
}

// ------------------------------------------------------------------ host

unsigned int *device_error_word();

static int stream_num_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

static size_t stream_cb_bytes(int d, int bits) {
    switch (geom_of(d, bits)) {
    case G_D2_B8: return SmemCB<2, 8>::BYTES;
    case G_D4_B8: return SmemCB<4, 8>::BYTES;
    case G_D8_B8: return SmemCB<8, 8>::BYTES;
    case G_D2_B12: return SmemCB<2, 12>::BYTES;
    case G_D4_B12: return SmemCB<4, 12>::BYTES;
    default: return SmemCB<8, 12>::BYTES;
    }
}

static size_t stream_smem(const StreamCfg &c, size_t cb) {
    return 128 + cb + (size_t)c.STAGES * (c.stage_code_bytes + c.stage_scale_bytes) +
           2 * (size_t)c.NG * c.WPG * c.RPG * sizeof(float) + 2 * (size_t)c.STAGES * 8;
}

template <int D, int BITS, typename XT, int RPG>
static vq_status stream_launch(const Mat &W, const void *x, void *y, int yt, const StreamCfg &c, size_t smem,
                               int grid, cudaStream_t s)
{
    auto k = gemv_stream_kernel<D, BITS, XT, RPG>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return VQ_ERR_CUDA;
    k<<<grid, 32 * (1 + c.NG * c.WPG), smem, s>>>(W, (const XT *)x, y, yt, c);
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

template <int D, int BITS, typename XT>
static vq_status stream_rpg(const Mat &W, const void *x, void *y, int yt, const StreamCfg &c, size_t smem, int grid,
                            cudaStream_t s)
{
    switch (c.RPG) {
    case 1: return stream_launch<D, BITS, XT, 1>(W, x, y, yt, c, smem, grid, s);
    case 2: return stream_launch<D, BITS, XT, 2>(W, x, y, yt, c, smem, grid, s);
    default: return stream_launch<D, BITS, XT, 4>(W, x, y, yt, c, smem, grid, s);
    }
}

template <typename XT>
static vq_status stream_geom(const Mat &W, const void *x, void *y, int yt, const StreamCfg &c, size_t smem,
                             int grid, cudaStream_t s)
{
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: return stream_rpg<2, 8, XT>(W, x, y, yt, c, smem, grid, s);
    case G_D4_B8: return stream_rpg<4, 8, XT>(W, x, y, yt, c, smem, grid, s);
    case G_D8_B8: return stream_rpg<8, 8, XT>(W, x, y, yt, c, smem, grid, s);
    case G_D2_B12: return stream_rpg<2, 12, XT>(W, x, y, yt, c, smem, grid, s);
    case G_D4_B12: return stream_rpg<4, 12, XT>(W, x, y, yt, c, smem, grid, s);
    case G_D8_B12: return stream_rpg<8, 12, XT>(W, x, y, yt, c, smem, grid, s);
    default: return VQ_ERR_UNSUPPORTED;
    }
}

// Batch-1 GEMV through the row-streaming kernel.  Returns VQ_ERR_UNSUPPORTED (nothing
// launched) for shapes it does not take: scale rows that are not whole 16-byte units,
// rows wider than 16 warps x 32 units, or too few rows to fill the GPU.
vq_status launch_gemv_stream(const Mat &W, const void *x, vq_dtype xt, void *y, vq_dtype yt, cudaStream_t s)
{
    const int64_t srow_bytes = W.scale_row_elems * 2;
    if (srow_bytes % 16 || ((uintptr_t)W.scales % 16)) return VQ_ERR_UNSUPPORTED;
    StreamCfg c{};
    c.U = W.cols / 64;
    c.WPG = (c.U + 31) / 32;
    if (c.WPG > 16) return VQ_ERR_UNSUPPORTED;
    const int nsm = stream_num_sms();
    if (W.rows < nsm) return VQ_ERR_UNSUPPORTED;
    c.NG = std::max(1, std::min(15, 16 / c.WPG));   // named barriers 1..15, one per group
    const int64_t row_bytes = W.code_row_bytes + srow_bytes;
    c.RPG = 4;
    while (c.RPG > 1 && (int64_t)c.NG * c.RPG * row_bytes > 24576) c.RPG /= 2;
    const size_t cb = stream_cb_bytes(W.d, W.bits);
    c.err = device_error_word();
    if (!c.err) return VQ_ERR_CUDA;
    for (;;) {
        const int RB = c.NG * c.RPG;
        c.stage_code_bytes = (int)(RB * W.code_row_bytes);
        c.stage_scale_bytes = (int)(RB * srow_bytes);
        c.STAGES = 8;
        while (c.STAGES > 2 && stream_smem(c, cb) > 232448) c.STAGES--;
        if (stream_smem(c, cb) <= 232448) break;
        if (c.RPG > 1) c.RPG /= 2;
        else if (c.NG > 1) c.NG--;
        else return VQ_ERR_UNSUPPORTED;
    }
    const int grid = nsm;
    c.rows_base = W.rows / grid;
    c.rows_extra = W.rows % grid;
    const size_t smem = stream_smem(c, cb);
    if (xt == VQ_F16) return stream_geom<__half>(W, x, y, (int)yt, c, smem, grid, s);
    if (xt == VQ_BF16) return stream_geom<__nv_bfloat16>(W, x, y, (int)yt, c, smem, grid, s);
    return stream_geom<float>(W, x, y, (int)yt, c, smem, grid, s);
}

}  // namespace vq

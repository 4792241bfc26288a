// vq_gemm.cu — prefill GEMM y[m][n] = sum_k x[m][k] W[n][k] on the tcgen05 tensor cores,
// with W expanded from its VQ codes inside the kernel.
//
// The pages' prefill path (paper "Data-Free Vector Quantization Beats Affine Quantization
// at Matched Bytes Below 5 Bits", §2.5 and §3.4: the prefill-shaped code path and the
// fused decode-and-matmul) is a dense contraction once the weights are expanded, so on
// sm_100a it runs on the 5th-generation tensor cores:
//
//   * one CTA computes a 128 (weight rows) x BT (tokens) output tile; the weight tile is
//     the MMA's A operand (M = 128), the activation tile its B operand (N = BT), so each
//     expanded weight is used by BT tokens;
//   * warp 0 (one thread) streams activation tiles [BT][64] into shared memory with TMA
//     (128-byte swizzle);
//   * where a row's codes for one 64-column stage are a whole number of 16-byte units
//     (d = 2 and d = 4 with 8-bit codes, d = 2 with 12-bit codes) the same TMA thread
//     loads the stage's [128 rows][code bytes] block with the activation tile, on the
//     same barrier; other geometries read the codes from global memory per thread;
//   * warps 2-13 (384 threads, three per weight row, each taking every third 64-column
//     stage, so each thread's prefetch runs several stages ahead and three expansions are
//     in flight per row) read the row's codes (shared
//     memory or global) and its scale (global), look the codes up in the shared-memory
//     codebook and multiply by the scale (one rounding to the tile type).  The expanded
//     128 x 64 tile goes to tensor memory: each thread writes its row (a warp may only
//     reach its own 32-lane quarter, so row = 32 (warp mod 4) + lane) as 32 columns with
//     one tcgen05.st, then signals an mbarrier.  Keeping the A tile out of shared memory
//     leaves the shared-memory bandwidth to the codebook lookups and the activation
//     tiles, which the MMA reads from there;
//   * warp 1 (one thread) issues tcgen05.mma (kind::f16, A from tensor memory, B from
//     shared memory, fp32 accumulation in tensor memory) for each 64-column stage and
//     frees the stage with tcgen05.commit;
//   * after the last stage, warps 2-13 read the accumulator out of tensor memory
//     (tcgen05.ld; the three warps of a 32-lane quarter share the columns) and store y.
// Stages are a ring of STAGES buffers guarded by mbarriers; every wait is bounded and a
// wait that runs out sets the library's device error word instead of hanging.
#include <string.h>

#include <algorithm>
#include <cmath>

#include "vq_codebook.cuh"
#include "vq_gemm_api.cuh"
#include "vq_internal.cuh"
#include "vq_mma.cuh"
#include "vq_sm100.cuh"

namespace vq {

__device__ unsigned int g_device_error;   // nonzero after a bounded wait ran out

constexpr int GEMM_BM = 128;       // weight rows per tile (UMMA M)
constexpr int GEMM_BK = 64;        // columns per stage (one 128-byte swizzle row of 16-bit)
constexpr int GEMM_NPAR = 3;      // expansion warp groups (each expands every GEMM_NPAR-th stage)
constexpr int GEMM_THREADS = 64 + 128 * GEMM_NPAR;   // warp 0 TMA, warp 1 MMA + TMEM, then the expansion + epilogue warps

// Code blocks go through TMA when a row's codes for one stage are whole 16-byte units.
__host__ __device__ constexpr bool gemm_code_tma(int d, int bits) { return ((64 / d) * bits / 8) % 16 == 0; }

// Tensor maps of the projections' codes (used where gemm_code_tma holds): uint8
// [experts][rows][code_row_bytes], box [1][128][code bytes of one stage].
struct GemmCodeMaps {
    CUtensorMap code[2];
};

// Packed codes of one row for one 64-column stage: 64/d codes.
template <int D, int BITS>
struct CodeBlock {
    static constexpr int BYTES = (64 / D) * BITS / 8;   // 32, 16, 8 (8-bit); 48, 24, 12 (12-bit)
    static constexpr int WORDS = BYTES / 4;
    uint32_t w[WORDS];

    __device__ __forceinline__ void load(const uint8_t *row, int kb) {
        const uint8_t *p = row + (int64_t)kb * BYTES;
        if constexpr (BYTES % 16 == 0) {
#pragma unroll
            for (int v = 0; v < BYTES / 16; v++) {
                uint4 u = ldg_stream_u4(p + 16 * v);
                w[4 * v] = u.x; w[4 * v + 1] = u.y; w[4 * v + 2] = u.z; w[4 * v + 3] = u.w;
            }
        } else if constexpr (BYTES % 8 == 0) {
#pragma unroll
            for (int v = 0; v < BYTES / 8; v++) {
                uint2 u = __ldg(reinterpret_cast<const uint2 *>(p) + v);
                w[2 * v] = u.x; w[2 * v + 1] = u.y;
            }
        } else {
#pragma unroll
            for (int v = 0; v < WORDS; v++) w[v] = __ldg(reinterpret_cast<const uint32_t *>(p) + v);
        }
    }
    // From a 16-byte aligned shared-memory copy of the row's block (TMA layout).
    __device__ __forceinline__ void load_smem(const uint8_t *p) {
        static_assert(BYTES % 16 == 0, "whole 16-byte units");
#pragma unroll
        for (int v = 0; v < BYTES / 16; v++) {
            const uint4 u = *reinterpret_cast<const uint4 *>(p + 16 * v);
            w[4 * v] = u.x; w[4 * v + 1] = u.y; w[4 * v + 2] = u.z; w[4 * v + 3] = u.w;
        }
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int v = 0; v < WORDS; v++) w[v] = 0u;
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

// scale * (two fp16 codebook values) -> two tile elements, one rounding.
template <bool BF16T>
__device__ __forceinline__ uint32_t scale_pair(uint32_t cb2, __half2 s2, float sf) {
    if constexpr (!BF16T) {
        __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&cb2), s2);
        return *reinterpret_cast<uint32_t *>(&r);
    } else {
        float2 f = __half22float2(*reinterpret_cast<__half2 *>(&cb2));
        __nv_bfloat162 r = __floats2bfloat162_rn(f.x * sf, f.y * sf);
        return *reinterpret_cast<uint32_t *>(&r);
    }
}

__device__ __forceinline__ void flag_error(volatile int *abort_flag) {
    *abort_flag = 1;
    atomicExch(&g_device_error, 1u);
}

// One CTA: output tile rows [n0, n0 + 128) of expert e's matrix W against activation rows
// [m0, m0 + mcount) of the tensor map; y[(m0 + j) * ldy + n] for j < mcount.
template <int D, int BITS, int BT, int STAGES, bool BF16T>
__device__ __forceinline__ void gemm_cta(const CUtensorMap *xmap, const CUtensorMap *cmap, const Mat &W, int e,
                                         int m0, int mcount, int n0, void *__restrict__ y, int64_t ldy, int yt,
                                         uint8_t *smem_raw)
{
    using CB = SmemCB<D, BITS>;
    using Blk = CodeBlock<D, BITS>;
    constexpr int B_TILE_BYTES = BT * GEMM_BK * 2;
    constexpr bool TMAC = gemm_code_tma(D, BITS);             // code blocks by TMA
    constexpr int C_TILE_BYTES = TMAC ? GEMM_BM * Blk::BYTES : 0;
    // tensor memory: fp32 accumulator (one column per token), then one 32-column A tile
    // per stage; the allocation is a power of two
    constexpr uint32_t TMEM_NEED = BT + 32 * STAGES;
    constexpr uint32_t TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256 : 512;
    static_assert(TMEM_NEED <= 512, "tensor memory holds 512 columns");

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sB = smem;
    uint8_t *sC = sB + STAGES * B_TILE_BYTES;                  // TMAC: [STAGES][128 rows][code bytes]
    uint8_t *sCB = sC + STAGES * C_TILE_BYTES;
    uint64_t *full_a = reinterpret_cast<uint64_t *>(sCB + CB::BYTES);
    uint64_t *full_b = full_a + STAGES;
    uint64_t *empty = full_b + STAGES;
    uint64_t *acc_bar = empty + STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *consumed = reinterpret_cast<volatile int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = W.cols / GEMM_BK;
    const uint8_t *codes_e = W.codes + (int64_t)e * W.expert_code_stride;
    const __half *scales_e = W.scales + (int64_t)e * W.expert_scale_stride;

    CB::stage(sCB, W.codebook + (int64_t)e * W.expert_codebook_stride);
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&full_a[s], 4);
            mbar_init(&full_b[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_bar, 1);
        *abort_flag = 0;
        *consumed = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer: activation tiles
        if (lane == 0) {
            tma_prefetch_map(xmap);
            if constexpr (TMAC) tma_prefetch_map(cmap);
            int issued = 0;
            for (int kb = 0; kb < nkb; kb++) {
                const int s = kb % STAGES, r = kb / STAGES;
                if (r > 0 && !mbar_wait_sleep(&empty[s], (r - 1) & 1)) { flag_error(abort_flag); break; }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(&full_b[s], B_TILE_BYTES + C_TILE_BYTES);
                tma_load_2d(sB + s * B_TILE_BYTES, xmap, &full_b[s], kb * GEMM_BK, m0);
                if constexpr (TMAC)   // rows past the end read as zeros
                    tma_load_3d(smem_u32(sC + s * C_TILE_BYTES), cmap, &full_b[s], kb * Blk::BYTES, n0, e);
                issued++;
            }
            // On an abort, wait (bounded) for the loads still in flight before leaving.
            if (*abort_flag) {
                for (int kb = *consumed; kb < issued; kb++)
                    mbar_wait(&full_b[kb % STAGES], (kb / STAGES) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(GEMM_BM, BT, BF16T);
            for (int kb = 0; kb < nkb; kb++) {
                const int s = kb % STAGES, r = kb / STAGES;
                if (!mbar_wait_sleep(&full_a[s], r & 1) || !mbar_wait_sleep(&full_b[s], r & 1)) {
                    flag_error(abort_flag);
                    break;
                }
                tc_fence_after();
                const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + s * B_TILE_BYTES));
#pragma unroll
                for (int k = 0; k < GEMM_BK / 16; k++)   // K = 16 per MMA: 8 A columns; +32 bytes = +2 in B's address field
                    umma_f16_ts(tmem, tmem + (uint32_t)(BT + 32 * s + 8 * k), bdesc + 2 * k, idesc,
                                (kb > 0 || k > 0) ? 1u : 0u);
                umma_commit(&empty[s]);
                *consumed = kb + 1;
            }
            umma_commit(acc_bar);
        }
    } else {
        // ---------------- expansion: thread t writes weight row n0 + t of every stage
        const int t = 32 * (warp & 3) + lane;    // tile row = tensor-memory lane
        const int par = (warp - 2) >> 2;         // this thread expands stages kb = par, par + NPAR, ...
        const int row = n0 + t;
        const bool rv = row < W.rows;
        const uint8_t *crow = codes_e + (int64_t)(rv ? row : 0) * W.code_row_bytes;
        const __half *srow = scales_e + (int64_t)(rv ? row : 0) * W.scale_row_elems;
        const uint8_t *cbl = sCB + (lane % CB::NREP) * CB::ENTRY;
        // 8-bit codes: the 32-bit shared address of this lane's codebook copy (laundered:
        // the lookups below must not move above the barrier that published the codebook);
        // entry e's copies start at e * 128, so one byte permute and a shift give the address
        const uint32_t cb32 = launder(smem_u32(cbl));
        auto ent = [&](const Blk &b, int q) -> uint32_t {
            return cb32 + (__byte_perm(b.w[q >> 2], 0u, 0x4440u | (uint32_t)(q & 3)) << 7);
        };
        const uint32_t tquarter = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's tensor-memory lanes

        // Scales (and, without TMAC, code blocks) of the stages kb = par + NPAR u (u < PF) are
        // kept in flight in a register ring; a slot is refilled (PF stages ahead) right
        // after it is expanded.  Rows past the end read row 0; their tile rows only reach
        // accumulator rows that are never stored.
        constexpr int PF = 5;
        constexpr int PFC = TMAC ? 1 : PF;
        Blk ring[PFC];
        __half sr[PF];
#pragma unroll
        for (int u = 0; u < PF; u++) {
            const int kbu = par + GEMM_NPAR * u;
            sr[u] = __float2half(0.f);
            if (kbu < nkb) sr[u] = srow[kbu];
            if constexpr (!TMAC) {
                if (kbu < nkb) ring[u].load(crow, kbu); else ring[u].zero();
            }
        }
        bool stop = false;
        for (int kb0 = par; kb0 < nkb && !stop; kb0 += GEMM_NPAR * PF) {
#pragma unroll
            for (int u = 0; u < PF; u++) {
                const int kb = kb0 + GEMM_NPAR * u;
                if (kb >= nkb || stop) break;                       // uniform over the warp
                const int s = kb % STAGES, r = kb / STAGES;
                bool ok = r == 0 || mbar_wait_sleep(&empty[s], (r - 1) & 1);
                if constexpr (TMAC) ok = ok && mbar_wait_sleep(&full_b[s], r & 1);   // the stage's codes landed
                if (__any_sync(0xffffffffu, !ok || *abort_flag)) {   // warp-uniform exit
                    if (lane == 0) flag_error(abort_flag);
                    stop = true;
                    break;
                }
                uint32_t av[32];                                     // the row's 64 tile elements
                const __half2 s2 = __half2half2(sr[u]);
                const float sf = __half2float(sr[u]);
                Blk tc;
                if constexpr (TMAC) tc.load_smem(sC + s * C_TILE_BYTES + t * Blk::BYTES);
                const Blk &cur = TMAC ? tc : ring[u % PFC];
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    uint32_t o[4];
                    if constexpr (D == 2) {
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            const uint32_t e = BITS == 8 ? ldsn32(ent(cur, 4 * c + j))
                                : *reinterpret_cast<const uint32_t *>(cbl + cur.code(4 * c + j) * CB::STRIDE);
                            o[j] = scale_pair<BF16T>(e, s2, sf);
                        }
                    } else if constexpr (D == 4) {
#pragma unroll
                        for (int j = 0; j < 2; j++) {
                            const uint2 e = BITS == 8 ? ldsn64(ent(cur, 2 * c + j))
                                : *reinterpret_cast<const uint2 *>(cbl + cur.code(2 * c + j) * CB::STRIDE);
                            o[2 * j] = scale_pair<BF16T>(e.x, s2, sf);
                            o[2 * j + 1] = scale_pair<BF16T>(e.y, s2, sf);
                        }
                    } else {
                        const uint4 e = BITS == 8 ? ldsn128(ent(cur, c))
                            : *reinterpret_cast<const uint4 *>(cbl + cur.code(c) * CB::STRIDE);
                        o[0] = scale_pair<BF16T>(e.x, s2, sf);
                        o[1] = scale_pair<BF16T>(e.y, s2, sf);
                        o[2] = scale_pair<BF16T>(e.z, s2, sf);
                        o[3] = scale_pair<BF16T>(e.w, s2, sf);
                    }
#pragma unroll
                    for (int j = 0; j < 4; j++) av[4 * c + j] = o[j];   // column 4c + j: elements 8c + 2j, +1
                }
                tmem_st_32x32b_x32(tmem + tquarter + (uint32_t)(BT + 32 * s), av);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_a[s]);
                const int nk = kb + GEMM_NPAR * PF;                  // refill this slot
                if (nk < nkb) {
                    sr[u] = srow[nk];
                    if constexpr (!TMAC) ring[u % PFC].load(crow, nk);
                }
            }
        }

        // ---------------- epilogue: TMEM -> registers -> y
        __syncwarp();
        const bool waited = mbar_wait_sleep(acc_bar, 0);
        if (!waited) flag_error(abort_flag);
        tc_fence_after();
        if (__all_sync(0xffffffffu, waited && !*abort_flag)) {   // warp-uniform: tcgen05.ld is .sync.aligned
            const int q = warp & 3;                  // TMEM lanes 32q..32q+31 belong to this warp
            const int erow = n0 + q * 32 + lane;
            const int cpar = (warp - 2) >> 2;        // GEMM_NPAR warps per quarter share the columns
#pragma unroll 1
            for (int c0 = 32 * cpar; c0 < BT; c0 += 32 * GEMM_NPAR) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
                tmem_ld_wait();
                if (erow < W.rows) {
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        if (c0 + j < mcount)
                            store_out(y, (int64_t)(m0 + c0 + j) * ldy + erow, __uint_as_float(v[j]), yt);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}


template <int BT, int STAGES, bool BF16T>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
vq_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ GemmArgs a,
               const __grid_constant__ GemmCodeMaps cm)
{
    extern __shared__ uint8_t smem_raw[];
    griddep_wait();   // the activations and (grouped) the tile list are the previous kernel's
    const int z = blockIdx.z;
    const Mat &W = a.W[z];
    const int n0 = blockIdx.y * GEMM_BM;
    if (n0 >= W.rows) return;                          // uniform over the CTA
    int e = 0, m0, mcount;
    if (a.t_exp) {
        const int tile = blockIdx.x;
        if (tile >= *a.ntiles) return;
        e = a.t_exp[tile];
        m0 = a.t_row[tile];
        mcount = a.t_cnt[tile];
    } else {
        m0 = blockIdx.x * BT;
        mcount = min(BT, a.M - m0);
    }
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: gemm_cta<2, 8, BT, STAGES, BF16T>(&xmap, &cm.code[z], W, e, m0, mcount, n0, a.y[z], a.ldy[z], a.yt, smem_raw); break;
    case G_D4_B8: gemm_cta<4, 8, BT, STAGES, BF16T>(&xmap, &cm.code[z], W, e, m0, mcount, n0, a.y[z], a.ldy[z], a.yt, smem_raw); break;
    case G_D8_B8: gemm_cta<8, 8, BT, STAGES, BF16T>(&xmap, &cm.code[z], W, e, m0, mcount, n0, a.y[z], a.ldy[z], a.yt, smem_raw); break;
    case G_D2_B12: gemm_cta<2, 12, BT, STAGES, BF16T>(&xmap, &cm.code[z], W, e, m0, mcount, n0, a.y[z], a.ldy[z], a.yt, smem_raw); break;
    case G_D4_B12: gemm_cta<4, 12, BT, STAGES, BF16T>(&xmap, &cm.code[z], W, e, m0, mcount, n0, a.y[z], a.ldy[z], a.yt, smem_raw); break;
    case G_D8_B12: gemm_cta<8, 12, BT, STAGES, BF16T>(&xmap, &cm.code[z], W, e, m0, mcount, n0, a.y[z], a.ldy[z], a.yt, smem_raw); break;
    default: break;
    }
}

// bf16 -> fp16 conversion of the activations (8 elements per thread).
__global__ void bf16_to_f16_kernel(const __nv_bfloat16 *__restrict__ in, __half *__restrict__ out, int64_t n8)
{
    griddep_wait();
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= n8) return;
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(in) + i);
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w[j]));
        __half2 h = __floats2half2_rn(f.x, f.y);
        w[j] = *reinterpret_cast<uint32_t *>(&h);
    }
    reinterpret_cast<uint4 *>(out)[i] = make_uint4(w[0], w[1], w[2], w[3]);
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

void *encode_tiled_fn();
static EncodeTiledFn encode_fn() { return reinterpret_cast<EncodeTiledFn>(encode_tiled_fn()); }

// cuTensorMapEncodeTiled from the driver (null if unavailable); shared with the GEMV.
void *encode_tiled_fn() {
    static void *fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = p;
    }
    return fn;
}

// Tensor map of activations [M][K] (16-bit, row stride K elements), box [BT][64], 128-B swizzle.
static bool make_x_map(CUtensorMap *map, const void *x, bool bf16, int M, int K, int BT) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {GEMM_BK, (cuuint32_t)BT};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                     const_cast<void *>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Shared memory of a launch whose largest codebook table takes cb_bytes and whose largest
// TMA code block takes ct_bytes per stage.
static size_t gemm_smem_bytes(int BT, int stages, size_t cb_bytes, size_t ct_bytes) {
    return 1024 + (size_t)stages * ((size_t)BT * GEMM_BK * 2 + ct_bytes) + cb_bytes + (3 * stages + 1) * 8 + 16;
}

static size_t code_tile_bytes(const Mat &W) {
    return gemm_code_tma(W.d, W.bits) ? (size_t)GEMM_BM * ((64 / W.d) * W.bits / 8) : 0;
}

// Code tensor map of W (3-D: bytes of a row, rows, experts).
static bool make_code_map(CUtensorMap *map, const Mat &W) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const int64_t E = W.num_experts > 1 ? W.num_experts : 1;
    const int64_t estride = E > 1 ? W.expert_code_stride : W.code_row_bytes * W.rows;
    cuuint64_t dims[3] = {(cuuint64_t)W.code_row_bytes, (cuuint64_t)W.rows, (cuuint64_t)E};
    cuuint64_t strides[2] = {(cuuint64_t)W.code_row_bytes, (cuuint64_t)estride};
    cuuint32_t box[3] = {(cuuint32_t)((64 / W.d) * W.bits / 8), (cuuint32_t)GEMM_BM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(W.codes), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static size_t cb_table_bytes(const Mat &W) {
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: return SmemCB<2, 8>::BYTES;
    case G_D4_B8: return SmemCB<4, 8>::BYTES;
    case G_D8_B8: return SmemCB<8, 8>::BYTES;
    case G_D2_B12: return SmemCB<2, 12>::BYTES;
    case G_D4_B12: return SmemCB<4, 12>::BYTES;
    default: return SmemCB<8, 12>::BYTES;
    }
}

template <int BT, int STAGES, bool BF16T>
static vq_status launch_gemm_cfg(const CUtensorMap &map, const GemmArgs &a, const GemmCodeMaps &cm, int nproj,
                                 int gx, size_t smem, cudaStream_t s)
{
    auto kern = vq_gemm_kernel<BT, STAGES, BF16T>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return VQ_ERR_CUDA;
    int rows = 0;
    for (int z = 0; z < nproj; z++) rows = std::max(rows, a.W[z].rows);
    dim3 grid(gx, (rows + GEMM_BM - 1) / GEMM_BM, nproj);
    if (launch_pdl(kern, grid, dim3(GEMM_THREADS), smem, s, map, a, cm) != cudaSuccess) return VQ_ERR_CUDA;
    return VQ_OK;
}

template <int BT, bool BF16T>
static vq_status launch_gemm_bt(const CUtensorMap &map, const GemmArgs &a, const GemmCodeMaps &cm, int nproj,
                                int gx, cudaStream_t s)
{
    size_t cb = 0, ct = 0;
    for (int z = 0; z < nproj; z++) {
        cb = std::max(cb, cb_table_bytes(a.W[z]));
        ct = std::max(ct, code_tile_bytes(a.W[z]));
    }
    // the deepest ring that fits (tensor memory: BT accumulator columns + 32 per stage)
    if (BT + 32 * 6 <= 512 && gemm_smem_bytes(BT, 6, cb, ct) <= 232448)
        return launch_gemm_cfg<BT, 6, BF16T>(map, a, cm, nproj, gx, gemm_smem_bytes(BT, 6, cb, ct), s);
    if (BT + 32 * 5 <= 512 && gemm_smem_bytes(BT, 5, cb, ct) <= 232448)
        return launch_gemm_cfg<BT, 5, BF16T>(map, a, cm, nproj, gx, gemm_smem_bytes(BT, 5, cb, ct), s);
    if (gemm_smem_bytes(BT, 4, cb, ct) <= 232448)
        return launch_gemm_cfg<BT, 4, BF16T>(map, a, cm, nproj, gx, gemm_smem_bytes(BT, 4, cb, ct), s);
    if (gemm_smem_bytes(BT, 3, cb, ct) <= 232448)
        return launch_gemm_cfg<BT, 3, BF16T>(map, a, cm, nproj, gx, gemm_smem_bytes(BT, 3, cb, ct), s);
    return VQ_ERR_UNSUPPORTED;
}

// Run the GEMM over activation rows held in x16 ([rows][K] 16-bit, K = W.cols): dense
// (a.t_exp == null, a.M rows) or grouped (tile list on the device, at most max_tiles).
vq_status run_vq_gemm(const GemmArgs &a, int nproj, const void *x16, int x_rows, bool bf16, int BT,
                      int max_tiles, cudaStream_t s)
{
    CUtensorMap map;
    if (!make_x_map(&map, x16, bf16, x_rows, a.W[0].cols, BT)) return VQ_ERR_CUDA;
    const int gx = a.t_exp ? max_tiles : (a.M + BT - 1) / BT;
    if (gx < 1) return VQ_OK;
    GemmCodeMaps cm;
    memset(&cm, 0, sizeof(cm));
    for (int z = 0; z < nproj; z++)
        if (gemm_code_tma(a.W[z].d, a.W[z].bits) && !make_code_map(&cm.code[z], a.W[z])) return VQ_ERR_UNSUPPORTED;
    if (bf16) {
        switch (BT) {
        case 32: return launch_gemm_bt<32, true>(map, a, cm, nproj, gx, s);
        case 64: return launch_gemm_bt<64, true>(map, a, cm, nproj, gx, s);
        case 128: return launch_gemm_bt<128, true>(map, a, cm, nproj, gx, s);
        case 192: return launch_gemm_bt<192, true>(map, a, cm, nproj, gx, s);
        default: return launch_gemm_bt<256, true>(map, a, cm, nproj, gx, s);
        }
    }
    switch (BT) {
    case 32: return launch_gemm_bt<32, false>(map, a, cm, nproj, gx, s);
    case 64: return launch_gemm_bt<64, false>(map, a, cm, nproj, gx, s);
    case 128: return launch_gemm_bt<128, false>(map, a, cm, nproj, gx, s);
    case 192: return launch_gemm_bt<192, false>(map, a, cm, nproj, gx, s);
    default: return launch_gemm_bt<256, false>(map, a, cm, nproj, gx, s);
    }
}

static int gemm_num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] <= 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 148;
    }
    return cache[dev];
}

// Tokens per tile of a dense GEMM with M tokens and N weight rows.  Large M: 256 tokens
// (the most reuse of each expanded weight tile) unless 192-token tiles fill the last wave
// of CTAs (one per SM) clearly better.
static int dense_bt(int M, int N) {
    if (M <= 128) return M <= 32 ? 32 : M <= 64 ? 64 : 128;
    const int nsm = gemm_num_sms(), rt = (N + GEMM_BM - 1) / GEMM_BM;
    auto fill = [&](int bt) {
        const double waves = (double)((M + bt - 1) / bt) * rt / nsm;
        return waves / std::ceil(waves);
    };
    return fill(192) > fill(256) + 0.05 ? 192 : 256;
}

size_t gemm_workspace_bytes(const Mat &W, vq_dtype xt, int M, uint32_t flags)
{
    if (xt == VQ_BF16 && !(flags & VQ_GEMM_BF16_TILES)) return ((size_t)M * W.cols * 2 + 255) / 256 * 256;
    return 0;
}

vq_status launch_gemm(const Mat &W, const void *x, vq_dtype xt, int M, void *y, vq_dtype yt, void *ws,
                      size_t ws_bytes, uint32_t flags, cudaStream_t s)
{
    (void)ws_bytes;
    GemmArgs a{};
    a.W[0] = W;
    a.y[0] = y;
    a.ldy[0] = W.rows;
    a.yt = (int)yt;
    a.M = M;
    const bool bf16_tiles = (flags & VQ_GEMM_BF16_TILES) != 0;
    const void *x16 = x;
    if (xt == VQ_BF16 && !bf16_tiles) {
        const int64_t n8 = (int64_t)M * W.cols / 8;
        if (launch_pdl(bf16_to_f16_kernel, dim3((unsigned)((n8 + 255) / 256)), dim3(256), 0, s,
                       (const __nv_bfloat16 *)x, (__half *)ws, n8) != cudaSuccess)
            return VQ_ERR_CUDA;
        x16 = ws;
    }
    return run_vq_gemm(a, 1, x16, M, bf16_tiles, dense_bt(M, W.rows), 0, s);
}

// Device address of the error word on the current device (looked up once per device).
unsigned int *device_error_word()
{
    static unsigned int *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<unsigned int *>(p);
    }
    return addr[dev];
}

vq_status read_device_error(cudaStream_t s, unsigned int *out)
{
    if (cudaStreamSynchronize(s) != cudaSuccess) return VQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(out, g_device_error, sizeof(unsigned int)) != cudaSuccess) return VQ_ERR_CUDA;
    return VQ_OK;
}

}  // namespace vq

// vq_gemv_mma.cu — decode GEMV (batch 1..16) with the multiply-adds on the tensor cores.
//
// The pages' fused decode-and-matmul (paper "Data-Free Vector Quantization Beats Affine
// Quantization at Matched Bytes Below 5 Bits", §3.4) spends, per code, one lookup and d
// multiply-adds.  Here the lookups stay on the shared-memory pipe and the multiply-adds
// move to mma.sync (m16n8k16, fp16 inputs, fp32 accumulation):
//
//   * weights are the MMA's A operand (16 m x 16 k): m = the 16 rows of a row block, and
//     lane (g = lane / 4, t = lane % 4) supplies rows g and g + 8.  An A register holds
//     two consecutive columns of one row — one d = 2 codebook entry, half of a d = 4
//     entry or a quarter of a d = 8 entry — so looked-up entries go straight into A
//     registers with no conversion;
//   * the activations are the B operand (16 k x 8 n): token n in column n (tokens 0..7;
//     a second MMA covers tokens 8..15); columns beyond the batch repeat a valid token
//     and are dropped, so a batch of up to 8 costs the same lookups as one token;
//   * k-slots are permuted so that in MMA s (s = 0..3) of a 64-column scale group lane t
//     covers columns [16t + 4s, 16t + 4s + 4): a lane's codes for a group are contiguous
//     (8, 4 or 2 bytes of 8-bit codes; 12, 6 or 3 bytes of 12-bit codes) and its
//     activations are 16 contiguous values;
//   * the four MMAs of a group produce a fresh fp32 partial per (row, token), which is
//     scaled by that row's group scale in fp32 and added to the running total — every
//     product is exact (fp16 x fp16 in fp32), nothing is rounded to 16 bits.
//
// Lookup addressing (K = 256): the table sits at a 64 KB-aligned shared address with one
// 256-byte line per entry, the lane's private copy at byte (lane * entry bytes) mod 256
// of the line.  The shared address of a lookup is then [table bits 16..31 | code | lane
// byte], so one byte permute of the packed code word forms it.  Lanes read distinct
// banks, so random codes never conflict.  K = 4096 tables are one plain copy.
//
// Data movement: one producer warp streams stages of (16 rows x a column chunk) codes and
// scales into a ring of shared-memory slots; each stage costs the copy engine as few
// operations as possible, because a bulk copy has a fixed cost of tens of nanoseconds.
// For 8-bit codes with rows a whole number of 128-byte segments, a stage is two TMA
// tensor loads: the codes as a 3-D box {128 bytes, 16 rows, segments} with the 128-byte
// swizzle, and the scales as a 2-D box.  Inside the MMA, row g of the block is stored
// row (2 (g mod 4) + g / 4), which together with the swizzle puts the lanes' code loads
// on distinct banks.  Other shapes use one bulk copy per row into padded row slots.
// The consumer warps split each stage's scale groups (the assignment rotates from one
// row block to the next) and keep per-(row, token) totals in registers across the chunks
// of a row block.  At the end of a row block one warp (rotating) adds the warps' totals
// in warp order.
//
// Load balance: a row block is 16 rows, so a matrix with few rows (5120 rows = 320
// blocks on 148 SMs) would leave SMs idle.  The launch therefore uses thread-block
// clusters of C CTAs: a cluster owns a contiguous range of row blocks and its C CTAs
// split the columns; each CTA keeps its per-block results in shared memory and, after a
// cluster barrier, the CTAs add the C partial results in rank order through distributed
// shared memory.  C is chosen on the host to minimise the largest per-CTA share.  Every
// sum runs in a fixed order, so results are deterministic.
#include <string.h>

#include <algorithm>
#include <mutex>

#include "vq_mma.cuh"

namespace vq {

constexpr int GV_RB = 16;                    // weight rows per block (the MMA's m)
// consumer warps: 16 for batches up to 8, 8 for batches 9..16 (whose reduction buffers
// are twice as large per warp)
template <int NT> __host__ __device__ constexpr int gv_nw() { return NT == 2 ? 8 : 16; }
template <int NT> __host__ __device__ constexpr int gv_threads() { return 32 * (gv_nw<NT>() + 1); }
constexpr int GV_MAX_STAGES = 10;
constexpr int GV_MAX_R = 14;                 // reduction buffers
static_assert(GV_MAX_STAGES <= 32 && GV_MAX_R <= 32, "barriers are initialised one per lane of a warp");
constexpr int GV_TBL = 65536;                // table region (64 KB)
constexpr int GV_BAR_BYTES = 512;            // mbarriers + abort word
constexpr int GV_DYN_SMEM = 232448;          // the per-block opt-in maximum (227 KB)
// Fixed shared-window placement: dynamic shared memory starts at a small offset (the
// window's reserved bytes; checked on the device), so everything is placed from GV_LO
// on: stages and buffers below the table, the table at 64 KB, the rest above it.
constexpr uint32_t GV_LO = 2048;
constexpr uint32_t GV_TBL_ADDR = 65536;

// Placement of everything in the shared window (byte addresses).
struct GvLayout {
    uint32_t s0, s1, bars, red, part, recv, xs, cbraw;
    int n0, stages, R;
    int ok;
};

// Columns are handled in units of `ug` scale groups (1 for row-slot copies; 8 or 16 — a
// whole number of 128-byte segments — for TMA boxes).  A cluster's C CTAs take
// contiguous unit ranges (slices) of every row; a slice is split into `nch` chunks of
// wl or wl + 1 units; a stage holds one chunk of 16 rows.
struct GvCfg {
    int C, ncl;        // CTAs per cluster, clusters
    int ug, U;         // groups per unit, units per row (the last may be partial)
    int nch, wl;       // chunks per slice, smaller chunk width (units)
    int useg;          // TMA: 128-byte segments per unit
    int sgw[2];        // TMA: scale box width (groups) for chunk widths wl, wl + 1
    int CS, SS;        // row-slot copies: bytes between code / scale row slots
    int SB, SOFF;      // bytes of a stage; offset of its scales
    int XR, XB;        // staged activations: bytes per token row (0: read from global), total
    int PB;            // per-block results kept for the cluster reduction (0 if C = 1)
    int RBB;           // bytes of one reduction buffer
    int lag;           // a block is reduced `lag` blocks after it is posted (so the wait is short)
    int CBB;           // bytes of the codebook as stored in global memory
    GvLayout L;
    unsigned int *err;
};

struct GvMaps {
    CUtensorMap code[2];    // chunk widths wl, wl + 1
    CUtensorMap scale[2];
};

struct GvBump {
    uint32_t p, e;
    bool take(uint32_t sz, uint32_t &out) {
        const uint32_t need = (sz + 127u) & ~127u;
        if (p + need > e) return false;
        out = p;
        p += need;
        return true;
    }
};

// Host: the deepest ring (at most GV_MAX_STAGES stages, 1 KB-aligned for the swizzled
// boxes) that fits with the other buffers.
inline GvLayout gv_layout(const GvCfg &c, bool raw_cb) {
    GvLayout L{};
    L.ok = 0;
    const uint32_t a = (GV_LO + 1023u) & ~1023u, end = (uint32_t)GV_DYN_SMEM;
    for (int S = GV_MAX_STAGES; S >= 2; S--) {
        // a warp can run S stages ahead of the slowest one, and a block is reduced `lag`
        // blocks late: the reduction ring covers both, plus one spare
        const int R = (S + 1 + c.nch - 1) / c.nch + c.lag + 1;
        GvBump r0{a, GV_TBL_ADDR}, r1{GV_TBL_ADDR + (uint32_t)GV_TBL, end};
        int n0 = (int)((GV_TBL_ADDR - a) / (uint32_t)c.SB);
        if (n0 > S) n0 = S;
        bool ok = R <= GV_MAX_R;
        uint32_t tmp = 0;
        L.s0 = a;
        for (int i = 0; i < n0; i++) ok = ok && r0.take((uint32_t)c.SB, tmp);
        L.s1 = r1.p;
        for (int i = n0; i < S; i++) ok = ok && r1.take((uint32_t)c.SB, tmp);
        auto put = [&](uint32_t sz, uint32_t &out) {
            out = 0;
            if (ok && sz > 0) ok = r0.take(sz, out) || r1.take(sz, out);
        };
        put((uint32_t)GV_BAR_BYTES, L.bars);
        put((uint32_t)(R * c.RBB), L.red);
        put((uint32_t)c.PB, L.part);
        put((uint32_t)(c.C > 1 ? (c.C - 1) * c.PB : 0), L.recv);
        put((uint32_t)c.XB, L.xs);
        put(raw_cb ? (uint32_t)c.CBB : 0u, L.cbraw);
        if (ok) {
            L.n0 = n0;
            L.stages = S;
            L.R = R;
            L.ok = 1;
            return L;
        }
    }
    return L;
}

// ------------------------------------------------------------------ device helpers

__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// fp32 store to shared address `addr` of the CTA with cluster rank `rank`.
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, uint32_t rank, float v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(addr), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t lds32_volatile(uint32_t a) {
    uint32_t v;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}

// Lookup address of code byte j of `w` (K = 256 layout): byte 1 <- w.byte[j], bytes 0,
// 2, 3 from the lane constant lb = table | lane byte.
__device__ __forceinline__ uint32_t gv_addr(uint32_t w, uint32_t lb, int j) {
    return __byte_perm(w, lb, 0x7604u | ((uint32_t)j << 4));
}

// One 64-column scale group of one 16-row block: four MMAs (eight for NT = 2).
//   ra, rb: 8-bit codes: shared addresses of this lane's code bytes of its two rows;
//           12-bit codes: shared addresses of the two rows at this group
//   lb: K = 256: table | lane byte; K = 4096: table address
//   xa, xb: the lane's 16 activations of tokens g and g + 8
//   d[n]: the lane's two rows x tokens 8n + 2t, 8n + 2t + 1, fresh partials
template <int D, int BITS, int NT>
__device__ __forceinline__ void gv_group(uint32_t ra, uint32_t rb, int t, uint32_t lb, const uint32_t (&xa)[8],
                                         const uint32_t (&xb)[8], float (&d)[NT][4])
{
    uint32_t a[4][4];   // [s][a0..a3]: a0/a2 first row, a1/a3 second row
    if constexpr (BITS == 8) {
        if constexpr (D == 2) {
            const uint2 ca = ldsn64(ra), cb = ldsn64(rb);
#pragma unroll
            for (int s = 0; s < 4; s++) {
                const uint32_t wa = s < 2 ? ca.x : ca.y, wb = s < 2 ? cb.x : cb.y;
                const int j = 2 * (s & 1);
                a[s][0] = ldsn32(gv_addr(wa, lb, j));
                a[s][1] = ldsn32(gv_addr(wb, lb, j));
                a[s][2] = ldsn32(gv_addr(wa, lb, j + 1));
                a[s][3] = ldsn32(gv_addr(wb, lb, j + 1));
            }
        } else if constexpr (D == 4) {
            const uint32_t wa = ldsn32(ra), wb = ldsn32(rb);
#pragma unroll
            for (int s = 0; s < 4; s++) {
                const uint2 ea = ldsn64(gv_addr(wa, lb, s)), eb = ldsn64(gv_addr(wb, lb, s));
                a[s][0] = ea.x; a[s][1] = eb.x; a[s][2] = ea.y; a[s][3] = eb.y;
            }
        } else {
            const uint32_t wa = ldsn16(ra), wb = ldsn16(rb);
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const uint4 ea = ldsn128(gv_addr(wa, lb, h)), eb = ldsn128(gv_addr(wb, lb, h));
                a[2 * h][0] = ea.x; a[2 * h][1] = eb.x; a[2 * h][2] = ea.y; a[2 * h][3] = eb.y;
                a[2 * h + 1][0] = ea.z; a[2 * h + 1][1] = eb.z; a[2 * h + 1][2] = ea.w; a[2 * h + 1][3] = eb.w;
            }
        }
    } else {
        constexpr uint32_t ENTRY = 2 * D;
        LaneCodes<D, BITS> ca, cb;
        ca.load(ra, t);
        cb.load(rb, t);
        if constexpr (D == 2) {
#pragma unroll
            for (int s = 0; s < 4; s++) {
                a[s][0] = ldsn32(lb + ca.code(2 * s) * ENTRY);
                a[s][1] = ldsn32(lb + cb.code(2 * s) * ENTRY);
                a[s][2] = ldsn32(lb + ca.code(2 * s + 1) * ENTRY);
                a[s][3] = ldsn32(lb + cb.code(2 * s + 1) * ENTRY);
            }
        } else if constexpr (D == 4) {
#pragma unroll
            for (int s = 0; s < 4; s++) {
                const uint2 ea = ldsn64(lb + ca.code(s) * ENTRY), eb = ldsn64(lb + cb.code(s) * ENTRY);
                a[s][0] = ea.x; a[s][1] = eb.x; a[s][2] = ea.y; a[s][3] = eb.y;
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const uint4 ea = ldsn128(lb + ca.code(h) * ENTRY), eb = ldsn128(lb + cb.code(h) * ENTRY);
                a[2 * h][0] = ea.x; a[2 * h][1] = eb.x; a[2 * h][2] = ea.y; a[2 * h][3] = eb.y;
                a[2 * h + 1][0] = ea.z; a[2 * h + 1][1] = eb.z; a[2 * h + 1][2] = ea.w; a[2 * h + 1][3] = eb.w;
            }
        }
    }
    mman_f16_f32_zero(d[0], a[0], xa[0], xa[1]);
#pragma unroll
    for (int s = 1; s < 4; s++) mman_f16_f32(d[0], a[s], xa[2 * s], xa[2 * s + 1]);
    if constexpr (NT == 2) {
        mman_f16_f32_zero(d[1], a[0], xb[0], xb[1]);
#pragma unroll
        for (int s = 1; s < 4; s++) mman_f16_f32(d[1], a[s], xb[2 * s], xb[2 * s + 1]);
    }
}

// NT = 1: tokens 0..7 (the MMA's columns); NT = 2: tokens 0..15 (two MMAs per k-step).
// XS: activations staged in shared memory (else read through L1 from global memory).
// TMA: stages arrive as tensor boxes (8-bit codes only), else as row-slot copies.
template <int D, int BITS, int NT, bool XS, bool TMA>
__global__ void __launch_bounds__(gv_threads<NT>(), 1)
gemv_mma_kernel(Mat W, const __half *__restrict__ x, int batch, void *__restrict__ y, int yt,
                const __grid_constant__ GvCfg cfg, const __grid_constant__ GvMaps maps)
{
    static_assert(!TMA || BITS == 8, "tensor boxes carry 8-bit codes only");
    constexpr int GB = (64 / D) * BITS / 8;   // code bytes of one row per scale group
    constexpr int GPS = 128 / GB;             // TMA: groups per 128-byte segment
    constexpr int NWK = gv_nw<NT>();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    const GvLayout &L = cfg.L;
    auto sptr = [&](uint32_t a) { return smem_raw + (a - base); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = cfg.C;
    const int q = (int)(blockIdx.x % (unsigned)C);          // rank in the cluster (1-D clusters)
    const int ci = (int)(blockIdx.x / (unsigned)C);         // cluster index
    const int NB = (W.rows + GV_RB - 1) / GV_RB;
    const int b0 = ci * NB / cfg.ncl, b1 = (ci + 1) * NB / cfg.ncl;   // (fits 32 bits: ci < 2^10, NB < 2^21)
    const int nb = b1 - b0;
    const int G = W.cols / 64;
    const int ua0 = q * cfg.U / C, ua1 = (q + 1) * cfg.U / C;
    const int su = ua1 - ua0;                               // >= nch (host)
    const int gs0 = ua0 * cfg.ug, gs1 = min(ua1 * cfg.ug, G);
    const int SG = gs1 - gs0;
    const int nch = cfg.nch;
    const int cbw = su / nch, cxw = su % nch;               // chunk c: cbw + (c < cxw) units

    // The placement is fixed relative to the 64 KB-aligned start of this CTA's window (in
    // a cluster, rank r's window starts at r x 16 MB); the window's reserved bytes must
    // lie below GV_LO.
    if ((base & 0xFFFFu) > GV_LO) {
        if (threadIdx.x == 0) atomicExch(cfg.err, 1u);
        return;           // (uniform over the grid)
    }
    const uint32_t wb = base & 0xFFFF0000u;
    const uint32_t A_s0 = wb + L.s0, A_s1 = wb + L.s1, A_bars = wb + L.bars, A_red = wb + L.red;
    const uint32_t A_part = wb + L.part, A_recv = wb + L.recv, A_xs = wb + L.xs, A_cbraw = wb + L.cbraw;
    const uint32_t A_tbl = wb + GV_TBL_ADDR;
    uint64_t *full = reinterpret_cast<uint64_t *>(sptr(A_bars));
    uint64_t *empty = full + GV_MAX_STAGES;
    uint64_t *red_bar = empty + GV_MAX_STAGES;
    uint64_t *setup_bar = red_bar + GV_MAX_R;               // codebook and activations landed
    const uint32_t abort_a = A_bars + (uint32_t)((2 * GV_MAX_STAGES + GV_MAX_R + 1) * 8);
    const int S = L.stages, R = L.R;

    if (warp == 0) {   // one barrier of each kind per lane (S, R <= 32)
        if (lane < S) {
            mbar_init(&full[lane], 1);
            mbar_init(&empty[lane], NWK);
        }
        if (lane < R) mbar_init(&red_bar[lane], NWK);
        if (lane == 0) {
            mbar_init(setup_bar, 1);
            *reinterpret_cast<volatile uint32_t *>(sptr(abort_a)) = 0u;
        }
        mbar_fence_init();
    }
    __syncthreads();
    griddep_wait();   // inputs and outputs are the previous kernel's until here

    auto stage_addr = [&](int slot) -> uint32_t {
        return slot < L.n0 ? A_s0 + (uint32_t)(slot * cfg.SB) : A_s1 + (uint32_t)((slot - L.n0) * cfg.SB);
    };
    auto aborted = [&]() { return lds32_volatile(abort_a) != 0u; };
    auto fail = [&]() {
        *reinterpret_cast<volatile uint32_t *>(sptr(abort_a)) = 1u;
        atomicExch(cfg.err, 1u);
    };

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            // the codebook (raw, or the whole K = 4096 table) and this CTA's activations
            const uint32_t xbytes = XS ? (uint32_t)(SG * 128) : 0u;
            mbar_arrive_expect_tx(setup_bar, (uint32_t)cfg.CBB + (uint32_t)batch * xbytes);
            bulk_copy_g2s(BITS == 8 ? A_cbraw : A_tbl, W.codebook, (uint32_t)cfg.CBB, setup_bar);
            if constexpr (XS)
                for (int tok = 0; tok < batch; tok++)
                    bulk_copy_g2s(A_xs + (uint32_t)(tok * cfg.XR), x + (int64_t)tok * W.cols + gs0 * 64, xbytes, setup_bar);
            if constexpr (TMA) {
                tma_prefetch_map(&maps.code[0]);
                tma_prefetch_map(&maps.code[1]);
                tma_prefetch_map(&maps.scale[0]);
                tma_prefetch_map(&maps.scale[1]);
            }
        }
        // one stage per (row block, chunk)
        int slot = 0, k = 0;
        uint32_t ph = 0;
        bool stop = false;
        for (int kb = 0; kb < nb && !stop; kb++) {
            const int r0 = (b0 + kb) * GV_RB;
            const int nrows = min(GV_RB, W.rows - r0);
            int ua = ua0;
            for (int c = 0; c < nch; c++, k++) {
                const int ue = ua + cbw + (c < cxw ? 1 : 0);
                bool ok = true;
                if (lane == 0) ok = !aborted() && (k < S || mbar_wait_sleep(&empty[slot], ph ^ 1u));
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    if (lane == 0) fail();
                    stop = true;
                    break;
                }
                const uint32_t st = stage_addr(slot);
                if constexpr (TMA) {
                    if (lane == 0) {
                        const int mi = (ue - ua) > cfg.wl ? 1 : 0;
                        const uint32_t cbytes = (uint32_t)(GV_RB * 128 * (cfg.wl + mi) * cfg.useg);
                        const uint32_t sbytes = (uint32_t)(GV_RB * (mi ? cfg.sgw[1] : cfg.sgw[0]) * 2);
                        mbar_arrive_expect_tx(&full[slot], cbytes + sbytes);
                        tma_load_3d(st, mi ? &maps.code[1] : &maps.code[0], &full[slot], 0, r0, ua * cfg.useg);
                        tma_load_2d_u32(st + (uint32_t)cfg.SOFF, mi ? &maps.scale[1] : &maps.scale[0], &full[slot],
                                        ua * cfg.ug, r0);
                    }
                } else {
                    const int ga = ua * cfg.ug, ge = min(ue * cfg.ug, G);
                    const uint32_t lo = (uint32_t)(ga * GB) & ~15u, hi = ((uint32_t)(ge * GB) + 15u) & ~15u;
                    const uint32_t slo = (uint32_t)(2 * ga) & ~15u, shi = ((uint32_t)(2 * ge) + 15u) & ~15u;
                    if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)nrows * ((hi - lo) + (shi - slo)));
                    __syncwarp();
                    if (lane < nrows)
                        bulk_copy_g2s(st + (uint32_t)(lane * cfg.CS),
                                      W.codes + (int64_t)(r0 + lane) * W.code_row_bytes + lo, hi - lo, &full[slot]);
                    else if (lane >= GV_RB && lane - GV_RB < nrows)
                        bulk_copy_g2s(st + (uint32_t)(cfg.SOFF + (lane - GV_RB) * cfg.SS),
                                      reinterpret_cast<const uint8_t *>(W.scales + (int64_t)(r0 + lane - GV_RB) * W.scale_row_elems) + slo,
                                      shi - slo, &full[slot]);
                }
                if (++slot == S) { slot = 0; ph ^= 1u; }
                ua = ue;
            }
        }
        if (lane == 0) griddep_launch_dependents();   // every load is issued: the next kernel may be scheduled
    } else {
        // ---------------- consumers
        const int cw = warp - 1, ctid = threadIdx.x - 32, nct = 32 * NWK;
        const int g = lane >> 2, t = lane & 3;
        // the lane's rows of the block: rho and rho + 8
        const int rho = TMA ? (((g & 3) << 1) | (g >> 2)) : g;
        bool stop = false;
        {
            const bool ok = mbar_wait_sleep(setup_bar, 0);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) fail();
                stop = true;
            }
        }
        if constexpr (BITS == 8) {
            // K = 256: expand the raw codebook into the replicated table (one entry per
            // thread or two threads per entry, each writing its share of the 16 lines)
            if (!stop) {
                constexpr int PER = NWK * 32 / 256;
                const int e = ctid & 255, u0 = (ctid >> 8) * (16 / PER);
                uint4 v;
                if constexpr (D == 2) {
                    const uint32_t w = ldsn32(launder(A_cbraw) + (uint32_t)(e * 4));
                    v = make_uint4(w, w, w, w);
                } else if constexpr (D == 4) {
                    const uint2 w = ldsn64(launder(A_cbraw) + (uint32_t)(e * 8));
                    v = make_uint4(w.x, w.y, w.x, w.y);
                } else {
                    v = ldsn128(launder(A_cbraw) + (uint32_t)(e * 16));
                }
#pragma unroll
                for (int u = 0; u < 16 / PER; u++) sts128(A_tbl + (uint32_t)(e * 256 + (u0 + u) * 16), v);
            }
        }
        bar_sync_named(1, nct);

        // (laundered: the table and activation loads below must not move above the barrier)
        const uint32_t lb = launder(BITS == 8 ? (A_tbl | (uint32_t)((lane * 2 * D) & 255)) : A_tbl);
        const int tok0 = min(g, batch - 1), tok1 = min(g + 8, batch - 1);
        const uint32_t xs0 = launder(A_xs + (uint32_t)(tok0 * cfg.XR + 32 * t));
        const uint32_t xs1 = launder(A_xs + (uint32_t)(tok1 * cfg.XR + 32 * t));
        const __half *xg0 = x + (int64_t)tok0 * W.cols + gs0 * 64 + 16 * t;
        const __half *xg1 = x + (int64_t)tok1 * W.cols + gs0 * 64 + 16 * t;
        // TMA layout: lane-constant part of the code address (row rho, byte within the
        // 16-byte chunk) and its swizzle
        const uint32_t lane_row = (uint32_t)(rho * 128) +
                                  (D == 2 ? (uint32_t)((t & 1) << 3) : D == 4 ? (uint32_t)(t << 2) : (uint32_t)(t << 1));
        const int nout = batch * GV_RB;
        float *const part = reinterpret_cast<float *>(sptr(A_part));
        // sum block kb's partials over the warps, in warp order, and store (or keep) them
        auto reduce = [&](int kb) -> bool {
            const int rbk = kb % R;
            const uint32_t rphk = (uint32_t)((kb / R) & 1);
            const float *rbr = reinterpret_cast<const float *>(sptr(A_red + (uint32_t)(rbk * cfg.RBB)));
            const bool ok = !aborted() && mbar_wait_sleep(&red_bar[rbk], rphk);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) fail();
                return false;
            }
            for (int o = lane; o < nout; o += 32) {
                float v = 0.f;
#pragma unroll 4
                for (int w = 0; w < NWK; w++) v += rbr[w * nout + o];
                if (C == 1) {
                    const int tok = o / GV_RB, r = (b0 + kb) * GV_RB + o % GV_RB;
                    if (r < W.rows) store_out(y, (int64_t)tok * W.rows + r, v, yt);
                } else if (q == 0) {
                    part[kb * nout + o] = v;
                } else {   // straight into rank 0's receive buffer
                    st_cluster_f32(A_recv + (uint32_t)(((q - 1) * nb * nout + kb * nout + o) * 4), 0u, v);
                }
            }
            return true;
        };
        int slot = 0, rbi = 0;
        uint32_t ph = 0;
        for (int kb = 0; kb < nb && !stop; kb++) {
            float acc[NT][4];
#pragma unroll
            for (int n = 0; n < NT; n++) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
            float *const rb = reinterpret_cast<float *>(sptr(A_red + (uint32_t)(rbi * cfg.RBB)));
            int ua = 0;   // slice-relative
            for (int c = 0; c < nch; c++) {
                const int ue = ua + cbw + (c < cxw ? 1 : 0);
                const int ga = ua * cfg.ug, ge = min(ue * cfg.ug, SG);   // slice-relative groups
                const bool ok = !aborted() && mbar_wait_sleep(&full[slot], ph);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0) fail();
                    stop = true;
                    break;
                }
                const uint32_t st = launder(stage_addr(slot));   // stage loads stay below the wait
                uint32_t rowa, sca, scb;
                if constexpr (TMA) {
                    const int sgw = (ue - ua) > cfg.wl ? cfg.sgw[1] : cfg.sgw[0];
                    rowa = st + lane_row;
                    sca = st + (uint32_t)(cfg.SOFF + rho * sgw * 2);
                    scb = sca + (uint32_t)(8 * sgw * 2);
                } else {
                    const uint32_t off_c = (uint32_t)((gs0 + ga) * GB) & 15u, off_s = (uint32_t)(2 * (gs0 + ga)) & 15u;
                    rowa = st + (uint32_t)(rho * cfg.CS) + off_c;
                    sca = st + (uint32_t)(cfg.SOFF + rho * cfg.SS) + off_s;
                    scb = sca + (uint32_t)(8 * cfg.SS);
                }
                // one group's fresh partials and its two row scales
                auto group = [&](int i, float (&d)[NT][4], float &sa, float &sb) {
                    const uint32_t gr = (uint32_t)(i - ga);   // within the chunk
                    uint32_t xa[8], xb[8];
                    if constexpr (XS) ldsn_x16(xs0 + (uint32_t)i * 128u, xa);
                    else ldg_x16(xg0 + i * 64, xa);
                    if constexpr (NT == 2) {
                        if constexpr (XS) ldsn_x16(xs1 + (uint32_t)i * 128u, xb);
                        else ldg_x16(xg1 + i * 64, xb);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; j++) xb[j] = xa[j];
                    }
                    uint32_t ca, cb;
                    if constexpr (TMA) {
                        // segment gr / GPS holds [16 rows][128 bytes], 16-byte chunks swizzled
                        // by the row's low three bits (rho < 8 for both rows)
                        const uint32_t c16 = D == 2 ? (((gr & 3u) << 1) | (uint32_t)(t >> 1))
                                           : D == 4 ? (gr & 7u)
                                                    : ((gr & 15u) >> 1);
                        ca = rowa + (gr / GPS) * 2048u + ((c16 ^ (uint32_t)rho) << 4) + (D == 8 ? ((gr & 1u) << 3) : 0u);
                        cb = ca + 1024u;
                    } else if constexpr (BITS == 8) {
                        ca = rowa + gr * GB + (uint32_t)(t * (16 / D));
                        cb = ca + (uint32_t)(8 * cfg.CS);
                    } else {
                        ca = rowa + gr * GB;
                        cb = ca + (uint32_t)(8 * cfg.CS);
                    }
                    gv_group<D, BITS, NT>(ca, cb, t, lb, xa, xb, d);
                    sa = __half2float(__ushort_as_half((unsigned short)ldsn16(sca + 2u * gr)));
                    sb = __half2float(__ushort_as_half((unsigned short)ldsn16(scb + 2u * gr)));
                };
                auto accumulate = [&](const float (&d)[NT][4], float sa, float sb) {
#pragma unroll
                    for (int n = 0; n < NT; n++) {
                        acc[n][0] = fmaf(sa, d[n][0], acc[n][0]);
                        acc[n][1] = fmaf(sa, d[n][1], acc[n][1]);
                        acc[n][2] = fmaf(sb, d[n][2], acc[n][2]);
                        acc[n][3] = fmaf(sb, d[n][3], acc[n][3]);
                    }
                };
                // this warp's groups of the chunk: slice index i with (i + kb) mod NW = cw,
                // two at a time (independent chains), in increasing order
                int i = ga + ((cw - kb - ga) & (NWK - 1));
                for (; i + NWK < ge; i += 2 * NWK) {
                    float d0[NT][4], d1[NT][4], sa0, sb0, sa1, sb1;
                    group(i, d0, sa0, sb0);
                    group(i + NWK, d1, sa1, sb1);
                    accumulate(d0, sa0, sb0);
                    accumulate(d1, sa1, sb1);
                }
                if (i < ge) {
                    float d0[NT][4], sa0, sb0;
                    group(i, d0, sa0, sb0);
                    accumulate(d0, sa0, sb0);
                }
                if (c == nch - 1) {
                    // post this warp's totals [cw][token][row] (tokens < batch) before the
                    // block's last stage is released
                    float *p = rb + cw * nout;
#pragma unroll
                    for (int n = 0; n < NT; n++) {
                        const int tk = 8 * n + 2 * t;
                        if (tk < batch) { p[tk * GV_RB + rho] = acc[n][0]; p[tk * GV_RB + rho + 8] = acc[n][2]; }
                        if (tk + 1 < batch) { p[(tk + 1) * GV_RB + rho] = acc[n][1]; p[(tk + 1) * GV_RB + rho + 8] = acc[n][3]; }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&red_bar[rbi]);
                }
                // every read of the stage is done before it is released
#pragma unroll
                for (int n = 0; n < NT; n++) {
                    consume(acc[n][0]); consume(acc[n][1]); consume(acc[n][2]); consume(acc[n][3]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
                if (++slot == S) { slot = 0; ph ^= 1u; }
                ua = ue;
            }
            if (stop) break;
            // reduce block kb - lag (posted long enough ago that the wait is short)
            if (kb >= cfg.lag && ((kb - cfg.lag) & (NWK - 1)) == cw && !reduce(kb - cfg.lag)) {
                stop = true;
                break;
            }
            if (++rbi == R) rbi = 0;
        }
        // the last `lag` blocks
        for (int kb = max(0, nb - cfg.lag); kb < nb && !stop; kb++)
            if ((kb & (NWK - 1)) == cw && !reduce(kb)) stop = true;
    }

    if (C > 1) {
        // the other ranks' results are in rank 0's receive buffer (the barrier orders the
        // remote stores before rank 0's reads); rank 0 adds them in rank order
        cluster_barrier();
        if (q == 0 && !aborted()) {
            const int nout = batch * GV_RB, total = nb * nout;
            const float *part = reinterpret_cast<const float *>(sptr(A_part));
            const float *recv = reinterpret_cast<const float *>(sptr(A_recv));
            for (int o = (int)threadIdx.x; o < total; o += (int)blockDim.x) {
                float v = part[o];
                for (int p = 1; p < C; p++) v += recv[(p - 1) * total + o];
                const int kb = o / nout, rem = o - kb * nout;
                const int tok = rem / GV_RB, r = (b0 + kb) * GV_RB + rem % GV_RB;
                if (r < W.rows) store_out(y, (int64_t)tok * W.rows + r, v, yt);
            }
        }
    }
}

// ------------------------------------------------------------------ host

unsigned int *device_error_word();
void *encode_tiled_fn();

namespace {

typedef CUresult (*EncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                             const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int gv_device() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}

int gv_num_sms(int dev) {
    static int cache[64] = {0};
    if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

void gv_cluster_attr(cudaLaunchConfig_t &lc, cudaLaunchAttribute *at, int C) {
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
}

// Programmatic dependent launch (see griddep_wait): appended as attribute n of at.
void gv_pdl_attr(cudaLaunchConfig_t &lc, cudaLaunchAttribute *at, int n) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = (unsigned)(n + 1);
}

// Tensor maps of one matrix, cached: a map holds only the address, shape, strides and
// box, so an entry stays valid for any matrix with the same key.
struct GvMapKey {
    const void *codes, *scales;
    int rows, G, wl, ug, useg, sgw0, sgw1;
    int64_t crb, srow;
    bool operator==(const GvMapKey &o) const {
        return codes == o.codes && scales == o.scales && rows == o.rows && G == o.G && wl == o.wl && ug == o.ug &&
               useg == o.useg && sgw0 == o.sgw0 && sgw1 == o.sgw1 && crb == o.crb && srow == o.srow;
    }
};

bool gv_encode(const GvMapKey &k, GvMaps &m) {
    EncodeFn enc = reinterpret_cast<EncodeFn>(encode_tiled_fn());
    if (!enc) return false;
    for (int i = 0; i < 2; i++) {
        const int w = k.wl + i;
        if (w < 1) {   // unused variant: keep a valid map of the other width
            continue;
        }
        cuuint64_t cdims[3] = {128, (cuuint64_t)k.rows, (cuuint64_t)(k.crb / 128)};
        cuuint64_t cstr[2] = {(cuuint64_t)k.crb, 128};
        cuuint32_t cbox[3] = {128, (cuuint32_t)GV_RB, (cuuint32_t)(w * k.useg)};
        cuuint32_t e3[3] = {1, 1, 1};
        if (enc(&m.code[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(k.codes), cdims, cstr, cbox, e3,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
        cuuint64_t sdims[2] = {(cuuint64_t)k.G, (cuuint64_t)k.rows};
        cuuint64_t sstr[1] = {(cuuint64_t)k.srow};
        cuuint32_t sbox[2] = {(cuuint32_t)(i == 0 ? k.sgw0 : k.sgw1), (cuuint32_t)GV_RB};
        cuuint32_t e2[2] = {1, 1};
        if (enc(&m.scale[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(k.scales), sdims, sstr, sbox, e2,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    if (k.wl < 1) {
        m.code[0] = m.code[1];
        m.scale[0] = m.scale[1];
    }
    return true;
}

bool gv_maps(const GvMapKey &k, GvMaps &out) {
    constexpr int N = 16;
    static GvMapKey keys[N];
    static GvMaps vals[N];
    static bool used[N] = {false};
    static int next = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < N; i++)
        if (used[i] && keys[i] == k) {
            out = vals[i];
            return true;
        }
    if (!gv_encode(k, out)) return false;
    keys[next] = k;
    vals[next] = out;
    used[next] = true;
    next = (next + 1) % N;
    return true;
}

template <int D, int BITS, int NT, bool XS, bool TMA>
vq_status gv_launch5(const Mat &W, const void *x, int batch, void *y, int yt, GvCfg c, int CHU, cudaStream_t s)
{
    auto k = gemv_mma_kernel<D, BITS, NT, XS, TMA>;
    const int dev = gv_device();
    // per-instantiation, per-device one-time setup: the shared-memory opt-in and the
    // number of clusters of 2, 4 and 8 CTAs that fit at once
    static uint64_t attr_done = 0;
    static int ncl_cache[64][4];
    const int nsm = gv_num_sms(dev);
    if (dev < 0 || dev >= 64) return VQ_ERR_UNSUPPORTED;
    if (!(attr_done >> dev & 1)) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, GV_DYN_SMEM) != cudaSuccess)
            return VQ_ERR_CUDA;
        for (int li = 0; li < 4; li++) {
            const int C = 1 << li;
            int n = nsm;
            if (C > 1) {
                cudaLaunchConfig_t lc{};
                cudaLaunchAttribute at[1];
                lc.gridDim = dim3((unsigned)(nsm / C * C));
                lc.blockDim = dim3(gv_threads<NT>());
                lc.dynamicSmemBytes = GV_DYN_SMEM;
                gv_cluster_attr(lc, at, C);
                n = 0;
                if (cudaOccupancyMaxActiveClusters(&n, k, &lc) != cudaSuccess) {
                    cudaGetLastError();
                    n = 0;
                }
            }
            ncl_cache[dev][li] = n;
        }
        attr_done |= uint64_t(1) << dev;
    }
    const int G = W.cols / 64, NB = (W.rows + GV_RB - 1) / GV_RB;
    // cluster size: candidates in order of their largest per-CTA share (row blocks x
    // units); the first whose shared-memory layout fits is launched
    int cand[4], ncand = 0;
    long long cost[4];
    for (int li = 0; li < 4; li++) {
        const int C = 1 << li;
        if (C > c.U) break;
        const int ncl = std::min(ncl_cache[dev][li], NB);
        if (ncl <= 0) continue;
        const int bpc = (NB + ncl - 1) / ncl;
        if (C > 1 && (long long)bpc * batch * GV_RB * 4 * C > 32768) continue;   // per-block results must fit
        cost[ncand] = (long long)bpc * (((c.U + C - 1) / C) * c.ug + 2);
        cand[ncand++] = li;
    }
    for (int i = 1; i < ncand; i++)   // stable insertion sort by cost
        for (int j = i; j > 0 && cost[j] < cost[j - 1]; j--) {
            std::swap(cost[j], cost[j - 1]);
            std::swap(cand[j], cand[j - 1]);
        }
    bool fits = false;
    for (int ic = 0; ic < ncand && !fits; ic++) {
        const int li = cand[ic];
        c.C = 1 << li;
        c.ncl = std::min(ncl_cache[dev][li], NB);
        const int bpc = (NB + c.ncl - 1) / c.ncl;
        const int su_min = c.U / c.C, su_max = (c.U + c.C - 1) / c.C;
        c.nch = std::max(1, std::min(su_min, (su_max + CHU - 1) / CHU));
        c.wl = su_min / c.nch;
        const int wmax = c.wl + 1;
        if (TMA) {
            for (int i = 0; i < 2; i++) {
                int w = (c.wl + i) * c.ug;
                if (w % 16 == 0) w += 8;   // scale rows of the box on distinct banks
                c.sgw[i] = w;
            }
            c.SOFF = GV_RB * 128 * wmax * c.useg;
            c.SB = (c.SOFF + GV_RB * c.sgw[1] * 2 + 1023) / 1024 * 1024;
        } else {
            const int GB = (64 / D) * BITS / 8;
            const int wg = wmax * c.ug;                         // most groups in a chunk
            const int pad = D == 2 ? 32 : 16;                   // row slots on distinct banks
            c.CS = (wg * GB + 32 + 127) / 128 * 128 + pad;
            c.SS = (2 * wg + 32 + 15) / 16 * 16;
            c.SOFF = GV_RB * c.CS;
            c.SB = (GV_RB * (c.CS + c.SS) + 1023) / 1024 * 1024;
        }
        const int sg_max = std::min(su_max * c.ug, G);
        c.XR = XS ? sg_max * 128 + 16 : 0;
        c.XB = XS ? batch * c.XR : 0;
        c.PB = c.C > 1 ? bpc * batch * GV_RB * 4 : 0;
        c.RBB = gv_nw<NT>() * batch * GV_RB * 4;
        c.lag = NT == 1 ? 2 : 0;   // (batches 9..16: buffers too large for a longer ring)
        c.CBB = (1 << BITS) * D * 2;
        c.L = gv_layout(c, BITS == 8);
        fits = c.L.ok && c.L.stages >= 3;
    }
    if (!fits) return VQ_ERR_UNSUPPORTED;

    GvMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (TMA) {
        GvMapKey key{W.codes, W.scales, W.rows, G, c.wl, c.ug, c.useg, c.sgw[0], c.sgw[1], W.code_row_bytes,
                     W.scale_row_elems * 2};
        if (!gv_maps(key, maps)) return VQ_ERR_UNSUPPORTED;
    }
    cudaLaunchConfig_t lc{};
    cudaLaunchAttribute at[2];
    lc.gridDim = dim3((unsigned)(c.ncl * c.C));
    lc.blockDim = dim3(gv_threads<NT>());
    lc.dynamicSmemBytes = GV_DYN_SMEM;
    lc.stream = s;
    int na = 0;
    if (c.C > 1) {
        gv_cluster_attr(lc, at, c.C);
        na = 1;
    }
    gv_pdl_attr(lc, at, na);
    if (cudaLaunchKernelEx(&lc, k, W, (const __half *)x, batch, y, yt, c, maps) != cudaSuccess) return VQ_ERR_CUDA;
    VQ_CHECK_LAUNCH();
    return VQ_OK;
}

template <int D, int BITS, bool TMA>
vq_status gv_launch(const Mat &W, const void *x, int batch, void *y, int yt, const GvCfg &c, int CHU, cudaStream_t s)
{
    const int G = W.cols / 64;
    // activations in shared memory when they take at most 48 KB at full width (a CTA
    // stages only its column slice)
    const bool xs = (size_t)batch * ((size_t)G * 128 + 16) <= 49152;
    vq_status st = VQ_ERR_UNSUPPORTED;
    if (batch <= 8) {
        if (xs) st = gv_launch5<D, BITS, 1, true, TMA>(W, x, batch, y, yt, c, CHU, s);
        if (st == VQ_ERR_UNSUPPORTED) st = gv_launch5<D, BITS, 1, false, TMA>(W, x, batch, y, yt, c, CHU, s);
        return st;
    }
    if (xs) st = gv_launch5<D, BITS, 2, true, TMA>(W, x, batch, y, yt, c, CHU, s);
    if (st == VQ_ERR_UNSUPPORTED) st = gv_launch5<D, BITS, 2, false, TMA>(W, x, batch, y, yt, c, CHU, s);
    return st;
}

template <int D>
vq_status gv_launch_8bit(const Mat &W, const void *x, int batch, void *y, int yt, GvCfg c, cudaStream_t s)
{
    constexpr int GB = 64 / D;   // 8-bit codes: bytes per scale group
    if (W.code_row_bytes % 128 == 0 && encode_tiled_fn()) {
        c.ug = GB * 8 >= 128 ? 8 : 128 / GB;   // d = 2, 4: 8 groups; d = 8: 16 groups (128 bytes)
        c.useg = c.ug * GB / 128;
        c.U = (W.cols / 64 + c.ug - 1) / c.ug;
        const int chu = std::min(std::max(1, 2560 / (c.ug * GB)), (256 - 8) / c.ug);
        const vq_status st = gv_launch<D, 8, true>(W, x, batch, y, yt, c, chu, s);
        if (st != VQ_ERR_UNSUPPORTED) return st;
    }
    c.ug = 1;
    c.useg = 0;
    c.U = W.cols / 64;
    return gv_launch<D, 8, false>(W, x, batch, y, yt, c, std::max(8, 1024 / GB), s);
}

template <int D>
vq_status gv_launch_12bit(const Mat &W, const void *x, int batch, void *y, int yt, GvCfg c, cudaStream_t s)
{
    constexpr int GB = (64 / D) * 12 / 8;
    c.ug = 1;
    c.useg = 0;
    c.U = W.cols / 64;
    return gv_launch<D, 12, false>(W, x, batch, y, yt, c, std::max(8, 1024 / GB), s);
}

}  // namespace

// fp16-activation GEMV (batch 1..16) on the tensor-core path.  VQ_ERR_UNSUPPORTED
// (nothing launched) when it does not apply: other activation types, activations or
// scales not 16-byte aligned, or scale rows that are not whole 16-byte units.
vq_status launch_gemv_mma(const Mat &W, const void *x, vq_dtype xt, int batch, void *y, vq_dtype yt, cudaStream_t s)
{
    if (xt != VQ_F16 || batch < 1 || batch > 16) return VQ_ERR_UNSUPPORTED;
    const int64_t srow = W.scale_row_elems * 2;
    if (srow % 16 || ((uintptr_t)W.scales % 16) || ((uintptr_t)x % 16)) return VQ_ERR_UNSUPPORTED;
    GvCfg c{};
    c.err = device_error_word();
    if (!c.err) return VQ_ERR_CUDA;
    switch (geom_of(W.d, W.bits)) {
    case G_D2_B8: return gv_launch_8bit<2>(W, x, batch, y, (int)yt, c, s);
    case G_D4_B8: return gv_launch_8bit<4>(W, x, batch, y, (int)yt, c, s);
    case G_D8_B8: return gv_launch_8bit<8>(W, x, batch, y, (int)yt, c, s);
    case G_D2_B12: return gv_launch_12bit<2>(W, x, batch, y, (int)yt, c, s);
    case G_D4_B12: return gv_launch_12bit<4>(W, x, batch, y, (int)yt, c, s);
    case G_D8_B12: return gv_launch_12bit<8>(W, x, batch, y, (int)yt, c, s);
    default: return VQ_ERR_UNSUPPORTED;
    }
}

}  // namespace vq

/*
 * vq.h — C ABI of the B200 (sm_100a) vector-quantized dequantize-and-multiply library.
 *
 * Weight format (the pages' format, restated):
 *   A weight matrix W has `rows` output features and `cols` input features (y = x W^T).
 *   Each run of d consecutive weights of a row is stored as one code (an index) into a
 *   per-tensor codebook of K = 2^bits fp16 entries of length d, and each (row, 64
 *   consecutive weights) group has one fp16 scale, so
 *       W[r][c] = scale[r][c / 64] * codebook[code(r, c / d)][c mod d].
 *   Sources: "Data-Free Vector Quantization Beats Affine Quantization at Matched Bytes
 *   Below 5 Bits", Abstract, §1 (Notation) and §2.2 (The fit); model card
 *   "Qwen3.5-397B-A17B-VQ-2.4bpw", Methodology.
 *
 * Packed code layout:
 *   Codes are packed at their true width, row-local, in blocks of 32 codes (model card
 *   "Qwen3.5-397B-A17B-VQ-2.4bpw", Methodology: Sub-byte bit-packing; paper §2.3).
 *   Each row is a little-endian, LSB-first bitstream: bit b of code i is stream bit
 *   bits*i + b, stream bit p is bit (p mod 8) of byte p/8.  8-bit codes are therefore
 *   plain uint8 arrays (same card, Runtime update 2026-08-20: uint8 codes already are
 *   the packed-8 layout); 12-bit codes take 48 bytes per 32 codes and straddle words.
 *   A packed row occupies vq_code_row_bytes(ncodes, bits) = ceil(ncodes/32)*4*bits
 *   bytes; padding codes are 0.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless stated.
 *     The library allocates no memory, never synchronises (except
 *     vq_read_device_status), and launches on `stream` only.
 *   - All arguments are validated on the host before anything is launched; on error
 *     nothing is launched and no output is touched.
 *   - Inputs are never modified.  Outputs are deterministic for fixed inputs on a given
 *     GPU: no floating-point atomics are used anywhere.
 *   - A CUDA launch failure is reported as VQ_ERR_CUDA.  Kernels never trap; bad data
 *     found on the device (an expert id out of range) is skipped and recorded in the
 *     workspace status word, read back with vq_read_device_status.
 *   - Rows of codes must start on 16-byte boundaries (codes base and code_row_bytes
 *     multiples of 16); activations and outputs must be 16-byte aligned with rows of a
 *     whole number of 16-byte units where stated.
 */
#ifndef VQ_B200_H
#define VQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so callers need no CUDA header. */
typedef struct CUstream_st *vq_stream_t;

typedef enum {
    VQ_OK = 0,
    VQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size or stride */
    VQ_ERR_UNSUPPORTED = 2,  /* geometry or dtype outside what is built */
    VQ_ERR_MISALIGNED = 3,   /* pointer or stride breaks an alignment rule */
    VQ_ERR_WORKSPACE = 4,    /* workspace null or smaller than the size query said */
    VQ_ERR_CUDA = 5,         /* a CUDA call or launch failed */
    VQ_ERR_DEVICE_FLAG = 6,  /* the device recorded bad input (expert id out of range) */
    VQ_ERR_TIMEOUT = 7       /* a bounded device-side wait ran out */
} vq_status;

typedef enum { VQ_F16 = 0, VQ_BF16 = 1, VQ_F32 = 2 } vq_dtype;

/* One VQ weight tensor, or a stack of `num_experts` tensors of the same shape and
 * geometry (one projection of a routed MoE layer). */
typedef struct {
    int32_t rows;                   /* output features N >= 1 */
    int32_t cols;                   /* input features Kin, a positive multiple of 64 */
    int32_t d;                      /* subvector length: 2, 4 or 8 */
    int32_t bits;                   /* code width: 8 (K = 256) or 12 (K = 4096) */
    const void *codebook;           /* fp16 [K][d] (per codebook) */
    const void *codes;              /* packed codes [rows][code_row_bytes] (per expert) */
    const void *scales;             /* fp16 [rows][scale_row_elems] (per expert) */
    int64_t code_row_bytes;         /* >= vq_code_row_bytes(cols/d, bits), multiple of 16 */
    int64_t scale_row_elems;        /* >= cols / 64 */
    int64_t expert_code_stride;     /* bytes between experts' codes (multiple of 16) */
    int64_t expert_scale_stride;    /* fp16 elements between experts' scales */
    int64_t expert_codebook_stride; /* fp16 elements between experts' codebooks;
                                       0 = one codebook shared by every expert (the
                                       pages' per-tensor codebook of a stacked tensor,
                                       model card "Qwen3.6-35B-A3B-MLX-VQ-2.4bpw", Recipe) */
    int32_t num_experts;            /* 1 for a dense tensor */
    int32_t reserved;               /* must be 0 */
} vq_matrix;

/* Bytes of one packed row of `ncodes` codes of width `bits`: ceil(ncodes/32)*4*bits.
 * Returns -1 for ncodes < 0 or bits outside 1..16. */
int64_t vq_code_row_bytes(int64_t ncodes, int32_t bits);

/* Pack codes [rows][ncodes] (uint16, each < 2^bits; bits 1..16) into rows of
 * code_row_bytes bytes at `packed` (code_row_bytes >= vq_code_row_bytes(ncodes, bits)).
 * Padding codes and padding bytes are written as 0.  Codes >= 2^bits are masked to
 * their low `bits` bits.  Definition: paper §2.3 (Packing); card
 * "Qwen3.5-397B-A17B-VQ-2.4bpw", Methodology. */
vq_status vq_pack(const uint16_t *codes, int32_t rows, int32_t ncodes, int32_t bits,
                  void *packed, int64_t code_row_bytes, vq_stream_t stream);

/* Inverse of vq_pack: codes [rows][ncodes] from packed rows.  Bit-exact. */
vq_status vq_unpack(const void *packed, int32_t rows, int32_t ncodes, int32_t bits,
                    int64_t code_row_bytes, uint16_t *codes, vq_stream_t stream);

/* Dequantize expert `expert` of W to a dense [rows][cols] matrix of type `out`
 * (VQ_F32 is exact: the product of two fp16 values is exact in fp32; 16-bit types are
 * rounded to nearest even once).  A test and inspection aid: the fast paths below
 * never build W.  Definition: paper §2.2; card "Qwen3.5-397B-A17B-VQ-2.4bpw". */
vq_status vq_dequant(const vq_matrix *W, int32_t expert, void *w_out, vq_dtype out,
                     vq_stream_t stream);

/* Decode GEMV: y[m][r] = sum_c W[r][c] * x[m][c] for m < batch (1..16), fp32
 * accumulation, expert 0 of W.  x is [batch][cols] of type xt (row stride cols,
 * 16-byte aligned base); y is [batch][rows] of type yt.  This is the pages' fused
 * decode-and-matmul (paper §3.4, Runtime performance and kernel support).
 * Needs no workspace: ws may be NULL with ws_bytes 0. */
vq_status vq_gemv(const vq_matrix *W, const void *x, vq_dtype xt, int32_t batch,
                  void *y, vq_dtype yt, void *ws, size_t ws_bytes, vq_stream_t stream);

/* Prefill GEMM: the same contraction for M >= 1 tokens on the tcgen05 tensor cores.
 * Codes and scales are expanded into fp16 weight tiles held in tensor memory and
 * multiplied with fp32 accumulation in tensor memory; the dense weights are never
 * written to device memory.  x is [M][cols] (fp16 or bf16, 16-byte aligned,
 * cols*2 bytes per row); bf16 activations are first converted to fp16 in the
 * workspace (exact for |x| >= 2^-14).  y is [M][rows] of type yt.
 * Prefill path of the pages: paper §2.5 and §3.4 (prefill-shaped code path). */
vq_status vq_gemm(const vq_matrix *W, const void *x, vq_dtype xt, int32_t M, void *y,
                  vq_dtype yt, void *ws, size_t ws_bytes, vq_stream_t stream);

/* vq_gemm with options.  VQ_GEMM_BF16_TILES: expand into bf16 tiles and multiply bf16
 * activations directly (no conversion, no workspace; weight rounding to bf16 gives
 * about 1.5e-3 normwise error, against about 2e-4 for fp16 tiles). */
#define VQ_GEMM_BF16_TILES 1u
vq_status vq_gemm_ex(const vq_matrix *W, const void *x, vq_dtype xt, int32_t M, void *y,
                     vq_dtype yt, void *ws, size_t ws_bytes, uint32_t flags,
                     vq_stream_t stream);

/* Workspace bytes vq_gemm / vq_gemm_ex need for these arguments (0 when none). */
vq_status vq_gemm_workspace_size(const vq_matrix *W, vq_dtype xt, int32_t M,
                                 uint32_t flags, size_t *bytes);

/* Workspace bytes vq_moe_grouped needs for T tokens routed top-k among E experts. */
vq_status vq_moe_workspace_size(int32_t T, int32_t topk, int32_t E, int32_t hidden,
                                int32_t inter, size_t *bytes);

/* Routed MoE layer over T tokens:
 *   for each token t and slot j < topk: e = expert_ids[t][j], weight = expert_w[t][j],
 *   h = silu(Gate_e x_t) * (Up_e x_t), o = Down_e h, y_t = sum_j weight * o (slot order).
 * gate and up are [inter][hidden] stacks, down is [hidden][inter], all with the same
 * num_experts E; each may use its own geometry (mixed tiers, card
 * "Qwen3.6-35B-A3B-MLX-VQ-2.4bpw", Recipe).  x is [T][hidden] fp16 or bf16, y is
 * [T][hidden] of type yt.  Pairs are bucketed by expert on the device and each stage
 * runs as one grouped launch over all routed experts.  A pair with an id outside
 * [0, E) contributes nothing and sets the status word (vq_read_device_status).
 * SwiGLU (silu(gate) * up) is this library's reading of the gate/up/down trio of
 * paper §2 (Method).  ws must hold vq_moe_workspace_size bytes, 256-byte aligned. */
vq_status vq_moe_grouped(const vq_matrix *gate, const vq_matrix *up, const vq_matrix *down,
                         const void *x, vq_dtype xt, int32_t T, const int32_t *expert_ids,
                         const float *expert_w, int32_t topk, void *y, vq_dtype yt,
                         void *ws, size_t ws_bytes, vq_stream_t stream);

/* vq_moe_grouped for callers that cannot allocate device memory (for example code that
 * runs where cudaMalloc is not allowed, or a caller without its own device allocator):
 * same arguments and results as vq_moe_grouped, minus the workspace.  There is no
 * counterpart on the pages; this is a convenience of this library.
 *   - The scratch is a fixed 16 MiB array inside the library's device image; every GPU
 *     that loads the library holds it until the process exits.  Calls whose
 *     vq_moe_workspace_size exceeds 16 MiB (about T * topk * (10 * inter + 6 * hidden)
 *     bytes plus small tables: decode-sized batches) return VQ_ERR_WORKSPACE and launch
 *     nothing.
 *   - The first call on each device looks up the array's device address (with that
 *     device current) and caches it; make that first call before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents (every call
 *     rewrites all it reads).  Calls that overlap on the GPU race on it: serialise them.
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - Bad expert ids are skipped as in vq_moe_grouped; their count stays in the shared
 *     scratch and is not reported by vq_read_device_status. */
vq_status vq_moe_grouped_noalloc(const vq_matrix *gate, const vq_matrix *up, const vq_matrix *down,
                                 const void *x, vq_dtype xt, int32_t T, const int32_t *expert_ids,
                                 const float *expert_w, int32_t topk, void *y, vq_dtype yt,
                                 vq_stream_t stream);

/* Synchronise `stream`, then report what the device recorded: VQ_ERR_TIMEOUT if any
 * kernel of this library gave up a bounded wait since the library was loaded (a bug
 * signal; the kernel ended instead of hanging), else, when ws is not NULL, the status
 * word a vq_moe_grouped call left in ws: VQ_ERR_DEVICE_FLAG if it skipped expert ids
 * outside [0, E); VQ_OK otherwise.  VQ_ERR_CUDA if the synchronisation failed. */
vq_status vq_read_device_status(const void *ws, vq_stream_t stream);

/* Static description of a status code (never NULL). */
const char *vq_status_string(vq_status s);

/* Library version as "major.minor.patch". */
const char *vq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VQ_B200_H */

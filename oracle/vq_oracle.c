/*
 * vq_oracle.c — plain, slow CPU oracle for the VQ dequantize-and-multiply path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  It shares no code, header, table or
 * helper with the CUDA library; it is the definition the CUDA path is checked
 * against, written out as directly as possible.
 *
 * What it computes, and where the definition comes from:
 *
 *   Format.  A weight matrix W is [rows][cols] (rows = output features, cols = input
 *   features).  Each run of d consecutive weights of a row (a "subvector") is stored
 *   as one index (a "code") into a per-tensor codebook of K = 2^bits fp16 entries of
 *   length d; each (row, 64 consecutive weights) group has one fp16 scale.
 *     - "Data-Free Vector Quantization Beats Affine Quantization at Matched Bytes
 *        Below 5 Bits", Abstract and §1 (Notation: geometry dN/KM, log2(K)/d bits).
 *     - model card "Qwen3.5-397B-A17B-VQ-2.4bpw", Methodology (per-tensor fp16
 *       codebook, one fp16 scale per (row, 64 weights)).
 *     - same paper §2.2 (The fit: each group of 64 scaled by its max-abs value, so
 *       the stored weight is scale x codebook entry).
 *
 *   Packing.  Codes are packed at their true bit width into uint32 words, row-local,
 *   in blocks of 32 codes; byte-wide codes are stored as plain bytes.
 *     - model card "Qwen3.5-397B-A17B-VQ-2.4bpw", Methodology (Sub-byte bit-packing)
 *       and Runtime update (2026-08-20) (uint8 codes are already the packed-8 layout).
 *     - paper §2.3 (Packing).
 *   Reading taken here: the row is one little-endian bitstream, LSB first: bit b of
 *   code i is stream bit bits*i + b, and stream bit p is bit (p mod 8) of byte p/8.
 *   This is the only order under which uint8 codes already are the packed-8 layout.
 *   Codes straddle word boundaries (12-bit codes: 8 codes per 3 words).  A row holds
 *   ceil(ncodes/32) blocks of 32 codes = ceil(ncodes/32)*4*bits bytes; padding codes
 *   are 0.
 *
 *   Dequantize.  W[r][c] = f32(scale[r][c/64]) * f32(codebook[code(r, c/d)][c mod d])
 *   computed in fp32 (the product of two fp16 values is exact in fp32).
 *
 *   Multiply.  y[m][r] = sum over c (ascending) of f64(W[r][c]) * f64(x[m][c]),
 *   accumulated in fp64.  This is the "dequantize, then matmul" reference path that
 *   the 35B card ("Qwen3.6-35B-A3B-MLX-VQ-2.4bpw", Run: pure-MLX reference path)
 *   describes as bit-identical to its fused kernels.
 *
 *   MoE layer.  For token t and routed slot j (expert e = ids[t][j], weight w[t][j]):
 *   g = Gate_e x_t, u = Up_e x_t, h = silu(g) * u = g / (1 + exp(-g)) * u,
 *   o = Down_e h, y_t = sum over j = 0..k-1 (in slot order) of w[t][j] * o.
 *     - paper §2 (Method: routed experts hold gate, up and down projections).
 *     - model card "Qwen3.6-35B-A3B-MLX-VQ-2.4bpw" (top-8 routed MoE).
 *   Reading taken here: the activation is SwiGLU (silu(gate) * up); the pages name
 *   the gate/up/down trio but print no formula.  All of g, u, h, o are fp64.
 *   A pair whose expert id lies outside [0, E) contributes nothing and is counted.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ number formats */

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.  Written
 * from the format's definition, value by value; subnormals are kept exactly. */
float orc_half_to_float(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);                 /* 0.frac x 2^-14 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + frac), expo - 25);  /* 1.frac x 2^(expo-15) */
    return (float)(sign ? -v : v);
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
float orc_bf16_to_float(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int expo = (b >> 7) & 0xff;
    int frac = b & 0x7f;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -133);                /* 0.frac x 2^-126 */
    else if (expo == 255)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + frac), expo - 134);  /* 1.frac x 2^(expo-127) */
    return (float)(sign ? -v : v);
}

void orc_half_to_float_n(const uint16_t *in, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_half_to_float(in[i]);
}

void orc_bf16_to_float_n(const uint16_t *in, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_bf16_to_float(in[i]);
}

/* Activation element c of row m; xt: 0 = fp16, 1 = bf16, 2 = fp32. */
static double orc_x_at(const void *x, int xt, int64_t idx)
{
    if (xt == 0) return (double)orc_half_to_float(((const uint16_t *)x)[idx]);
    if (xt == 1) return (double)orc_bf16_to_float(((const uint16_t *)x)[idx]);
    return (double)((const float *)x)[idx];
}

/* ------------------------------------------------------------------ packing */

/* Bytes of one packed row: ceil(ncodes / 32) blocks of 32 codes, each block
 * 32 * bits bits = 4 * bits bytes. */
int64_t orc_code_row_bytes(int64_t ncodes, int32_t bits)
{
    return ((ncodes + 31) / 32) * 4 * (int64_t)bits;
}

/* Code i of a packed row, read one bit at a time from the LSB-first bitstream. */
uint32_t orc_code_at(const uint8_t *row, int64_t i, int32_t bits)
{
    uint32_t v = 0;
    for (int b = 0; b < bits; b++) {
        int64_t p = (int64_t)bits * i + b;
        uint32_t bit = (row[p / 8] >> (p % 8)) & 1u;
        v |= bit << b;
    }
    return v;
}

/* Pack codes [rows][ncodes] (each < 2^bits) into rows of row_bytes bytes. */
void orc_pack(const uint16_t *codes, int64_t rows, int64_t ncodes, int32_t bits,
              uint8_t *packed, int64_t row_bytes)
{
    for (int64_t r = 0; r < rows; r++) {
        uint8_t *row = packed + r * row_bytes;
        memset(row, 0, (size_t)row_bytes);
        for (int64_t i = 0; i < ncodes; i++) {
            uint32_t code = codes[r * ncodes + i];
            for (int b = 0; b < bits; b++) {
                int64_t p = (int64_t)bits * i + b;
                if ((code >> b) & 1u) row[p / 8] |= (uint8_t)(1u << (p % 8));
            }
        }
    }
}

void orc_unpack(const uint8_t *packed, int64_t rows, int64_t ncodes, int32_t bits,
                int64_t row_bytes, uint16_t *codes)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t i = 0; i < ncodes; i++)
            codes[r * ncodes + i] = (uint16_t)orc_code_at(packed + r * row_bytes, i, bits);
}

/* ------------------------------------------------------------------ one VQ tensor */

/* The oracle's own description of one (possibly expert-stacked) VQ tensor. */
typedef struct {
    int32_t rows, cols, d, bits;
    const uint16_t *codebook;       /* fp16 [K][d] per codebook */
    const uint8_t *codes;           /* [rows][code_row_bytes] per expert */
    const uint16_t *scales;         /* fp16 [rows][scale_row_elems] per expert */
    int64_t code_row_bytes;
    int64_t scale_row_elems;
    int64_t expert_code_stride;     /* bytes */
    int64_t expert_scale_stride;    /* elements */
    int64_t expert_codebook_stride; /* elements; 0 = one codebook for all experts */
    int32_t num_experts;
    int32_t pad_;
} orc_mat;

/* Row r of expert e, dequantized to fp32: w[c] = scale * codebook entry. */
static void orc_dequant_row(const orc_mat *W, int32_t e, int64_t r, float *w)
{
    const uint8_t *row = W->codes + (int64_t)e * W->expert_code_stride + r * W->code_row_bytes;
    const uint16_t *srow = W->scales + (int64_t)e * W->expert_scale_stride + r * W->scale_row_elems;
    const uint16_t *cb = W->codebook + (int64_t)e * W->expert_codebook_stride;
    for (int64_t c = 0; c < W->cols; c++) {
        uint32_t code = orc_code_at(row, c / W->d, W->bits);
        float s = orc_half_to_float(srow[c / 64]);
        float v = orc_half_to_float(cb[(int64_t)code * W->d + c % W->d]);
        w[c] = s * v;
    }
}

/* Whole matrix of expert e to fp32 [rows][cols]. */
void orc_dequant(const orc_mat *W, int32_t e, float *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < W->rows; r++) orc_dequant_row(W, e, r, out + r * W->cols);
}

/* y[m][r] = sum_c W[r][c] x[m][c] in fp64, for all m < M and r < rows. */
void orc_linear(const orc_mat *W, int32_t e, const void *x, int32_t xt, int64_t M,
                int64_t x_row_stride, double *y)
{
#pragma omp parallel
    {
        float *w = (float *)malloc(sizeof(float) * (size_t)W->cols);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < W->rows; r++) {
            orc_dequant_row(W, e, r, w);
            for (int64_t m = 0; m < M; m++) {
                double acc = 0.0;
                for (int64_t c = 0; c < W->cols; c++)
                    acc += (double)w[c] * orc_x_at(x, xt, m * x_row_stride + c);
                y[m * W->rows + r] = acc;
            }
        }
        free(w);
    }
}

/* The same sum for a list of (m, r) output positions only. */
void orc_linear_sampled(const orc_mat *W, int32_t e, const void *x, int32_t xt,
                        int64_t x_row_stride, int64_t n, const int64_t *ms,
                        const int64_t *rs, double *out)
{
#pragma omp parallel
    {
        float *w = (float *)malloc(sizeof(float) * (size_t)W->cols);
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < n; i++) {
            orc_dequant_row(W, e, rs[i], w);
            double acc = 0.0;
            for (int64_t c = 0; c < W->cols; c++)
                acc += (double)w[c] * orc_x_at(x, xt, ms[i] * x_row_stride + c);
            out[i] = acc;
        }
        free(w);
    }
}

/* ------------------------------------------------------------------ MoE layer */

/* Expert FFN of one token through expert e, fp64 throughout; o has hidden entries.
 * x_t has gate->cols (= hidden) entries starting at element x_off of x. */
static void orc_expert_ffn(const orc_mat *gate, const orc_mat *up, const orc_mat *down,
                           int32_t e, const void *x, int32_t xt, int64_t x_off,
                           float *wbuf, double *h, double *o)
{
    int64_t inter = gate->rows, hidden = gate->cols;
    for (int64_t i = 0; i < inter; i++) {
        double g = 0.0, u = 0.0;
        orc_dequant_row(gate, e, i, wbuf);
        for (int64_t c = 0; c < hidden; c++) g += (double)wbuf[c] * orc_x_at(x, xt, x_off + c);
        orc_dequant_row(up, e, i, wbuf);
        for (int64_t c = 0; c < hidden; c++) u += (double)wbuf[c] * orc_x_at(x, xt, x_off + c);
        h[i] = g / (1.0 + exp(-g)) * u;
    }
    for (int64_t r = 0; r < hidden; r++) {
        double acc = 0.0;
        orc_dequant_row(down, e, r, wbuf);
        for (int64_t c = 0; c < inter; c++) acc += (double)wbuf[c] * h[c];
        o[r] = acc;
    }
}

/* y[t][hidden] for the listed tokens (ntok of them, indices in toks) of a routed MoE
 * layer: ids and w are [T][topk].  Returns the number of skipped (invalid) pairs. */
int64_t orc_moe_tokens(const orc_mat *gate, const orc_mat *up, const orc_mat *down,
                       const void *x, int32_t xt, int64_t ntok, const int64_t *toks,
                       const int32_t *ids, const float *w, int32_t topk, double *y)
{
    int64_t hidden = gate->cols, inter = gate->rows;
    int64_t bad = 0;
#pragma omp parallel reduction(+ : bad)
    {
        int64_t wl = hidden > inter ? hidden : inter;
        float *wbuf = (float *)malloc(sizeof(float) * (size_t)wl);
        double *h = (double *)malloc(sizeof(double) * (size_t)inter);
        double *o = (double *)malloc(sizeof(double) * (size_t)hidden);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < ntok; i++) {
            int64_t t = toks[i];
            double *yt = y + i * hidden;
            for (int64_t c = 0; c < hidden; c++) yt[c] = 0.0;
            for (int32_t j = 0; j < topk; j++) {
                int32_t e = ids[t * topk + j];
                if (e < 0 || e >= gate->num_experts) { bad++; continue; }
                orc_expert_ffn(gate, up, down, e, x, xt, t * hidden, wbuf, h, o);
                double wt = (double)w[t * topk + j];
                for (int64_t c = 0; c < hidden; c++) yt[c] += wt * o[c];
            }
        }
        free(wbuf); free(h); free(o);
    }
    return bad;
}

/* Number of host threads the parallel loops above use. */
int32_t orc_num_threads(void)
{
#ifdef _OPENMP
    return (int32_t)omp_get_max_threads();
#else
    return 1;
#endif
}

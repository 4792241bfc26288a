// vq_gemm_api.cuh — launch interface of the tcgen05 VQ GEMM, shared by the dense prefill
// entry point and the grouped MoE path.
#pragma once

#include "vq_internal.cuh"

namespace vq {

// Up to two projections (selected by blockIdx.z) against the same activation rows.
// Dense: t_exp == nullptr, activation rows [0, M).  Grouped: tile i covers activation
// rows [t_row[i], t_row[i] + t_cnt[i]) of expert t_exp[i]; *ntiles tiles are valid.
struct GemmArgs {
    Mat W[2];
    void *y[2];       // outputs, row j of the activations -> y[j * ldy + n]
    int64_t ldy[2];
    int yt;           // vq_dtype of y
    int M;
    const int *t_exp, *t_row, *t_cnt, *ntiles;
};

// x16: 16-bit activations [x_rows][W.cols] (bf16 when `bf16`, else fp16); BT tokens per
// tile (32, 64, 128 or 256); grouped launches use a grid of max_tiles tiles.
vq_status run_vq_gemm(const GemmArgs &a, int nproj, const void *x16, int x_rows, bool bf16, int BT,
                      int max_tiles, cudaStream_t s);

}  // namespace vq

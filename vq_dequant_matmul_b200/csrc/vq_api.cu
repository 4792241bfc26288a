// vq_api.cu — the extern "C" entry points declared in include/vq.h: argument
// validation on the host, then dispatch to the kernels.  Nothing is launched when an
// argument is rejected.
#include <string.h>

#include "vq_internal.cuh"

namespace vq {
vq_status launch_pack(const uint16_t *, int32_t, int32_t, int32_t, void *, int64_t, cudaStream_t);
vq_status launch_unpack(const void *, int32_t, int32_t, int32_t, int64_t, uint16_t *, cudaStream_t);
vq_status launch_dequant(const Mat &, int32_t, void *, vq_dtype, cudaStream_t);
vq_status launch_gemv(const Mat &, const void *, vq_dtype, int, void *, vq_dtype, cudaStream_t);
vq_status launch_gemm(const Mat &, const void *, vq_dtype, int, void *, vq_dtype, void *, size_t,
                      uint32_t, cudaStream_t);
size_t gemm_workspace_bytes(const Mat &, vq_dtype, int, uint32_t);
vq_status moe_workspace_bytes(int32_t, int32_t, int32_t, int32_t, int32_t, size_t *);
vq_status launch_moe(const Mat &, const Mat &, const Mat &, const void *, vq_dtype, int32_t,
                     const int32_t *, const float *, int32_t, void *, vq_dtype, void *, size_t,
                     cudaStream_t);
vq_status read_moe_status(const void *, cudaStream_t);
vq_status read_device_error(cudaStream_t, unsigned int *);
size_t moe_static_scratch_bytes();
void *moe_static_scratch();
}  // namespace vq

namespace {

inline bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }
inline bool valid_dtype(vq_dtype t) { return t == VQ_F16 || t == VQ_BF16 || t == VQ_F32; }
inline size_t dtype_bytes(vq_dtype t) { return t == VQ_F32 ? 4 : 2; }

// Checks shared by every entry point that takes a vq_matrix.
vq_status check_matrix(const vq_matrix *W)
{
    if (!W) return VQ_ERR_INVALID_ARG;
    if (W->rows < 1 || W->cols < 64 || W->cols % 64) return VQ_ERR_INVALID_ARG;
    if (W->num_experts < 1 || W->reserved != 0) return VQ_ERR_INVALID_ARG;
    if (vq::geom_of(W->d, W->bits) < 0) return VQ_ERR_UNSUPPORTED;
    if (!W->codebook || !W->codes || !W->scales) return VQ_ERR_INVALID_ARG;
    const int64_t need = vq_code_row_bytes(W->cols / W->d, W->bits);
    if (W->code_row_bytes < need || W->scale_row_elems < W->cols / 64) return VQ_ERR_INVALID_ARG;
    if (W->code_row_bytes % 16 || !aligned(W->codes, 16) || !aligned(W->codebook, 16) ||
        !aligned(W->scales, 2))
        return VQ_ERR_MISALIGNED;
    if (W->num_experts > 1) {
        if (W->expert_code_stride < W->code_row_bytes * W->rows ||
            W->expert_scale_stride < W->scale_row_elems * W->rows ||
            W->expert_codebook_stride < 0 ||
            (W->expert_codebook_stride > 0 &&
             W->expert_codebook_stride < ((int64_t)1 << W->bits) * W->d))
            return VQ_ERR_INVALID_ARG;
        if (W->expert_code_stride % 16 || W->expert_codebook_stride % 8) return VQ_ERR_MISALIGNED;
    }
    return VQ_OK;
}

}  // namespace

extern "C" {

int64_t vq_code_row_bytes(int64_t ncodes, int32_t bits)
{
    if (ncodes < 0 || bits < 1 || bits > 16) return -1;
    return ((ncodes + 31) / 32) * 4 * (int64_t)bits;
}

vq_status vq_pack(const uint16_t *codes, int32_t rows, int32_t ncodes, int32_t bits, void *packed,
                  int64_t code_row_bytes, vq_stream_t stream)
{
    if (rows < 0 || ncodes < 0 || bits < 1 || bits > 16) return VQ_ERR_INVALID_ARG;
    if (code_row_bytes < vq_code_row_bytes(ncodes, bits)) return VQ_ERR_INVALID_ARG;
    if ((int64_t)rows * ncodes > 0 && !codes) return VQ_ERR_INVALID_ARG;
    if (rows > 0 && code_row_bytes > 0 && !packed) return VQ_ERR_INVALID_ARG;
    if (code_row_bytes % 4 || !aligned(packed, 4) || !aligned(codes, 2)) return VQ_ERR_MISALIGNED;
    return vq::launch_pack(codes, rows, ncodes, bits, packed, code_row_bytes, (cudaStream_t)stream);
}

vq_status vq_unpack(const void *packed, int32_t rows, int32_t ncodes, int32_t bits,
                    int64_t code_row_bytes, uint16_t *codes, vq_stream_t stream)
{
    if (rows < 0 || ncodes < 0 || bits < 1 || bits > 16) return VQ_ERR_INVALID_ARG;
    if (code_row_bytes < vq_code_row_bytes(ncodes, bits)) return VQ_ERR_INVALID_ARG;
    if ((int64_t)rows * ncodes > 0 && (!codes || !packed)) return VQ_ERR_INVALID_ARG;
    if (code_row_bytes % 4 || !aligned(packed, 4) || !aligned(codes, 2)) return VQ_ERR_MISALIGNED;
    return vq::launch_unpack(packed, rows, ncodes, bits, code_row_bytes, codes, (cudaStream_t)stream);
}

vq_status vq_dequant(const vq_matrix *W, int32_t expert, void *w_out, vq_dtype out, vq_stream_t stream)
{
    vq_status st = check_matrix(W);
    if (st != VQ_OK) return st;
    if (expert < 0 || expert >= W->num_experts || !w_out || !valid_dtype(out)) return VQ_ERR_INVALID_ARG;
    if (!aligned(w_out, dtype_bytes(out))) return VQ_ERR_MISALIGNED;
    return vq::launch_dequant(vq::to_mat(*W), expert, w_out, out, (cudaStream_t)stream);
}

vq_status vq_gemv(const vq_matrix *W, const void *x, vq_dtype xt, int32_t batch, void *y, vq_dtype yt,
                  void *ws, size_t ws_bytes, vq_stream_t stream)
{
    (void)ws; (void)ws_bytes;
    vq_status st = check_matrix(W);
    if (st != VQ_OK) return st;
    if (batch < 1 || batch > 16 || !x || !y || !valid_dtype(xt) || !valid_dtype(yt)) return VQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, dtype_bytes(yt))) return VQ_ERR_MISALIGNED;
    return vq::launch_gemv(vq::to_mat(*W), x, xt, batch, y, yt, (cudaStream_t)stream);
}

vq_status vq_gemm_workspace_size(const vq_matrix *W, vq_dtype xt, int32_t M, uint32_t flags, size_t *bytes)
{
    vq_status st = check_matrix(W);
    if (st != VQ_OK) return st;
    if (!bytes || M < 1 || (xt != VQ_F16 && xt != VQ_BF16)) return VQ_ERR_INVALID_ARG;
    *bytes = vq::gemm_workspace_bytes(vq::to_mat(*W), xt, M, flags);
    return VQ_OK;
}

vq_status vq_gemm_ex(const vq_matrix *W, const void *x, vq_dtype xt, int32_t M, void *y, vq_dtype yt,
                     void *ws, size_t ws_bytes, uint32_t flags, vq_stream_t stream)
{
    vq_status st = check_matrix(W);
    if (st != VQ_OK) return st;
    if (M < 1 || !x || !y || (xt != VQ_F16 && xt != VQ_BF16) || !valid_dtype(yt)) return VQ_ERR_INVALID_ARG;
    if (flags & ~VQ_GEMM_BF16_TILES) return VQ_ERR_INVALID_ARG;
    if ((flags & VQ_GEMM_BF16_TILES) && xt != VQ_BF16) return VQ_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(y, 16)) return VQ_ERR_MISALIGNED;
    const size_t need = vq::gemm_workspace_bytes(vq::to_mat(*W), xt, M, flags);
    if (need > 0 && (!ws || ws_bytes < need)) return VQ_ERR_WORKSPACE;
    if (need > 0 && !aligned(ws, 256)) return VQ_ERR_MISALIGNED;
    return vq::launch_gemm(vq::to_mat(*W), x, xt, M, y, yt, ws, ws_bytes, flags, (cudaStream_t)stream);
}

vq_status vq_gemm(const vq_matrix *W, const void *x, vq_dtype xt, int32_t M, void *y, vq_dtype yt,
                  void *ws, size_t ws_bytes, vq_stream_t stream)
{
    return vq_gemm_ex(W, x, xt, M, y, yt, ws, ws_bytes, 0u, stream);
}

vq_status vq_moe_workspace_size(int32_t T, int32_t topk, int32_t E, int32_t hidden, int32_t inter,
                                size_t *bytes)
{
    if (!bytes) return VQ_ERR_INVALID_ARG;
    return vq::moe_workspace_bytes(T, topk, E, hidden, inter, bytes);
}

vq_status vq_moe_grouped(const vq_matrix *gate, const vq_matrix *up, const vq_matrix *down, const void *x,
                         vq_dtype xt, int32_t T, const int32_t *expert_ids, const float *expert_w,
                         int32_t topk, void *y, vq_dtype yt, void *ws, size_t ws_bytes, vq_stream_t stream)
{
    vq_status st;
    if ((st = check_matrix(gate)) != VQ_OK || (st = check_matrix(up)) != VQ_OK ||
        (st = check_matrix(down)) != VQ_OK)
        return st;
    const int32_t E = gate->num_experts, hidden = gate->cols, inter = gate->rows;
    if (up->num_experts != E || down->num_experts != E || up->rows != inter || up->cols != hidden ||
        down->rows != hidden || down->cols != inter)
        return VQ_ERR_INVALID_ARG;
    if (T < 1 || topk < 1 || topk > E || !x || !expert_ids || !expert_w || !y || !ws) return VQ_ERR_INVALID_ARG;
    if ((xt != VQ_F16 && xt != VQ_BF16) || !valid_dtype(yt)) return VQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ws, 256) || !aligned(expert_ids, 4) ||
        !aligned(expert_w, 4))
        return VQ_ERR_MISALIGNED;
    size_t need = 0;
    if ((st = vq::moe_workspace_bytes(T, topk, E, hidden, inter, &need)) != VQ_OK) return st;
    if (ws_bytes < need) return VQ_ERR_WORKSPACE;
    return vq::launch_moe(vq::to_mat(*gate), vq::to_mat(*up), vq::to_mat(*down), x, xt, T, expert_ids,
                          expert_w, topk, y, yt, ws, ws_bytes, (cudaStream_t)stream);
}

vq_status vq_moe_grouped_noalloc(const vq_matrix *gate, const vq_matrix *up, const vq_matrix *down,
                                 const void *x, vq_dtype xt, int32_t T, const int32_t *expert_ids,
                                 const float *expert_w, int32_t topk, void *y, vq_dtype yt, vq_stream_t stream)
{
    vq_status st;
    if ((st = check_matrix(gate)) != VQ_OK || (st = check_matrix(up)) != VQ_OK ||
        (st = check_matrix(down)) != VQ_OK)
        return st;
    size_t need = 0;
    if ((st = vq_moe_workspace_size(T, topk, gate->num_experts, gate->cols, gate->rows, &need)) != VQ_OK)
        return st;
    if (need > vq::moe_static_scratch_bytes()) return VQ_ERR_WORKSPACE;
    void *scratch = vq::moe_static_scratch();
    if (!scratch) return VQ_ERR_CUDA;
    return vq_moe_grouped(gate, up, down, x, xt, T, expert_ids, expert_w, topk, y, yt, scratch,
                          vq::moe_static_scratch_bytes(), stream);
}

vq_status vq_read_device_status(const void *ws, vq_stream_t stream)
{
    unsigned int err = 0;
    vq_status st = vq::read_device_error((cudaStream_t)stream, &err);
    if (st != VQ_OK) return st;
    if (err) return VQ_ERR_TIMEOUT;
    return ws ? vq::read_moe_status(ws, (cudaStream_t)stream) : VQ_OK;
}

const char *vq_status_string(vq_status s)
{
    switch (s) {
    case VQ_OK: return "ok";
    case VQ_ERR_INVALID_ARG: return "invalid argument";
    case VQ_ERR_UNSUPPORTED: return "unsupported geometry or dtype";
    case VQ_ERR_MISALIGNED: return "misaligned pointer or stride";
    case VQ_ERR_WORKSPACE: return "workspace missing or too small";
    case VQ_ERR_CUDA: return "CUDA error";
    case VQ_ERR_DEVICE_FLAG: return "device recorded bad input (expert id out of range)";
    case VQ_ERR_TIMEOUT: return "bounded device wait ran out";
    }
    return "unknown status";
}

const char *vq_version(void) { return "0.1.0"; }

}  // extern "C"

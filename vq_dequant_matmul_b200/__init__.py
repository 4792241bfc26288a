"""Python binding of the B200 VQ dequantize-and-multiply library (libvq_b200.so).

Argument marshalling only: every step of the computation runs in the CUDA kernels of
the shared library, whose C ABI is declared in include/vq.h.  The functions keep the C
names (vq_pack, vq_gemv, ...), take torch tensors that live on a CUDA device, and
launch on torch's current stream.  There is no fallback: if the library is not built,
importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvq_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python vq_dequant_matmul_b200/build.py` "
                      "(nvcc, sm_100a); there is no CPU fallback")

_lib = ctypes.CDLL(LIB_PATH)

VQ_OK, VQ_ERR_INVALID_ARG, VQ_ERR_UNSUPPORTED, VQ_ERR_MISALIGNED = 0, 1, 2, 3
VQ_ERR_WORKSPACE, VQ_ERR_CUDA, VQ_ERR_DEVICE_FLAG, VQ_ERR_TIMEOUT = 4, 5, 6, 7
VQ_F16, VQ_BF16, VQ_F32 = 0, 1, 2
VQ_GEMM_BF16_TILES = 1

_TORCH_TO_VQ = {torch.float16: VQ_F16, torch.bfloat16: VQ_BF16, torch.float32: VQ_F32}
VQ_TO_TORCH = {v: k for k, v in _TORCH_TO_VQ.items()}


class vq_matrix(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int32), ("cols", ctypes.c_int32),
        ("d", ctypes.c_int32), ("bits", ctypes.c_int32),
        ("codebook", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("code_row_bytes", ctypes.c_int64), ("scale_row_elems", ctypes.c_int64),
        ("expert_code_stride", ctypes.c_int64), ("expert_scale_stride", ctypes.c_int64),
        ("expert_codebook_stride", ctypes.c_int64),
        ("num_experts", ctypes.c_int32), ("reserved", ctypes.c_int32),
    ]


_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_M = ctypes.POINTER(vq_matrix)
_SIGS = {
    "vq_code_row_bytes": (_I64, [_I64, _I32]),
    "vq_pack": (_I32, [_P, _I32, _I32, _I32, _P, _I64, _P]),
    "vq_unpack": (_I32, [_P, _I32, _I32, _I32, _I64, _P, _P]),
    "vq_dequant": (_I32, [_M, _I32, _P, _I32, _P]),
    "vq_gemv": (_I32, [_M, _P, _I32, _I32, _P, _I32, _P, _SZ, _P]),
    "vq_gemm": (_I32, [_M, _P, _I32, _I32, _P, _I32, _P, _SZ, _P]),
    "vq_gemm_ex": (_I32, [_M, _P, _I32, _I32, _P, _I32, _P, _SZ, ctypes.c_uint32, _P]),
    "vq_gemm_workspace_size": (_I32, [_M, _I32, _I32, ctypes.c_uint32, ctypes.POINTER(_SZ)]),
    "vq_moe_workspace_size": (_I32, [_I32, _I32, _I32, _I32, _I32, ctypes.POINTER(_SZ)]),
    "vq_moe_grouped": (_I32, [_M, _M, _M, _P, _I32, _I32, _P, _P, _I32, _P, _I32, _P, _SZ, _P]),
    "vq_moe_grouped_noalloc": (_I32, [_M, _M, _M, _P, _I32, _I32, _P, _P, _I32, _P, _I32, _P]),
    "vq_read_device_status": (_I32, [_P, _P]),
    "vq_status_string": (ctypes.c_char_p, [_I32]),
    "vq_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args

EXPORTED = tuple(_SIGS)


class VQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.vq_status_string(status).decode()} (status {status})")


def _check(st: int, where: str) -> None:
    if st != VQ_OK:
        raise VQError(st, where)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    """Device address of a CUDA tensor (None passes through as NULL).  Host tensors are
    refused here: every pointer the library takes is a device pointer."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}: the library takes device pointers only")
    return ctypes.c_void_p(t.data_ptr())


def status_string(st: int) -> str:
    return _lib.vq_status_string(st).decode()


def version() -> str:
    return _lib.vq_version().decode()


def vq_code_row_bytes(ncodes: int, bits: int) -> int:
    return int(_lib.vq_code_row_bytes(ncodes, bits))


# ----------------------------------------------------------------------------- tensors

def _as_device_bits(a, device):
    """numpy uint8/uint16/float16 array or torch tensor -> device tensor with the same bits
    (uint16 becomes int16, since the bits are all that matter)."""
    if isinstance(a, torch.Tensor):
        return a.to(device)
    import numpy as np

    a = np.ascontiguousarray(a)
    if a.dtype in (np.uint16, np.float16):
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


class VQMatrix:
    """Device tensors of one VQ tensor (or expert stack) plus its vq_matrix descriptor.

    codebook: fp16 [n_cb][K][d]; codes: uint8 packed [E][rows][code_row_bytes];
    scales: fp16 [E][rows][scale_row_elems]."""

    def __init__(self, codebook: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                 rows: int, cols: int, d: int, bits: int):
        assert codebook.dtype == torch.float16 and scales.dtype == torch.float16
        assert codes.dtype == torch.uint8 and codes.dim() == 3
        for t in (codebook, codes, scales):
            if not t.is_cuda or t.device != codes.device:
                raise ValueError(f"codebook, codes and scales must be CUDA tensors on one device (got {t.device})")
        self.codebook, self.codes, self.scales = codebook, codes, scales
        self.rows, self.cols, self.d, self.bits = rows, cols, d, bits
        E = codes.shape[0]
        self.num_experts = E
        self.desc = vq_matrix(
            rows=rows, cols=cols, d=d, bits=bits,
            codebook=codebook.data_ptr(), codes=codes.data_ptr(), scales=scales.data_ptr(),
            code_row_bytes=codes.shape[2], scale_row_elems=scales.shape[2],
            expert_code_stride=codes.stride(0), expert_scale_stride=scales.stride(0),
            expert_codebook_stride=0 if codebook.shape[0] == 1 else codebook.stride(0),
            num_experts=E, reserved=0)

    @property
    def ptr(self):
        return ctypes.byref(self.desc)

    @classmethod
    def from_unpacked(cls, codebook_bits, codes, scales_bits, rows: int, cols: int, d: int, bits: int,
                      device="cuda", stream=None) -> "VQMatrix":
        """Upload raw arrays (fp16 bit patterns as uint16 numpy arrays or fp16 tensors; codes
        [E][rows][ncodes] as uint8/uint16) and pack the codes on the device with vq_pack."""
        cb = _as_device_bits(codebook_bits, device).view(torch.float16).contiguous()
        sc = _as_device_bits(scales_bits, device).view(torch.float16).contiguous()
        E, ncodes = codes.shape[0], codes.shape[2]
        rb = (vq_code_row_bytes(ncodes, bits) + 15) // 16 * 16
        packed = torch.empty((E, rows, rb), dtype=torch.uint8, device=device)
        for e in range(E):
            c16 = _as_device_bits(codes[e], device)
            if c16.dtype == torch.uint8:
                c16 = c16.to(torch.int16)
            vq_pack(c16.contiguous(), rows, ncodes, bits, packed[e], rb, stream)
        return cls(cb, packed, sc, rows, cols, d, bits)

    @classmethod
    def from_data(cls, data, device="cuda", stream=None) -> "VQMatrix":
        """From a workloads.VQTensorData (raw synthetic arrays)."""
        return cls.from_unpacked(data.codebook, data.codes, data.scales, data.rows, data.cols,
                                 data.d, data.bits, device, stream)


# ----------------------------------------------------------------------------- entry points

def vq_pack(codes: torch.Tensor, rows: int, ncodes: int, bits: int, packed: torch.Tensor,
            code_row_bytes: int, stream=None) -> None:
    _check(_lib.vq_pack(_ptr(codes), rows, ncodes, bits, _ptr(packed), code_row_bytes, _stream(stream)), "vq_pack")


def vq_unpack(packed: torch.Tensor, rows: int, ncodes: int, bits: int, code_row_bytes: int,
              codes: torch.Tensor, stream=None) -> None:
    _check(_lib.vq_unpack(_ptr(packed), rows, ncodes, bits, code_row_bytes, _ptr(codes), _stream(stream)),
           "vq_unpack")


def vq_dequant(W: VQMatrix, expert: int, out: torch.Tensor, stream=None) -> None:
    _check(_lib.vq_dequant(W.ptr, expert, _ptr(out), _TORCH_TO_VQ[out.dtype], _stream(stream)), "vq_dequant")


def vq_gemv(W: VQMatrix, x: torch.Tensor, y: torch.Tensor, ws: torch.Tensor | None = None,
            stream=None) -> None:
    """y [batch][rows] = x [batch][cols] @ W^T."""
    batch = x.shape[0] if x.dim() == 2 else 1
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.vq_gemv(W.ptr, _ptr(x), _TORCH_TO_VQ[x.dtype], batch, _ptr(y), _TORCH_TO_VQ[y.dtype],
                        _ptr(ws), ws_bytes, _stream(stream)), "vq_gemv")


def vq_gemm_workspace_size(W: VQMatrix, x_dtype: torch.dtype, M: int, flags: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.vq_gemm_workspace_size(W.ptr, _TORCH_TO_VQ[x_dtype], M, flags, ctypes.byref(n)),
           "vq_gemm_workspace_size")
    return int(n.value)


def vq_gemm(W: VQMatrix, x: torch.Tensor, y: torch.Tensor, ws: torch.Tensor | None = None,
            flags: int = 0, stream=None) -> None:
    """y [M][rows] = x [M][cols] @ W^T on the tensor cores."""
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.vq_gemm_ex(W.ptr, _ptr(x), _TORCH_TO_VQ[x.dtype], x.shape[0], _ptr(y), _TORCH_TO_VQ[y.dtype],
                           _ptr(ws), ws_bytes, flags, _stream(stream)), "vq_gemm")


def vq_moe_workspace_size(T: int, topk: int, E: int, hidden: int, inter: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.vq_moe_workspace_size(T, topk, E, hidden, inter, ctypes.byref(n)), "vq_moe_workspace_size")
    return int(n.value)


def vq_moe_grouped(gate: VQMatrix, up: VQMatrix, down: VQMatrix, x: torch.Tensor, expert_ids: torch.Tensor,
                   expert_w: torch.Tensor, y: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    T, topk = expert_ids.shape
    _check(_lib.vq_moe_grouped(gate.ptr, up.ptr, down.ptr, _ptr(x), _TORCH_TO_VQ[x.dtype], T,
                               _ptr(expert_ids), _ptr(expert_w), topk, _ptr(y), _TORCH_TO_VQ[y.dtype],
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "vq_moe_grouped")


def vq_moe_grouped_noalloc(gate: VQMatrix, up: VQMatrix, down: VQMatrix, x: torch.Tensor,
                           expert_ids: torch.Tensor, expert_w: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """vq_moe_grouped without a workspace: for callers that cannot allocate device memory.
    Uses the library's fixed 16 MiB device scratch (decode-sized batches only)."""
    T, topk = expert_ids.shape
    _check(_lib.vq_moe_grouped_noalloc(gate.ptr, up.ptr, down.ptr, _ptr(x), _TORCH_TO_VQ[x.dtype], T,
                                       _ptr(expert_ids), _ptr(expert_w), topk, _ptr(y), _TORCH_TO_VQ[y.dtype],
                                       _stream(stream)), "vq_moe_grouped_noalloc")


def vq_read_device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream; returns the raw status (0 = ok, 6 = bad expert ids seen)."""
    return int(_lib.vq_read_device_status(_ptr(ws), _stream(stream)))

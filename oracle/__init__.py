"""CPU oracle for the VQ dequantize-and-multiply path — TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import this
package.  It loads `liboracle.so`, built from `vq_oracle.c` with gcc, which shares no
code with the CUDA library.  See `vq_oracle.c` for the definitions and the passages
of the pages each one follows.

Parity status: every function here is pinned by `tests/test_oracle_pins.py` against
values fixed by the pages or by mathematics (closed-form sizes, hand-derived byte
patterns, exact integer brute force, reductions to a library matmul, MoE invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile vq_oracle.c into liboracle.so (gcc, OpenMP, strict fp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


class OrcMat(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int32), ("cols", ctypes.c_int32),
        ("d", ctypes.c_int32), ("bits", ctypes.c_int32),
        ("codebook", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("code_row_bytes", ctypes.c_int64), ("scale_row_elems", ctypes.c_int64),
        ("expert_code_stride", ctypes.c_int64), ("expert_scale_stride", ctypes.c_int64),
        ("expert_codebook_stride", ctypes.c_int64),
        ("num_experts", ctypes.c_int32), ("pad_", ctypes.c_int32),
    ]


def configure(L):
    """Declare the C signatures on a loaded copy of the oracle library."""
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    L.orc_half_to_float.restype = ctypes.c_float
    L.orc_half_to_float.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_float.restype = ctypes.c_float
    L.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
    L.orc_half_to_float_n.argtypes = [P, i64, P]
    L.orc_bf16_to_float_n.argtypes = [P, i64, P]
    L.orc_code_row_bytes.restype = i64
    L.orc_code_row_bytes.argtypes = [i64, i32]
    L.orc_code_at.restype = ctypes.c_uint32
    L.orc_code_at.argtypes = [P, i64, i32]
    L.orc_pack.argtypes = [P, i64, i64, i32, P, i64]
    L.orc_unpack.argtypes = [P, i64, i64, i32, i64, P]
    L.orc_dequant.argtypes = [ctypes.POINTER(OrcMat), i32, P]
    L.orc_linear.argtypes = [ctypes.POINTER(OrcMat), i32, P, i32, i64, i64, P]
    L.orc_linear_sampled.argtypes = [ctypes.POINTER(OrcMat), i32, P, i32, i64, i64, P, P, P]
    L.orc_moe_tokens.restype = i64
    L.orc_moe_tokens.argtypes = [ctypes.POINTER(OrcMat)] * 3 + [P, i32, i64, P, P, P, i32, P]
    L.orc_num_threads.restype = i32
    return L


def load(path: str):
    """Load an oracle library from `path` (the mutation test builds altered copies)."""
    return configure(ctypes.CDLL(path))


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads(L=None) -> int:
    return int((L or lib()).orc_num_threads())


def code_row_bytes(ncodes: int, bits: int, L=None) -> int:
    return int((L or lib()).orc_code_row_bytes(ncodes, bits))


def half_to_float(bits16: np.ndarray, L=None) -> np.ndarray:
    a = np.ascontiguousarray(bits16, dtype=np.uint16)
    out = np.empty(a.shape, np.float32)
    (L or lib()).orc_half_to_float_n(_p(a), a.size, _p(out))
    return out


def bf16_to_float(bits16: np.ndarray, L=None) -> np.ndarray:
    a = np.ascontiguousarray(bits16, dtype=np.uint16)
    out = np.empty(a.shape, np.float32)
    (L or lib()).orc_bf16_to_float_n(_p(a), a.size, _p(out))
    return out


def pack(codes: np.ndarray, bits: int, row_bytes: int | None = None, L=None) -> np.ndarray:
    """codes [rows][ncodes] -> packed uint8 [rows][row_bytes]."""
    c = np.ascontiguousarray(codes, dtype=np.uint16)
    rows, ncodes = c.shape
    rb = code_row_bytes(ncodes, bits, L) if row_bytes is None else row_bytes
    out = np.empty((rows, rb), np.uint8)
    (L or lib()).orc_pack(_p(c), rows, ncodes, bits, _p(out), rb)
    return out


def unpack(packed: np.ndarray, ncodes: int, bits: int, L=None) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    rows, rb = p.shape
    out = np.empty((rows, ncodes), np.uint16)
    (L or lib()).orc_unpack(_p(p), rows, ncodes, bits, rb, _p(out))
    return out


class Tensor:
    """A VQ tensor in the oracle's own packed form (packed by `pack` above)."""

    def __init__(self, data, L=None, experts=None):
        """`experts`: pack only these experts (the others stay zero) — for full-size
        checks that evaluate a sample of tokens."""
        self.L = L or lib()
        self.data = data
        E, rows = data.num_experts, data.rows
        self.row_bytes = code_row_bytes(data.ncodes, data.bits, self.L)
        self.codes = np.zeros((E, rows, self.row_bytes), np.uint8)
        for e in (range(E) if experts is None else sorted(set(int(v) for v in experts))):
            self.codes[e] = pack(data.codes[e], data.bits, self.row_bytes, self.L)
        self.codebook = np.ascontiguousarray(data.codebook, dtype=np.uint16)
        self.scales = np.ascontiguousarray(data.scales, dtype=np.uint16)
        self.mat = OrcMat(
            rows=rows, cols=data.cols, d=data.d, bits=data.bits,
            codebook=self.codebook.ctypes.data, codes=self.codes.ctypes.data,
            scales=self.scales.ctypes.data, code_row_bytes=self.row_bytes,
            scale_row_elems=self.scales.shape[2],
            expert_code_stride=rows * self.row_bytes,
            expert_scale_stride=rows * self.scales.shape[2],
            expert_codebook_stride=0 if self.codebook.shape[0] == 1 else self.codebook.shape[1] * data.d,
            num_experts=E, pad_=0)

    def dequant(self, expert: int = 0) -> np.ndarray:
        out = np.empty((self.data.rows, self.data.cols), np.float32)
        self.L.orc_dequant(ctypes.byref(self.mat), expert, _p(out))
        return out

    def linear(self, x: np.ndarray, xt: int, expert: int = 0) -> np.ndarray:
        """y [M][rows] (fp64) for activations x [M][cols] given as raw bits of type xt."""
        x = np.ascontiguousarray(x)
        M = x.shape[0]
        y = np.empty((M, self.data.rows), np.float64)
        self.L.orc_linear(ctypes.byref(self.mat), expert, _p(x), xt, M, x.shape[1], _p(y))
        return y

    def linear_sampled(self, x: np.ndarray, xt: int, ms, rs, expert: int = 0) -> np.ndarray:
        x = np.ascontiguousarray(x)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        rs = np.ascontiguousarray(rs, dtype=np.int64)
        out = np.empty(ms.shape[0], np.float64)
        self.L.orc_linear_sampled(ctypes.byref(self.mat), expert, _p(x), xt, x.shape[1],
                                 ms.shape[0], _p(ms), _p(rs), _p(out))
        return out


def moe_tokens(gate: Tensor, up: Tensor, down: Tensor, x: np.ndarray, xt: int,
               tokens, ids: np.ndarray, w: np.ndarray):
    """y [len(tokens)][hidden] (fp64) and the count of skipped (invalid) pairs."""
    x = np.ascontiguousarray(x)
    toks = np.ascontiguousarray(tokens, dtype=np.int64)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    topk = ids.shape[1]
    y = np.empty((toks.shape[0], gate.data.cols), np.float64)
    bad = gate.L.orc_moe_tokens(ctypes.byref(gate.mat), ctypes.byref(up.mat), ctypes.byref(down.mat),
                               _p(x), xt, toks.shape[0], _p(toks), _p(ids), _p(w), topk, _p(y))
    return y, int(bad)

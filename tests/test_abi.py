"""The C-ABI library loads on a machine without a GPU, exports every entry point the
header declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vq.h")


def header_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(vq_\w+)\s*\(", src, re.M)))


def test_header_declares_the_boundary():
    names = header_functions()
    for n in ("vq_pack", "vq_unpack", "vq_gemv", "vq_gemm", "vq_moe_grouped"):
        assert n in names


def test_library_exports_every_declared_symbol(vqlib):
    out = subprocess.run(["nm", "-D", "--defined-only", vqlib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (vq_\w+)$", out, re.M))
    missing = [n for n in header_functions() if n not in exported]
    assert not missing, missing
    for n in header_functions():
        assert hasattr(vqlib._lib, n)
    assert set(vqlib.EXPORTED) == set(header_functions())


def test_host_functions(vqlib):
    assert vqlib.vq_code_row_bytes(2560, 8) == 2560
    assert vqlib.vq_code_row_bytes(256, 12) == 384
    assert vqlib.vq_code_row_bytes(33, 12) == 96
    assert vqlib.vq_code_row_bytes(1, 3) == 12
    assert vqlib.vq_code_row_bytes(-1, 8) == -1
    assert vqlib.vq_code_row_bytes(10, 17) == -1
    for s in range(8):
        assert vqlib.status_string(s)
    assert re.match(r"^\d+\.\d+\.\d+$", vqlib.version())


def _mat(vqlib, **kw):
    # Fake, 256-aligned, never-dereferenced addresses: every case below is rejected by the
    # host-side checks before any CUDA call.
    base = dict(rows=16, cols=128, d=4, bits=8, codebook=0x10000, codes=0x20000, scales=0x30000,
                code_row_bytes=32, scale_row_elems=2, expert_code_stride=0, expert_scale_stride=0,
                expert_codebook_stride=0, num_experts=1, reserved=0)
    base.update(kw)
    return vqlib.vq_matrix(**base)


@pytest.mark.parametrize("kw,want", [
    (dict(rows=0), 1), (dict(cols=100), 1), (dict(cols=0), 1), (dict(d=3), 2), (dict(bits=10), 2),
    (dict(codes=0), 1), (dict(code_row_bytes=16), 1), (dict(scale_row_elems=1), 1),
    (dict(codes=0x20008), 3), (dict(code_row_bytes=40), 3), (dict(reserved=1), 1),
    (dict(num_experts=2, expert_code_stride=16), 1),
])
def test_gemv_rejects_bad_matrix(vqlib, kw, want):
    W = _mat(vqlib, **kw)
    st = vqlib._lib.vq_gemv(ctypes.byref(W), ctypes.c_void_p(0x40000), 0, 1, ctypes.c_void_p(0x50000), 2,
                            None, 0, None)
    assert st == want


@pytest.mark.parametrize("args,want", [
    (dict(batch=0), 1), (dict(batch=17), 1), (dict(x=0), 1), (dict(x=0x40008), 3), (dict(xt=7), 1),
])
def test_gemv_rejects_bad_call(vqlib, args, want):
    W = _mat(vqlib)
    a = dict(x=0x40000, xt=0, batch=1, y=0x50000, yt=2)
    a.update(args)
    st = vqlib._lib.vq_gemv(ctypes.byref(W), ctypes.c_void_p(a["x"]), a["xt"], a["batch"],
                            ctypes.c_void_p(a["y"]), a["yt"], None, 0, None)
    assert st == want


def test_moe_rejects_bad_args(vqlib):
    """vq_moe_grouped validates shapes, sizes, alignment and the workspace on the host and
    launches nothing when they are wrong (fake addresses, never dereferenced)."""
    L = vqlib._lib
    P = ctypes.c_void_p
    E, hidden, inter = 4, 128, 64
    gate = _mat(vqlib, rows=inter, cols=hidden, num_experts=E, expert_code_stride=inter * 32,
                expert_scale_stride=inter * 2)
    up = _mat(vqlib, rows=inter, cols=hidden, num_experts=E, expert_code_stride=inter * 32,
              expert_scale_stride=inter * 2)
    down = _mat(vqlib, rows=hidden, cols=inter, scale_row_elems=1, num_experts=E,
                expert_code_stride=hidden * 32, expert_scale_stride=hidden)
    n = ctypes.c_size_t(0)
    assert L.vq_moe_workspace_size(2, 2, E, hidden, inter, ctypes.byref(n)) == 0 and n.value > 0

    def call(g=gate, u=up, dn=down, x=0x40000, xt=0, T=2, ids=0x60000, w=0x70000, topk=2, y=0x80000, yt=2,
             ws=0x100000, wsb=None):
        return L.vq_moe_grouped(ctypes.byref(g), ctypes.byref(u), ctypes.byref(dn), P(x), xt, T, P(ids), P(w),
                                topk, P(y), yt, P(ws), n.value if wsb is None else wsb, None)

    assert call(topk=E + 1) == 1                  # more slots than experts
    assert call(T=0) == 1
    assert call(x=0) == 1
    assert call(xt=2) == 1                        # fp32 activations
    assert call(u=_mat(vqlib, rows=inter + 16, cols=hidden, num_experts=E, expert_code_stride=(inter + 16) * 32,
                       expert_scale_stride=(inter + 16) * 2)) == 1   # up shape differs from gate
    assert call(dn=_mat(vqlib, rows=hidden, cols=inter, scale_row_elems=1, num_experts=E - 1,
                        expert_code_stride=hidden * 32, expert_scale_stride=hidden)) == 1
    assert call(ws=0x100010) == 3                 # workspace not 256-byte aligned
    assert call(ids=0x60002) == 3                 # expert ids not 4-byte aligned
    assert call(wsb=n.value - 1) == 4             # workspace too small


def test_binding_refuses_host_tensors(vqlib):
    """The Python binding passes device pointers only: a host tensor is refused before any
    call into the library (a host address handed to a kernel would fault the GPU)."""
    import torch

    with pytest.raises(ValueError):
        vqlib._ptr(torch.zeros(4))
    assert vqlib._ptr(None) is None
    cb = torch.zeros((1, 256, 2), dtype=torch.float16)
    codes = torch.zeros((1, 4, 16), dtype=torch.uint8)
    sc = torch.zeros((1, 4, 1), dtype=torch.float16)
    with pytest.raises(ValueError):
        vqlib.VQMatrix(cb, codes, sc, 4, 64, 2, 8)

    class _W:   # a descriptor stand-in: the activations are checked before the stream is read
        ptr = None

    with pytest.raises(ValueError):
        vqlib.vq_gemv(_W(), torch.zeros((1, 64), dtype=torch.float16), torch.zeros((1, 4)))


def test_pack_rejects_bad_args(vqlib):
    L = vqlib._lib
    P = ctypes.c_void_p
    assert L.vq_pack(P(0x1000), 4, 32, 17, P(0x2000), 68, None) == 1
    assert L.vq_pack(P(0x1000), 4, 32, 12, P(0x2000), 47, None) == 1
    assert L.vq_pack(P(0x1000), 4, 32, 12, P(0x2002), 48, None) == 3
    assert L.vq_unpack(P(0x1000), 4, 32, 12, 50, P(0x2000), None) == 3
    assert L.vq_unpack(None, 4, 32, 12, 48, P(0x2000), None) == 1


def test_gemm_and_moe_reject_bad_args(vqlib):
    L = vqlib._lib
    P = ctypes.c_void_p
    W = _mat(vqlib)
    assert L.vq_gemm(ctypes.byref(W), P(0x40000), 2, 16, P(0x50000), 2, None, 0, None) == 1  # f32 x
    assert L.vq_gemm(ctypes.byref(W), P(0x40000), 0, 0, P(0x50000), 2, None, 0, None) == 1
    assert L.vq_gemm_ex(ctypes.byref(W), P(0x40000), 0, 16, P(0x50000), 2, None, 0, 1, None) == 2
    assert L.vq_gemm_ex(ctypes.byref(W), P(0x40000), 0, 16, P(0x50000), 2, None, 0, 4, None) == 1
    n = ctypes.c_size_t(0)
    assert L.vq_moe_workspace_size(0, 8, 256, 2048, 512, ctypes.byref(n)) == 1

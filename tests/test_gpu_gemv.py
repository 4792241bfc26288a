"""Decode GEMV (vq_gemv) against the CPU oracle on seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_util import assert_out, normwise, x_tensor, GEMV_F32_TOL

pytestmark = pytest.mark.gpu

GEOMS = [(2, 8), (4, 8), (8, 8), (2, 12), (4, 12), (8, 12)]
TORCH_OUT = {wl.F32: torch.float32, wl.F16: torch.float16, wl.BF16: torch.bfloat16}


def run_gemv(vqlib, data, xbits, xt, yt=wl.F32):
    W = vqlib.VQMatrix.from_data(data)
    x = x_tensor(xbits, xt)
    y = torch.full((xbits.shape[0], data.rows), float("nan"), dtype=TORCH_OUT[yt], device="cuda")
    vqlib.vq_gemv(W, x, y)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("d,bits", GEOMS)
@pytest.mark.parametrize("rows,cols", [(37, 64), (130, 320), (96, 2048), (24, 17408)])
@pytest.mark.parametrize("batch", [1, 2, 3, 8, 16])
def test_gemv_shapes(vqlib, d, bits, rows, cols, batch):
    data = wl.uniform_tensor(rows, cols, d, bits, seed=rows + cols + d + bits)
    x = wl.activations(batch, cols, seed=batch + 7, dtype=wl.F16)
    ref = oracle.Tensor(data).linear(x, wl.F16)
    assert_out(run_gemv(vqlib, data, x, wl.F16), ref)


@pytest.mark.parametrize("xt", [wl.F16, wl.BF16, wl.F32])
@pytest.mark.parametrize("yt", [wl.F32, wl.F16, wl.BF16])
@pytest.mark.parametrize("batch", [1, 5])
def test_gemv_dtypes(vqlib, xt, yt, batch):
    data = wl.uniform_tensor(200, 512, 4, 8, seed=5)
    x = wl.activations(batch, 512, seed=6, dtype=xt)
    ref = oracle.Tensor(data).linear(x, xt)
    assert_out(run_gemv(vqlib, data, x, xt, yt), ref)


def test_gemv_zero_and_extreme_inputs(vqlib):
    data = wl.uniform_tensor(64, 256, 2, 8, seed=8)
    x = np.zeros((1, 256), np.float16).view(np.uint16)
    y = run_gemv(vqlib, data, x, wl.F16)
    assert (y == 0).all()
    # fp16 subnormal and max-magnitude activations stay exact in the oracle comparison
    xv = np.full((1, 256), 6.0e-8, np.float32)
    xv[0, ::3] = 60000.0
    xb = wl.activation_bits(xv, wl.F16)
    ref = oracle.Tensor(data).linear(xb, wl.F16)
    assert_out(run_gemv(vqlib, data, xb, wl.F16), ref)


def test_c1_single_gemv(vqlib):
    data, x = wl.c1_single_gemv()
    ref = oracle.Tensor(data).linear(x, wl.F16)
    assert_out(run_gemv(vqlib, data, x, wl.F16), ref)


@pytest.mark.parametrize("batch", [1, 8])
def test_c3_expert_gemv(vqlib, batch):
    data, x = wl.c3_expert_gemv(batch=batch)
    ref = oracle.Tensor(data).linear(x, wl.F16)
    assert_out(run_gemv(vqlib, data, x, wl.F16), ref)


def test_c2_mlp_decode_full(vqlib):
    """Dense MLP trio (gate/up 17408x5120, down 5120x17408, d2/K256 k-means codebooks),
    batch-1 decode: every output against the oracle."""
    gate, up, down = wl.c2_mlp_tensors(device="cuda")
    for i, data in enumerate((gate, up, down)):
        x = wl.activations(1, data.cols, seed=wl.BASE_SEED + 10 + i, dtype=wl.F16)
        ref = oracle.Tensor(data).linear(x, wl.F16)
        y = run_gemv(vqlib, data, x, wl.F16)
        assert_out(y, ref)
        assert normwise(y.cpu().numpy(), ref) <= GEMV_F32_TOL


@pytest.mark.parametrize("d,bits", GEOMS)
@pytest.mark.parametrize("rows", [8, 148, 301, 1000])
@pytest.mark.parametrize("cols", [512, 1536, 4608, 17408])
@pytest.mark.parametrize("batch", [1, 9])
def test_gemv_tensor_core_path(vqlib, d, bits, rows, cols, batch):
    """Shapes taken by the tensor-core GEMV (fp16 activations, scale rows of whole 16-byte
    units): ragged 8-row blocks per CTA, 8 to 272 scale groups per row, tokens in the
    MMA's first and second row halves, activations from shared and from global memory."""
    data = wl.uniform_tensor(rows, cols, d, bits, seed=rows * 3 + cols + d * 5 + bits + batch)
    x = wl.activations(batch, cols, seed=cols + batch, dtype=wl.F16)
    ref = oracle.Tensor(data).linear(x, wl.F16)
    assert_out(run_gemv(vqlib, data, x, wl.F16), ref)


@pytest.mark.parametrize("xt", [wl.BF16, wl.F32])
def test_gemv_non_fp16_activations_large(vqlib, xt):
    data = wl.uniform_tensor(400, 1024, 8, 12, seed=31)
    x = wl.activations(1, 1024, seed=32, dtype=xt)
    ref = oracle.Tensor(data).linear(x, xt)
    assert_out(run_gemv(vqlib, data, x, xt), ref)

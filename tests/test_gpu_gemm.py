"""Prefill GEMM (vq_gemm, tcgen05 tensor cores) against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_util import NORMWISE_TOL, normwise, to_np, x_tensor
from oracle_pins import encode_dense

pytestmark = pytest.mark.gpu

GEOMS = [(2, 8), (4, 8), (8, 8), (2, 12), (4, 12), (8, 12)]
# fp16 tiles: each weight is rounded once to fp16 (relative 2^-11); the normwise error of
# an fp32-accumulated product is then ~2e-4, an order below the 2e-3 gate.
F16_TILE_EXPECT = 6e-4
# bf16 tiles: weights rounded to bf16 (relative 2^-8): ~1.5e-3 normwise (documented option).
BF16_TILE_BOUND = 3e-3


def run_gemm(vqlib, W, xbits, xt, out=torch.float32, flags=0):
    x = x_tensor(xbits, xt)
    M = xbits.shape[0]
    y = torch.full((M, W.rows), float("nan"), dtype=out, device="cuda")
    n = vqlib.vq_gemm_workspace_size(W, x.dtype, M, flags)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device="cuda") if n else None
    vqlib.vq_gemm(W, x, y, ws, flags)
    torch.cuda.synchronize()
    assert vqlib.vq_read_device_status(None) == 0
    return y


@pytest.mark.parametrize("d,bits", GEOMS)
@pytest.mark.parametrize("M", [1, 16, 33, 128, 256, 300])
def test_gemm_integer_exact(vqlib, d, bits, M):
    """Integer weights and activations: every partial sum is an integer below 2^24, so the
    fp16 tiles and the fp32 tensor-core accumulation are exact and the result must equal
    the exact integer product bit for bit (any misplaced tile element changes it)."""
    rng = np.random.default_rng(M * 7 + d + bits)
    rows, cols = 200, 512
    pool = rng.integers(-6, 7, (min(1 << bits, 200), d))          # <= K distinct subvectors
    Wi = pool[rng.integers(0, pool.shape[0], (rows, cols // d))].reshape(rows, cols).astype(np.int64)
    xi = rng.integers(-8, 9, (M, cols)).astype(np.int64)
    data = encode_dense(Wi.astype(np.float32), d, bits)
    W = vqlib.VQMatrix.from_data(data)
    y = run_gemm(vqlib, W, wl.activation_bits(xi.astype(np.float32), wl.F16), wl.F16)
    assert np.array_equal(to_np(y), (xi @ Wi.T).astype(np.float64))


@pytest.mark.parametrize("d,bits", GEOMS)
def test_gemm_integer_exact_192_token_tiles(vqlib, d, bits):
    """2048 weight rows x 512 tokens: on 148 SMs 192-token tiles fill the CTA waves better
    than 256-token ones (48 vs 32 CTAs), so this shape takes the 192-token tiles, with a
    ragged last tile of 128 tokens; integer data makes the result exact."""
    rng = np.random.default_rng(d * 31 + bits)
    rows, cols, M = 2048, 512, 512
    pool = rng.integers(-6, 7, (min(1 << bits, 200), d))
    Wi = pool[rng.integers(0, pool.shape[0], (rows, cols // d))].reshape(rows, cols).astype(np.int64)
    xi = rng.integers(-8, 9, (M, cols)).astype(np.int64)
    data = encode_dense(Wi.astype(np.float32), d, bits)
    W = vqlib.VQMatrix.from_data(data)
    y = run_gemm(vqlib, W, wl.activation_bits(xi.astype(np.float32), wl.F16), wl.F16)
    assert np.array_equal(to_np(y), (xi @ Wi.T).astype(np.float64))


@pytest.mark.parametrize("d,bits", GEOMS)
@pytest.mark.parametrize("rows,cols,M", [(128, 64, 40), (200, 320, 256), (384, 1024, 513), (130, 2048, 64),
                                         (2048, 1024, 500)])
def test_gemm_vs_oracle(vqlib, d, bits, rows, cols, M):
    data = wl.uniform_tensor(rows, cols, d, bits, seed=rows + cols + M + d)
    x = wl.activations(M, cols, seed=M, dtype=wl.F16)
    ref = oracle.Tensor(data).linear(x, wl.F16)
    y = run_gemm(vqlib, vqlib.VQMatrix.from_data(data), x, wl.F16)
    e = normwise(to_np(y), ref)
    assert e <= min(NORMWISE_TOL, F16_TILE_EXPECT), e


@pytest.mark.parametrize("out", [torch.float32, torch.float16, torch.bfloat16])
def test_gemm_bf16_activations_and_outputs(vqlib, out):
    data = wl.uniform_tensor(256, 512, 4, 8, seed=3)
    x = wl.activations(96, 512, seed=4, dtype=wl.BF16)
    ref = oracle.Tensor(data).linear(x, wl.BF16)
    y = run_gemm(vqlib, vqlib.VQMatrix.from_data(data), x, wl.BF16, out=out)
    e = normwise(to_np(y), ref)
    bound = {torch.float32: F16_TILE_EXPECT, torch.float16: 1e-3, torch.bfloat16: 5e-3}[out]
    assert e <= bound, e


def test_gemm_bf16_tiles_option(vqlib):
    data = wl.uniform_tensor(256, 1024, 2, 8, seed=5)
    x = wl.activations(256, 1024, seed=6, dtype=wl.BF16)
    ref = oracle.Tensor(data).linear(x, wl.BF16)
    y = run_gemm(vqlib, vqlib.VQMatrix.from_data(data), x, wl.BF16, flags=vqlib.VQ_GEMM_BF16_TILES)
    e = normwise(to_np(y), ref)
    assert e <= BF16_TILE_BOUND, e


def test_gemm_workspace_rules(vqlib):
    data = wl.uniform_tensor(128, 256, 4, 8, seed=7)
    W = vqlib.VQMatrix.from_data(data)
    assert vqlib.vq_gemm_workspace_size(W, torch.float16, 100) == 0
    assert vqlib.vq_gemm_workspace_size(W, torch.bfloat16, 100) >= 100 * 256 * 2
    assert vqlib.vq_gemm_workspace_size(W, torch.bfloat16, 100, vqlib.VQ_GEMM_BF16_TILES) == 0
    x = torch.zeros((100, 256), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((100, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(vqlib.VQError) as e:
        vqlib.vq_gemm(W, x, y, None)
    assert e.value.status == vqlib.VQ_ERR_WORKSPACE


def test_c2_mlp_prefill_sampled(vqlib):
    """Dense MLP trio, 2048-token bf16 prefill (the bench launch configuration): 4096
    sampled outputs per projection against the oracle, plus finiteness of all outputs."""
    gate, up, down = wl.c2_mlp_tensors(device="cuda")
    rng = np.random.default_rng(0)
    for i, data in enumerate((gate, up, down)):
        x = wl.activations(2048, data.cols, seed=wl.BASE_SEED + 20 + i, dtype=wl.BF16)
        W = vqlib.VQMatrix.from_data(data)
        y = run_gemm(vqlib, W, x, wl.BF16)
        assert torch.isfinite(y).all()
        ms, rs = rng.integers(0, 2048, 4096), rng.integers(0, data.rows, 4096)
        ref = oracle.Tensor(data).linear_sampled(x, wl.BF16, ms, rs)
        got = to_np(y)[ms, rs]
        e = normwise(got, ref)
        assert e <= min(NORMWISE_TOL, F16_TILE_EXPECT), (i, e)

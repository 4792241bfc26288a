"""vq_pack / vq_unpack / vq_dequant on the GPU against the CPU oracle: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from workloads import uniform_tensor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits", [8, 12, 1, 3, 4, 5, 7, 9, 10, 11, 13, 16])
@pytest.mark.parametrize("ncodes", [1, 31, 32, 33, 1000])
def test_pack_unpack_bit_exact(vqlib, bits, ncodes):
    rng = np.random.default_rng(bits * 1000 + ncodes)
    rows = 7
    codes = rng.integers(0, 1 << bits, (rows, ncodes), dtype=np.uint32).astype(np.uint16)
    want = oracle.pack(codes, bits)
    rb = want.shape[1]
    rb_pad = (rb + 15) // 16 * 16 + 16                     # extra padding bytes must be 0
    dcodes = torch.from_numpy(codes.view(np.int16)).cuda()
    packed = torch.full((rows, rb_pad), 0xAB, dtype=torch.uint8, device="cuda")
    vqlib.vq_pack(dcodes, rows, ncodes, bits, packed, rb_pad)
    got = packed.cpu().numpy()
    assert np.array_equal(got[:, :rb], want)
    assert not got[:, rb:].any()
    back = torch.zeros((rows, ncodes), dtype=torch.int16, device="cuda")
    vqlib.vq_unpack(packed, rows, ncodes, bits, rb_pad, back)
    assert np.array_equal(back.cpu().numpy().view(np.uint16), codes)


def test_pack8_is_zero_copy(vqlib):
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 256, (5, 256), dtype=np.uint16)
    packed = torch.empty((5, 256), dtype=torch.uint8, device="cuda")
    vqlib.vq_pack(torch.from_numpy(codes.view(np.int16)).cuda(), 5, 256, 8, packed, 256)
    assert np.array_equal(packed.cpu().numpy(), codes.astype(np.uint8))


GEOMS = [(2, 8), (4, 8), (8, 8), (2, 12), (4, 12), (8, 12)]


@pytest.mark.parametrize("d,bits", GEOMS)
@pytest.mark.parametrize("rows,cols", [(5, 64), (33, 192), (16, 1024)])
def test_dequant_bit_exact(vqlib, d, bits, rows, cols):
    data = uniform_tensor(rows, cols, d, bits, seed=17 * d + bits + rows, experts=3, per_expert_codebook=True)
    ot = oracle.Tensor(data)
    W = vqlib.VQMatrix.from_data(data)
    for e in (0, 2):
        ref = ot.dequant(e)
        out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
        vqlib.vq_dequant(W, e, out)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        for dt in (torch.float16, torch.bfloat16):
            out16 = torch.empty((rows, cols), dtype=dt, device="cuda")
            vqlib.vq_dequant(W, e, out16)
            want = torch.from_numpy(ref).to(dt)                     # round to nearest even
            assert torch.equal(out16.cpu().view(torch.int16), want.view(torch.int16))


def test_codes_roundtrip_through_matrix(vqlib):
    data = uniform_tensor(40, 640, 4, 12, seed=99)
    W = vqlib.VQMatrix.from_data(data)
    ncodes = 640 // 4
    back = torch.empty((40, ncodes), dtype=torch.int16, device="cuda")
    vqlib.vq_unpack(W.codes[0], 40, ncodes, 12, W.codes.shape[2], back)
    assert np.array_equal(back.cpu().numpy().view(np.uint16), data.codes[0])
    want = oracle.Tensor(data).codes[0]
    assert np.array_equal(W.codes[0].cpu().numpy()[:, : want.shape[1]], want)

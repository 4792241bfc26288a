"""Pins of the CPU oracle to values the pages or mathematics fix.

Each `pin_*` function takes a loaded oracle library (ctypes handle) and raises
AssertionError when the oracle disagrees.  `tests/test_oracle_pins.py` runs them on the
real oracle; `tests/test_oracle_mutants.py` runs them on copies of the oracle with a
planted mistake and requires that some pin fails for every mistake.

None of these recomputes the oracle's formulas: expected values come from the golden
files (the pages' printed numbers, hand-derived bytes, hand-multiplied weights), from
exact integer arithmetic on a dense matrix built first and encoded afterwards (so the
check runs the encoding backwards), from numpy/torch library routines, or from
identities of the SiLU function.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle
from workloads import F16, BF16, F32, VQTensorData

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def f16(vals) -> np.ndarray:
    return np.asarray(vals, np.float32).astype(np.float16).view(np.uint16)


# ---------------------------------------------------------------- encoding from dense W

def encode_dense(W: np.ndarray, d: int, bits: int, scales: np.ndarray | None = None) -> VQTensorData:
    """Build codebook/codes/scales that reproduce the dense matrix W exactly.

    W [rows][cols] must be exactly representable as scale * fp16 entry.  The codebook
    is the list of distinct scaled-down subvectors (so it needs <= 2^bits of them)."""
    rows, cols = W.shape
    if scales is None:
        scales = np.ones((rows, cols // 64), np.float32)
    S = np.repeat(scales, 64, axis=1)
    V = (W / S).reshape(rows, cols // d, d).astype(np.float16)
    assert np.array_equal(V.astype(np.float32).reshape(rows, cols) * S, W), "W not encodable"
    flat = V.reshape(-1, d)
    uniq, inv = np.unique(flat.view(np.uint16), axis=0, return_inverse=True)
    K = 1 << bits
    assert uniq.shape[0] <= K
    cb = np.zeros((1, K, d), np.uint16)
    cb[0, : uniq.shape[0]] = uniq
    codes = inv.reshape(1, rows, cols // d).astype(np.uint16)
    return VQTensorData(rows, cols, d, bits, cb, codes, f16(scales).reshape(1, rows, cols // 64))


# ---------------------------------------------------------------- pins: sizes and rates

def pin_bpw(L):
    """Bits per weight of each printed geometry from the oracle's row size."""
    for line in _golden_lines("bpw.txt"):
        spec = line.split("|")[0].split()
        d, K, kind, val = int(spec[0]), int(spec[1]), spec[2], float(spec[3])
        bits = int(round(math.log2(K)))
        cols = 64 * 32 * 8                      # whole 32-code blocks for every d
        code_bits = 8 * oracle.code_row_bytes(cols // d, bits, L) / cols
        got = code_bits + (16 / 64 if kind == "total" else 0.0)
        assert got == val, (line, got)


def pin_tensor_bytes(L):
    """Stored bytes of every workload tensor equal rows*cols*bpw/8."""
    for line in _golden_lines("tensor_bytes.txt"):
        name, rows, cols, d, K, bpw = line.split()
        rows, cols, d, K, bpw = int(rows), int(cols), int(d), int(K), float(bpw)
        bits = int(round(math.log2(K)))
        stored = rows * oracle.code_row_bytes(cols // d, bits, L) + rows * (cols // 64) * 2
        assert stored * 8 == rows * cols * bpw, (name, stored)


# ---------------------------------------------------------------- pins: packing

def pin_pack_bytes(L):
    """Hand-derived packed bytes (golden) and their inverse."""
    for line in _golden_lines("pack_bytes.txt"):
        bits_s, codes_s, bytes_s = (p.strip() for p in line.split("|"))
        bits = int(bits_s)
        codes = np.array([int(c, 16) for c in codes_s.split()], np.uint16)[None, :]
        want = [int(b, 16) for b in bytes_s.split()]
        packed = oracle.pack(codes, bits, L=L)
        rb = ((codes.shape[1] + 31) // 32) * 4 * bits
        assert packed.shape == (1, rb), (line, packed.shape)
        assert list(packed[0, : len(want)]) == want, (line, packed[0, : len(want)])
        assert not packed[0, len(want):].any(), line
        assert np.array_equal(oracle.unpack(packed, codes.shape[1], bits, L=L), codes), line


def pin_pack8_zero_copy(L):
    """uint8 codes are their own packed-8 layout (and read as LSB-first uint32 words)."""
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (3, 96), dtype=np.uint16)
    packed = oracle.pack(codes, 8, L=L)
    assert np.array_equal(packed, codes.astype(np.uint8))
    words = packed.view("<u4")
    for i in range(96):
        assert ((words[:, i // 4] >> (8 * (i % 4))) & 0xFF == codes[:, i]).all()


def pin_pack12_bigint(L):
    """12-bit rows read back as one little-endian integer: code i = (v >> 12 i) & 0xfff,
    over every 12-bit value, with a ragged row length."""
    rng = np.random.default_rng(6)
    codes = np.concatenate([np.arange(4096, dtype=np.uint16),
                            rng.integers(0, 4096, 4 * 1043 - 4096, dtype=np.uint16)]).reshape(4, 1043)
    packed = oracle.pack(codes, 12, L=L)
    assert packed.shape[1] == 33 * 48
    for r in range(4):
        v = int.from_bytes(packed[r].tobytes(), "little")
        got = [(v >> (12 * i)) & 0xFFF for i in range(1043)]
        assert got == codes[r].tolist()
        assert v >> (12 * 1043) == 0               # padding codes are zero
    assert np.array_equal(oracle.unpack(packed, 1043, 12, L=L), codes)


def pin_pack_roundtrip_widths(L):
    """pack then unpack is the identity for every width 1..16 and ragged rows."""
    rng = np.random.default_rng(7)
    for bits in range(1, 17):
        for ncodes in (1, 31, 32, 33, 100):
            codes = rng.integers(0, 1 << bits, (3, ncodes), dtype=np.uint32).astype(np.uint16)
            packed = oracle.pack(codes, bits, L=L)
            assert packed.shape[1] == ((ncodes + 31) // 32) * 4 * bits
            v = int.from_bytes(packed[1].tobytes(), "little")
            assert [(v >> (bits * i)) & ((1 << bits) - 1) for i in range(ncodes)] == codes[1].tolist()
            assert np.array_equal(oracle.unpack(packed, ncodes, bits, L=L), codes)


# ---------------------------------------------------------------- pins: number formats

def pin_half_all(L):
    """All 65,536 fp16 patterns against numpy's conversion."""
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.half_to_float(h, L)
    want = h.view(np.float16).astype(np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


def pin_bf16_all(L):
    """All 65,536 bf16 patterns against torch's conversion."""
    import torch

    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_float(b, L)
    want = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


# ---------------------------------------------------------------- pins: dequantize

def pin_dequant_tiny(L):
    """The hand-multiplied tensor of golden/dequant_tiny.json, bit for bit."""
    with open(os.path.join(GOLDEN, "dequant_tiny.json")) as f:
        g = json.load(f)
    d, bits, cols = g["d"], g["bits"], g["cols"]
    cb = np.zeros((1, 1 << bits, d), np.float32)
    for k, v in g["codebook_entries"].items():
        cb[0, int(k)] = v
    rows = len(g["rows"])
    codes = np.zeros((1, rows, cols // d), np.uint16)
    scales = np.zeros((1, rows, cols // 64), np.float32)
    want = np.zeros((rows, cols), np.float32)
    for r, row in enumerate(g["rows"]):
        pat = row["codes_pattern"]
        codes[0, r] = np.tile(pat, (cols // d) // len(pat))
        scales[0, r] = row["scales"]
        for gi, key in enumerate(("expected_first_group_pattern", "expected_second_group_pattern")):
            p = row[key]
            want[r, 64 * gi: 64 * gi + 64] = np.tile(p, 64 // len(p))
    data = VQTensorData(rows, cols, d, bits, f16(cb), codes, f16(scales))
    got = oracle.Tensor(data, L).dequant()
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]


def _dyadic_dense(rng, rows, cols, d, bits, pool=24):
    """Dense W whose subvectors come from a small pool of dyadic vectors, with
    power-of-two group scales; returns (W, scales)."""
    vecs = rng.integers(-8, 9, (pool, d)).astype(np.float32) / 4.0
    pick = rng.integers(0, pool, (rows, cols // d))
    V = vecs[pick].reshape(rows, cols)
    scales = (2.0 ** rng.integers(-3, 3, (rows, cols // 64))).astype(np.float32)
    return V * np.repeat(scales, 64, axis=1), scales


def pin_dequant_reconstructs(L):
    """Encoding a dense matrix and dequantizing it gives the matrix back exactly, for
    every geometry the library builds (codebook = the matrix's own subvectors)."""
    rng = np.random.default_rng(8)
    for d in (2, 4, 8):
        for bits in (8, 12):
            W, s = _dyadic_dense(rng, 6, 192, d, bits)
            got = oracle.Tensor(encode_dense(W, d, bits, s), L).dequant()
            assert np.array_equal(got, W), (d, bits)


# ---------------------------------------------------------------- pins: multiply

def pin_linear_bruteforce_8x64(L):
    """8x64 integer-valued W and x: the exact integer product (numpy int64)."""
    rng = np.random.default_rng(9)
    for d, bits in ((4, 8), (2, 8), (8, 12)):
        Wi = rng.integers(-6, 7, (8, 64)).astype(np.int64)
        xi = rng.integers(-8, 9, (8, 64)).astype(np.int64)
        data = encode_dense(Wi.astype(np.float32), d, bits)
        want = xi @ Wi.T
        for xt in (F16, BF16, F32):
            from workloads import activation_bits
            xb = activation_bits(xi.astype(np.float32), xt)
            got = oracle.Tensor(data, L).linear(xb, xt)
            assert np.array_equal(got, want.astype(np.float64)), (d, bits, xt)


def pin_linear_matches_library_matmul(L):
    """Codebook = the exact fp16 subvectors, scales = 1: the product reduces to a plain
    dense matmul (numpy float64), for real-valued data and a ragged shape."""
    rng = np.random.default_rng(10)
    for d, bits, rows, cols in ((2, 8, 4, 128), (4, 8, 7, 128), (8, 12, 33, 320)):
        W = rng.standard_normal((rows, cols)).astype(np.float16).astype(np.float32)
        data = encode_dense(W, d, bits)
        x = rng.standard_normal((5, cols)).astype(np.float16)
        want = x.astype(np.float64) @ W.astype(np.float64).T
        got = oracle.Tensor(data, L).linear(x.view(np.uint16), F16)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12), (d, bits)
        ms, rs = rng.integers(0, 5, 17), rng.integers(0, rows, 17)
        smp = oracle.Tensor(data, L).linear_sampled(x.view(np.uint16), F16, ms, rs)
        assert np.array_equal(smp, got[ms, rs])


# ---------------------------------------------------------------- pins: MoE layer

def _eye_tensor(rows, cols, d, bits, col_of_row, gain=1.0, experts=1):
    """Selection matrix W[i][col_of_row[i]] = gain (others 0), encoded exactly."""
    W = np.zeros((rows, cols), np.float32)
    W[np.arange(rows), col_of_row] = gain
    data = encode_dense(W, d, bits)
    if experts > 1:
        data = VQTensorData(rows, cols, d, bits, data.codebook,
                            np.repeat(data.codes, experts, 0), np.repeat(data.scales, experts, 0))
    return data


def pin_moe_silu_identities(L):
    """Gate = identity, up = ones, down = identity -> y = silu(x).  SiLU satisfies
    silu(a) - silu(-a) = a and silu(a) + silu(-a) = a tanh(a/2); silu(0) = 0.  Mixed
    geometries per projection (d8/12-bit gate, d4/8-bit up, d2/8-bit down)."""
    H = 64
    a = np.array([0.0, 0.25, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0, 0.125, 6.0, 7.0, 8.0, 0.75, 1.25, 2.5,
                  3.5, 0.375, 9.0, 10.0, 0.0625, 11.0, 12.0, 1.75, 2.25, 13.0, 14.0, 15.0, 0.875, 5.5, 6.5],
                 np.float32)
    x = np.zeros((1, H), np.float32)
    x[0, 0:62:2], x[0, 1:62:2] = a, -a
    x[0, 62], x[0, 63] = 0.0, 1.0
    gate = oracle.Tensor(_eye_tensor(H, H, 8, 12, np.arange(H)), L)
    up = oracle.Tensor(_eye_tensor(H, H, 4, 8, np.full(H, 63)), L)
    down = oracle.Tensor(_eye_tensor(H, H, 2, 8, np.arange(H)), L)
    y, bad = oracle.moe_tokens(gate, up, down, f16(x), F16, [0],
                               np.zeros((1, 1), np.int32), np.ones((1, 1), np.float32))
    assert bad == 0
    y = y[0]
    assert np.allclose(y[0:62:2] - y[1:62:2], a, rtol=1e-12, atol=1e-12)
    assert np.allclose(y[0:62:2] + y[1:62:2], a * np.tanh(a.astype(np.float64) / 2), rtol=1e-12, atol=1e-12)
    assert y[62] == 0.0


def pin_moe_combine(L):
    """Two experts differing only in the up projection (gain 1 vs 2), routing weights
    0.25 / 0.75: y = (0.25 + 2*0.75) * y_single.  An out-of-range id is skipped and
    counted; the remaining slot still contributes."""
    H = 64
    x = f16(np.linspace(-3, 3, H, dtype=np.float32)[None, :])
    gate = oracle.Tensor(_eye_tensor(H, H, 4, 8, np.arange(H), experts=2), L)
    up1 = _eye_tensor(H, H, 4, 8, np.arange(H))
    up2 = _eye_tensor(H, H, 4, 8, np.arange(H), gain=2.0)
    up = oracle.Tensor(VQTensorData(H, H, 4, 8, np.concatenate([up1.codebook, up2.codebook]),
                                    np.concatenate([up1.codes, up2.codes]),
                                    np.concatenate([up1.scales, up2.scales])), L)
    down = oracle.Tensor(_eye_tensor(H, H, 4, 8, np.arange(H), experts=2), L)
    one, _ = oracle.moe_tokens(gate, up, down, x, F16, [0], np.zeros((1, 1), np.int32),
                               np.ones((1, 1), np.float32))
    both, bad = oracle.moe_tokens(gate, up, down, x, F16, [0], np.array([[0, 1]], np.int32),
                                  np.array([[0.25, 0.75]], np.float32))
    assert bad == 0 and np.allclose(both, 1.75 * one, rtol=1e-12, atol=1e-14)
    skip, bad = oracle.moe_tokens(gate, up, down, x, F16, [0], np.array([[0, 7]], np.int32),
                                  np.array([[0.25, 0.75]], np.float32))
    assert bad == 1 and np.allclose(skip, 0.25 * one, rtol=1e-12, atol=1e-14)


def pin_moe_structure(L):
    """Identical experts with weights summing to 1 equal one dense FFN; permuting the
    tokens permutes the outputs; top-1 with weight 1 equals the expert's FFN built from
    three linear calls."""
    from workloads import uniform_tensor, routing

    rng = np.random.default_rng(11)
    E, H, I, T, k = 4, 128, 64, 5, 3
    g1 = uniform_tensor(I, H, 4, 8, 21)
    u1 = uniform_tensor(I, H, 8, 12, 22)
    d1 = uniform_tensor(H, I, 2, 8, 23)
    rep = lambda t: VQTensorData(t.rows, t.cols, t.d, t.bits, t.codebook,
                                 np.repeat(t.codes, E, 0), np.repeat(t.scales, E, 0))
    G, U, D = (oracle.Tensor(rep(t), L) for t in (g1, u1, d1))
    x = f16(rng.standard_normal((T, H)).astype(np.float32))
    ids, _ = routing(T, E, k, 31)
    w = np.tile(np.array([0.5, 0.25, 0.25], np.float32), (T, 1))   # sums to 1 exactly
    y, _ = oracle.moe_tokens(G, U, D, x, F16, np.arange(T), ids, w)
    y1, _ = oracle.moe_tokens(G, U, D, x, F16, np.arange(T), np.zeros((T, 1), np.int32),
                              np.ones((T, 1), np.float32))
    assert np.allclose(y, y1, rtol=1e-10, atol=1e-12)
    perm = rng.permutation(T)
    yp, _ = oracle.moe_tokens(G, U, D, x[perm], F16, np.arange(T), ids[perm], w[perm])
    assert np.array_equal(yp, y[perm])
    g = G.linear(x, F16)
    u = U.linear(x, F16)
    h = g / (1.0 + np.exp(-g)) * u
    o = h @ D.dequant().astype(np.float64).T
    assert np.allclose(y1, o, rtol=1e-9, atol=1e-12)


ALL_PINS = [pin_bpw, pin_tensor_bytes, pin_pack_bytes, pin_pack8_zero_copy, pin_pack12_bigint,
            pin_pack_roundtrip_widths, pin_half_all, pin_bf16_all, pin_dequant_tiny,
            pin_dequant_reconstructs, pin_linear_bruteforce_8x64,
            pin_linear_matches_library_matmul, pin_moe_silu_identities, pin_moe_combine,
            pin_moe_structure]

"""Seeded synthetic inputs for the VQ dequantize-and-multiply path.

This module is the one piece both the CUDA path's tests/benchmark and the CPU oracle
consume.  It produces raw inputs only (unpacked codes, fp16 codebooks and scales as
uint16 bit patterns, activations, routing) and holds none of the path's arithmetic:
no packing, no dequantization, no matmul, no MoE evaluation.

Recipes (the pages' workloads are real Qwen checkpoints, which are not available;
these synthetic tensors take the shapes of the five workloads and stand in for them):

* Uniform tensors: codebook entries ~ N(0, 1) rounded to fp16, scales = |N(0, 0.02)|
  rounded to fp16, codes uniform on [0, K).
* k-means tensors (the dense MLP trio): weights ~ N(0, 0.02^2); per (row, 64) group
  the scale is the group's max-abs value rounded to fp16 (paper "Data-Free Vector
  Quantization Beats Affine Quantization at Matched Bytes Below 5 Bits", §2.2 The
  fit); the weights divided by their scale are cut into d-vectors; a K-entry codebook
  is fit by k-means++ seeding and 10 Lloyd iterations on a seeded subsample of 65,536
  subvectors (seed 1234, §2.6), rounded to fp16; every subvector takes the index of
  its nearest codebook entry.  This is input synthesis, not part of the checked path.
* Activations ~ N(0, 1) rounded to the requested 16-bit type.
* Routing: logits ~ N(0, 1) of shape [T][E]; softmax; top-k experts by probability
  (ties to the lower id); the k weights renormalised to sum to 1.

Seeds: base 1234; every tensor of a workload draws from base + its ordinal.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

BASE_SEED = 1234

F16, BF16, F32 = 0, 1, 2          # activation / output type codes used by both sides
DTYPE_NAMES = {F16: "f16", BF16: "bf16", F32: "f32"}


@dataclasses.dataclass
class VQTensorData:
    """Raw contents of one VQ tensor (or an expert stack of them), unpacked."""

    rows: int
    cols: int
    d: int
    bits: int
    codebook: np.ndarray      # uint16 fp16 bits, [n_codebooks][K][d]
    codes: np.ndarray         # uint8 (bits <= 8) or uint16, [E][rows][cols // d]
    scales: np.ndarray        # uint16 fp16 bits, [E][rows][cols // 64]

    @property
    def num_experts(self) -> int:
        return int(self.codes.shape[0])

    @property
    def K(self) -> int:
        return 1 << self.bits

    @property
    def ncodes(self) -> int:
        return self.cols // self.d

    @property
    def shared_codebook(self) -> bool:
        return self.codebook.shape[0] == 1


def _f16_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a.astype(np.float16)).view(np.uint16)


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def activation_bits(a: np.ndarray, dtype: int) -> np.ndarray:
    """fp32 array -> raw bits of the requested activation type (uint16 or float32)."""
    if dtype == F16:
        return _f16_bits(a)
    if dtype == BF16:
        return _bf16_bits(a)
    return np.ascontiguousarray(a, dtype=np.float32)


def uniform_tensor(rows: int, cols: int, d: int, bits: int, seed: int,
                   experts: int = 1, per_expert_codebook: bool = False) -> VQTensorData:
    """Codebook ~ N(0,1), scales = |N(0,0.02)|, codes uniform (fp16 where stored)."""
    if cols % 64 or 64 % d:
        raise ValueError("cols must be a multiple of 64 and d must divide 64")
    rng = np.random.default_rng(seed)
    K = 1 << bits
    ncb = experts if per_expert_codebook else 1
    codebook = _f16_bits(rng.standard_normal((ncb, K, d), dtype=np.float32))
    scales = _f16_bits(np.abs(rng.normal(0.0, 0.02, (experts, rows, cols // 64))).astype(np.float32))
    codes = rng.integers(0, K, (experts, rows, cols // d), dtype=np.uint8 if bits <= 8 else np.uint16)
    return VQTensorData(rows, cols, d, bits, codebook, codes, scales)


def _kmeanspp(pts, K, rng, torch):
    """k-means++ seeding on a (small) point set held as a torch tensor."""
    n = pts.shape[0]
    centers = torch.empty((K, pts.shape[1]), dtype=pts.dtype, device=pts.device)
    first = int(rng.integers(0, n))
    centers[0] = pts[first]
    dist = ((pts - centers[0]) ** 2).sum(1)
    for k in range(1, K):
        p = dist.double().cpu().numpy()
        tot = p.sum()
        idx = int(rng.choice(n, p=p / tot)) if tot > 0 else int(rng.integers(0, n))
        centers[k] = pts[idx]
        dist = torch.minimum(dist, ((pts - centers[k]) ** 2).sum(1))
    return centers


def _nearest(pts, centers, torch, chunk=1 << 20):
    """Index of the nearest center (squared distance in fp32, ties to lower index)."""
    out = torch.empty(pts.shape[0], dtype=torch.int64, device=pts.device)
    cc = (centers * centers).sum(1)
    for s in range(0, pts.shape[0], chunk):
        p = pts[s:s + chunk]
        dist = cc[None, :] - 2.0 * (p @ centers.T) + (p * p).sum(1, keepdim=True)
        out[s:s + chunk] = torch.argmin(dist, dim=1)
    return out


def kmeans_tensor(rows: int, cols: int, d: int, bits: int, seed: int,
                  device: str = "cpu", sample: int = 65536, iters: int = 10) -> VQTensorData:
    """Gaussian weights fit by k-means on normalised subvectors (see module doc)."""
    import torch

    rng = np.random.default_rng(seed)
    K = 1 << bits
    w = rng.normal(0.0, 0.02, (rows, cols)).astype(np.float32)
    g = w.reshape(rows, cols // 64, 64)
    s16 = np.abs(g).max(axis=2).astype(np.float16)
    s32 = s16.astype(np.float32)
    s32[s32 == 0] = 1.0
    norm = (g / s32[:, :, None]).reshape(-1, d)
    del w, g
    pts = torch.from_numpy(norm).to(device)
    sub_idx = torch.from_numpy(rng.choice(pts.shape[0], size=min(sample, pts.shape[0]), replace=False)).to(device)
    sub = pts[sub_idx]
    centers = _kmeanspp(sub, K, rng, torch)
    for _ in range(iters):
        a = _nearest(sub, centers, torch)
        sums = torch.zeros_like(centers).index_add_(0, a, sub)
        cnt = torch.bincount(a, minlength=K).to(centers.dtype)
        keep = cnt > 0
        centers[keep] = sums[keep] / cnt[keep, None]
    cb16 = centers.cpu().numpy().astype(np.float16)
    codes = _nearest(pts, torch.from_numpy(cb16.astype(np.float32)).to(device), torch)
    codes = codes.to(torch.int32).cpu().numpy().astype(np.uint8 if bits <= 8 else np.uint16)
    codes = codes.reshape(1, rows, cols // d)
    return VQTensorData(rows, cols, d, bits, cb16.view(np.uint16).reshape(1, K, d),
                        codes, s16.view(np.uint16).reshape(1, rows, cols // 64))


def activations(M: int, cols: int, seed: int, dtype: int = F16) -> np.ndarray:
    """x ~ N(0, 1) of shape [M][cols] as raw bits of `dtype`."""
    rng = np.random.default_rng(seed)
    return activation_bits(rng.standard_normal((M, cols), dtype=np.float32), dtype)


def routing(T: int, E: int, topk: int, seed: int):
    """Seeded softmax top-k routing: (ids int32 [T][k], weights float32 [T][k])."""
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E))
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    order = np.argsort(-p, axis=1, kind="stable")[:, :topk]
    w = np.take_along_axis(p, order, axis=1)
    w = w / w.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w.astype(np.float32)


# ----------------------------------------------------------------------------- workloads

@dataclasses.dataclass
class MoEWorkload:
    gate: VQTensorData
    up: VQTensorData
    down: VQTensorData
    E: int
    topk: int
    hidden: int
    inter: int


def c1_single_gemv(seed: int = BASE_SEED):
    """Single VQ GEMV: W 1024x1024, d4/K256 uint8, x fp16 1x1024."""
    W = uniform_tensor(1024, 1024, 4, 8, seed)
    x = activations(1, 1024, seed + 1, F16)
    return W, x


def c2_mlp_tensors(seed: int = BASE_SEED, device: str = "cpu", scale: int = 1):
    """Dense MLP trio at d2/K256 with k-means codebooks: gate, up [17408][5120] and
    down [5120][17408].  `scale` > 1 divides both dimensions (small parity cases)."""
    inter, hidden = 17408 // scale, 5120 // scale
    gate = kmeans_tensor(inter, hidden, 2, 8, seed, device)
    up = kmeans_tensor(inter, hidden, 2, 8, seed + 1, device)
    down = kmeans_tensor(hidden, inter, 2, 8, seed + 2, device)
    return gate, up, down


def c3_expert_gemv(seed: int = BASE_SEED, batch: int = 1):
    """Expert GEMV at the 1.5-bit tier: W 512x2048, d8/K4096 12-bit, x fp16."""
    W = uniform_tensor(512, 2048, 8, 12, seed)
    x = activations(batch, 2048, seed + 1, F16)
    return W, x


def c4_moe(seed: int = BASE_SEED, E: int = 256, hidden: int = 2048, inter: int = 512):
    """MoE layer: 256 experts, top-8, gate d8/K4096, up d4/K256, down d4/K4096."""
    gate = uniform_tensor(inter, hidden, 8, 12, seed, experts=E)
    up = uniform_tensor(inter, hidden, 4, 8, seed + 1, experts=E)
    down = uniform_tensor(hidden, inter, 4, 12, seed + 2, experts=E)
    return MoEWorkload(gate, up, down, E, 8, hidden, inter)


def c5_moe_large(seed: int = BASE_SEED, E: int = 512, hidden: int = 4096, inter: int = 1024):
    """Large MoE layer: 512 experts, top-10, all d4/K256 uint8."""
    gate = uniform_tensor(inter, hidden, 4, 8, seed, experts=E)
    up = uniform_tensor(inter, hidden, 4, 8, seed + 1, experts=E)
    down = uniform_tensor(hidden, inter, 4, 8, seed + 2, experts=E)
    return MoEWorkload(gate, up, down, E, 10, hidden, inter)


def moe_inputs(wl: MoEWorkload, T: int, seed: int, dtype: int = F16):
    x = activations(T, wl.hidden, seed, dtype)
    ids, w = routing(T, wl.E, wl.topk, seed + 1)
    return x, ids, w

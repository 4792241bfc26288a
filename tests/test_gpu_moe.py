"""Routed MoE layer (vq_moe_grouped) against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_util import NORMWISE_TOL, normwise, to_np, x_tensor

pytestmark = pytest.mark.gpu

TORCH_OUT = {wl.F32: torch.float32, wl.F16: torch.float16, wl.BF16: torch.bfloat16}


def run_moe(vqlib, mw, x, xt, ids, w, yt=wl.F32):
    T = x.shape[0]
    G, U, D = (vqlib.VQMatrix.from_data(t) for t in (mw.gate, mw.up, mw.down))
    xd = x_tensor(x, xt)
    idd = torch.from_numpy(ids).cuda()
    wd = torch.from_numpy(w).cuda()
    y = torch.full((T, mw.hidden), float("nan"), dtype=TORCH_OUT[yt], device="cuda")
    n = vqlib.vq_moe_workspace_size(T, ids.shape[1], mw.E, mw.hidden, mw.inter)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    vqlib.vq_moe_grouped(G, U, D, xd, idd, wd, y, ws)
    st = vqlib.vq_read_device_status(ws)
    return y, st


def oracle_moe(mw, x, xt, ids, w, tokens):
    used = np.unique(ids[tokens])
    used = used[(used >= 0) & (used < mw.E)]
    ts = [oracle.Tensor(t, experts=used) for t in (mw.gate, mw.up, mw.down)]
    return oracle.moe_tokens(*ts, x, xt, tokens, ids, w)


def small_moe(E=8, hidden=256, inter=128, topk=2, geoms=((8, 12), (4, 8), (4, 12)), seed=1, per_expert_cb=False):
    (gd, gb), (ud, ub), (dd, db) = geoms
    gate = wl.uniform_tensor(inter, hidden, gd, gb, seed, experts=E, per_expert_codebook=per_expert_cb)
    up = wl.uniform_tensor(inter, hidden, ud, ub, seed + 1, experts=E, per_expert_codebook=per_expert_cb)
    down = wl.uniform_tensor(hidden, inter, dd, db, seed + 2, experts=E, per_expert_codebook=per_expert_cb)
    return wl.MoEWorkload(gate, up, down, E, topk, hidden, inter)


@pytest.mark.parametrize("T", [1, 3, 40, 300])
@pytest.mark.parametrize("geoms", [((8, 12), (4, 8), (4, 12)), ((2, 8), (2, 8), (2, 8)), ((4, 12), (8, 8), (2, 12))])
def test_moe_small(vqlib, T, geoms):
    mw = small_moe(geoms=geoms, seed=T)
    x, ids, w = wl.moe_inputs(mw, T, seed=T + 100)
    y, st = run_moe(vqlib, mw, x, wl.F16, ids, w)
    assert st == 0
    ref, bad = oracle_moe(mw, x, wl.F16, ids, w, np.arange(T))
    assert bad == 0
    assert normwise(to_np(y), ref) <= NORMWISE_TOL


@pytest.mark.parametrize("xt", [wl.F16, wl.BF16])
@pytest.mark.parametrize("yt", [wl.F32, wl.F16, wl.BF16])
def test_moe_dtypes_and_per_expert_codebooks(vqlib, xt, yt):
    mw = small_moe(per_expert_cb=True, seed=7, topk=3)
    x, ids, w = wl.moe_inputs(mw, 24, seed=8, dtype=xt)
    y, st = run_moe(vqlib, mw, x, xt, ids, w, yt)
    assert st == 0
    ref, _ = oracle_moe(mw, x, xt, ids, w, np.arange(24))
    bound = {wl.F32: NORMWISE_TOL, wl.F16: NORMWISE_TOL, wl.BF16: 6e-3}[yt]   # bf16 output rounding: 2^-8
    assert normwise(to_np(y), ref) <= bound


def test_moe_invalid_ids_are_skipped_and_flagged(vqlib):
    mw = small_moe(seed=9)
    x, ids, w = wl.moe_inputs(mw, 10, seed=10)
    ids[2, 0] = -1
    ids[5, 1] = mw.E
    ids[7, :] = 1000
    y, st = run_moe(vqlib, mw, x, wl.F16, ids, w)
    assert st == vqlib.VQ_ERR_DEVICE_FLAG
    ref, bad = oracle_moe(mw, x, wl.F16, ids, w, np.arange(10))
    assert bad == 4
    assert normwise(to_np(y), ref) <= NORMWISE_TOL
    assert (to_np(y)[7] == 0).all()
    # a clean call afterwards clears the flag
    x2, ids2, w2 = wl.moe_inputs(mw, 10, seed=11)
    _, st2 = run_moe(vqlib, mw, x2, wl.F16, ids2, w2)
    assert st2 == 0


def test_moe_all_tokens_one_expert(vqlib):
    mw = small_moe(seed=12, E=4, topk=1)
    x, _, _ = wl.moe_inputs(mw, 70, seed=13)
    ids = np.full((70, 1), 3, np.int32)
    w = np.ones((70, 1), np.float32)
    y, st = run_moe(vqlib, mw, x, wl.F16, ids, w)
    ref, _ = oracle_moe(mw, x, wl.F16, ids, w, np.arange(70))
    assert st == 0 and normwise(to_np(y), ref) <= NORMWISE_TOL


@pytest.mark.parametrize("T", [1, 16, 512])
def test_c4_moe_layer(vqlib, T):
    """256 experts, top-8, hidden 2048, inter 512, gate d8/K4096, up d4/K256, down
    d4/K4096; up to 16 sampled tokens compared with the oracle."""
    mw = wl.c4_moe()
    x, ids, w = wl.moe_inputs(mw, T, seed=wl.BASE_SEED + 50 + T)
    y, st = run_moe(vqlib, mw, x, wl.F16, ids, w)
    assert st == 0 and torch.isfinite(y).all()
    toks = np.arange(T) if T <= 16 else np.random.default_rng(T).choice(T, 16, replace=False)
    ref, _ = oracle_moe(mw, x, wl.F16, ids, w, toks)
    assert normwise(to_np(y)[toks], ref) <= NORMWISE_TOL


@pytest.mark.parametrize("T", [1, 1024])
def test_c5_moe_layer(vqlib, T):
    """512 experts, top-10, hidden 4096, inter 1024, all d4/K256; sampled tokens."""
    mw = wl.c5_moe_large()
    x, ids, w = wl.moe_inputs(mw, T, seed=wl.BASE_SEED + 60 + T)
    y, st = run_moe(vqlib, mw, x, wl.F16, ids, w)
    assert st == 0 and torch.isfinite(y).all()
    toks = np.arange(T) if T <= 8 else np.random.default_rng(T).choice(T, 8, replace=False)
    ref, _ = oracle_moe(mw, x, wl.F16, ids, w, toks)
    assert normwise(to_np(y)[toks], ref) <= NORMWISE_TOL


def test_moe_decode_path_token_chunks(vqlib):
    """Few tokens per expert on average (the tensor-core GEMV route) but one expert holds
    40 tokens: its tokens go through the MMA rows in chunks of 16."""
    mw = small_moe(E=64, seed=14, topk=1, hidden=512, inter=512)
    x, _, _ = wl.moe_inputs(mw, 40, seed=15)
    ids = np.full((40, 1), 3, np.int32)
    ids[::7, 0] = 5
    w = np.ones((40, 1), np.float32)
    y, st = run_moe(vqlib, mw, x, wl.F16, ids, w)
    ref, _ = oracle_moe(mw, x, wl.F16, ids, w, np.arange(40))
    assert st == 0 and normwise(to_np(y), ref) <= NORMWISE_TOL


@pytest.mark.parametrize("T", [1, 2, 7])
def test_moe_decode_path_bf16(vqlib, T):
    mw = small_moe(seed=16 + T, topk=2, E=16, hidden=512, inter=512)
    x, ids, w = wl.moe_inputs(mw, T, seed=17, dtype=wl.BF16)
    y, st = run_moe(vqlib, mw, x, wl.BF16, ids, w)
    ref, _ = oracle_moe(mw, x, wl.BF16, ids, w, np.arange(T))
    assert st == 0 and normwise(to_np(y), ref) <= NORMWISE_TOL


@pytest.mark.parametrize("T", [1, 3, 6])
@pytest.mark.parametrize("geoms", [((8, 12), (4, 8), (4, 12)), ((2, 8), (2, 8), (2, 8)), ((4, 12), (8, 8), (2, 12))])
def test_moe_decode_path_geometries(vqlib, T, geoms):
    """Layers whose scale rows are whole 16-byte units, few tokens per expert: the grouped
    tensor-core GEMV route, mixed tiers in one launch."""
    mw = small_moe(geoms=geoms, seed=20 + T, E=16, hidden=1024, inter=512)
    x, ids, w = wl.moe_inputs(mw, T, seed=T + 200)
    y, st = run_moe(vqlib, mw, x, wl.F16, ids, w)
    ref, bad = oracle_moe(mw, x, wl.F16, ids, w, np.arange(T))
    assert st == 0 and bad == 0
    assert normwise(to_np(y), ref) <= NORMWISE_TOL

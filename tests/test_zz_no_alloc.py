"""The allocation-free MoE entry point (vq_moe_grouped_noalloc) against the regular one.

Some callers cannot allocate device memory — for example code running where cudaMalloc
is not allowed, or a host without its own device allocator — so the library offers a
variant of the MoE layer that uses a fixed scratch array compiled into the library
instead of a caller-provided workspace.  This file is collected last on purpose; it must
pass both alone in a fresh process and after every other test."""
import numpy as np
import pytest
import torch

import workloads as wl
from gpu_util import NORMWISE_TOL, normwise, to_np, x_tensor

pytestmark = pytest.mark.gpu


def _layer(seed, E=16, hidden=512, inter=256):
    gate = wl.uniform_tensor(inter, hidden, 8, 12, seed, experts=E)
    up = wl.uniform_tensor(inter, hidden, 4, 8, seed + 1, experts=E)
    down = wl.uniform_tensor(hidden, inter, 4, 12, seed + 2, experts=E)
    return wl.MoEWorkload(gate, up, down, E, 4, hidden, inter)


def test_noalloc_matches_workspace_entry_twice(vqlib):
    mw = _layer(seed=71)
    G, U, D = (vqlib.VQMatrix.from_data(t) for t in (mw.gate, mw.up, mw.down))
    for call, (T, seed) in enumerate(((16, 72), (5, 73))):          # two calls in a row
        x, ids, w = wl.moe_inputs(mw, T, seed=seed)
        xd = x_tensor(x, wl.F16)
        idd, wd = torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda()
        ref = torch.empty((T, mw.hidden), dtype=torch.float32, device="cuda")
        ws = torch.empty(vqlib.vq_moe_workspace_size(T, mw.topk, mw.E, mw.hidden, mw.inter),
                         dtype=torch.uint8, device="cuda")
        vqlib.vq_moe_grouped(G, U, D, xd, idd, wd, ref, ws)
        got = torch.full((T, mw.hidden), float("nan"), dtype=torch.float32, device="cuda")
        vqlib.vq_moe_grouped_noalloc(G, U, D, xd, idd, wd, got)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all(), call
        assert normwise(to_np(got), to_np(ref)) <= NORMWISE_TOL, call
        assert torch.equal(got, ref), call          # same kernels, deterministic


def test_noalloc_rejects_oversized_calls(vqlib):
    mw = _layer(seed=74)
    G, U, D = (vqlib.VQMatrix.from_data(t) for t in (mw.gate, mw.up, mw.down))
    T = 4096                                               # needs far more than 16 MiB
    assert vqlib.vq_moe_workspace_size(T, mw.topk, mw.E, mw.hidden, mw.inter) > (16 << 20)
    x = torch.zeros((T, mw.hidden), dtype=torch.float16, device="cuda")
    ids = torch.zeros((T, mw.topk), dtype=torch.int32, device="cuda")
    w = torch.zeros((T, mw.topk), dtype=torch.float32, device="cuda")
    y = torch.zeros((T, mw.hidden), dtype=torch.float32, device="cuda")
    with pytest.raises(vqlib.VQError) as e:
        vqlib.vq_moe_grouped_noalloc(G, U, D, x, ids, w, y)
    assert e.value.status == vqlib.VQ_ERR_WORKSPACE

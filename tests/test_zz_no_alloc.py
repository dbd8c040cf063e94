"""The allocation-free entry point, vsa_forward_noalloc.

It serves callers that may not allocate device memory (strict memory
budgets, allocators that must own every byte, loops where cudaMalloc's
implicit synchronisation is not allowed). Its workspace is a fixed device
array inside libvsa.so. These checks call it through the C ABI and compare
it with the plan-based entry point on the same inputs, on two calls in a row
(the second with different inputs, so leftovers of the first call in the
shared array cannot leak into the result). This file is collected last and
passes both alone and after the other tests.
"""
import ctypes

import pytest
import torch

from trainable_block_sparse_cube_b200 import build as vsa_build
from trainable_block_sparse_cube_b200 import synth, vsa

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module")
def lib():
    vsa_build.build()
    assert torch.cuda.is_available(), "needs a CUDA device"
    return vsa.load()


def _noalloc(lib, wl, q, k, v, gc, gf):
    out = torch.empty_like(q)
    idx = torch.empty((wl.B, wl.heads, wl.C, wl.kcap), dtype=torch.int32, device=q.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    code = lib.vsa_forward_noalloc(p(q), p(k), p(v), p(gc), p(gf), wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, wl.topk,
                                   ctypes.c_float(wl.top_p), p(out), p(idx), stream)
    return code, out, idx


def test_noalloc_matches_plan_entry_point_twice(lib):
    wls = [
        synth.WORKLOADS["pretrain16k"].with_(name="na_a", heads=3, T=8, H=16, W=24, topk=5),
        synth.WORKLOADS["pretrain16k"].with_(name="na_b", heads=3, T=8, H=16, W=24, topk=5, seed=9),
    ]
    for wl in wls:  # two calls in a row on the same shape, different inputs
        q, k, v, gc, gf = (t.cuda() for t in synth.make_inputs(wl))
        plan = vsa.Plan(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, wl.topk)
        ref_out, ref_idx, _ = plan.run(q, k, v, gc, gf)
        plan.check()
        code, out, idx = _noalloc(lib, wl, q, k, v, gc, gf)
        torch.cuda.synchronize()
        assert code == 0, vsa.STATUS.get(code, code)
        assert torch.equal(idx, ref_idx)
        d = (out.float() - ref_out.float()).abs()
        assert d.max().item() <= MAX_ABS and d.mean().item() <= MEAN_ABS


def test_noalloc_topp_and_no_new_device_memory(lib):
    wl = synth.WORKLOADS["dynamic61k"].with_(name="na_p", heads=2, T=8, H=16, W=16)
    q, k, v, gc, gf = (t.cuda() for t in synth.make_inputs(wl))
    wl = wl.with_(kmin=4, kmax=min(128, wl.C))   # the one-call form's top-p clamp
    code, out0, idx0 = _noalloc(lib, wl, q, k, v, gc, gf)   # first call: device address set-up
    torch.cuda.synchronize()
    assert code == 0
    out = torch.empty_like(q)
    idx = torch.empty_like(idx0)
    free_before = torch.cuda.mem_get_info()[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    code = lib.vsa_forward_noalloc(p(q), p(k), p(v), p(gc), p(gf), wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, 0,
                                   ctypes.c_float(wl.top_p), p(out), p(idx), stream)
    torch.cuda.synchronize()
    assert code == 0
    assert torch.cuda.mem_get_info()[0] == free_before
    assert torch.equal(idx, idx0) and torch.equal(out, out0)
    plan = vsa.Plan(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, 0, wl.top_p, wl.kmin, wl.kmax)
    ref_out, ref_idx, _ = plan.run(q, k, v, gc, gf)
    plan.check()
    assert torch.equal(idx, ref_idx)
    d = (out.float() - ref_out.float()).abs()
    assert d.max().item() <= MAX_ABS and d.mean().item() <= MEAN_ABS


def test_noalloc_rejects_workspace_beyond_limit(lib):
    wl = synth.WORKLOADS["long61k_k32"]        # ~1.3 GB of workspace, far above the fixed array
    cfg = vsa.make_config(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, wl.topk)
    assert vsa.workspace_bytes(cfg) > (64 << 20)
    dummy = torch.empty(16, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    code = lib.vsa_forward_noalloc(p, p, p, p, p, wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, wl.topk,
                                   ctypes.c_float(0.0), p, p, None)
    assert code == 3   # VSA_ERR_UNSUPPORTED, nothing enqueued

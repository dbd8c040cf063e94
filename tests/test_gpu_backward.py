"""GPU parity of the backward pass (through the C ABI) against the fp64
backward oracle, with the selection held fixed.

The training forward must return the same output and selection as the plain
forward and save the fine output and the per-token log-sum-exp, both
compared with the oracle. The backward gradients (dq, dk, dv, dgate_c,
dgate_f) are compared element by element with the oracle's chain rule on the
GPU's own lists, on the small workloads in full and on the full-size
workloads at sampled query and KV cubes of a sampled head.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.vsa_oracle_backward import backward_head, fine_lse
from parity import assert_close, assert_close_rel, grad_tolerance, oracle_head
from test_gpu_parity import SMALL
from trainable_block_sparse_cube_b200 import build as vsa_build
from trainable_block_sparse_cube_b200 import synth, vsa

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _built():
    vsa_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    vsa.load()


def _plan(wl):
    return vsa.Plan(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, wl.topk, wl.top_p, wl.kmin, wl.kmax)


def _f64(x, b, h):
    return x[b, h].double().numpy()


def _train_and_backward(wl):
    inputs = synth.make_inputs(wl)
    dout = synth.make_dout(wl)
    dev = tuple(t.cuda() for t in inputs)
    plan = _plan(wl)
    out, idx, cnt, of, lse = plan.run_train(*dev)
    plan.check()
    grads = plan.run_backward(*dev, idx, cnt, of, lse, dout.cuda())
    plan.check()
    return plan, inputs, dout, dev, (out, idx, cnt, of, lse), grads


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_backward_small(wl):
    plan, inputs, dout, dev, fw, grads = _train_and_backward(wl)
    q, k, v, gc, gf = inputs
    out, idx, cnt, of, lse = fw
    out2, idx2, cnt2 = plan.run(*dev)
    plan.check()
    assert torch.equal(out, out2) and torch.equal(idx, idx2) and torch.equal(cnt, cnt2)
    dq, dk, dv, dgc, dgf = (t.float().cpu().numpy() for t in grads)
    of, lse = of.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.heads):
            idx_h, cnt_h = idx[b, h].cpu().numpy(), cnt[b, h].cpu().numpy()
            r = oracle_head(wl, q, k, v, gc, gf, b, h, lists_in=idx_h, counts_in=cnt_h)
            assert_close(of[b, h], r["Of"], "saved fine output")
            lse_ref = fine_lse(_f64(q, b, h), _f64(k, b, h), r["perm"], idx_h, cnt_h)
            assert_close(lse[b, h], lse_ref, "saved lse", max_abs=5e-4, mean_abs=5e-5)
            g = backward_head(_f64(q, b, h), _f64(k, b, h), _f64(v, b, h), _f64(gc, b, h), _f64(gf, b, h),
                              _f64(dout, b, h), wl.T, wl.H, wl.W, idx_h, cnt_h)
            for name, got in (("dq", dq), ("dk", dk), ("dv", dv), ("dgate_c", dgc), ("dgate_f", dgf)):
                assert_close_rel(got[b, h], g[name], f"{wl.name} {name}", *grad_tolerance(wl, name))


def test_backward_is_deterministic():
    wl = SMALL[3]
    plan, inputs, dout, dev, fw, grads = _train_and_backward(wl)
    out, idx, cnt, of, lse = fw
    for _ in range(2):
        again = plan.run_backward(*dev, idx, cnt, of, lse, dout.cuda())
        plan.check()
        for a, b in zip(grads, again):
            assert torch.equal(a, b)


def test_backward_reports_malformed_selection():
    wl = SMALL[1]
    plan, inputs, dout, dev, fw, grads = _train_and_backward(wl)
    out, idx, cnt, of, lse = fw
    bad = idx.clone()
    bad[0, 0, 2, 1] = bad[0, 0, 2, 0]       # not strictly ascending
    bad[0, 1, 3, 0] = wl.C + 3               # out of range
    plan.run_backward(*dev, bad, cnt, of, lse, dout.cuda())
    with pytest.raises(vsa.VSAError) as e:
        plan.check()
    assert e.value.code == 1
    again = plan.run_backward(*dev, idx, cnt, of, lse, dout.cuda())
    plan.check()
    for a, b in zip(grads, again):
        assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["pretrain16k", "long61k_k32", "dynamic61k"])
def test_backward_full_size_sampled(name):
    """Full-size workload, one sampled head: dq at sampled query cubes, dk and
    dv at sampled KV cubes (summed over every query cube that selected them),
    the gate gradients at every token."""
    wl = W[name]
    plan, inputs, dout, dev, fw, grads = _train_and_backward(wl)
    q, k, v, gc, gf = inputs
    out, idx, cnt, of, lse = fw
    h = wl.heads // 2
    rng = np.random.default_rng(5)
    qc = sorted({0, wl.C - 1, *rng.choice(wl.C, 6, replace=False).tolist()})
    kc = sorted({1, wl.C - 2, *rng.choice(wl.C, 3, replace=False).tolist()})
    idx_h, cnt_h = idx[0, h].cpu().numpy(), cnt[0, h].cpu().numpy()
    g = backward_head(_f64(q, 0, h), _f64(k, 0, h), _f64(v, 0, h), _f64(gc, 0, h), _f64(gf, 0, h), _f64(dout, 0, h),
                      wl.T, wl.H, wl.W, idx_h, cnt_h, query_cubes=qc, kv_cubes=kc)
    perm = oracle.cube_perm(wl.T, wl.H, wl.W)
    qt = np.concatenate([perm[64 * c: 64 * c + 64] for c in qc])
    kt = np.concatenate([perm[64 * c: 64 * c + 64] for c in kc])
    dq, dk, dv, dgc, dgf = grads
    assert_close_rel(dq[0, h, torch.from_numpy(qt).cuda()].float().cpu().numpy(), g["dq"][qt], f"{name} dq",
                     *grad_tolerance(wl, "dq"))
    assert_close_rel(dk[0, h, torch.from_numpy(kt).cuda()].float().cpu().numpy(), g["dk"][kt], f"{name} dk",
                     *grad_tolerance(wl, "dk"))
    assert_close_rel(dv[0, h, torch.from_numpy(kt).cuda()].float().cpu().numpy(), g["dv"][kt], f"{name} dv",
                     *grad_tolerance(wl, "dv"))
    assert_close_rel(dgc[0, h].cpu().numpy(), g["dgate_c"], f"{name} dgate_c", *grad_tolerance(wl, "dgate_c"))
    assert_close_rel(dgf[0, h].cpu().numpy(), g["dgate_f"], f"{name} dgate_f", *grad_tolerance(wl, "dgate_f"))

"""The gradient tolerances of the GPU backward tests, tied to the arithmetic.

The backward kernels round every product operand to bf16 (unit roundoff
2^-8) and accumulate in fp32; the forward that feeds them computes its fine
output with bf16 probabilities in the P.V product. This CPU test replays
those rounding steps in numpy (torch only for the bf16 casts) on seeded
inputs of the two kinds of workload -- the block-correlated `cube` inputs and
the ill-conditioned `cluster` inputs -- and measures the errors they produce
against the fp64 backward oracle, in units of the reference's RMS as the GPU
tests measure them. The tolerances in tests/parity.py must cover these
errors with a margin (>= 1.5x) and must not be vacuous (<= 8x).
"""
import math

import numpy as np
import torch

import oracle
from oracle.vsa_oracle_backward import backward_head
from parity import grad_tolerance
from trainable_block_sparse_cube_b200 import synth


def _bf(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _replay(wl, b=0, h=0):
    """Gradients of one head computed with the kernels' rounding steps."""
    q, k, v, gc, gf = (t[b, h].double().numpy() for t in synth.make_inputs(wl))
    dout = synth.make_dout(wl)[b, h].double().numpy()
    kmax = wl.kmax or None
    r = oracle.forward_head(q, k, v, gc, gf, wl.T, wl.H, wl.W, topk=wl.topk, top_p=wl.top_p,
                            kmin=max(wl.kmin, 1), kmax=kmax, query_cubes=[])
    lists, counts, perm = r["lists"], r["counts"], r["perm"]
    ref = backward_head(q, k, v, gc, gf, dout, wl.T, wl.H, wl.W, lists, counts)
    N, D = q.shape
    C = N // 64
    ct = perm.reshape(C, 64)
    sc = 1.0 / math.sqrt(D)
    dq = np.zeros((N, D))
    dk = np.zeros((N, D))
    dv = np.zeros((N, D))
    for i in range(C):
        kv = ct[lists[i, : counts[i]]].reshape(-1)
        qi = ct[i]
        S = _f32(q[qi] @ k[kv].T * sc)
        m = S.max(axis=1, keepdims=True)
        Pu = _f32(np.exp(S - m))
        l = _f32(Pu.sum(axis=1, keepdims=True))
        O = _f32(_bf(Pu) @ v[kv] / l)                     # forward: bf16 P in the P.V product
        lse = m + np.log(l)
        dOb = _bf(gf[qi, None] * dout[qi])                # bf16 cube-major dO
        dP = _f32(dOb @ v[kv].T)
        P = _f32(np.exp(S - lse))
        delta = _f32((dOb * O).sum(axis=1, keepdims=True))
        dS = _bf(P * (dP - delta))
        dq[qi] += _f32(dS @ k[kv]) * sc
        np.add.at(dk, kv, _f32(dS.T @ q[qi]) * sc)
        np.add.at(dv, kv, _f32(_bf(P).T @ dOb))
    # the coarse path and the bf16 outputs
    coarse = {n: ref[n] - _fine_only(ref, n, q, k, v, gc, gf, dout, wl, lists, counts) for n in ("dq", "dk", "dv")}
    out = {"dq": _bf(dq + coarse["dq"]), "dk": _bf(dk + coarse["dk"]), "dv": _bf(dv + coarse["dv"])}
    return out, ref


def _fine_only(ref, name, q, k, v, gc, gf, dout, wl, lists, counts):
    # the fine part of the oracle's gradient: the full gradient minus the
    # gradient with the fine gate set to zero (which leaves only the coarse path)
    zero = backward_head(q, k, v, gc, np.zeros_like(gf), dout, wl.T, wl.H, wl.W, lists, counts)
    return ref[name] - zero[name]


def _errors(got, ref):
    rms = math.sqrt(float(np.mean(ref * ref)))
    d = np.abs(got - ref) / rms
    return float(d.max()), float(d.mean())


def _check(wl, names=("dq", "dk", "dv")):
    got, ref = _replay(wl)
    for n in names:
        emax, emean = _errors(got[n], ref[n])
        tmax, tmean = grad_tolerance(wl, n)
        print(f"{wl.name} {n}: replayed max {emax:.3e} mean {emean:.3e}; tolerance {tmax} / {tmean}")
        assert 1.5 * emax <= tmax <= 8 * emax, (wl.name, n, emax, tmax)
        assert 1.5 * emean <= tmean <= 8 * emean, (wl.name, n, emean, tmean)


def test_tolerances_cover_the_cube_workload_arithmetic():
    _check(synth.WORKLOADS["pretrain16k"].with_(name="em_cube", heads=1, T=8, H=16, W=16, topk=8))


def test_tolerances_cover_the_cluster_workload_arithmetic():
    _check(synth.WORKLOADS["dynamic61k"].with_(name="em_cluster", heads=1, T=8, H=16, W=32, kmin=4, kmax=24))

"""Pins of the fp64 backward oracle (CPU).

The backward oracle writes out the chain rule of the forward oracle. It is
checked here against things other than itself: central finite differences of
the forward oracle (selection held fixed), and torch.autograd through torch's
scaled_dot_product_attention for the attention block. A dropped term, a
wrong sign or a transposed operand in any step fails one of these.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle.vsa_oracle_backward import attention_backward, backward_head, fine_lse

T = H = W = 8          # 512 tokens, 8 cubes
D = 8
K = 3


def _inputs(seed):
    rng = np.random.default_rng(seed)
    N = T * H * W
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    gc, gf = 1.0 / (1.0 + np.exp(-rng.standard_normal((2, N))))
    dout = rng.standard_normal((N, D))
    return q, k, v, gc, gf, dout


def _loss(q, k, v, gc, gf, dout, lists, counts):
    r = oracle.forward_head(q, k, v, gc, gf, T, H, W, lists_in=lists, counts_in=counts)
    return float((r["out"] * dout).sum())


@pytest.mark.parametrize("odd_counts", [False, True], ids=["topk3", "mixed_counts"])
def test_gradients_match_central_differences(odd_counts):
    q, k, v, gc, gf, dout = _inputs(7)
    r = oracle.forward_head(q, k, v, gc, gf, T, H, W, topk=K)
    lists, counts = r["lists"], r["counts"]
    if odd_counts:  # a variable number of cubes per query cube, as top-p produces
        counts = np.array([1, 2, 3, 1, 3, 2, 1, 3])
    g = backward_head(q, k, v, gc, gf, dout, T, H, W, lists, counts)
    rng = np.random.default_rng(3)
    h = 1e-5
    args = {"q": q, "k": k, "v": v, "gc": gc, "gf": gf}
    grads = {"q": g["dq"], "k": g["dk"], "v": g["dv"], "gc": g["dgate_c"], "gf": g["dgate_f"]}
    for name, x in args.items():
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            a = {**args, name: xp}
            b = {**args, name: xm}
            fd = (_loss(a["q"], a["k"], a["v"], a["gc"], a["gf"], dout, lists, counts)
                  - _loss(b["q"], b["k"], b["v"], b["gc"], b["gf"], dout, lists, counts)) / (2 * h)
            an = grads[name][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), f"d{name}{idx}: fd {fd} vs {an}"


def test_attention_block_matches_torch_autograd():
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((64, 16)) for _ in range(3))
    k, v = rng.standard_normal((192, 16)), rng.standard_normal((192, 16))
    dout = rng.standard_normal((64, 16))
    scale = 1.0 / math.sqrt(16)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None])[0]
    o.backward(torch.tensor(dout))
    dq, dk, dv = attention_backward(q, k, v, dout, scale)
    for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(a, b.numpy(), rtol=1e-10, atol=1e-12)


def test_zero_fine_gate_leaves_only_the_coarse_path():
    """gate_f = 0: the fine stage receives no gradient, so q, k and v get only
    the pooled coarse gradient, identical for all 64 tokens of a cube."""
    q, k, v, gc, gf, dout = _inputs(5)
    gf = np.zeros_like(gf)
    r = oracle.forward_head(q, k, v, gc, gf, T, H, W, topk=K)
    g = backward_head(q, k, v, gc, gf, dout, T, H, W, r["lists"], r["counts"])
    perm = oracle.cube_perm(T, H, W)
    for name in ("dq", "dk", "dv"):
        per_cube = g[name][perm].reshape(-1, 64, D)
        assert np.allclose(per_cube, per_cube[:, :1, :], atol=1e-14)
    assert np.allclose(g["dgate_f"], (dout * r["Of"]).sum(axis=1))


def test_fine_lse_matches_torch_logsumexp():
    q, k, v, gc, gf, dout = _inputs(11)
    r = oracle.forward_head(q, k, v, gc, gf, T, H, W, topk=K)
    perm = oracle.cube_perm(T, H, W)
    counts = np.array([1, 2, 3, 1, 3, 2, 1, 3])
    lse = fine_lse(q, k, perm, r["lists"], counts)
    N = T * H * W
    cube_of = np.empty(N, dtype=np.int64)
    cube_of[perm] = np.arange(N) // 64
    # torch.logsumexp over the full logits with -inf outside each token's selection
    mask = np.zeros((N, N), dtype=bool)
    for n in range(N):
        for j in r["lists"][cube_of[n], : counts[cube_of[n]]]:
            mask[n, perm[64 * j: 64 * j + 64]] = True
    logits = torch.from_numpy(q @ k.T / math.sqrt(D)).masked_fill(torch.from_numpy(~mask), float("-inf"))
    ref = torch.logsumexp(logits, dim=1).numpy()
    assert np.allclose(lse, ref, rtol=1e-12, atol=1e-12)
    # the softmax rebuilt from lse sums to one over the selection
    assert np.allclose(np.where(mask, np.exp(logits.numpy() - lse[:, None]), 0).sum(axis=1), 1.0)
    # a planted mistake (missing 1/sqrt(D)) fails the pin
    bad = fine_lse(q * math.sqrt(D), k, perm, r["lists"], counts)
    assert not np.allclose(bad, ref, rtol=1e-6)


def test_sampled_backward_equals_full_on_sampled_rows():
    q, k, v, gc, gf, dout = _inputs(5)
    r = oracle.forward_head(q, k, v, gc, gf, T, H, W, topk=K)
    counts = np.array([1, 2, 3, 1, 3, 2, 1, 3])
    full = backward_head(q, k, v, gc, gf, dout, T, H, W, r["lists"], counts)
    part = backward_head(q, k, v, gc, gf, dout, T, H, W, r["lists"], counts, query_cubes=[1, 6], kv_cubes=[0, 5])
    perm = oracle.cube_perm(T, H, W)
    cube_of = np.empty(T * H * W, dtype=np.int64)
    cube_of[perm] = np.arange(T * H * W) // 64
    qrows = np.isin(cube_of, [1, 6])
    kvrows = np.isin(cube_of, [0, 5])
    assert np.array_equal(part["dq"][qrows], full["dq"][qrows]) or np.allclose(part["dq"][qrows], full["dq"][qrows])
    assert np.allclose(part["dk"][kvrows], full["dk"][kvrows], rtol=1e-13, atol=1e-13)
    assert np.allclose(part["dv"][kvrows], full["dv"][kvrows], rtol=1e-13, atol=1e-13)
    assert np.isnan(part["dq"][~qrows]).all() and np.isnan(part["dk"][~kvrows]).all()

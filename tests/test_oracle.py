"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each pin is written as a check function taking the oracle functions it
tests, so the same checks can be run against deliberately broken copies
(see test_pins_catch_planted_mistakes): a pin that cannot fail pins nothing.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from trainable_block_sparse_cube_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers
def _box_perm(T, H, W):
    """Cube-major order built by enumeration: cubes in (t,h,w) row-major order,
    tokens of a cube in (dt,dh,dw) row-major order."""
    out = []
    for ct in range(T // 4):
        for ch in range(H // 4):
            for cw in range(W // 4):
                for dt in range(4):
                    for dh in range(4):
                        for dw in range(4):
                            t, h, w = 4 * ct + dt, 4 * ch + dh, 4 * cw + dw
                            out.append((t * H + h) * W + w)
    return np.array(out)


def _sdpa(q, k, v, mask=None):
    """torch's own attention routine in float64 on the CPU."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x))[None, None] for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return F.scaled_dot_product_attention(tq, tk, tv, attn_mask=m)[0, 0].numpy()


def _brute_topk(s_row, K):
    chosen = []
    for _ in range(K):
        best = None
        for j in range(len(s_row)):
            if j in chosen:
                continue
            if best is None or s_row[j] > s_row[best]:
                best = j
        chosen.append(best)
    return sorted(chosen)


def _brute_topp(s_row, P_row, p, kmin, kmax):
    C = len(s_row)
    order = sorted(range(C), key=lambda j: (-s_row[j], j))
    mass, n = 0.0, C
    for m in range(C):
        mass += P_row[order[m]]
        if mass >= p:
            n = m + 1
            break
    n = min(max(n, kmin), kmax)
    return sorted(order[:n]), n


# ----------------------------------------------------------------- pins
def check_perm(cube_perm):
    for T, H, W in [(4, 4, 4), (8, 8, 8), (4, 8, 12), (12, 4, 8)]:
        perm = cube_perm(T, H, W)
        N = T * H * W
        assert sorted(perm.tolist()) == list(range(N)), "not a bijection"
        for c in range(N // 64):
            toks = perm[64 * c: 64 * c + 64]
            t, h, w = toks // (H * W), (toks // W) % H, toks % W
            assert t.max() - t.min() == 3 and h.max() - h.min() == 3 and w.max() - w.min() == 3
            assert t.min() % 4 == 0 and h.min() % 4 == 0 and w.min() % 4 == 0
            assert len(set(zip(t.tolist(), h.tolist(), w.tolist()))) == 64
        assert np.array_equal(perm, _box_perm(T, H, W)), "enumeration convention"


def check_pool(cube_perm, pool_cubes):
    rng = np.random.default_rng(1)
    T, H, W, D = 8, 4, 12, 5
    vals = rng.normal(size=(T // 4, H // 4, W // 4, D))
    x = np.empty((T * H * W, D))
    for t in range(T):
        for h in range(H):
            for w in range(W):
                x[(t * H + h) * W + w] = vals[t // 4, h // 4, w // 4]
    pooled = pool_cubes(x, cube_perm(T, H, W))
    assert np.allclose(pooled, vals.reshape(-1, D), atol=1e-14)
    # random tokens: explicit means over each box, in raster coordinates
    x = rng.normal(size=(T * H * W, D))
    pooled = pool_cubes(x, cube_perm(T, H, W))
    c = 0
    for ct in range(T // 4):
        for ch in range(H // 4):
            for cw in range(W // 4):
                acc = np.zeros(D)
                for dt in range(4):
                    for dh in range(4):
                        for dw in range(4):
                            acc += x[((4 * ct + dt) * H + 4 * ch + dh) * W + 4 * cw + dw]
                assert np.allclose(pooled[c], acc / 64, atol=1e-13)
                c += 1


def check_coarse(coarse_attention):
    rng = np.random.default_rng(2)
    for C, D in [(8, 64), (37, 128), (3, 16)]:
        qb, kb, vb = rng.normal(size=(C, D)), rng.normal(size=(C, D)), rng.normal(size=(C, D))
        s, P, Oc = coarse_attention(qb, kb, vb)
        assert np.allclose(Oc, _sdpa(qb, kb, vb), atol=1e-12)
        assert np.allclose(P.sum(axis=1), 1.0, atol=1e-12)
        # logits: the row argmax of P is the best-aligned key
        assert np.array_equal(np.argmax(P, axis=1), np.argmax(qb @ kb.T, axis=1))
        # uniform keys -> uniform weights -> mean of the values
        s, P, Oc = coarse_attention(qb, np.tile(kb[:1], (C, 1)), vb)
        assert np.allclose(Oc, np.tile(vb.mean(axis=0), (C, 1)), atol=1e-12)
    # scale: two keys whose dot products differ by sqrt(D)*ln(3) -> weights 3:1
    D = 16
    qb = np.zeros((1, D)); qb[0, 0] = 1.0
    kb = np.zeros((2, D)); kb[0, 0] = math.sqrt(D) * math.log(3.0)
    vb = np.array([[1.0] + [0.0] * (D - 1), [0.0] * D])
    _, P, Oc = coarse_attention(qb, kb, vb)
    assert np.allclose(P[0], [0.75, 0.25], atol=1e-12)


def check_topk(select_topk):
    rng = np.random.default_rng(3)
    for C, K in [(8, 2), (20, 5), (33, 33), (50, 1)]:
        s = rng.integers(0, 4, size=(C, C)).astype(np.float64)   # many ties
        got = select_topk(s, K)
        for i in range(C):
            assert got[i].tolist() == _brute_topk(s[i].tolist(), K)
        s = rng.normal(size=(C, C))
        got = select_topk(s, K)
        for i in range(C):
            assert got[i].tolist() == _brute_topk(s[i].tolist(), K)
    s = np.zeros((6, 10))
    assert select_topk(s, 4).tolist() == [[0, 1, 2, 3]] * 6
    assert select_topk(rng.normal(size=(5, 5)), 5).tolist() == [list(range(5))] * 5


def check_topp(select_topp):
    rng = np.random.default_rng(4)
    C = 40
    s = rng.normal(size=(C, C))
    e = np.exp(s - s.max(axis=1, keepdims=True))
    P = e / e.sum(axis=1, keepdims=True)
    lists, cnt = select_topp(s, P, 1.0, 1, C)
    assert (cnt == C).all()
    lists, cnt = select_topp(s, P, 1.0, 1, 17)
    assert (cnt == 17).all()
    lists, cnt = select_topp(s, P, 1e-12, 4, 30)
    assert (cnt == 4).all()
    for i in range(C):
        assert lists[i, :4].tolist() == _brute_topk(s[i].tolist(), 4)
        assert (lists[i, 4:] == -1).all()
    # one dominant cube per row
    s2 = np.zeros((C, C)); s2[np.arange(C), (np.arange(C) * 7) % C] = 60.0
    e2 = np.exp(s2 - s2.max(axis=1, keepdims=True)); P2 = e2 / e2.sum(axis=1, keepdims=True)
    lists, cnt = select_topp(s2, P2, 0.9, 3, 10)
    assert (cnt == 3).all()
    for i in range(C):
        assert (i * 7) % C in lists[i, :3].tolist()
    # brute-force prefix scan, including ties
    s3 = rng.integers(0, 6, size=(C, C)).astype(np.float64) * 0.7
    e3 = np.exp(s3 - s3.max(axis=1, keepdims=True)); P3 = e3 / e3.sum(axis=1, keepdims=True)
    for p, kmin, kmax in [(0.9, 4, 30), (0.5, 1, C), (0.99, 2, 12)]:
        lists, cnt = select_topp(s3, P3, p, kmin, kmax)
        for i in range(C):
            ref, n = _brute_topp(s3[i].tolist(), P3[i].tolist(), p, kmin, kmax)
            assert cnt[i] == n and lists[i, :n].tolist() == ref
            assert (lists[i, n:] == -1).all()


def check_fine(cube_perm, fine_attention):
    rng = np.random.default_rng(5)
    T, H, W, D = 8, 8, 4, 32
    N, C = T * H * W, T * H * W // 64
    q, k, v = (rng.normal(size=(N, D)) for _ in range(3))
    perm = cube_perm(T, H, W)
    allc = np.tile(np.arange(C), (C, 1))
    Of = fine_attention(q, k, v, perm, allc, np.full(C, C), None)
    assert np.allclose(Of, _sdpa(q, k, v), atol=1e-12)
    # sparse selection == masked dense attention
    K = 3
    lists = np.array([np.sort(rng.choice(C, K, replace=False)) for _ in range(C)])
    cube_of = np.empty(N, dtype=np.int64)
    for c in range(C):
        cube_of[perm[64 * c: 64 * c + 64]] = c
    mask = np.zeros((N, N), dtype=bool)
    for n in range(N):
        for j in lists[cube_of[n]]:
            mask[n, cube_of == j] = True
    Of = fine_attention(q, k, v, perm, lists, np.full(C, K), None)
    assert np.allclose(Of, _sdpa(q, k, v, mask), atol=1e-12)


def check_combine(cube_perm, gated_combine):
    rng = np.random.default_rng(6)
    T, H, W, D = 4, 8, 8, 8
    N, C = T * H * W, T * H * W // 64
    perm = cube_perm(T, H, W)
    Oc, Of = rng.normal(size=(C, D)), rng.normal(size=(N, D))
    zeros, ones = np.zeros(N), np.ones(N)
    assert np.allclose(gated_combine(Oc, Of, zeros, ones, perm), Of)
    got = gated_combine(Oc, Of, ones, zeros, perm)
    for t in range(T):
        for h in range(H):
            for w in range(W):
                c = ((t // 4) * (H // 4) + h // 4) * (W // 4) + w // 4
                assert np.allclose(got[(t * H + h) * W + w], Oc[c])
    g1, g2, g3, g4 = (rng.uniform(size=N) for _ in range(4))
    lhs = gated_combine(Oc, Of, 2 * g1 + 3 * g3, 2 * g2 + 3 * g4, perm)
    rhs = 2 * gated_combine(Oc, Of, g1, g2, perm) + 3 * gated_combine(Oc, Of, g3, g4, perm)
    assert np.allclose(lhs, rhs, atol=1e-12)


def check_single_cube(forward_head):
    """One 4x4x4 cube: coarse output is mean(v); fine stage is full attention."""
    rng = np.random.default_rng(7)
    D = 16
    q, k, v = (rng.normal(size=(64, D)) for _ in range(3))
    gc, gf = rng.uniform(size=64), rng.uniform(size=64)
    r = forward_head(q, k, v, gc, gf, 4, 4, 4, topk=1)
    ref = gc[:, None] * v.mean(axis=0)[None] + gf[:, None] * _sdpa(q, k, v)
    assert np.allclose(r["out"], ref, atol=1e-12)
    assert r["lists"].tolist() == [[0]]


ALL_PINS = {
    "perm": lambda o: check_perm(o.cube_perm),
    "pool": lambda o: check_pool(o.cube_perm, o.pool_cubes),
    "coarse": lambda o: check_coarse(o.coarse_attention),
    "topk": lambda o: check_topk(o.select_topk),
    "topp": lambda o: check_topp(o.select_topp),
    "fine": lambda o: check_fine(o.cube_perm, o.fine_attention),
    "combine": lambda o: check_combine(o.cube_perm, o.gated_combine),
    "single_cube": lambda o: check_single_cube(o.forward_head),
}


@pytest.mark.parametrize("name", list(ALL_PINS))
def test_oracle_pin(name):
    ALL_PINS[name](oracle)


# ----------------------------------------------------------------- planted mistakes
class _Mutant:
    """The oracle with one function replaced by a plausible mistake."""

    def __init__(self, **over):
        for n in oracle.__all__:
            setattr(self, n, getattr(oracle, n))
        for n, f in over.items():
            setattr(self, n, f)


def _perm_swapped_hw(T, H, W):
    # cube enumeration with w-cubes before h-cubes (a transposed index)
    n = np.arange(T * H * W)
    t, h, w = n // (H * W), (n // W) % H, n % W
    c = ((t // 4) * (W // 4) + w // 4) * (H // 4) + h // 4
    r = ((t % 4) * 4 + h % 4) * 4 + w % 4
    perm = np.empty_like(n); perm[64 * c + r] = n
    return perm


def _coarse_no_scale(qb, kb, vb):
    s = qb @ kb.T
    e = np.exp(s - s.max(axis=1, keepdims=True)); P = e / e.sum(axis=1, keepdims=True)
    return s, P, P @ vb


def _coarse_transposed(qb, kb, vb):
    s = (kb @ qb.T) / math.sqrt(qb.shape[1])
    e = np.exp(s - s.max(axis=1, keepdims=True)); P = e / e.sum(axis=1, keepdims=True)
    return s, P, P @ vb


def _topk_ties_high(s, K):
    out = np.empty((s.shape[0], K), dtype=np.int64)
    for i in range(s.shape[0]):
        order = np.argsort(-s[i][::-1], kind="stable")
        out[i] = np.sort((s.shape[1] - 1 - order)[:K])
    return out


def _topp_exclusive(s, P, p, kmin, kmax):
    C = s.shape[0]
    lists = np.full((C, kmax), -1, dtype=np.int64); cnt = np.empty(C, dtype=np.int64)
    for i in range(C):
        order = np.argsort(-s[i], kind="stable"); cum = np.cumsum(P[i, order])
        hit = np.nonzero(cum > p)[0]
        n = int(hit[0]) + 2 if hit.size else C          # off by one
        n = min(max(n, kmin), kmax); cnt[i] = n; lists[i, :n] = np.sort(order[:n])
    return lists, cnt


def _fine_per_tile_softmax(q, k, v, perm, lists, counts, query_cubes=None):
    # softmax normalised per selected cube instead of over their union
    N, D = q.shape; C = N // 64; ct = perm.reshape(C, 64); out = np.full((N, D), np.nan)
    for i in range(C) if query_cubes is None else query_cubes:
        acc = 0
        for j in lists[i, : counts[i]]:
            lg = q[ct[i]] @ k[ct[j]].T / math.sqrt(D)
            e = np.exp(lg - lg.max(axis=1, keepdims=True))
            acc = acc + (e / e.sum(axis=1, keepdims=True)) @ v[ct[j]]
        out[ct[i]] = acc / counts[i]
    return out


def _combine_swapped(Oc, Of, gc, gf, perm):
    return oracle.gated_combine(Oc, Of, gf, gc, perm)


MUTANTS = [
    ("perm", dict(cube_perm=_perm_swapped_hw)),
    ("coarse", dict(coarse_attention=_coarse_no_scale)),
    ("coarse", dict(coarse_attention=_coarse_transposed)),
    ("topk", dict(select_topk=_topk_ties_high)),
    ("topp", dict(select_topp=_topp_exclusive)),
    ("fine", dict(fine_attention=_fine_per_tile_softmax)),
    ("combine", dict(gated_combine=_combine_swapped)),
]


@pytest.mark.parametrize("pin,over", MUTANTS, ids=[f"{p}-{list(o.values())[0].__name__}" for p, o in MUTANTS])
def test_pins_catch_planted_mistakes(pin, over):
    with pytest.raises(AssertionError):
        ALL_PINS[pin](_Mutant(**over))


# ----------------------------------------------------------------- page facts
def test_workloads_match_page_facts():
    facts = json.load(open(os.path.join(GOLDEN, "page_facts.json")))
    assert facts["cube_shape"]["value"] == [4, 4, 4]
    assert oracle.cube_perm(4, 4, 4).size == 4 * 4 * 4 == 64
    sp = facts["sparsity_matching_full_attention"]["value"]
    w = synth.WORKLOADS
    assert w["pretrain16k"].N == facts["pretraining_sequence_length"]["value"]
    assert 1 - w["pretrain16k"].topk / w["pretrain16k"].C == sp
    assert 1 - w["large77k"].topk / w["large77k"].C == sp
    assert w["long61k_k32"].N == w["long61k_k16"].N == facts["long_sequence_tokens"]["value"]
    assert sorted([w["long61k_k16"].topk, w["long61k_k32"].topk]) == facts["topk_compared_at_long_sequence"]["value"]


# ----------------------------------------------------------------- end-to-end properties
def test_forward_tiny_properties():
    wl = synth.WORKLOADS["tiny"]
    q, k, v, gc, gf = synth.make_inputs(wl)
    for h in range(wl.heads):
        r = oracle.forward_head(q[0, h].double().numpy(), k[0, h].double().numpy(), v[0, h].double().numpy(),
                                gc[0, h].double().numpy(), gf[0, h].double().numpy(), wl.T, wl.H, wl.W,
                                topk=wl.topk)
        assert r["out"].shape == (512, 64) and r["lists"].shape == (8, 2)
        assert np.isfinite(r["out"]).all()
        assert (np.diff(r["lists"], axis=-1) > 0).all()            # ascending, distinct
        assert (r["counts"] == 2).all()


def test_topp_mass_property():
    wl = synth.WORKLOADS["dynamic61k"].with_(T=8, H=16, W=16, heads=1)
    q, k, v, gc, gf = synth.make_inputs(wl)
    r = oracle.forward_head(q[0, 0].double().numpy(), k[0, 0].double().numpy(), v[0, 0].double().numpy(),
                            gc[0, 0].numpy(), gf[0, 0].numpy(), wl.T, wl.H, wl.W, topk=0, top_p=0.9,
                            kmin=4, kmax=32, query_cubes=[])
    P, s = r["P"], r["s"]
    for i in range(P.shape[0]):
        n = r["counts"][i]
        sel = r["lists"][i, :n]
        mass = P[i, sel].sum()
        if n < 32:
            assert mass >= 0.9 - 1e-12
        if n > 4:
            weakest = sel[np.argmin(s[i, sel])]
            assert mass - P[i, weakest] < 0.9

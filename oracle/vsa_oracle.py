"""Plain fp64 CPU statement of the VSA forward pass -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this module. The CUDA library never calls it, and it shares no
code with the CUDA library: the only thing both sides use is the seeded input
generator module, which holds no step of the method.

Sources (web pages about the method; cited by title and section):
  [VSA-Approach]  "Faster Video Diffusion with Trainable Sparse Attention",
                  section "Approach" (atlas.scime.ai summary, NeurIPS 2025).
  [VSA-Abstract]  "VSA: Faster Video Diffusion with Trainable Sparse
                  Attention", section "Abstract (arXiv)".
  [VSA-Limits]    same summary page as [VSA-Approach], section "Limitations".
  [VSA-Findings]  same summary page, section "Surprising findings".
  [VSA2-Abstract] "Improving Video Sparse Attention with Fine-grained Router
                  and Sparse Rebasing", section "Abstract (arXiv)".

The pages give the method in words only (no formulas, no listing). Each step
below is the plainest reading of those words; every reading that fills a gap
is marked READING. Everything is computed in float64 from the bf16 inputs,
which convert to float64 exactly.

Pinned by tests/test_oracle.py against: brute-force index maps, closed forms
(constant cubes, single-cube problems, uniform scores), torch's CPU
scaled_dot_product_attention (full and masked attention), brute-force
selection loops, and the gate special cases. The end-to-end result has no
printed worked example on the pages; see the pins listed per function.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "cube_perm", "pool_cubes", "coarse_attention", "select_topk", "select_topp",
    "fine_attention", "gated_combine", "forward_head",
]


def cube_perm(T: int, H: int, W: int) -> np.ndarray:
    """Cube-major order of a T x H x W token grid.

    [VSA-Approach]: tokens are grouped into 4x4x4 cubes, each cube one GPU
    tile; [VSA-Limits]: T, H and W must be multiples of 4.
    READING (cube enumeration, in-cube order): both row-major in (t, h, w):
      raster index      n = (t*H + h)*W + w
      cube index        c = ((t//4)*(H//4) + h//4)*(W//4) + w//4
      in-cube offset    r = ((t%4)*4 + h%4)*4 + w%4
      cube-major slot   p = 64*c + r
    Returns perm with perm[p] = n (so x[perm] is the cube-major copy of x).
    Pinned by: every cube's 64 tokens form one 4x4x4 box; perm is a bijection.
    """
    if T % 4 or H % 4 or W % 4:
        raise ValueError("T, H, W must be multiples of 4")
    n = np.arange(T * H * W, dtype=np.int64)
    t = n // (H * W)
    h = (n // W) % H
    w = n % W
    c = ((t // 4) * (H // 4) + h // 4) * (W // 4) + w // 4
    r = ((t % 4) * 4 + h % 4) * 4 + w % 4
    p = 64 * c + r
    perm = np.empty_like(n)
    perm[p] = n
    return perm


def pool_cubes(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Mean of the 64 tokens of every cube: [N, D] -> [C, D].

    [VSA-Approach] "mean-pool tokens into 4x4x4 cubes"; [VSA-Findings] mean
    pooling is the variant kept (over max and conv pooling).
    Pinned by: a constant cube pools to that constant; explicit box means.
    """
    N, D = x.shape
    return x[perm].reshape(N // 64, 64, D).mean(axis=1)


def coarse_attention(qbar: np.ndarray, kbar: np.ndarray, vbar: np.ndarray):
    """Dense cube-to-cube attention on pooled tokens.

    [VSA-Approach] "a coarse cube-to-cube dense attention ... output a coarse
    context"; [VSA-Abstract] "a lightweight coarse stage pools tokens into
    tiles". READING: scale 1/sqrt(D); attention is dense over all C cubes.
    Returns (s, P, Oc): logits s = qbar kbar^T / sqrt(D) [C, C], row softmax
    P [C, C] (max-subtracted) and coarse output Oc = P vbar [C, D].
    Pinned by: torch scaled_dot_product_attention on the pooled tokens;
    uniform scores give the mean of vbar.
    """
    D = qbar.shape[1]
    s = (qbar @ kbar.T) / math.sqrt(D)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    P = e / e.sum(axis=1, keepdims=True)
    return s, P, P @ vbar


def _rank_order(s_row: np.ndarray) -> np.ndarray:
    """Cube ids sorted by descending score, ties to the lowest id.

    READING: ranking uses the coarse logits (same order as P); equal scores
    are broken toward the lower cube index."""
    return np.argsort(-s_row, kind="stable")


def select_topk(s: np.ndarray, K: int) -> np.ndarray:
    """Top-K critical cubes per query cube, listed in ascending cube id.

    [VSA-Approach] "select top-K critical cubes". READING: list order is
    ascending cube id. Returns int64 [C, K].
    Pinned by: a brute-force max-extraction loop; all-equal scores give
    0..K-1; K = C gives every cube.
    """
    C = s.shape[0]
    if not 1 <= K <= s.shape[1]:
        raise ValueError("K out of range")
    out = np.empty((C, K), dtype=np.int64)
    for i in range(C):
        out[i] = np.sort(_rank_order(s[i])[:K])
    return out


def select_topp(s: np.ndarray, P: np.ndarray, p: float, kmin: int, kmax: int):
    """Variable-size selection: smallest score-ranked prefix with mass >= p.

    [VSA2-Abstract] lets "each query ... attend to a variable number of
    key-value pairs"; the page does not define the rule. READING: for query
    cube i rank cubes as in top-K, take the smallest n with cumulative coarse
    probability (fp64) >= p, inclusive; if no prefix reaches p, n = C; then
    clamp n to [kmin, kmax]. Returns (lists [C, kmax] ascending, padded -1;
    counts [C]).
    Pinned by: p = 1 -> min(C, kmax); tiny p -> kmin; one dominant cube ->
    kmin; a brute-force prefix scan.
    """
    C = s.shape[0]
    lists = np.full((C, kmax), -1, dtype=np.int64)
    cnt = np.empty(C, dtype=np.int64)
    for i in range(C):
        order = _rank_order(s[i])
        cum = np.cumsum(P[i, order])
        hit = np.nonzero(cum >= p)[0]
        n = int(hit[0]) + 1 if hit.size else C
        n = min(max(n, kmin), kmax)
        cnt[i] = n
        lists[i, :n] = np.sort(order[:n])
    return lists, cnt


def fine_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, perm: np.ndarray,
                   lists: np.ndarray, counts: np.ndarray, query_cubes=None) -> np.ndarray:
    """Token-level attention of each query cube over its selected cubes only.

    [VSA-Approach] "block-sparse token-level fine attention only over selected
    cubes"; [VSA-Abstract] "a fine stage computes token-level attention only
    inside those tiles". READING: one softmax over the union of the selected
    cubes' tokens, scale 1/sqrt(D), no forced local window ([VSA-Findings]:
    injected local priors gave negligible benefit).
    Inputs in raster order [N, D]; result in raster order [N, D] (rows of
    query cubes not in `query_cubes` are left as NaN).
    Pinned by: with every cube selected it equals torch's full attention;
    otherwise torch's masked attention with -inf outside the selection.
    """
    N, D = q.shape
    C = N // 64
    cube_tok = perm.reshape(C, 64)            # raster ids of each cube's tokens
    out = np.full((N, D), np.nan)
    scale = 1.0 / math.sqrt(D)
    qc = range(C) if query_cubes is None else query_cubes
    for i in qc:
        sel = lists[i, : counts[i]]
        kv_tok = cube_tok[sel].reshape(-1)
        qi = q[cube_tok[i]]
        logits = (qi @ k[kv_tok].T) * scale
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        out[cube_tok[i]] = (e / e.sum(axis=1, keepdims=True)) @ v[kv_tok]
    return out


def gated_combine(Oc: np.ndarray, Of: np.ndarray, gate_c: np.ndarray, gate_f: np.ndarray,
                  perm: np.ndarray) -> np.ndarray:
    """out[n] = gate_c[n] * Oc[cube(n)] + gate_f[n] * Of[n]   (raster order).

    [VSA-Approach] "combine both via learned gates". READING: one scalar gate
    per token and head for each branch, used as given (no sigmoid inside, no
    normalisation); the coarse output of a cube is shared by its 64 tokens.
    Pinned by: (gate_c, gate_f) = (0, 1) gives the fine output, (1, 0) the
    broadcast coarse output, and the result is linear in the gates.
    """
    N = Of.shape[0]
    cube_of = np.empty(N, dtype=np.int64)
    cube_of[perm] = np.arange(N) // 64
    return gate_c[:, None] * Oc[cube_of] + gate_f[:, None] * Of


def forward_head(q, k, v, gate_c, gate_f, T, H, W, topk=0, top_p=0.0, kmin=1, kmax=None,
                 query_cubes=None, lists_in=None, counts_in=None):
    """The whole forward pass for one (batch, head): the steps above in order.

    q, k, v: [N, D] (any float dtype; converted to float64); gates: [N].
    topk > 0 selects top-K, otherwise top-p with clamp [kmin, kmax].
    lists_in / counts_in, if given, replace the selection step (used to run
    the fine stage on another selection).
    Returns a dict with perm, qbar, kbar, vbar, s, P, Oc, lists, counts, Of, out.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    gate_c = np.asarray(gate_c, dtype=np.float64)
    gate_f = np.asarray(gate_f, dtype=np.float64)
    perm = cube_perm(T, H, W)
    C = q.shape[0] // 64
    qbar, kbar, vbar = (pool_cubes(x, perm) for x in (q, k, v))
    s, P, Oc = coarse_attention(qbar, kbar, vbar)
    if lists_in is not None:
        lists = np.asarray(lists_in, dtype=np.int64)
        counts = (np.asarray(counts_in, dtype=np.int64) if counts_in is not None
                  else np.full(C, lists.shape[1], dtype=np.int64))
    elif topk > 0:
        lists = select_topk(s, topk)
        counts = np.full(C, topk, dtype=np.int64)
    else:
        kmax = C if kmax is None else kmax
        lists, counts = select_topp(s, P, top_p, kmin, kmax)
    Of = fine_attention(q, k, v, perm, lists, counts, query_cubes)
    out = gated_combine(Oc, Of, gate_c, gate_f, perm)
    return dict(perm=perm, qbar=qbar, kbar=kbar, vbar=vbar, s=s, P=P, Oc=Oc,
                lists=lists, counts=counts, Of=Of, out=out)

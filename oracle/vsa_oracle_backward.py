"""Plain fp64 CPU statement of the VSA backward pass -- TEST INFRASTRUCTURE ONLY.

Only the tests may import this module; the CUDA library never calls it and
shares no code with it.

Source: "Faster Video Diffusion with Trainable Sparse Attention", section
"Approach": the whole hierarchy (coarse stage, selection, fine stage, gated
combine) is one differentiable kernel trained end to end. The pages give no
formulas for the gradients, so this module writes out the chain rule of the
forward pass in vsa_oracle.py, step by step.
READING: the selection (top-K or top-p lists) is an index choice and is held
fixed: no gradient flows through it. The gates are inputs of the kernel, so
their gradients are returned and not propagated further.

Pinned by tests/test_oracle_backward.py against central finite differences of
the forward oracle (each input perturbed coordinate by coordinate, selection
held fixed) and, for the attention block, against torch.autograd through
torch's CPU scaled_dot_product_attention in float64.
"""
from __future__ import annotations

import math

import numpy as np

from .vsa_oracle import coarse_attention, cube_perm, fine_attention, pool_cubes

__all__ = ["attention_backward", "backward_head", "fine_lse"]


def attention_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, dout: np.ndarray, scale: float):
    """Gradients of O = softmax_rows(q k^T * scale) v with respect to q, k, v.

    With P the row softmax and dO the upstream gradient (chain rule):
      dV = P^T dO,  dP = dO V^T,  dS_ij = P_ij (dP_ij - sum_l P_il dP_il),
      dQ = dS K * scale,  dK = dS^T Q * scale.
    Pinned by: torch.autograd through scaled_dot_product_attention (float64).
    """
    logits = (q @ k.T) * scale
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    P = e / e.sum(axis=1, keepdims=True)
    dv = P.T @ dout
    dP = dout @ v.T
    dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
    return dS @ k * scale, dS.T @ q * scale, dv


def fine_lse(q: np.ndarray, k: np.ndarray, perm: np.ndarray, lists: np.ndarray, counts: np.ndarray,
             query_cubes=None) -> np.ndarray:
    """Per query token n, the natural log of its fine softmax denominator,
    log sum_m exp(q_n . k_m / sqrt(D)) over the tokens m of its query cube's
    selected cubes (the normaliser of the fine attention in vsa_oracle.py, the
    forward statistic the backward pass reuses). Raster order [N]; tokens of
    query cubes not in `query_cubes` are NaN.
    Pinned by: torch.logsumexp over the masked logits (-inf outside the
    selection), and exp(logits - lse) rows summing to one.
    """
    N, D = q.shape
    C = N // 64
    cube_tok = perm.reshape(C, 64)
    out = np.full(N, np.nan)
    for i in (range(C) if query_cubes is None else query_cubes):
        kv_tok = cube_tok[lists[i, : counts[i]]].reshape(-1)
        logits = (q[cube_tok[i]] @ k[kv_tok].T) / math.sqrt(D)
        m = logits.max(axis=1)
        out[cube_tok[i]] = m + np.log(np.exp(logits - m[:, None]).sum(axis=1))
    return out


def backward_head(q, k, v, gate_c, gate_f, dout, T, H, W, lists, counts, query_cubes=None, kv_cubes=None):
    """Gradients of one (batch, head) of the gated forward pass.

    Forward (vsa_oracle.forward_head with the selection `lists`/`counts`):
      qbar, kbar, vbar = cube means;  Oc = coarse attention of the means;
      Of = fine attention of every query cube over its selected cubes' tokens;
      out_n = gate_c[n] Oc[cube(n)] + gate_f[n] Of_n.
    Backward, in reverse order:
      dgate_c[n] = dout_n . Oc[cube(n)],   dgate_f[n] = dout_n . Of_n;
      dOc[c] = sum over the cube's tokens of gate_c[n] dout_n;  dOf_n = gate_f[n] dout_n;
      fine: attention_backward per query cube over its selected tokens, the key
            and value gradients summed over every query cube that selected them;
      coarse: attention_backward of the means;
      pooling: every token of cube c receives 1/64 of the mean's gradient.
    Inputs [N, D] and [N] in raster order, fp64. Returns a dict with
    dq, dk, dv [N, D] and dgate_c, dgate_f [N].
    query_cubes / kv_cubes (optional) restrict the work to sampled outputs:
    dq only for the tokens of query_cubes, dk and dv only for the tokens of
    kv_cubes (each still summed over every query cube that selected it); the
    other rows of those arrays are NaN. The fine terms are the only ones
    restricted; the result on the sampled rows is the same.
    Pinned by: central finite differences of the forward oracle; the sampled
    rows equal the unrestricted result.
    """
    N, D = q.shape
    C = N // 64
    perm = cube_perm(T, H, W)
    cube_tok = perm.reshape(C, 64)
    cube_of = np.empty(N, dtype=np.int64)
    cube_of[perm] = np.repeat(np.arange(C), 64)
    scale = 1.0 / math.sqrt(D)

    qbar, kbar, vbar = pool_cubes(q, perm), pool_cubes(k, perm), pool_cubes(v, perm)
    _, _, Oc = coarse_attention(qbar, kbar, vbar)
    Of = fine_attention(q, k, v, perm, lists, counts)

    dgate_c = (dout * Oc[cube_of]).sum(axis=1)
    dgate_f = (dout * Of).sum(axis=1)
    dOc = np.zeros((C, D))
    np.add.at(dOc, cube_of, gate_c[:, None] * dout)
    dOf = gate_f[:, None] * dout

    dq = np.zeros((N, D))
    dk = np.zeros((N, D))
    dv = np.zeros((N, D))
    qset = None if query_cubes is None else set(int(x) for x in query_cubes)
    kvset = None if kv_cubes is None else set(int(x) for x in kv_cubes)
    for i in range(C):
        sel = lists[i, : counts[i]]
        want_q = qset is None or i in qset
        want_kv = kvset is None or any(int(j) in kvset for j in sel)
        if not (want_q or want_kv):
            continue
        kv_tok = cube_tok[sel].reshape(-1)
        qi = cube_tok[i]
        gq, gk, gv = attention_backward(q[qi], k[kv_tok], v[kv_tok], dOf[qi], scale)
        dq[qi] += gq
        np.add.at(dk, kv_tok, gk)
        np.add.at(dv, kv_tok, gv)

    gqb, gkb, gvb = attention_backward(qbar, kbar, vbar, dOc, scale)
    dq += gqb[cube_of] / 64.0
    dk += gkb[cube_of] / 64.0
    dv += gvb[cube_of] / 64.0
    if qset is not None:
        dq[~np.isin(cube_of, list(qset))] = np.nan
    if kvset is not None:
        keep = np.isin(cube_of, list(kvset))
        dk[~keep] = np.nan
        dv[~keep] = np.nan
    return dict(dq=dq, dk=dk, dv=dv, dgate_c=dgate_c, dgate_f=dgate_f)

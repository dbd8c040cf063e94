"""The GPU parity workloads reach the fine kernel's rarely taken branches.

The fine kernel's online softmax keeps a lazy reference maximum per row: the
first step of a query cube sets it to the exact row maximum (log2 units), and
a later step moves it, rescaling the O accumulator held in tensor memory,
only when a score exceeds it by more than 8 (a factor 2^8). On the smooth
workloads that never happens after the first step, so the rescale branch is
covered only if some parity workload has a late KV cube that dominates. This
replays the reference rule on CPU over the oracle's own selection lists (in
the kernel's step order: ascending cube ids, two cubes per step) and checks
that the `cluster_topp` parity workload, tokens clustered around shared
centres, moves the reference after the first step in some rows.
"""
import numpy as np

import oracle
from trainable_block_sparse_cube_b200 import synth

MARGIN_LOG2 = 8.0


def late_reference_moves(wl, heads):
    q, k, v, gc, gf = synth.make_inputs(wl)
    perm = oracle.cube_perm(wl.T, wl.H, wl.W)
    scale_log2 = np.log2(np.e) / np.sqrt(wl.D)
    moves = steps = 0
    for h in range(heads):
        r = oracle.forward_head(q[0, h].double().numpy(), k[0, h].double().numpy(), v[0, h].double().numpy(),
                                gc[0, h].double().numpy(), gf[0, h].double().numpy(), wl.T, wl.H, wl.W,
                                topk=wl.topk, top_p=wl.top_p, kmin=max(wl.kmin, 1), kmax=(wl.kmax or None))
        qc = q[0, h].float().numpy()[perm].reshape(-1, 64, wl.D)
        kc = k[0, h].float().numpy()[perm].reshape(-1, 64, wl.D)
        for i in range(qc.shape[0]):
            sel = r["lists"][i][: r["counts"][i]]
            ref = None
            for t in range((len(sel) + 1) // 2):
                x = (qc[i] @ np.concatenate([kc[c] for c in sel[2 * t: 2 * t + 2]]).T) * scale_log2
                xm = x.max(axis=1)
                if ref is None:
                    ref = xm
                    continue
                steps += 1
                up = xm > ref + MARGIN_LOG2
                moves += int(up.any())
                ref = np.where(up, xm, ref)
    return moves, steps


def test_cluster_workload_moves_the_reference_after_the_first_step():
    from test_gpu_parity import SMALL  # the GPU parity workloads themselves (only their definitions are used)

    wl = next(w for w in SMALL if w.name == "cluster_topp")
    moves, steps = late_reference_moves(wl, wl.heads)
    assert steps > 0
    assert moves >= 1, "no parity workload exercises the O rescale after an item's first step"

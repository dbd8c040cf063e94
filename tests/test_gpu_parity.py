"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Per stage: the cube gather is compared bit for bit, the pooled means and
coarse output numerically, the selections bit for bit outside the score tie
band, the fine stage on the oracle's own lists, and the whole pass on the
GPU's own (validated) lists. Small workloads span several tiles and ragged
tails (odd counts, partial 64-cube blocks); the full-size workloads are
checked on sampled heads and query cubes.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, check_lists, oracle_head
from trainable_block_sparse_cube_b200 import build as vsa_build
from trainable_block_sparse_cube_b200 import synth, vsa

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS

SMALL = [
    W["tiny"],
    W["pretrain16k"].with_(name="cube_k5_odd", heads=3, T=8, H=16, W=24, topk=5),
    W["pretrain16k"].with_(name="cube_b2", B=2, heads=2, T=12, H=8, W=16, topk=8),
    W["large77k"].with_(name="sin_k12", heads=2, T=8, H=16, W=20, topk=12),
    W["dynamic61k"].with_(name="cluster_topp", heads=2, T=8, H=16, W=32, kmin=4, kmax=24),
    W["tiny"].with_(name="tiny_topp_d64", heads=3, topk=0, top_p=0.9, kmin=1, kmax=8),
    W["pretrain16k"].with_(name="d64_k7", D=64, heads=2, T=8, H=8, W=24, topk=7),
    W["pretrain16k"].with_(name="k_eq_c", heads=1, T=4, H=8, W=12, topk=6),
    W["tiny"].with_(name="single_cube", T=4, H=4, W=4, heads=2, topk=1),
    W["large77k"].with_(name="sin_k40_c80", heads=2, T=8, H=16, W=40, topk=40),
    # odd cube counts (the select kernel's unpaired score loads); 243 cubes put
    # 65..256 keys above the lane-maxima bound (its wider candidate sets)
    W["pretrain16k"].with_(name="odd_c27_k5", heads=2, T=12, H=12, W=12, topk=5),
    W["pretrain16k"].with_(name="odd_c243_k32", heads=1, T=36, H=36, W=12, topk=32),
]


@pytest.fixture(scope="module", autouse=True)
def _built():
    vsa_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    vsa.load()


def _run(wl, inputs, cube_copies=False):
    q, k, v, gc, gf = (t.cuda() for t in inputs)
    plan = vsa.Plan(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, wl.topk, wl.top_p, wl.kmin, wl.kmax)
    plan.set_cube_major_copies(cube_copies)
    out, idx, cnt = plan.run(q, k, v, gc, gf)
    plan.check()
    return plan, (q, k, v, gc, gf), out, idx, cnt


def _padded(lists, counts, kcap):
    C = lists.shape[0]
    a = np.full((C, kcap), -1, dtype=np.int32)
    a[:, : lists.shape[1]] = lists[:, :kcap]
    return a, counts.astype(np.int32)


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_small_all_stages(wl):
    inputs = synth.make_inputs(wl)
    q, k, v, gc, gf = inputs
    plan, dev_in, out, idx, cnt = _run(wl, inputs, cube_copies=True)
    perm = oracle.cube_perm(wl.T, wl.H, wl.W)
    BH = wl.B * wl.heads
    qc = plan.cube_major("q").cpu().view(wl.B, wl.heads, wl.C * 64, wl.D)
    vcm = plan.cube_major("v").cpu().view(wl.B, wl.heads, wl.C * 64, wl.D)
    qpool = plan.pooled("q").cpu().view(wl.B, wl.heads, wl.C, wl.D)
    kpool = plan.pooled("k").cpu().view(wl.B, wl.heads, wl.C, wl.D)
    vpool = plan.pooled("v").cpu().view(wl.B, wl.heads, wl.C, wl.D)
    idx_h, cnt_h, out_h = idx.cpu().numpy(), cnt.cpu().numpy(), out.float().cpu().numpy()
    ref_idx = np.zeros((wl.B, wl.heads, wl.C, wl.kcap), dtype=np.int32)
    ref_cnt = np.zeros((wl.B, wl.heads, wl.C), dtype=np.int32)
    refs = {}
    for b in range(wl.B):
        for h in range(wl.heads):
            # a1 gather: bit-exact copies
            assert torch.equal(qc[b, h], q[b, h][torch.from_numpy(perm)])
            assert torch.equal(vcm[b, h], v[b, h][torch.from_numpy(perm)])
            r = oracle_head(wl, q, k, v, gc, gf, b, h)
            refs[b, h] = r
            # a2 pool
            assert_close(qpool[b, h].numpy(), r["qbar"], "pooled q", max_abs=1e-5, mean_abs=1e-6)
            assert_close(kpool[b, h].numpy(), r["kbar"], "pooled k", max_abs=1e-5, mean_abs=1e-6)
            assert_close(vpool[b, h].numpy(), r["vbar"], "pooled v", max_abs=1e-5, mean_abs=1e-6)
            # a4 selection
            check_lists(wl, r, idx_h[b, h], cnt_h[b, h])
            ref_idx[b, h], ref_cnt[b, h] = _padded(r["lists"], r["counts"], wl.kcap)
    # a3 / a5 / a6 on the oracle's own lists
    out2, oc, of = plan.run_fixed_idx(*dev_in, torch.from_numpy(ref_idx).cuda(), torch.from_numpy(ref_cnt).cuda(),
                                      want_coarse=True, want_fine=True)
    plan.check()
    oc, of, out2 = oc.cpu().numpy(), of.cpu().numpy(), out2.float().cpu().numpy()
    for (b, h), r in refs.items():
        assert_close(oc[b, h], r["Oc"], "coarse output", max_abs=1e-4, mean_abs=1e-5)
        assert_close(of[b, h], r["Of"], "fine output")
        assert_close(out2[b, h], r["out"], "gated output")
        # whole pass on the GPU's own (validated) lists
        n = cnt_h[b, h]
        r2 = oracle_head(wl, q, k, v, gc, gf, b, h, lists_in=idx_h[b, h], counts_in=n)
        assert_close(out_h[b, h], r2["out"], "end-to-end output")
    assert BH == len(refs)


@pytest.mark.parametrize("name", ["pretrain16k", "long61k_k32", "long61k_k16", "large77k", "dynamic61k"])
def test_full_size_sampled(name):
    """Full-size workloads, sampled heads.

    Per sampled head: every selection row against the oracle's fp64 scores;
    the whole pass on the GPU's own lists at sampled query cubes; then the
    fixed-selection path on the oracle's own lists (the other heads keep the
    GPU's lists), which at these sizes gives each CTA several items: the
    coarse output of every cube, and the fine output before gating and the
    gated output at the sampled cubes, element by element."""
    wl = W[name]
    inputs = synth.make_inputs(wl)
    q, k, v, gc, gf = inputs
    plan, dev_in, out, idx, cnt = _run(wl, inputs)
    heads = sorted({0, wl.heads // 2, wl.heads - 1})
    rng = np.random.default_rng(11)
    exact = exempt = 0
    idx_or = idx.clone()
    cnt_or = cnt.clone()
    sampled = {}
    for h in heads:
        idx_h = idx[0, h].cpu().numpy()
        cnt_h = cnt[0, h].cpu().numpy()
        cubes = sorted({0, wl.C - 1, *rng.choice(wl.C, 10, replace=False).tolist()})
        r = oracle_head(wl, q, k, v, gc, gf, 0, h, query_cubes=cubes, lists_in=idx_h, counts_in=cnt_h)
        # selection of every row of the head against the oracle's scores
        rsel = oracle_head(wl, q, k, v, gc, gf, 0, h, query_cubes=[])
        e1, e2 = check_lists(wl, rsel, idx_h, cnt_h)
        exact += e1
        exempt += e2
        toks = np.concatenate([r["perm"][64 * c: 64 * c + 64] for c in cubes])
        got = out[0, h, torch.from_numpy(toks).cuda()].float().cpu().numpy()
        assert_close(got, r["out"][toks], f"{name} head {h} sampled output")
        ref_idx, ref_cnt = _padded(rsel["lists"], rsel["counts"], wl.kcap)
        idx_or[0, h] = torch.from_numpy(ref_idx).cuda()
        cnt_or[0, h] = torch.from_numpy(ref_cnt).cuda()
        sampled[h] = (cubes, toks, rsel, ref_idx, ref_cnt)
    # fixed-selection path on the oracle's lists
    out2, oc, of = plan.run_fixed_idx(*dev_in, idx_or, cnt_or, want_coarse=True, want_fine=True)
    plan.check()
    for h, (cubes, toks, rsel, ref_idx, ref_cnt) in sampled.items():
        assert_close(oc[0, h].cpu().numpy(), rsel["Oc"], f"{name} head {h} coarse output", max_abs=1e-4,
                     mean_abs=1e-5)
        r = oracle_head(wl, q, k, v, gc, gf, 0, h, query_cubes=cubes, lists_in=ref_idx, counts_in=ref_cnt)
        t = torch.from_numpy(toks).cuda()
        assert_close(of[0, h, t].cpu().numpy(), r["Of"][toks], f"{name} head {h} fine output (oracle lists)")
        assert_close(out2[0, h, t].float().cpu().numpy(), r["out"][toks], f"{name} head {h} gated output (oracle lists)")
    print(f"{name}: exact rows {exact}, exempt rows {exempt} ({exempt / (exact + exempt):.4f})")
    assert exact > 0


def test_flat_forward_matches_plan():
    wl = SMALL[1]
    inputs = synth.make_inputs(wl)
    plan, dev_in, out, idx, cnt = _run(wl, inputs)
    out2, idx2 = vsa.forward(*dev_in, wl.T, wl.H, wl.W, topk=wl.topk)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    assert torch.equal(out, out2)


def test_repeat_runs_are_deterministic():
    wl = SMALL[4]
    inputs = synth.make_inputs(wl)
    plan, dev_in, out, idx, cnt = _run(wl, inputs)
    for _ in range(3):
        o2, i2, c2 = plan.run(*dev_in)
        plan.check()
        assert torch.equal(i2, idx) and torch.equal(c2, cnt) and torch.equal(o2, out)


def test_timeout_path_reports_and_recovers():
    """A wait on a barrier nothing signals gives up, reports VSA_ERR_TIMEOUT,
    and the context stays usable for the next run."""
    wl = SMALL[1]
    inputs = synth.make_inputs(wl)
    plan, dev_in, out, idx, cnt = _run(wl, inputs)
    plan.set_wait_limit_ns(20_000_000)
    plan.set_debug_stall(True)
    plan.run(*dev_in)
    with pytest.raises(vsa.VSAError) as e:
        plan.check()
    assert e.value.code == 6
    plan.set_debug_stall(False)
    o2, i2, _ = plan.run(*dev_in)
    plan.check()
    assert torch.equal(o2, out) and torch.equal(i2, idx)


def test_out_of_range_index_is_reported_not_read():
    wl = SMALL[1]
    inputs = synth.make_inputs(wl)
    plan, dev_in, out, idx, cnt = _run(wl, inputs)
    bad = idx.clone()
    bad[0, 0, 3, 1] = wl.C + 5
    bad[0, 1, 0, 0] = -7
    plan.run_fixed_idx(*dev_in, bad, cnt)
    with pytest.raises(vsa.VSAError) as e:
        plan.check()
    assert e.value.code == 1
    badc = cnt.clone()
    badc[0, 0, 0] = 0
    plan.run_fixed_idx(*dev_in, idx, badc)
    with pytest.raises(vsa.VSAError):
        plan.check()
    o2, i2, _ = plan.run(*dev_in)
    plan.check()
    assert torch.equal(o2, out)


@pytest.mark.parametrize("wl", [SMALL[1], SMALL[6]], ids=["cube_k5_odd", "d64_k7"])
def test_coarse_scores_keep_fp32_accuracy(wl):
    """The coarse products run on the tensor cores with every fp32 operand
    written as three bf16 terms; the scores must stay at fp32 accuracy (a
    single bf16 term would be off by ~1e-3)."""
    inputs = synth.make_inputs(wl)
    plan, dev_in, out, idx, cnt = _run(wl, inputs)
    q, k, v, gc, gf = inputs
    BH = wl.B * wl.heads
    s_gpu = plan.workspace_view("s_coarse", torch.float32, (BH, wl.C, wl.C)).cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.heads):
            r = oracle_head(wl, q, k, v, gc, gf, b, h)
            assert_close(s_gpu[b * wl.heads + h], r["s"], "coarse scores", max_abs=1e-5, mean_abs=1e-6)


@pytest.mark.parametrize("T,H,W_", [(8, 32, 32), (16, 32, 48)], ids=["C128_candidates", "C384_fallback"])
def test_all_equal_scores_select_lowest_ids(T, H, W_):
    """q = 0 makes every coarse score equal: top-K must take cubes 0..K-1 in
    every row (ties to the lower id). With C = 384 every score is a candidate
    above the lane-maxima bound (more than 256), which exercises the full bit
    search of the shared-memory select kernel."""
    wl = W["tiny"].with_(name="zero_q", heads=1, D=64, T=T, H=H, W=W_, topk=8)
    q, k, v, gc, gf = synth.make_inputs(wl)
    q = torch.zeros_like(q)
    plan, dev_in, out, idx, cnt = _run(wl, (q, k, v, gc, gf))
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    assert (cnt_h == 8).all()
    assert (idx_h[0, 0] == np.arange(8, dtype=np.int32)[None, :]).all()
    sample = np.array([0, 1, wl.C // 2, wl.C - 1])
    r = oracle_head(wl, q, k, v, gc, gf, 0, 0, query_cubes=sample)
    perm = oracle.cube_perm(wl.T, wl.H, wl.W)
    toks = perm.reshape(wl.C, 64)[sample].reshape(-1)
    assert_close(out[0, 0].float().cpu().numpy()[toks], r["out"][toks], "output, all-equal scores")


@pytest.mark.parametrize("wl", [SMALL[2], SMALL[5]], ids=["cube_b2", "tiny_topp_d64"])
def test_host_buffers_match_device_run(wl):
    """vsa_run_host (pinned host tensors in and out, per-(batch, head) slices
    pipelined over copy streams) returns exactly what vsa_run returns on the
    same inputs in device memory."""
    inputs = synth.make_inputs(wl)
    plan, dev_in, out, idx, cnt = _run(wl, inputs)
    hin = [t.pin_memory() for t in inputs]
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hidx = torch.full(idx.shape, -5, dtype=idx.dtype).pin_memory()
    hcnt = torch.full(cnt.shape, -5, dtype=cnt.dtype).pin_memory()
    for _ in range(2):  # the second call reuses the device copies and streams
        plan.run_host(*hin, hout, hidx, hcnt)
        plan.check()
        assert torch.equal(hout, out.cpu()) and torch.equal(hidx, idx.cpu()) and torch.equal(hcnt, cnt.cpu())
        hout.zero_()
        hidx.fill_(-5)


@pytest.mark.parametrize("mode", ["topk_all", "topp_kmax1024"])
def test_maximum_cube_count(mode):
    """C = 4096 cubes, the largest the library accepts: every select kernel
    holds a whole 4096-key row in shared memory. topk_all selects every cube
    (K = C, the degenerate case where the fine stage is dense attention over
    all 262,144 keys); topp_kmax1024 runs top-p with the largest kmax."""
    if mode == "topk_all":
        wl = W["pretrain16k"].with_(name="max_c_all", heads=1, D=64, T=16, H=64, W=256, topk=4096)
    else:
        wl = W["dynamic61k"].with_(name="max_c_topp", heads=1, D=64, T=16, H=64, W=256, kmin=4, kmax=1024)
    assert wl.C == 4096
    inputs = synth.make_inputs(wl)
    q, k, v, gc, gf = inputs
    plan, dev_in, out, idx, cnt = _run(wl, inputs)
    idx_h, cnt_h = idx[0, 0].cpu().numpy(), cnt[0, 0].cpu().numpy()
    if mode == "topk_all":
        assert (cnt_h == 4096).all()
        assert (idx_h == np.arange(4096, dtype=np.int32)[None, :]).all()
    else:
        rsel = oracle_head(wl, q, k, v, gc, gf, 0, 0, query_cubes=[])
        check_lists(wl, rsel, idx_h, cnt_h)
    cubes = [0, 1777, 4095]
    r = oracle_head(wl, q, k, v, gc, gf, 0, 0, query_cubes=cubes, lists_in=idx_h, counts_in=cnt_h)
    toks = np.concatenate([r["perm"][64 * c: 64 * c + 64] for c in cubes])
    got = out[0, 0, torch.from_numpy(toks).cuda()].float().cpu().numpy()
    assert_close(got, r["out"][toks], f"{mode} sampled output")


def test_work_order_is_longest_first_per_head():
    """With variable counts the fine step's items are handed out from an order
    array: each head's query cubes by descending count, ties by ascending id,
    heads in sequence (a permutation of all items)."""
    wl = SMALL[4]                                   # top-p, variable counts
    plan, dev_in, out, idx, cnt = _run(wl, synth.make_inputs(wl))
    BH = wl.B * wl.heads
    order = plan.workspace_view("order", torch.int32, (BH * wl.C,)).cpu().numpy()
    counts = cnt.cpu().numpy().reshape(BH, wl.C)
    assert sorted(order.tolist()) == list(range(BH * wl.C))
    for bh in range(BH):
        ids = np.arange(wl.C)
        want = bh * wl.C + ids[np.lexsort((ids, -counts[bh]))]
        assert np.array_equal(order[bh * wl.C:(bh + 1) * wl.C], want)

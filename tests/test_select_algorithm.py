"""CPU replay of the GPU top-K selection's algorithm (top-K <= 32, C <= 1024).

The register-resident select kernel does not sort. Per row of fp32 coarse
scores it:
  1. maps each score to an order-preserving uint32 key;
  2. takes as a lower bound of the K-th largest key the minimum over the 32
     lanes of each lane's largest key (lane t holds columns 64u + 2t, +1; a
     lane that holds no column contributes 0);
  3. keeps the keys at or above that bound as candidates;
  4. finds the K-th largest key T by an MSB-first count search over the
     candidates, starting below the bits the bound and the row maximum share;
  5. emits the ids of the keys above T, then the lowest ids of the keys equal
     to T, ascending (through two 32-word bitmaps);
and with more than 256 candidates it searches all keys instead.

This replays those integer steps with numpy on the same fp32 scores and
checks the lists against the oracle's select_topk (score-ranked, ties to the
lowest id, listed ascending). It pins the algorithm's claims (the bound, the
search window, the tie rule, the fallback) on rows the GPU parity workloads
do not reach: heavy exact ties at the threshold, all-equal rows at every C,
C below 64, K = C. The kernel itself is checked against the oracle by the
GPU parity tests.
"""
import numpy as np
import pytest

import oracle

CAND_CAP = 256


def order_keys(s32):
    """Larger float -> larger uint32 (sign-magnitude to biased order)."""
    u = s32.astype(np.float32).view(np.uint32)
    return np.where(u & np.uint32(0x80000000), ~u, u | np.uint32(0x80000000)).astype(np.uint32)


def lane_of_columns(C):
    """Lane holding each column: column j is in lane (j % 64) // 2."""
    return (np.arange(C) % 64) // 2


def kth_largest(keys, K, start=0, first_bit=31):
    """MSB-first search: the largest T (with the given high bits) such that #{key >= T} >= K."""
    T = start
    for b in range(first_bit, -1, -1):
        c = T | (1 << b)
        if int(np.count_nonzero(keys >= c)) >= K:
            T = c
    return T


def emit(keys, ids, K, T):
    """Ids of the keys above T, then the lowest ids equal to T, ascending."""
    above = ids[keys > T]
    need = K - above.size
    equal = np.sort(ids[keys == T])[:need]
    return np.sort(np.concatenate([above, equal]))


def gpu_select_row(s_row32, K):
    C = s_row32.shape[0]
    keys = order_keys(s_row32)
    lanes = lane_of_columns(C)
    lkmax = np.zeros(32, dtype=np.uint64)
    for t in range(32):
        own = keys[lanes == t]
        if own.size:
            lkmax[t] = own.max()
    lo, hi = int(lkmax.min()), int(lkmax.max())
    cand = np.nonzero(keys >= lo)[0]
    if cand.size <= CAND_CAP:
        ck = keys[cand].astype(np.int64)
        if lo == hi:
            T = lo
        else:
            hb = (lo ^ hi).bit_length() - 1
            T = kth_largest(ck, K, start=hi & ~((2 << hb) - 1) & 0xFFFFFFFF, first_bit=hb)
        return emit(ck, cand, K, T), cand.size
    ka = keys.astype(np.int64)
    return emit(ka, np.arange(C), K, kth_largest(ka, K)), cand.size


def check_rows(s32, K):
    ref = oracle.select_topk(s32.astype(np.float64), K)
    sizes = []
    for i in range(s32.shape[0]):
        got, n = gpu_select_row(s32[i], K)
        sizes.append(n)
        assert np.array_equal(got, ref[i]), (i, K, got, ref[i])
    return np.array(sizes)


@pytest.mark.parametrize("C", [1, 6, 8, 27, 48, 63, 64, 65, 100, 243, 256, 960, 1024])
def test_random_rows_match_oracle(C):
    rng = np.random.default_rng(C)
    s = rng.standard_normal((12, C)).astype(np.float32)
    for K in sorted({1, min(5, C), min(32, C), C if C <= 32 else 32}):
        check_rows(s, K)


@pytest.mark.parametrize("C", [6, 27, 64, 100, 243, 960])
def test_exact_ties_at_the_threshold(C):
    # scores from a handful of values: most rows have many keys equal to T
    rng = np.random.default_rng(1000 + C)
    s = rng.integers(-3, 4, size=(16, C)).astype(np.float32) * 0.25
    for K in sorted({1, min(7, C), min(32, C)}):
        check_rows(s, K)


@pytest.mark.parametrize("C", [5, 40, 64, 200, 257, 960, 1024])
def test_all_equal_rows_take_the_lowest_ids(C):
    s = np.full((3, C), 0.5, dtype=np.float32)
    K = min(32, C)
    sizes = check_rows(s, K)
    assert (sizes == C).all()  # every key sits on the bound
    for i in range(3):
        assert np.array_equal(gpu_select_row(s[i], K)[0], np.arange(K))


def test_candidate_sets_span_every_width():
    # 960 cubes: the bound leaves ~60 candidates; 243 cubes: 65..256; all equal: the fallback
    rng = np.random.default_rng(7)
    widths = []
    for C in (960, 243, 100):
        s = rng.standard_normal((64, C)).astype(np.float32)
        widths.append(check_rows(s, 32))
    w = np.concatenate(widths)
    assert (w > 32).any() and (w > 64).any() and (w > 128).any()
    assert (w <= CAND_CAP).all()


def test_bound_never_excludes_a_selected_key():
    # the K-th largest key is never below the minimum of the lane maxima (K <= 32)
    rng = np.random.default_rng(11)
    for C in (64, 65, 130, 960, 1024):
        s = rng.standard_normal((50, C)).astype(np.float32)
        keys = order_keys(s)
        lanes = lane_of_columns(C)
        for i in range(s.shape[0]):
            lo = min(int(keys[i][lanes == t].max()) for t in range(32))
            kth = np.sort(keys[i])[::-1][31]
            assert kth >= lo


def test_planted_mistake_is_caught():
    # excluding lanes without keys from the bound (instead of letting them
    # contribute 0) breaks rows with fewer than 64 cubes and K near C
    s = np.random.default_rng(3).standard_normal((4, 20)).astype(np.float32)
    K = 20
    ref = oracle.select_topk(s.astype(np.float64), K)
    keys = order_keys(s[0])
    lanes = lane_of_columns(20)
    lo_wrong = min(int(keys[lanes == t].max()) for t in range(32) if (lanes == t).any())
    assert np.count_nonzero(keys >= lo_wrong) < K  # the wrong bound would drop selected cubes
    assert np.array_equal(gpu_select_row(s[0], K)[0], ref[0])

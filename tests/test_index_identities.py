"""The identities the fused index path rests on, checked on the host against the oracle.

The fused path keeps, per 32-token tile and per column (a rank r < R, or an expert slot
R + q), the bit mask of the tile's tokens that reach it. From those masks alone it takes:

* the co-activation histogram: hist[a][b] = sum over the tiles of
  popcount(mask(slot(a)) & mask(slot(b)));
* the dispatched-row counter: per_rank[r] = the popcount total of rank column r,
  total = C_T, and remote = C_T less the own-rank hits, where the hits are the bits of
  rank column r among the tokens t of rank r's batch slice, floor(t * R / T) = r.

These tests build the masks from routings in plain numpy, the way the definitions
read, and compare the counts with the oracle's direct definitions on the ids. The
routings include pruned (empty, -1) slots and permuted placements.
"""
import numpy as np
import pytest

import oracle


def routing(T, E, k, seed, empty_frac=0.0):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    if empty_frac:
        drop = rng.random((T, k)) < empty_frac
        drop[:, 0] = False  # every token keeps at least one expert
        idx[drop] = -1
    return idx


def masks_from_routing(idx, slot_of, E, R):
    """[R + E, n_tiles] uint32 masks: bit l of tile b is token 32 b + l."""
    T, k = idx.shape
    L = E // R
    n_tiles = (T + 31) // 32
    m = np.zeros((R + E, n_tiles), np.uint64)
    for t in range(T):
        b, bit = divmod(t, 32)
        for e in idx[t]:
            if e < 0:
                continue
            q = int(slot_of[e])
            m[R + q, b] |= np.uint64(1) << np.uint64(bit)
            m[q // L, b] |= np.uint64(1) << np.uint64(bit)
    return m


def popcount(x):
    return int(bin(int(x)).count("1"))


CASES = [
    (1000, 64, 8, 8, 0.0, 1),
    (777, 16, 4, 4, 0.3, 2),   # pruned slots; T not a multiple of 32 or R
    (300, 8, 2, 8, 0.0, 3),    # one expert per rank
    (5, 8, 2, 8, 0.0, 4),      # fewer tokens than ranks
    (513, 64, 6, 1, 0.2, 5),   # one rank
]


@pytest.mark.parametrize("T,E,k,R,empty,seed", CASES)
@pytest.mark.parametrize("permuted", [False, True])
def test_histogram_from_masks(T, E, k, R, empty, seed, permuted):
    idx = routing(T, E, k, seed, empty)
    slot_of = (np.random.default_rng(seed + 100).permutation(E) if permuted
               else np.arange(E)).astype(np.int32)
    m = masks_from_routing(idx, slot_of, E, R)
    hist = np.zeros((E, E), np.int64)
    for a in range(E):
        ma = m[R + slot_of[a]]
        for b in range(E):
            mb = m[R + slot_of[b]]
            hist[a, b] = sum(popcount(x & y) for x, y in zip(ma, mb))
    assert np.array_equal(hist, oracle.coact_histogram(idx, E).astype(np.int64))


@pytest.mark.parametrize("T,E,k,R,empty,seed", CASES)
@pytest.mark.parametrize("permuted", [False, True])
def test_counter_from_masks(T, E, k, R, empty, seed, permuted):
    idx = routing(T, E, k, seed, empty)
    slot_of = (np.random.default_rng(seed + 200).permutation(E) if permuted
               else np.arange(E)).astype(np.int32)
    m = masks_from_routing(idx, slot_of, E, R)
    per_rank = np.array([sum(popcount(x) for x in m[r]) for r in range(R)])
    c_t = int(per_rank.sum())
    own = 0
    for r in range(R):
        lo, hi = -(-r * T // R), -(-(r + 1) * T // R)  # ceil: the tokens with floor(t R / T) = r
        assert all(t * R // T == r for t in range(lo, hi))
        for t in range(lo, hi):
            b, bit = divmod(t, 32)
            own += int((int(m[r, b]) >> bit) & 1)
    ref_per_rank, ref_total, ref_remote = oracle.count_dispatched(idx, slot_of, E, R)
    assert np.array_equal(per_rank, ref_per_rank)
    assert c_t == ref_total
    assert c_t - own == ref_remote

"""Pins for the oracle's token-shuffling statistics (no GPU): the inter-layer
pair histogram, the rank affinity table, the predicted home rank, the count of
assignments served on the token's home rank, and the shuffle order."""
import json
import os

import numpy as np
import pytest

import oracle
from expert_warp_top_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _two_layers(T=300, seed=3, follow_p=0.8):
    cfg = inputs.CONFIGS["corr_prefill"].with_(T=T, seed=seed)
    l1, l2 = inputs.make_layer_pair_logits(cfg, follow_p=follow_p)
    i1, _ = oracle.route(l1.numpy(), cfg.k, 0)
    i2, _ = oracle.route(l2.numpy(), cfg.k, 0)
    return cfg, i1, i2


def test_hand_worked_fixture():
    with open(os.path.join(GOLDEN, "shuffle_small.json")) as fh:
        g = json.load(fh)
    a = np.array(g["idx_l"], np.int32)
    b = np.array(g["idx_next"], np.int32)
    slot = np.array(g["slot_of_next"], np.int32)
    H = oracle.interlayer_histogram(a, b, g["E"])
    assert H.tolist() == g["H"]
    A = oracle.rank_affinity(H, slot, g["R"])
    assert A.tolist() == g["A"]
    home = oracle.predict_home(a, A)
    assert home.tolist() == g["home"]
    assert oracle.count_local(b, slot, g["E"], g["R"], home) == tuple(g["local_predicted"])
    assert oracle.count_local(b, slot, g["E"], g["R"]) == tuple(g["local_contiguous"])


def test_same_layer_histogram_is_the_coactivation_histogram():
    _, i1, _ = _two_layers()
    E = 64
    assert np.array_equal(oracle.interlayer_histogram(i1, i1, E), oracle.coact_histogram(i1, E))


def test_histogram_margins():
    cfg, i1, i2 = _two_layers()
    H = oracle.interlayer_histogram(i1, i2, cfg.E).astype(np.int64)
    # every token gives k x k pairs; row a sums to k x (tokens with a at layer l)
    assert H.sum() == cfg.T * cfg.k * cfg.k
    assert np.array_equal(H.sum(1), cfg.k * np.bincount(i1.ravel(), minlength=cfg.E))
    assert np.array_equal(H.sum(0), cfg.k * np.bincount(i2.ravel(), minlength=cfg.E))
    # empty slots count nothing
    i1e = i1.copy()
    i1e[::2, -1] = -1
    He = oracle.interlayer_histogram(i1e, i2, cfg.E).astype(np.int64)
    assert He.sum() == cfg.T * cfg.k * cfg.k - ((cfg.T + 1) // 2) * cfg.k


def test_affinity_special_cases():
    cfg, i1, i2 = _two_layers()
    H = oracle.interlayer_histogram(i1, i2, cfg.E)
    perm = np.random.default_rng(1).permutation(cfg.E).astype(np.int32)
    A = oracle.rank_affinity(H, perm, cfg.R)
    assert np.array_equal(A.sum(1), H.astype(np.uint64).sum(1))  # ranks partition the experts
    assert np.array_equal(oracle.rank_affinity(H, perm, 1)[:, 0], H.astype(np.uint64).sum(1))
    ident = np.arange(cfg.E, dtype=np.int32)
    assert np.array_equal(oracle.rank_affinity(H, ident, cfg.E), H.astype(np.uint64))  # L = 1
    # one expert per rank, permuted: A's columns are H's columns in slot order
    A1 = oracle.rank_affinity(H, perm, cfg.E)
    assert np.array_equal(A1[:, perm], H.astype(np.uint64))


def test_predicted_home_is_the_argmax():
    cfg, i1, i2 = _two_layers(T=500)
    calib_cfg, c1, c2 = _two_layers(T=2000, seed=9)
    slot = np.random.default_rng(4).permutation(cfg.E).astype(np.int32)
    A = oracle.rank_affinity(oracle.interlayer_histogram(c1, c2, cfg.E), slot, cfg.R)
    home = oracle.predict_home(i1, A)
    scores = A[i1.astype(np.int64)].sum(axis=1)          # [T, R]
    expect = np.argmax(scores, axis=1)                    # first maximum = lower rank
    zero = scores.max(axis=1) == 0
    expect[zero] = (np.arange(cfg.T) * cfg.R // cfg.T)[zero]
    assert np.array_equal(home, expect)
    # equal scores on every rank: the lower rank wins
    assert np.array_equal(oracle.predict_home(i1, np.ones_like(A)), np.zeros(cfg.T, np.int32))
    A2 = np.zeros_like(A)
    A2[:, 2] = A2[:, 5] = 7
    assert np.array_equal(oracle.predict_home(i1, A2), np.full(cfg.T, 2, np.int32))
    # a table of zeros leaves every token at its contiguous home
    assert np.array_equal(oracle.predict_home(i1, np.zeros_like(A)),
                          np.arange(cfg.T) * cfg.R // cfg.T)


def test_count_local_closed_forms():
    cfg, i1, i2 = _two_layers()
    slot = np.random.default_rng(5).permutation(cfg.E).astype(np.int32)
    L = cfg.E // cfg.R
    top1 = np.ascontiguousarray(i2[:, :1])
    # k = 1 with the contiguous home: local = T - remote rows of the counter
    _, total, remote = oracle.count_dispatched(top1, slot, cfg.E, cfg.R)
    assert oracle.count_local(top1, slot, cfg.E, cfg.R) == (total - remote, cfg.T)
    # home = the rank of the token's only expert: everything is local
    home = (slot[top1[:, 0]] // L).astype(np.int32)
    assert oracle.count_local(top1, slot, cfg.E, cfg.R, home) == (cfg.T, cfg.T)
    # empty slots are not assignments
    i2e = i2.copy()
    i2e[::3, -1] = -1
    assert oracle.count_local(i2e, slot, cfg.E, cfg.R)[1] == cfg.T * cfg.k - (cfg.T + 2) // 3
    # summed over every possible home, each assignment is local exactly once
    tot = sum(oracle.count_local(i2, slot, cfg.E, cfg.R, np.full(cfg.T, r, np.int32))[0]
              for r in range(cfg.R))
    assert tot == cfg.T * cfg.k


def test_shuffle_order_is_a_stable_sort_by_home():
    cfg, i1, i2 = _two_layers(T=777)
    home = np.random.default_rng(7).integers(0, cfg.R, cfg.T).astype(np.int32)
    # the shuffle is a BRIM_0 over one "expert" per rank: k = 1, E = R
    b = oracle.brim(home[:, None], np.ones((cfg.T, 1)), np.arange(cfg.R, dtype=np.int32),
                    cfg.R, cfg.R)
    assert np.array_equal(b["sfd_token"], np.argsort(home, kind="stable"))
    assert np.array_equal(np.diff(b["sfd_off"]), np.bincount(home, minlength=cfg.R))


def test_planted_affinity_raises_the_local_share():
    cfg, i1, i2 = _two_layers(T=4000, follow_p=1.0)
    _, c1, c2 = _two_layers(T=8000, seed=11, follow_p=1.0)
    # layer l+1 placed by its own co-activation: its planted groups land on ranks
    slot2 = oracle.place_greedy(oracle.coact_histogram(c2, cfg.E), cfg.R)
    A = oracle.rank_affinity(oracle.interlayer_histogram(c1, c2, cfg.E), slot2, cfg.R)
    home = oracle.predict_home(i1, A)
    base, n = oracle.count_local(i2, slot2, cfg.E, cfg.R)
    shuf, _ = oracle.count_local(i2, slot2, cfg.E, cfg.R, home)
    assert abs(base / n - 1 / cfg.R) < 0.03          # contiguous home: ~1/R
    assert shuf / n > 0.6                              # predicted home: most are local

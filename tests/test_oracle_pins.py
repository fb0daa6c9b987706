"""Pins for the CPU oracle (no GPU): each test ties the oracle to something
other than itself -- a hand-worked example, brute force over every k-subset,
a closed form, a library routine on a special case, or an invariant -- so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit, softmax

import oracle
from expert_warp_top_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bfloat16 tensor -> its raw uint16 bits (the oracle widens them)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------
# routing: brute force over all C(E, k) subsets
# --------------------------------------------------------------------------
def _brute_topk_set(row, k):
    """Among all k-subsets with the maximal logit sum, the one whose sorted id
    tuple is lexicographically smallest (= the 'lower id wins ties' rule)."""
    best = None
    for sub in itertools.combinations(range(len(row)), k):
        s = sum(float(row[i]) for i in sub)
        key = (-s, sub)
        if best is None or key < best:
            best = key
    return set(best[1])


@pytest.mark.parametrize("renorm", [0, 1])
def test_route_matches_bruteforce_tiny(renorm):
    cfg = inputs.CONFIGS["tiny"]
    logits = inputs.make_logits(cfg).numpy()
    # plant ties: round a quarter of the rows to one decimal so equal logits occur
    logits[::4] = np.round(logits[::4], 1)
    logits[1::16, :] = 0.5  # whole rows of equal logits
    idx, w = oracle.route(logits, cfg.k, renorm)
    for t in range(cfg.T):
        row = logits[t]
        assert set(idx[t].tolist()) == _brute_topk_set(row, cfg.k), t
        # output order: descending logit, equal logits by ascending id
        keys = [(-float(row[e]), int(e)) for e in idx[t]]
        assert keys == sorted(keys)
        # gate weights against scipy's softmax (a library routine)
        if renorm:
            ref = softmax(row[idx[t]].astype(np.float64))
        else:
            ref = softmax(row.astype(np.float64))[idx[t]]
        np.testing.assert_allclose(w[t], ref, rtol=1e-13, atol=0)


def test_route_weight_sums():
    cfg = inputs.CONFIGS["olmoe"].with_(T=512)
    logits = inputs.make_logits(cfg).numpy()
    _, w0 = oracle.route(logits, cfg.k, 0)
    _, w1 = oracle.route(logits, cfg.k, 1)
    assert np.all(w0.sum(1) <= 1 + 1e-12) and np.all(w0 > 0)
    np.testing.assert_allclose(w1.sum(1), 1.0, rtol=1e-13)
    # renormalising is a per-row rescale of the full-softmax weights
    np.testing.assert_allclose(w1, w0 / w0.sum(1, keepdims=True), rtol=1e-12)


def test_route_k_equals_e_and_k_one():
    logits = np.array([[0.1, 3.0, -2.0, 3.0]], np.float32)
    idx, w = oracle.route(logits, 4, 0)
    assert idx.tolist() == [[1, 3, 0, 2]]
    np.testing.assert_allclose(w.sum(), 1.0, rtol=1e-14)
    idx1, w1 = oracle.route(logits, 1, 1)
    assert idx1.tolist() == [[1]] and w1[0, 0] == 1.0


# --------------------------------------------------------------------------
# BRIMs, counter and histogram: the hand-worked example
# --------------------------------------------------------------------------
def _golden():
    with open(os.path.join(GOLDEN, "brim_small.json")) as fh:
        return json.load(fh)


@pytest.mark.parametrize("case", [0, 1])
def test_brim_hand_worked(case):
    g = _golden()
    c = g["cases"][case]
    idx = np.array(g["topk_idx"], np.int32)
    w = np.array(g["topk_w"], np.float64)
    b = oracle.brim(idx, w, np.array(c["slot_of"], np.int32), g["E"], g["R"])
    assert b["c_t"] == c["c_t"]
    assert b["sfd_off"].tolist() == c["sfd_off"]
    assert b["brim0"].tolist() == c["brim0"]
    assert b["sfd_token"].tolist() == c["sfd_token"]
    assert b["epd_off"].tolist() == c["epd_off"]
    assert b["brim1"].tolist() == c["brim1"]
    assert b["epd_sfd"].tolist() == c["epd_sfd"]
    assert b["epd_gate"].tolist() == c["epd_gate"]
    per_rank, total, remote = oracle.count_dispatched(idx, np.array(c["slot_of"], np.int32),
                                                      g["E"], g["R"])
    assert per_rank.tolist() == c["per_rank"] and total == c["total"] and remote == c["remote"]


def test_histogram_hand_worked():
    g = _golden()
    h = oracle.coact_histogram(np.array(g["topk_idx"], np.int32), g["E"])
    assert h.tolist() == g["coact_hist"]
    h2 = oracle.coact_histogram(np.array(g["topk_idx"], np.int32), g["E"], hist=h.copy())
    assert (h2 == 2 * h).all()


# --------------------------------------------------------------------------
# BRIM invariants and closed forms on random routings
# --------------------------------------------------------------------------
def _check_brim_invariants(idx, b, slot_of, E, R):
    T, k = idx.shape
    L = E // R
    c_t = b["c_t"]
    assert c_t <= T * min(k, R)
    # each SFD row appears exactly once in BRIM_0
    pos = b["brim0"][b["brim0"] >= 0]
    assert sorted(pos.tolist()) == list(range(c_t))
    # sfd_token is the inverse of BRIM_0, ascending inside each segment
    for r in range(R):
        seg = b["sfd_token"][b["sfd_off"][r]:b["sfd_off"][r + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.array_equal(b["brim0"][r, seg], np.arange(b["sfd_off"][r], b["sfd_off"][r + 1]))
    # exactly T*k non-negative BRIM_1 entries in the first C_T columns, a bijection onto EPD rows
    valid = b["brim1"][:, :c_t]
    ent = valid[valid >= 0]
    assert sorted(ent.tolist()) == list(range(T * k))
    assert np.all(b["brim1"][:, c_t:] == -1)
    # epd_sfd is the inverse of BRIM_1; the SFD row's token selected that expert
    expert_at_slot = np.empty(E, np.int64)
    expert_at_slot[slot_of] = np.arange(E)
    for l in range(L):
        for s in np.nonzero(valid[l] >= 0)[0]:
            p = valid[l, s]
            assert b["epd_sfd"][p] == s
            q = np.searchsorted(b["epd_off"], p, side="right") - 1
            assert q % L == l
            r = q // L
            assert b["sfd_off"][r] <= s < b["sfd_off"][r + 1]
            assert expert_at_slot[q] in idx[b["sfd_token"][s]]


@pytest.mark.parametrize("T,E,k,R", [(1, 8, 2, 4), (7, 8, 2, 4), (300, 64, 8, 8),
                                     (257, 64, 6, 8), (100, 16, 4, 16), (64, 256, 16, 8)])
def test_brim_invariants_random(T, E, k, R):
    idx = inputs.random_topk(T, E, k, seed=T + E).numpy()
    w = np.random.default_rng(0).random((T, k))
    rng = np.random.default_rng(1)
    for slot_of in (np.arange(E, dtype=np.int32), rng.permutation(E).astype(np.int32)):
        b = oracle.brim(idx, w, slot_of, E, R)
        _check_brim_invariants(idx, b, slot_of, E, R)
        per_rank, total, _ = oracle.count_dispatched(idx, slot_of, E, R)
        assert total == b["c_t"]
        assert np.array_equal(per_rank, np.diff(b["sfd_off"]))


def test_c_t_closed_forms():
    T, E, k = 333, 16, 4
    idx = inputs.random_topk(T, E, k, seed=3).numpy()
    w = np.ones((T, k))
    ident = np.arange(E, dtype=np.int32)
    # one rank: every token is sent exactly once
    assert oracle.brim(idx, w, ident, E, 1)["c_t"] == T
    # one expert per rank: every (token, expert) pair is its own row
    assert oracle.brim(idx, w, ident, E, E)["c_t"] == T * k
    # all tokens to one expert
    same = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    b = oracle.brim(same, w, ident, E, 4)
    assert b["c_t"] == T and b["epd_off"][1] == T and b["epd_off"][k] == T * k


def test_c_t_matches_uniform_expectation():
    # E[C_T] = T * R * (1 - C(E-L, k) / C(E, k)) under uniform routing
    for (T, E, k, R) in [(4096, 64, 8, 8), (4096, 64, 6, 8)]:
        L = E // R
        idx = inputs.random_topk(T, E, k, seed=11).numpy()
        b = oracle.brim(idx, np.ones((T, k)), np.arange(E, dtype=np.int32), E, R)
        expect = T * R * (1 - math.comb(E - L, k) / math.comb(E, k))
        sigma_bound = math.sqrt(T) * (min(k, R) - 1) / 2  # Popoviciu per-token bound
        assert abs(b["c_t"] - expect) < 4 * sigma_bound, (b["c_t"], expect)


def test_remote_rows_closed_forms():
    T, E, k, R = 240, 32, 3, 8
    L = E // R
    ident = np.arange(E, dtype=np.int32)
    src = (np.arange(T) * R) // T
    # every token picks k experts on its own source rank: nothing is remote
    own = np.stack([src * L + j for j in range(k)], 1).astype(np.int32)
    per_rank, total, remote = oracle.count_dispatched(own, ident, E, R)
    assert total == T and remote == 0 and per_rank.tolist() == [T // R] * R
    # every token picks experts on the next rank only: every row is remote
    nxt = np.stack([((src + 1) % R) * L + j for j in range(k)], 1).astype(np.int32)
    _, total, remote = oracle.count_dispatched(nxt, ident, E, R)
    assert total == T and remote == T
    # one rank: nothing can be remote
    idx = inputs.random_topk(T, E, k, seed=9).numpy()
    _, total, remote = oracle.count_dispatched(idx, ident, E, 1)
    assert total == T and remote == 0


def test_greedy_placement_hand_worked():
    # seed = largest diagonal (expert 2); candidates 0 and 1 tie on score 2, the
    # larger diagonal (expert 0) wins; rank 1 is seeded by expert 1 (diag 4 > 3)
    h = np.array([[5, 0, 2, 0], [0, 4, 2, 0], [2, 2, 6, 1], [0, 0, 1, 3]], np.uint32)
    assert oracle.place_greedy(h, 2).tolist() == [1, 2, 0, 3]
    # equal score and equal diagonal: the lower id wins
    h2 = h.copy(); h2[1, 1] = 5
    assert oracle.place_greedy(h2, 2).tolist() == [1, 2, 0, 3]
    h3 = h.copy(); h3[0, 0] = 3; h3[1, 1] = 5
    assert oracle.place_greedy(h3, 2).tolist() == [2, 1, 0, 3]


def test_histogram_invariants():
    T, E, k = 1000, 64, 6
    idx = inputs.random_topk(T, E, k, seed=5).numpy()
    h = oracle.coact_histogram(idx, E).astype(np.int64)
    assert np.array_equal(h, h.T)
    assert np.trace(h) == T * k
    assert np.triu(h, 1).sum() == T * k * (k - 1) // 2
    # brute force on a handful of pairs
    for (a, bb) in [(0, 1), (5, 9), (63, 2), (7, 7)]:
        n = sum(1 for t in range(T) if a in idx[t] and bb in idx[t])
        assert h[a, bb] == n


# --------------------------------------------------------------------------
# dispatch / combine: round trip and identity experts
# --------------------------------------------------------------------------
def test_permute_unpermute_roundtrip():
    cfg = inputs.CONFIGS["tiny"]
    inp = inputs.make_inputs(cfg, weights=False)
    x = bf16_bits(inp["x"])
    idx, w = oracle.route(inp["logits"].numpy(), cfg.k, 0)
    slot_of = np.random.default_rng(2).permutation(cfg.E).astype(np.int32)
    b = oracle.brim(idx, w, slot_of, cfg.E, cfg.R)
    x_sfd = oracle.gather_rows(x, b["sfd_token"])
    x_epd = oracle.gather_rows(x_sfd, b["epd_sfd"])
    # unpermute SFD through BRIM_0: every copy equals its ORI row bit for bit
    for r in range(cfg.R):
        for t in range(cfg.T):
            s = b["brim0"][r, t]
            if s >= 0:
                assert np.array_equal(x_sfd[s], x[t])
    # EPD rows are the ORI rows of their tokens
    assert np.array_equal(x_epd, x[b["sfd_token"][b["epd_sfd"]]])


@pytest.mark.parametrize("renorm", [0, 1])
def test_identity_experts_return_gate_sum_times_x(renorm):
    cfg = inputs.CONFIGS["tiny"].with_(dtype="f32")
    inp = inputs.make_inputs(cfg, weights=False)
    x = inp["x"].numpy()
    idx, w = oracle.route(inp["logits"].numpy(), cfg.k, renorm)
    slot_of = np.arange(cfg.E, dtype=np.int32)
    b = oracle.brim(idx, w, slot_of, cfg.E, cfg.R)
    _, y = oracle.occult_layer(x, slot_of, cfg.E, cfg.R, cfg.k, b, None, None, None,
                               kind=oracle.KIND_IDENTITY)
    ref = w.sum(1, keepdims=True) * x.astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=4 * np.finfo(np.float64).eps, atol=1e-300)


# --------------------------------------------------------------------------
# the expert FFN: closed forms on structured weights
# --------------------------------------------------------------------------
def test_swiglu_closed_form_structured_weights():
    # Wg = c*I, Wu = I, Wd = P (a non-symmetric permutation):
    #   o = P (silu(c a) * a), silu(z) = z * sigmoid(z)   (sigmoid via scipy)
    d = 8
    rng = np.random.default_rng(7)
    a = rng.standard_normal(d)
    c = 1.75
    perm = np.roll(np.arange(d), 3)
    P = np.eye(d)[perm]
    wg = np.ascontiguousarray(c * np.eye(d))
    wu = np.eye(d)
    o = oracle.expert_row(a, wg, wu, np.ascontiguousarray(P))
    z = c * a
    expect = P @ (z * expit(z) * a)
    np.testing.assert_allclose(o, expect, rtol=1e-14, atol=1e-15)
    # swapping the roles of gate and up changes the answer (c != 1)
    o_swapped = oracle.expert_row(a, wu, wg, np.ascontiguousarray(P))
    assert not np.allclose(o_swapped, o)


def test_swiglu_rectangular_rank_one():
    # Wg = g1 * e_0^T (f x d), Wu = u1 * e_1^T, Wd = v * e_2^T (d x f):
    #   gate_i = g1_i a_0, up_i = u1_i a_1, o = v * silu(g1_2 a_0) * u1_2 a_1
    d, f = 6, 5
    rng = np.random.default_rng(8)
    a = rng.standard_normal(d)
    g1, u1, v = rng.standard_normal(f), rng.standard_normal(f), rng.standard_normal(d)
    wg = np.zeros((f, d)); wg[:, 0] = g1
    wu = np.zeros((f, d)); wu[:, 1] = u1
    wd = np.zeros((d, f)); wd[:, 2] = v
    o = oracle.expert_row(a, wg, wu, wd)
    z = g1[2] * a[0]
    expect = v * (z * expit(z)) * (u1[2] * a[1])
    np.testing.assert_allclose(o, expect, rtol=1e-14, atol=1e-16)


def test_bf16_widening_is_exact():
    vals = torch.tensor([1.0, -2.5, 3.140625, 1e-3, 65280.0], dtype=torch.bfloat16)
    a = np.zeros(5); a[0] = 1.0
    # Wd = I (5x5), Wg picks column 0 with weight vals, Wu picks col 0 with weight 1
    wg = torch.zeros(5, 5, dtype=torch.bfloat16); wg[:, 0] = vals
    wu = torch.zeros(5, 5, dtype=torch.bfloat16); wu[:, 0] = 1
    wd = torch.eye(5, dtype=torch.bfloat16)
    o = oracle.expert_row(a, bf16_bits(wg), bf16_bits(wu), bf16_bits(wd))
    z = vals.double().numpy()
    np.testing.assert_allclose(o, z * expit(z), rtol=1e-14)


# --------------------------------------------------------------------------
# the BRIM-guided layer equals the dense definition; shared experts add exactly
# --------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,renorm,perm", [("f32", 0, False), ("bf16", 1, True),
                                               ("bf16", 0, True)])
def test_occult_emulation_equals_dense(dtype, renorm, perm):
    cfg = inputs.CONFIGS["tiny"].with_(dtype=dtype, T=96, S=1, fs=64)
    inp = inputs.make_inputs(cfg)
    conv = bf16_bits if dtype == "bf16" else (lambda t: t.numpy())
    x = conv(inp["x"])
    wg, wu, wd = conv(inp["wg"]), conv(inp["wu"]), conv(inp["wd"])
    shared = (conv(inp["sg"]), conv(inp["su"]), conv(inp["sd"]))
    idx, w = oracle.route(inp["logits"].numpy(), cfg.k, renorm)
    slot_of = (np.random.default_rng(4).permutation(cfg.E) if perm
               else np.arange(cfg.E)).astype(np.int32)
    b = oracle.brim(idx, w, slot_of, cfg.E, cfg.R)
    y_sfd, y = oracle.occult_layer(x, slot_of, cfg.E, cfg.R, cfg.k, b, wg, wu, wd,
                                   shared=shared)
    y_dense = oracle.dense_layer(x, idx, w, wg, wu, wd, shared=shared)
    scale = np.abs(y_dense).max(1, keepdims=True)
    assert np.all(np.abs(y - y_dense) <= 1e-12 * scale)
    # the return rows summed per token give back the routed output
    y_routed = np.zeros_like(y)
    for r in range(cfg.R):
        for t in range(cfg.T):
            s = b["brim0"][r, t]
            if s >= 0:
                y_routed[t] += y_sfd[s]
    y_nos = oracle.dense_layer(x, idx, w, wg, wu, wd)
    assert np.all(np.abs(y_routed - y_nos) <= 1e-12 * scale)
    # token subset of the dense definition = the same rows of the full run
    sub = np.array([5, 0, 95, 17], np.int32)
    np.testing.assert_array_equal(oracle.dense_layer(x, idx, w, wg, wu, wd, shared=shared,
                                                     tokens=sub), y_dense[sub])


def test_shared_experts_add_exactly():
    cfg = inputs.CONFIGS["tiny"].with_(T=32, S=2, fs=64)
    inp = inputs.make_inputs(cfg)
    x = bf16_bits(inp["x"])
    wg, wu, wd = bf16_bits(inp["wg"]), bf16_bits(inp["wu"]), bf16_bits(inp["wd"])
    sg, su, sd = bf16_bits(inp["sg"]), bf16_bits(inp["su"]), bf16_bits(inp["sd"])
    idx, w = oracle.route(inp["logits"].numpy(), cfg.k, 0)
    slot_of = np.arange(cfg.E, dtype=np.int32)
    b = oracle.brim(idx, w, slot_of, cfg.E, cfg.R)
    _, y_routed = oracle.occult_layer(x, slot_of, cfg.E, cfg.R, cfg.k, b, wg, wu, wd)
    _, y_all = oracle.occult_layer(x, slot_of, cfg.E, cfg.R, cfg.k, b, wg, wu, wd,
                                   shared=(sg, su, sd))
    xd = inp["x"].double().numpy()
    expect = y_routed.copy()
    for t in range(cfg.T):
        for s in range(cfg.S):
            expect[t] += oracle.expert_row(xd[t], sg[s], su[s], sd[s])
    assert np.array_equal(y_all, expect)


# --------------------------------------------------------------------------
# correlated placement recovers planted groups
# --------------------------------------------------------------------------
def test_greedy_placement_recovers_planted_groups():
    cfg = inputs.CONFIGS["corr_prefill"].with_(T=4096, seed=1)
    logits = inputs.make_logits(cfg).numpy()
    idx, _ = oracle.route(logits, cfg.k, 0)
    h = oracle.coact_histogram(idx, cfg.E)
    slot_of = oracle.place_greedy(h, cfg.R)
    assert sorted(slot_of.tolist()) == list(range(cfg.E))
    member = inputs.group_members(cfg.E, cfg.groups).numpy()
    for r in range(cfg.R):
        experts = np.nonzero(slot_of // cfg.L == r)[0]
        assert len(set(member[experts].tolist())) == 1, (r, experts, member[experts])
    # fewer dispatched rows than contiguous placement, close to 0.8 + 0.2 * E[ranks]
    _, c_contig, _ = oracle.count_dispatched(idx, np.arange(cfg.E, dtype=np.int32), cfg.E, cfg.R)
    _, c_corr, _ = oracle.count_dispatched(idx, slot_of, cfg.E, cfg.R)
    assert c_corr < 0.5 * c_contig
    L = cfg.L
    uniform = cfg.R * (1 - math.comb(cfg.E - L, cfg.k) / math.comb(cfg.E, cfg.k))
    assert abs(c_corr / cfg.T - (0.8 + 0.2 * uniform)) < 0.05


# --------------------------------------------------------------------------
# routing-score-based collaboration pruning
# --------------------------------------------------------------------------
def test_prune_hand_worked():
    with open(os.path.join(GOLDEN, "prune_small.json")) as fh:
        g = json.load(fh)
    idx = np.array(g["topk_idx"], np.int32)
    w = np.array(g["topk_w"], np.float64)
    ident = np.arange(g["E"], dtype=np.int32)
    assert oracle.brim(idx, w, ident, g["E"], g["R"])["c_t"] == g["c_t_before"]
    pi, pw = oracle.prune(idx, w, ident, g["E"], g["R"], g["m"])
    assert pi.tolist() == g["pruned_idx"]
    np.testing.assert_allclose(pw, np.array(g["pruned_w"]), rtol=1e-15)
    assert oracle.brim(pi, pw, ident, g["E"], g["R"])["c_t"] == g["c_t_after"]
    # m = R keeps everything
    pi2, pw2 = oracle.prune(idx, w, ident, g["E"], g["R"], g["R"])
    assert np.array_equal(pi2, idx) and np.array_equal(pw2, w)


@pytest.mark.parametrize("m", [1, 2, 3, 8])
def test_prune_properties(m):
    cfg = inputs.CONFIGS["olmoe"].with_(T=600)
    idx, w = oracle.route(inputs.make_logits(cfg).numpy(), cfg.k, 0)
    slot_of = np.random.default_rng(6).permutation(cfg.E).astype(np.int32)
    pi, pw = oracle.prune(idx, w, slot_of, cfg.E, cfg.R, m)
    L = cfg.L
    # gate sums are preserved; dropped entries carry no weight
    np.testing.assert_allclose(pw.sum(1), w.sum(1), rtol=1e-13)
    assert np.all(pw[pi == -1] == 0)
    # kept entries are unchanged ids in their places; at most m ranks per token;
    # the top-1 expert is always kept
    keep = pi != -1
    assert np.array_equal(pi[keep], idx[keep])
    assert np.all(pi[:, 0] == idx[:, 0])
    for t in range(cfg.T):
        ranks = {slot_of[e] // L for e in pi[t] if e != -1}
        assert len(ranks) <= m
        # a kept rank is one of the first m distinct ranks of the original order
        first = []
        for e in idx[t]:
            r = slot_of[e] // L
            if r not in first:
                first.append(r)
        assert ranks == set(first[:m])
    # BRIMs and counter with empty slots: one EPD row per kept assignment
    b = oracle.brim(pi, pw, slot_of, cfg.E, cfg.R)
    _check_brim_invariants_with_empty(pi, b, cfg.E, cfg.R)
    _, total, _ = oracle.count_dispatched(pi, slot_of, cfg.E, cfg.R)
    assert total == b["c_t"] <= cfg.T * m
    if m == 1:
        assert b["c_t"] == cfg.T


def _check_brim_invariants_with_empty(idx, b, E, R):
    n_valid = int((idx != -1).sum())
    assert b["epd_off"][E] == n_valid
    valid = b["brim1"][:, :b["c_t"]]
    assert sorted(valid[valid >= 0].tolist()) == list(range(n_valid))
    assert sorted(b["brim0"][b["brim0"] >= 0].tolist()) == list(range(b["c_t"]))


def test_pruned_layer_emulation_equals_dense():
    cfg = inputs.CONFIGS["tiny"].with_(T=64, E=8, k=4, R=4)
    inp = inputs.make_inputs(cfg)
    x = bf16_bits(inp["x"])
    wg, wu, wd = bf16_bits(inp["wg"]), bf16_bits(inp["wu"]), bf16_bits(inp["wd"])
    idx, w = oracle.route(inp["logits"].numpy(), cfg.k, 0)
    slot_of = np.arange(cfg.E, dtype=np.int32)
    pi, pw = oracle.prune(idx, w, slot_of, cfg.E, cfg.R, 1)
    b = oracle.brim(pi, pw, slot_of, cfg.E, cfg.R)
    _, y = oracle.occult_layer(x, slot_of, cfg.E, cfg.R, cfg.k, b, wg, wu, wd)
    y_dense = oracle.dense_layer(x, pi, pw, wg, wu, wd)
    scale = np.abs(y_dense).max(1, keepdims=True)
    assert np.all(np.abs(y - y_dense) <= 1e-12 * scale)
    # identity experts: a pruned token returns its (preserved) gate sum times x
    _, yi = oracle.occult_layer(inp["x"].float().numpy(), slot_of, cfg.E, cfg.R, cfg.k, b,
                                None, None, None, kind=oracle.KIND_IDENTITY)
    np.testing.assert_allclose(yi, w.sum(1, keepdims=True) * inp["x"].double().numpy(),
                               rtol=1e-12)

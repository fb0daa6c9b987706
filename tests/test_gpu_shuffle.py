"""Token shuffling across layers on the GPU against the oracle: the inter-layer
histogram, the rank affinity table, the predicted home rank, the count of
assignments served on the home rank and the shuffled token order and rows.
All integer work: compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _routes(cfg, follow_p=0.8, seed=None):
    l1, l2 = inputs.make_layer_pair_logits(cfg, follow_p=follow_p, seed=seed)
    i1, _ = oracle.route(l1.numpy(), cfg.k, 0)
    i2, _ = oracle.route(l2.numpy(), cfg.k, 0)
    return i1, i2


def _t(a, dtype=torch.int32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).to(DEV)


CASES = [
    inputs.CONFIGS["corr_prefill"].with_(name="small", T=777, seed=3),
    inputs.CONFIGS["corr_prefill"].with_(name="e256", T=500, E=256, k=16, R=64, seed=4),
    inputs.CONFIGS["corr_prefill"].with_(name="e8", T=300, E=8, k=2, R=4, groups=2, seed=5),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_statistics_match_oracle(cfg):
    i1, i2 = _routes(cfg)
    i1[::7, -1] = -1  # empty slots count nothing
    slot = np.random.default_rng(cfg.seed).permutation(cfg.E).astype(np.int32)
    H_ref = oracle.interlayer_histogram(i1, i2, cfg.E)
    hist = torch.full((cfg.E, cfg.E), 7, dtype=torch.int32, device=DEV)
    moe.moe_interlayer_histogram(_t(i1), _t(i2), cfg.E, hist, accumulate=0)
    moe.moe_interlayer_histogram(_t(i1), _t(i2), cfg.E, hist, accumulate=1)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert np.array_equal(hist.cpu().numpy().astype(np.int64), 2 * H_ref.astype(np.int64))
    A_ref = oracle.rank_affinity(H_ref, slot, cfg.R)
    table = torch.empty(cfg.E, cfg.R, dtype=torch.int32, device=DEV)
    moe.moe_rank_affinity(_t(H_ref.astype(np.int32)), _t(slot), cfg.R, table)
    torch.cuda.synchronize()
    assert np.array_equal(table.cpu().numpy().astype(np.uint64), A_ref)
    home_ref = oracle.predict_home(i1, A_ref)
    home = torch.empty(cfg.T, dtype=torch.int32, device=DEV)
    moe.moe_predict_home(_t(i1), table, home)
    out = torch.empty(2, dtype=torch.int64, device=DEV)
    moe.moe_count_local(_t(i2), _t(slot), cfg.E, cfg.R, out, home=home)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert np.array_equal(home.cpu().numpy(), home_ref)
    assert tuple(out.cpu().tolist()) == oracle.count_local(i2, slot, cfg.E, cfg.R, home_ref)
    moe.moe_count_local(_t(i2), _t(slot), cfg.E, cfg.R, out)
    torch.cuda.synchronize()
    assert tuple(out.cpu().tolist()) == oracle.count_local(i2, slot, cfg.E, cfg.R)


def test_predict_home_ties_and_zeros():
    cfg = CASES[0]
    i1, _ = _routes(cfg)
    eq = np.full((cfg.E, cfg.R), 5, np.uint64)           # equal scores: rank 0
    two = np.zeros((cfg.E, cfg.R), np.uint64)
    two[:, 3] = two[:, 6] = 9                            # tie between 3 and 6: rank 3
    zero = np.zeros((cfg.E, cfg.R), np.uint64)           # no information: contiguous home
    for A in (eq, two, zero):
        home = torch.empty(cfg.T, dtype=torch.int32, device=DEV)
        moe.moe_predict_home(_t(i1), _t(A.astype(np.int32)), home)
        torch.cuda.synchronize()
        assert np.array_equal(home.cpu().numpy(), oracle.predict_home(i1, A))


@pytest.mark.parametrize("T,R", [(1, 8), (31, 4), (1000, 8), (4097, 64)])
def test_token_shuffle_order_and_rows(T, R):
    rng = np.random.default_rng(T + R)
    home = rng.integers(0, R, T).astype(np.int32)
    x = torch.randn(T, 256, generator=torch.Generator().manual_seed(T)).to(torch.bfloat16)
    perm = torch.empty(T, dtype=torch.int32, device=DEV)
    inv = torch.empty(T, dtype=torch.int32, device=DEV)
    rank_off = torch.empty(R + 1, dtype=torch.int32, device=DEV)
    x_out = torch.empty(T, 256, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(moe.moe_token_shuffle_workspace_size(T, R), dtype=torch.uint8, device=DEV)
    moe.moe_token_shuffle(_t(home), R, perm, rank_off, ws, x=x.to(DEV), x_out=x_out, inv=inv)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    # the order: BRIM_0 over one "expert" per rank in the oracle (k = 1, E = R)
    b = oracle.brim(home[:, None], np.ones((T, 1)), np.arange(R, dtype=np.int32), R, R)
    p = perm.cpu().numpy()
    assert np.array_equal(p, b["sfd_token"])
    assert np.array_equal(rank_off.cpu().numpy(), b["sfd_off"])
    assert np.array_equal(inv.cpu().numpy()[p], np.arange(T))
    assert torch.equal(x_out.cpu(), x[torch.from_numpy(p).long()])


def test_full_size_pipeline_matches_oracle():
    """Calibration batch -> layer-(l+1) placement from its co-activation ->
    affinity -> predicted homes of the evaluation batch -> served-locally
    counts, every step on the GPU, against the oracle on the same routes."""
    cfg = inputs.CONFIGS["corr_prefill"]
    calib = cfg.with_(seed=1)
    c1, c2 = _routes(calib)
    i1, i2 = _routes(cfg)
    E, R = cfg.E, cfg.R
    coact = torch.zeros(E, E, dtype=torch.int32, device=DEV)
    moe.moe_coact_histogram(_t(c2), E, coact, 0)
    slot = moe.moe_place_greedy(coact.cpu(), R)
    slot_ref = oracle.place_greedy(oracle.coact_histogram(c2, E), R)
    assert np.array_equal(slot.numpy(), slot_ref)
    hist = torch.empty(E, E, dtype=torch.int32, device=DEV)
    moe.moe_interlayer_histogram(_t(c1), _t(c2), E, hist, 0)
    table = torch.empty(E, R, dtype=torch.int32, device=DEV)
    moe.moe_rank_affinity(hist, slot.to(DEV), R, table)
    home = torch.empty(cfg.T, dtype=torch.int32, device=DEV)
    moe.moe_predict_home(_t(i1), table, home)
    out = torch.empty(2, dtype=torch.int64, device=DEV)
    moe.moe_count_local(_t(i2), slot.to(DEV), E, R, out, home=home)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    A_ref = oracle.rank_affinity(oracle.interlayer_histogram(c1, c2, E), slot_ref, R)
    home_ref = oracle.predict_home(i1, A_ref)
    assert np.array_equal(home.cpu().numpy(), home_ref)
    got = tuple(out.cpu().tolist())
    assert got == oracle.count_local(i2, slot_ref, E, R, home_ref)
    base = oracle.count_local(i2, slot_ref, E, R)
    assert got[0] / got[1] > 2 * base[0] / base[1]   # the shuffle serves far more locally


def test_empty_batch():
    hist = torch.full((8, 8), 5, dtype=torch.int32, device=DEV)
    e = torch.empty(0, 2, dtype=torch.int32, device=DEV)
    moe.moe_interlayer_histogram(e, e, 8, hist, 0)
    out = torch.full((2,), 9, dtype=torch.int64, device=DEV)
    moe.moe_count_local(e, torch.arange(8, dtype=torch.int32, device=DEV), 8, 4, out)
    rank_off = torch.full((5,), 9, dtype=torch.int32, device=DEV)
    perm = torch.empty(0, dtype=torch.int32, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    moe.moe_token_shuffle(torch.empty(0, dtype=torch.int32, device=DEV), 4, perm, rank_off, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert not hist.any() and not out.any() and not rank_off.any()

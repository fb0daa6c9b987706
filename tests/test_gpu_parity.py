"""CUDA path vs the CPU oracle, through the C ABI, on seeded synthetic inputs.

Indices, counts, BRIMs and C_T must match bit for bit; copies must be bit
exact; gate weights match to fp32 rounding; layer outputs match within the
per-row normwise tolerance OUT_RTOL (bf16 data, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import oracle
import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs
from expert_warp_top_b200.layer import MoELayer
from helpers import OUT_RTOL, expert_at_slot, oracle_route, rowwise_rel_err, to_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def softmax_rtol(E: int) -> float:
    # fp32 expf (a few ulp) + an fp32 sum of E terms + one division, vs double
    return (E + 8) * 2.0 ** -23


def make_layer(cfg, inp, slot_of=None, ffn_kind=moe.MOE_FFN_SWIGLU, epd_mode="auto", prune_m=0):
    dt = inputs.torch_dtype(cfg)
    kw = {}
    if ffn_kind == moe.MOE_FFN_SWIGLU:
        kw = dict(wg=inp["wg"].to(DEV), wu=inp["wu"].to(DEV), wd=inp["wd"].to(DEV))
        if cfg.S:
            kw.update(sg=inp["sg"].to(DEV), su=inp["su"].to(DEV), sd=inp["sd"].to(DEV))
    return MoELayer(T=cfg.T, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k, R=cfg.R, renorm=cfg.renorm,
                    dtype=dt, S=cfg.S if ffn_kind == moe.MOE_FFN_SWIGLU else 0, fs=cfg.fs,
                    slot_of=slot_of, ffn_kind=ffn_kind, device=DEV, epd_mode=epd_mode,
                    prune_m=prune_m, **kw)


def check_indices(layer, idx_ref, w_ref, cfg, slot_of):
    """Route, BRIMs, counts and histogram against the oracle, bit for bit."""
    torch.cuda.synchronize()
    idx = layer.topk_idx.cpu().numpy()
    assert np.array_equal(idx, idx_ref)
    w = layer.topk_w.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(w, w_ref, rtol=softmax_rtol(cfg.E), atol=1e-30)
    # BRIMs from the GPU's own (fp32) weights so that epd_gate is comparable bit for bit
    b = oracle.brim(idx, layer.topk_w.cpu().numpy().astype(np.float64), slot_of, cfg.E, cfg.R)
    c_t = int(layer.c_t.item())
    assert c_t == b["c_t"]
    assert np.array_equal(layer.brim0.cpu().numpy(), b["brim0"])
    assert np.array_equal(layer.sfd_off.cpu().numpy(), b["sfd_off"])
    assert np.array_equal(layer.sfd_token[:c_t].cpu().numpy(), b["sfd_token"])
    assert np.array_equal(layer.brim1[:, :c_t].cpu().numpy(), b["brim1"][:, :c_t])
    assert np.array_equal(layer.epd_off.cpu().numpy(), b["epd_off"])
    n_epd = int(b["epd_off"][-1])  # T*k, or fewer with empty (pruned) slots
    assert np.array_equal(layer.epd_sfd[:n_epd].cpu().numpy(), b["epd_sfd"][:n_epd])
    assert np.array_equal(layer.epd_gate[:n_epd].cpu().numpy().astype(np.float64),
                          b["epd_gate"][:n_epd])
    per_rank, total, remote = oracle.count_dispatched(idx, slot_of, cfg.E, cfg.R)
    assert np.array_equal(layer.per_rank.cpu().numpy(), per_rank)
    assert int(layer.total.item()) == total == c_t
    assert int(layer.remote.item()) == remote
    return b


def run_and_check_small(cfg, slot_of=None, ffn_kind=moe.MOE_FFN_SWIGLU, seed=None,
                        epd_mode="auto", fused_index=True, prune_m=0):
    inp = inputs.make_inputs(cfg, seed=seed)
    if slot_of is None:
        slot_of = np.arange(cfg.E, dtype=np.int32)
    layer = make_layer(cfg, inp, torch.from_numpy(slot_of), ffn_kind, epd_mode, prune_m)
    logits, x = inp["logits"].to(DEV), inp["x"].to(DEV)
    layer.hist.zero_()
    y = layer.forward(logits, x, fused_index=fused_index)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    idx_ref, w_ref = oracle_route(inp["logits"], cfg.k, cfg.renorm)
    if prune_m:
        idx_ref, w_ref = oracle.prune(idx_ref, w_ref, slot_of, cfg.E, cfg.R, prune_m)
    b = check_indices(layer, idx_ref, w_ref, cfg, slot_of)
    assert np.array_equal(layer.hist.cpu().numpy().astype(np.uint32),
                          oracle.coact_histogram(idx_ref, cfg.E))
    # dispatch: bit-exact copies
    c_t = b["c_t"]
    xo = to_oracle(inp["x"])
    x_sfd_ref = oracle.gather_rows(xo, b["sfd_token"])
    assert np.array_equal(to_oracle(layer.x_sfd[:c_t]), x_sfd_ref)
    if layer.x_epd is not None:
        n_epd = int(b["epd_off"][-1])
        assert np.array_equal(to_oracle(layer.x_epd[:n_epd]),
                              oracle.gather_rows(x_sfd_ref, b["epd_sfd"][:n_epd]))
    # outputs against the BRIM-guided oracle and against the dense definition
    kind = oracle.KIND_IDENTITY if ffn_kind == moe.MOE_FFN_IDENTITY else oracle.KIND_SWIGLU
    w_ = (None, None, None) if kind == oracle.KIND_IDENTITY else \
        (to_oracle(inp["wg"]), to_oracle(inp["wu"]), to_oracle(inp["wd"]))
    shared = None
    if cfg.S and kind == oracle.KIND_SWIGLU:
        shared = (to_oracle(inp["sg"]), to_oracle(inp["su"]), to_oracle(inp["sd"]))
    b64 = oracle.brim(idx_ref, w_ref, slot_of, cfg.E, cfg.R)
    y_sfd_ref, y_ref = oracle.occult_layer(xo, slot_of, cfg.E, cfg.R, cfg.k, b64, *w_,
                                           kind=kind, shared=shared)
    y_dense = oracle.dense_layer(xo, idx_ref, w_ref, *w_, kind=kind, shared=shared)
    assert rowwise_rel_err(y_ref, y_dense) < 1e-10
    err_y = rowwise_rel_err(y.float().cpu().numpy(), y_ref)
    assert err_y <= OUT_RTOL, err_y
    # y_sfd rows: compare only where the oracle's return row is not all ~0
    # (rank rows whose routed sum cancels are compared against the row scale of y)
    ys = layer.y_sfd[:c_t].float().cpu().numpy()
    tok = b["sfd_token"]
    scale = np.maximum(np.abs(y_ref[tok]).max(1), np.abs(y_sfd_ref).max(1))
    err_sfd = (np.abs(ys - y_sfd_ref).max(1) / np.maximum(scale, 1e-30)).max()
    assert err_sfd <= OUT_RTOL, err_sfd
    return layer, err_y


# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("renorm", [0, 1])
def test_tiny_layer(dtype, renorm):
    cfg = inputs.CONFIGS["tiny"].with_(dtype=dtype, renorm=renorm)
    run_and_check_small(cfg)


@pytest.mark.parametrize("cfg", [
    inputs.CONFIGS["tiny"],
    inputs.LayerConfig("sep", T=1000, d=256, f=192, E=16, k=4, R=4, seed=5),
    inputs.LayerConfig("sep16", T=300, d=128, f=128, E=256, k=16, R=8, seed=3),
], ids=["tiny", "sep", "sep16"])
def test_separate_index_entry_points(cfg):
    """moe_route_topk + moe_brim_build + counter + histogram called one by one."""
    run_and_check_small(cfg, fused_index=False)


def test_fused_index_equals_separate():
    cfg = inputs.LayerConfig("fz", T=3000, d=128, f=128, E=64, k=6, R=8, bias_std=1.0, seed=17)
    inp = inputs.make_inputs(cfg)
    a = make_layer(cfg, inp)
    b = make_layer(cfg, inp)
    logits, x = inp["logits"].to(DEV), inp["x"].to(DEV)
    a.hist.zero_(); b.hist.zero_()
    ya = a.forward(logits, x, fused_index=True)
    yb = b.forward(logits, x, fused_index=False)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    c_t = int(a.c_t.item())
    assert c_t == int(b.c_t.item())
    for name in ("topk_idx", "topk_w", "brim0", "sfd_off", "epd_off", "epd_sfd", "epd_gate",
                 "per_rank", "total", "remote", "hist"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert torch.equal(a.sfd_token[:c_t], b.sfd_token[:c_t])
    assert torch.equal(a.brim1[:, :c_t], b.brim1[:, :c_t])
    assert torch.equal(ya, yb)


@pytest.mark.parametrize("E", [64, 8, 160, 6])
@pytest.mark.parametrize("renorm", [0, 1])
def test_routing_does_not_depend_on_batch_size(E, renorm):
    """The lanes per token (G = 1, 2, 4 or 8) follow the batch size; the routes and gates
    of a token do not: the same rows routed inside batches of 40000, 30000, 15000 and 300
    tokens (G = 1, 2, 4, 8 on a 148-SM part) come out bit for bit equal, and match the
    oracle."""
    k = min(6, E)
    g = torch.Generator().manual_seed(11 + E)
    big = torch.randn(40000, E, generator=g, dtype=torch.float32) * 2.0
    ref_idx = ref_w = None
    for T in (40000, 30000, 15000, 300):
        logits = big[:T].contiguous().to(DEV)
        idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
        w = torch.empty(T, k, dtype=torch.float32, device=DEV)
        moe.moe_route_topk(logits, k, renorm, idx, w)
        torch.cuda.synchronize()
        if ref_idx is None:
            ref_idx, ref_w = idx[:300].cpu(), w[:300].cpu()
        else:
            assert torch.equal(idx[:300].cpu(), ref_idx), T
            assert torch.equal(w[:300].cpu(), ref_w), T
    idx_o, w_o = oracle_route(big[:300], k, renorm)
    assert np.array_equal(ref_idx.numpy(), idx_o)
    np.testing.assert_allclose(ref_w.numpy().astype(np.float64), w_o, rtol=softmax_rtol(E),
                               atol=1e-30)


@pytest.mark.parametrize("epd_mode", ["stored", "gather"])
def test_tiny_layer_permuted_placement(epd_mode):
    cfg = inputs.CONFIGS["tiny"]
    slot_of = np.random.default_rng(3).permutation(cfg.E).astype(np.int32)
    run_and_check_small(cfg, slot_of, epd_mode=epd_mode)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gathered_epd_rows(dtype):
    """The GEMM gathering its EPD rows out of the SFD payload (TMA gather4)."""
    cfg = inputs.LayerConfig("gather", T=900, d=256, f=128, E=16, k=4, R=4, dtype=dtype, seed=13)
    run_and_check_small(cfg, epd_mode="gather")


@pytest.mark.parametrize("epd_mode", ["direct", "stored"])
def test_one_expert_per_rank(epd_mode):
    """L = 1: the EPD state equals the SFD state; "direct" runs the GEMM on the payload."""
    cfg = inputs.LayerConfig("l1", T=700, d=256, f=256, E=8, k=2, R=8, renorm=1, seed=14)
    layer, _ = run_and_check_small(cfg, epd_mode=epd_mode)
    c_t = int(layer.c_t.item())
    assert c_t == cfg.T * cfg.k
    assert torch.equal(layer.epd_sfd[:c_t].cpu(), torch.arange(c_t, dtype=torch.int32))
    assert torch.equal(layer.epd_off.cpu(), layer.sfd_off.cpu())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_identity_experts(dtype):
    cfg = inputs.CONFIGS["tiny"].with_(dtype=dtype, T=300)
    run_and_check_small(cfg, ffn_kind=moe.MOE_FFN_IDENTITY)


@pytest.mark.parametrize("cfg", [
    # several M tiles per expert, ragged tails, BN=128 for GEMM 1 (2f % 256 != 0)
    inputs.LayerConfig("multi", T=1000, d=256, f=192, E=16, k=4, R=4, seed=5),
    # d % 256 != 0 (BN=128 in GEMM 2) and shared experts
    inputs.LayerConfig("shared", T=777, d=384, f=256, E=8, k=2, R=2, S=2, fs=128, seed=6),
    # d = 192 (BN=64 in GEMM 2), one expert per rank
    inputs.LayerConfig("narrow", T=515, d=192, f=128, E=8, k=3, R=8, seed=7),
    # fp32 / TF32 with several tiles
    inputs.LayerConfig("f32", T=600, d=256, f=256, E=8, k=2, R=4, dtype="f32", seed=8),
    # biased routing (empty and overfull experts)
    inputs.LayerConfig("skew", T=900, d=128, f=128, E=32, k=4, R=8, bias_std=2.0, seed=9),
])
def test_multi_tile_layers(cfg):
    run_and_check_small(cfg)


# test-only switches of the library: force the single-CTA GEMM, the CTA-pair
# GEMM alone, or CTA pairs plus single-CTA tiles for groups' short tails; and
# the CTA-pair GEMM with one K chunk per stage (2-D loads) where two would run
FORCE_SINGLE, FORCE_PAIR, FORCE_HYBRID = 2, 4, 8
FORCE_PAIR_ONE_CHUNK = 4 | 65536


@pytest.fixture
def gemm_variant(request):
    moe.moe_set_debug(request.param, 4000.0)
    yield request.param
    moe.moe_set_debug(0, 4000.0)


@pytest.mark.parametrize("gemm_variant", [FORCE_SINGLE, FORCE_PAIR, FORCE_HYBRID,
                                          FORCE_PAIR_ONE_CHUNK], indirect=True)
@pytest.mark.parametrize("cfg", [
    # 256-row pair tiles over ragged groups, BN = 256 / 256
    inputs.LayerConfig("pair", T=1500, d=256, f=256, E=8, k=2, R=4, seed=21),
    # BN = 128 in both GEMMs (2f = 384, d = 384), skewed groups, shared experts
    inputs.LayerConfig("pair128", T=1100, d=384, f=192, E=16, k=4, R=4, bias_std=1.5,
                       S=1, fs=128, seed=22),
    # TF32 on pairs
    inputs.LayerConfig("pairf32", T=800, d=256, f=128, E=4, k=2, R=2, dtype="f32", seed=23),
    # tiny groups: most pair tiles are mostly empty
    inputs.LayerConfig("pairsmall", T=40, d=128, f=128, E=16, k=4, R=4, seed=24),
], ids=["pair", "pair128", "pairf32", "pairsmall"])
def test_gemm_variants(cfg, gemm_variant):
    run_and_check_small(cfg)


@pytest.mark.parametrize("T,E,k,R", [(1, 8, 2, 4), (2, 64, 6, 8), (257, 8, 2, 1),
                                     (300, 8, 2, 8), (100, 256, 16, 8), (513, 64, 8, 64),
                                     # several histogram chunks with E > 128 (4-tile chunks), and
                                     # an E that is no power of two
                                     (2000, 256, 16, 8), (1500, 160, 6, 8)])
def test_edge_shapes(T, E, k, R):
    cfg = inputs.LayerConfig("edge", T=T, d=128, f=128, E=E, k=k, R=R, seed=T)
    run_and_check_small(cfg)


def test_all_tokens_to_one_expert_group():
    # every token's logits favour experts 0..k-1: one overfull group per expert, the rest empty
    cfg = inputs.LayerConfig("one", T=400, d=128, f=128, E=16, k=2, R=4, seed=2)
    inp = inputs.make_inputs(cfg)
    inp["logits"][:, :2] += 100.0
    layer = make_layer(cfg, inp)
    y = layer.forward(inp["logits"].to(DEV), inp["x"].to(DEV))
    torch.cuda.synchronize()
    idx_ref, w_ref = oracle_route(inp["logits"], cfg.k, 0)
    check_indices(layer, idx_ref, w_ref, cfg, np.arange(cfg.E, dtype=np.int32))
    y_ref = oracle.dense_layer(to_oracle(inp["x"]), idx_ref, w_ref, to_oracle(inp["wg"]),
                               to_oracle(inp["wu"]), to_oracle(inp["wd"]))
    assert rowwise_rel_err(y.float().cpu().numpy(), y_ref) <= OUT_RTOL


def test_empty_batch():
    cfg = inputs.LayerConfig("empty", T=0, d=128, f=128, E=8, k=2, R=4)
    inp = inputs.make_inputs(cfg)
    layer = make_layer(cfg, inp)
    layer.forward(inp["logits"].to(DEV), inp["x"].to(DEV))
    torch.cuda.synchronize()
    assert int(layer.c_t.item()) == 0
    assert layer.sfd_off.cpu().tolist() == [0] * 5
    assert moe.moe_get_device_status() == moe.MOE_OK


def test_expert_ffn_ragged_groups():
    """The grouped GEMM alone on hand-made groups: empty, 1 row, tile +/- 1, several tiles."""
    torch.manual_seed(0)
    d, f, G = 256, 192, 8
    sizes = [0, 1, 127, 128, 129, 300, 0, 64]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    m = int(off[-1])
    a = torch.randn(m + 5, d).to(torch.bfloat16)
    wg = (torch.randn(G, f, d) * 0.05).to(torch.bfloat16)
    wu = (torch.randn(G, f, d) * 0.05).to(torch.bfloat16)
    wd = (torch.randn(G, d, f) * 0.05).to(torch.bfloat16)
    scale = torch.rand(m + 5)
    w_gu = torch.empty(G, 2 * f, d, dtype=torch.bfloat16, device=DEV)
    w_dn = torch.empty(G, d, f, dtype=torch.bfloat16, device=DEV)
    moe.moe_prepare_weights(wg.to(DEV), wu.to(DEV), wd.to(DEV), None, w_gu, w_dn)
    out = torch.full((m + 5, d), 7.0, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(moe.moe_expert_ffn_workspace_size(m + 5, f, moe.MOE_BF16), dtype=torch.uint8,
                     device=DEV)
    moe.moe_expert_ffn(a.to(DEV), torch.from_numpy(off).to(DEV), w_gu, w_dn, f, scale.to(DEV),
                       moe.MOE_FFN_SWIGLU, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    out = out.float().cpu().numpy()
    ao, sc = a.double().numpy(), scale.double().numpy()
    ref = np.zeros((m, d))
    for g in range(G):
        for r in range(off[g], off[g + 1]):
            ref[r] = sc[r] * oracle.expert_row(ao[r], to_oracle(wg[g]), to_oracle(wu[g]),
                                               to_oracle(wd[g]))
    assert rowwise_rel_err(out[:m], ref) <= OUT_RTOL
    assert np.all(out[m:] == 7.0)  # rows outside every group are not written


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_expert_ffn_gathered_rows(dtype):
    """The grouped GEMM reading its rows through a row index (TMA gather4)."""
    g = torch.Generator().manual_seed(1)
    d, f, G, a_rows = 128, 256, 4, 1000
    sizes = [129, 0, 3, 300]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    m = int(off[-1])
    a = torch.randn(a_rows, d, generator=g).to(dtype)
    ridx = torch.randint(0, a_rows, (m,), generator=g, dtype=torch.int32)
    wg = (torch.randn(G, f, d, generator=g) * 0.05).to(dtype)
    wu = (torch.randn(G, f, d, generator=g) * 0.05).to(dtype)
    wd = (torch.randn(G, d, f, generator=g) * 0.05).to(dtype)
    w_gu = torch.empty(G, 2 * f, d, dtype=dtype, device=DEV)
    w_dn = torch.empty(G, d, f, dtype=dtype, device=DEV)
    moe.moe_prepare_weights(wg.to(DEV), wu.to(DEV), wd.to(DEV), None, w_gu, w_dn)
    out = torch.zeros(m, d, dtype=dtype, device=DEV)
    ws = torch.empty(moe.moe_expert_ffn_workspace_size(m, f, moe.dtype_code(dtype)),
                     dtype=torch.uint8, device=DEV)
    moe.moe_expert_ffn(a.to(DEV), torch.from_numpy(off).to(DEV), w_gu, w_dn, f, None,
                       moe.MOE_FFN_SWIGLU, out, ws, a_row_index=ridx.to(DEV))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    out = out.float().cpu().numpy()
    ao = a.double().numpy()
    ref = np.zeros((m, d))
    for gi in range(G):
        for r in range(off[gi], off[gi + 1]):
            ref[r] = oracle.expert_row(ao[int(ridx[r])], to_oracle(wg[gi]), to_oracle(wu[gi]),
                                       to_oracle(wd[gi]))
    assert rowwise_rel_err(out, ref) <= OUT_RTOL


def test_bad_expert_id_raises_device_check():
    cfg = inputs.CONFIGS["tiny"]
    idx = inputs.random_topk(cfg.T, cfg.E, cfg.k, seed=1).to(DEV)
    idx[17, 1] = 99      # out of range
    idx[40, 1] = idx[40, 0]  # repeated expert
    layer = MoELayer(T=cfg.T, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k, R=cfg.R,
                     ffn_kind=moe.MOE_FFN_IDENTITY, device=DEV)
    layer.topk_idx.copy_(idx)
    layer.topk_w.fill_(0.5)
    layer.build_brims()
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE_CHECK
    assert moe.moe_get_device_status() == moe.MOE_OK  # reading clears it
    # the bad tokens are not sent anywhere; everything else is intact
    b0 = layer.brim0.cpu().numpy()
    assert np.all(b0[:, 17] == -1) and np.all(b0[:, 40] == -1)


def test_outputs_are_deterministic():
    cfg = inputs.LayerConfig("det", T=700, d=256, f=256, E=16, k=4, R=4, seed=4)
    inp = inputs.make_inputs(cfg)
    layer = make_layer(cfg, inp)
    logits, x = inp["logits"].to(DEV), inp["x"].to(DEV)
    y1 = layer.forward(logits, x).clone()
    s1 = layer.y_sfd.clone()
    y2 = layer.forward(logits, x).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(s1, layer.y_sfd)



# ---------------------------------------------------------------------------
# routing-score-based collaboration pruning
@pytest.mark.parametrize("m", [1, 2, 3])
@pytest.mark.parametrize("fused", [True, False], ids=["fused", "separate"])
def test_pruned_layer(m, fused):
    cfg = inputs.LayerConfig("prune", T=700, d=128, f=128, E=32, k=6, R=8, bias_std=0.5,
                             seed=40 + m)
    slot_of = np.random.default_rng(m).permutation(cfg.E).astype(np.int32)
    layer, _ = run_and_check_small(cfg, slot_of, fused_index=fused, prune_m=m)
    c_t = int(layer.c_t.item())
    assert c_t <= cfg.T * m
    if m == 1:
        assert c_t == cfg.T


def test_prune_kernel_equals_fused_prune():
    cfg = inputs.LayerConfig("prunek", T=2000, d=128, f=128, E=64, k=8, R=8, seed=44)
    inp = inputs.make_inputs(cfg, weights=False)
    a = make_layer(cfg, inp, ffn_kind=moe.MOE_FFN_IDENTITY, prune_m=2)
    logits = inp["logits"].to(DEV)
    a.route_brim(logits)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    moe.moe_route_topk(logits, cfg.k, 0, idx, w)
    moe.moe_prune_topk(idx, w, a.slot_of, cfg.E, cfg.R, 2)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert torch.equal(idx, a.topk_idx) and torch.equal(w, a.topk_w)
    assert (idx == -1).any()

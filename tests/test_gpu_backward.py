"""The training path on the GPU against the oracle's backward.

moe_expert_ffn_train / moe_expert_ffn_backward (grouped input- and
weight-gradient GEMMs on tcgen05), moe_route_backward and the whole-layer
moe_layer_forward_train / moe_layer_backward are compared with
oracle.dense_layer_backward and oracle.route_backward (double precision, no
BRIMs), on seeded inputs.

Tolerances (bf16 operands, fp32 accumulation; the backward rounds the saved
pre-activations, dZ and w*h to bf16, each <= 2^-9 relative):
  dx                per-row normwise <= 2e-2 (as the forward's outputs)
  weight gradients  per-expert normwise (max error / max |ref|) <= 2e-2
  gate gradients    |dw - ref| <= 2e-2 * (sum of |terms| of ref): the bf16
                    rounding of h perturbs each term of the dot product
                    dw = sum_i (W_d^T dy)_i h_i by <= ~3 * 2^-9 of its size, so
                    the error scales with the terms, not with a sum that may
                    cancel (the oracle reports that sum as dw_abs)
  d_logits          per row, max error / max_e q_e (c(e) + sum_j c_j w_j) <= 2e-2,
                    with c the gate gradients' term magnitudes: the softmax
                    backward carries the gate gradients' errors through q
"""
import numpy as np
import pytest
import torch

import oracle
import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs, unpack_gate_up
from helpers import OUT_RTOL, oracle_route, rowwise_rel_err, to_oracle
from test_gpu_parity import make_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRAD_RTOL = 2e-2
FORCE_SINGLE, FORCE_PAIR, FORCE_HYBRID = 2, 4, 8


def normwise_err(a, ref) -> float:
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(a - ref).max() / max(np.abs(ref).max(), 1e-30))


def dlogits_err(got, ref, logits, idx, dw_abs, renorm) -> float:
    """Per-row error of d_logits relative to the magnitude its rounding error
    scales with: q_e (c(e) + sum_j c_j w_j), with c_j the condition magnitude of
    the gate gradient dw_j (the sum of |terms| of dw_j, from the oracle) and
    c(e) = c_j for e = e_j, else 0.  An entry that cancels to near zero is held
    to the accuracy of its terms, not to its own tiny value."""
    lg = np.asarray(logits, np.float64)
    ex = np.exp(lg - lg.max(axis=1, keepdims=True))
    rows = np.arange(lg.shape[0])[:, None]
    if renorm:
        mask = np.zeros_like(ex, dtype=bool)
        mask[rows, idx] = True
        ex = np.where(mask, ex, 0.0)
    q = ex / ex.sum(axis=1, keepdims=True)
    ce = np.zeros_like(q)
    ce[rows, idx] = dw_abs
    s_abs = (dw_abs * q[rows, idx]).sum(axis=1, keepdims=True)
    scale = (q * (ce + s_abs)).max(axis=1)
    err = np.abs(np.asarray(got, np.float64) - ref).max(axis=1)
    return float((err / np.maximum(scale, 1e-30)).max())


def gate_grad_err(got, ref, dw_abs) -> float:
    """max |dw - ref| / (sum of |terms| of ref): the gate gradient's error
    relative to its condition magnitude."""
    err = np.abs(np.asarray(got, np.float64) - ref)
    return float((err / np.maximum(dw_abs, 1e-30)).max())


def _bf16(t):
    return t.to(torch.bfloat16)


def _ffn_problem(sizes, d, f, seed):
    g = torch.Generator().manual_seed(seed)
    G, rows = len(sizes), int(sum(sizes))
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32)
    x = _bf16(torch.randn(rows, d, generator=g))
    wg = _bf16(torch.randn(G, f, d, generator=g) * 0.05)
    wu = _bf16(torch.randn(G, f, d, generator=g) * 0.05)
    wd = _bf16(torch.randn(G, d, f, generator=g) * 0.05)
    scale = torch.rand(rows, generator=g) * 0.9 + 0.1
    dout = _bf16(torch.randn(rows, d, generator=g))
    return off, x, wg, wu, wd, scale, dout


def _ffn_oracle(off, x, wg, wu, wd, scale, dout):
    """Each row is a token routed to its group's expert alone (k = 1)."""
    G = off.numel() - 1
    idx = np.repeat(np.arange(G, dtype=np.int32), np.diff(off.numpy()))[:, None]
    w = scale.double().numpy()[:, None]
    xs, dys = to_oracle(x), dout.float().double().numpy()
    y = oracle.dense_layer(xs, idx, w, to_oracle(wg), to_oracle(wu), to_oracle(wd))
    g = oracle.dense_layer_backward(xs, idx, w, to_oracle(wg), to_oracle(wu), to_oracle(wd), dys,
                                    experts=np.arange(G))
    return y, g


SHORT_SIZES = [0, 1, 64, 200, 413]  # an empty group, a one-row group, an exact tile, ragged
# groups averaging more than 1024 rows (the weight gradient's 128-row stages),
# with last blocks of 76, 1, 64 and 92 rows and an empty group
LONG_SIZES = [1100, 0, 2049, 1600, 1500]


@pytest.mark.parametrize("variant", [0, FORCE_SINGLE, FORCE_PAIR, FORCE_HYBRID],
                         ids=["auto", "single", "pair", "hybrid"])
@pytest.mark.parametrize("dw_dtype", [torch.float32, torch.bfloat16], ids=["dw_f32", "dw_bf16"])
@pytest.mark.parametrize("sizes", [SHORT_SIZES, LONG_SIZES], ids=["short", "long"])
def test_expert_ffn_backward_matches_oracle(variant, dw_dtype, sizes):
    d, f = 256, 256
    off, x, wg, wu, wd, scale, dout = _ffn_problem(sizes, d, f, seed=11)
    G, rows = len(sizes), int(sum(sizes))
    w_gu = torch.empty(G, 2 * f, d, dtype=torch.bfloat16, device=DEV)
    w_dn = torch.empty(G, d, f, dtype=torch.bfloat16, device=DEV)
    moe.moe_prepare_weights(wg.to(DEV), wu.to(DEV), wd.to(DEV), None, w_gu, w_dn)
    z = torch.empty(rows, 2 * f, dtype=torch.bfloat16, device=DEV)
    h = torch.empty(rows, f, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    dx = torch.empty_like(out)
    drs = torch.empty(rows, dtype=torch.float32, device=DEV)
    dw_gu = torch.full((G, 2 * f, d), float("nan"), dtype=dw_dtype, device=DEV)
    dw_dn = torch.full((G, d, f), float("nan"), dtype=dw_dtype, device=DEV)
    ws = torch.empty(moe.moe_expert_ffn_backward_workspace_size(rows, f), dtype=torch.uint8,
                     device=DEV)
    offd, xd, sd, dyd = off.to(DEV), x.to(DEV), scale.to(DEV), dout.to(DEV)
    moe.moe_set_debug(variant, 4000.0)
    try:
        moe.moe_expert_ffn_train(xd, offd, w_gu, w_dn, f, sd, z, h, out)
        moe.moe_expert_ffn_backward(dyd, xd, z, offd, w_gu, w_dn, f, sd, dx, drs, dw_gu, dw_dn, ws)
        torch.cuda.synchronize()
    finally:
        moe.moe_set_debug(0, 4000.0)
    assert moe.moe_get_device_status() == moe.MOE_OK
    y_ref, g = _ffn_oracle(off, x, wg, wu, wd, scale, dout)
    assert rowwise_rel_err(out.float().cpu().numpy(), y_ref) <= OUT_RTOL
    assert rowwise_rel_err(dx.float().cpu().numpy(), g["dx"]) <= GRAD_RTOL
    assert gate_grad_err(drs.cpu().numpy()[:rows], g["dw"][:, 0], g["dw_abs"][:, 0]) <= GRAD_RTOL
    dwg, dwu = unpack_gate_up(dw_gu.float().cpu())
    for e in range(G):
        if sizes[e] == 0:  # an expert without rows gets a zero gradient
            assert not dwg[e].any() and not dwu[e].any() and not dw_dn[e].float().any()
            continue
        assert normwise_err(dwg[e].numpy(), g["dwg"][e]) <= GRAD_RTOL, e
        assert normwise_err(dwu[e].numpy(), g["dwu"][e]) <= GRAD_RTOL, e
        assert normwise_err(dw_dn[e].float().cpu().numpy(), g["dwd"][e]) <= GRAD_RTOL, e


def test_gate_gradient_error_is_the_rounding_of_h():
    """What the gate-gradient tolerance covers.  The gate gradient of an EPD row
    is dw = sum_i (W_d^T dy)_i h_i; the GPU uses h rounded to bf16.  Fed that
    same bf16 h, the double-precision sum matches the GPU's to fp32 accumulation
    (<= 1e-4 of the terms' magnitude, 200x inside the 2e-2 bound), so the error
    against the oracle's unrounded h is the rounding of h and nothing else.
    (d_logits is a softmax backward of these gate gradients; fed the same gate
    gradients it matches the oracle to 1e-4: test_route_backward_matches_oracle.)"""
    sizes, d, f = [1, 64, 200, 413], 256, 256
    off, x, wg, wu, wd, scale, dout = _ffn_problem(sizes, d, f, seed=12)
    G, rows = len(sizes), int(sum(sizes))
    w_gu = torch.empty(G, 2 * f, d, dtype=torch.bfloat16, device=DEV)
    w_dn = torch.empty(G, d, f, dtype=torch.bfloat16, device=DEV)
    moe.moe_prepare_weights(wg.to(DEV), wu.to(DEV), wd.to(DEV), None, w_gu, w_dn)
    z = torch.empty(rows, 2 * f, dtype=torch.bfloat16, device=DEV)
    h = torch.empty(rows, f, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    dx = torch.empty_like(out)
    drs = torch.empty(rows, dtype=torch.float32, device=DEV)
    dw_gu = torch.empty(G, 2 * f, d, dtype=torch.float32, device=DEV)
    dw_dn = torch.empty(G, d, f, dtype=torch.float32, device=DEV)
    ws = torch.empty(moe.moe_expert_ffn_backward_workspace_size(rows, f), dtype=torch.uint8,
                     device=DEV)
    offd, xd, sd, dyd = off.to(DEV), x.to(DEV), scale.to(DEV), dout.to(DEV)
    moe.moe_expert_ffn_train(xd, offd, w_gu, w_dn, f, sd, z, h, out)
    moe.moe_expert_ffn_backward(dyd, xd, z, offd, w_gu, w_dn, f, sd, dx, drs, dw_gu, dw_dn, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    h_gpu = h.float().cpu().double().numpy()
    dy, wdn = dout.float().double().numpy(), wd.float().double().numpy()
    ref, terms = np.empty(rows), np.empty(rows)
    o = off.numpy()
    for g_ in range(G):
        dh = dy[o[g_]:o[g_ + 1]] @ wdn[g_]  # (W_d^T dy) per row, [rows_g, f]
        ref[o[g_]:o[g_ + 1]] = (dh * h_gpu[o[g_]:o[g_ + 1]]).sum(1)
        terms[o[g_]:o[g_ + 1]] = np.abs(dh * h_gpu[o[g_]:o[g_ + 1]]).sum(1)
    got = drs.cpu().numpy().astype(np.float64)
    matched = gate_grad_err(got, ref, terms)
    _, g = _ffn_oracle(off, x, wg, wu, wd, scale, dout)
    unmatched = gate_grad_err(got, g["dw"][:, 0], g["dw_abs"][:, 0])
    assert matched <= 1e-4, matched
    assert unmatched <= GRAD_RTOL, unmatched


def test_expert_ffn_backward_accumulates_and_is_deterministic():
    sizes, d, f = [37, 0, 300], 256, 192
    off, x, wg, wu, wd, scale, dout = _ffn_problem(sizes, d, f, seed=5)
    G, rows = len(sizes), int(sum(sizes))
    w_gu = torch.empty(G, 2 * f, d, dtype=torch.bfloat16, device=DEV)
    w_dn = torch.empty(G, d, f, dtype=torch.bfloat16, device=DEV)
    moe.moe_prepare_weights(wg.to(DEV), wu.to(DEV), wd.to(DEV), None, w_gu, w_dn)
    z = torch.empty(rows, 2 * f, dtype=torch.bfloat16, device=DEV)
    h = torch.empty(rows, f, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(moe.moe_expert_ffn_backward_workspace_size(rows, f), dtype=torch.uint8,
                     device=DEV)
    offd, xd, sd, dyd = off.to(DEV), x.to(DEV), scale.to(DEV), dout.to(DEV)
    moe.moe_expert_ffn_train(xd, offd, w_gu, w_dn, f, sd, z, h, out)

    def run(dw_gu, dw_dn, acc):
        dx = torch.empty_like(out)
        drs = torch.empty(rows, dtype=torch.float32, device=DEV)
        moe.moe_expert_ffn_backward(dyd, xd, z, offd, w_gu, w_dn, f, sd, dx, drs, dw_gu, dw_dn,
                                    ws, accumulate=acc)
        return dx, drs

    a_gu = torch.empty(G, 2 * f, d, device=DEV)
    a_dn = torch.empty(G, d, f, device=DEV)
    dx1, drs1 = run(a_gu, a_dn, 0)
    first_gu, first_dn = a_gu.clone(), a_dn.clone()
    dx2, drs2 = run(a_gu, a_dn, 1)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert torch.equal(dx1, dx2) and torch.equal(drs1, drs2)       # deterministic
    assert torch.equal(a_gu, 2 * first_gu) and torch.equal(a_dn, 2 * first_dn)  # accumulated
    assert not first_gu[1].any() and not first_dn[1].any()        # the empty group


def _brim_row_of(b, slot_of, E, R, T, k, idx):
    """EPD row of each (token, slot) from the oracle's BRIMs."""
    L = E // R
    cap = T * min(k, R)
    p = np.full((T, k), -1, np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            q = slot_of[e]
            s = b["brim0"][q // L, t]
            p[t, j] = b["brim1"].reshape(L, cap)[q % L, s]
    return p


ROUTE_CASES = [
    inputs.LayerConfig("route_tiny", T=256, d=128, f=128, E=8, k=2, R=4, seed=1),
    inputs.LayerConfig("route_tiny_renorm", T=256, d=128, f=128, E=8, k=2, R=4, renorm=1, seed=2),
    inputs.LayerConfig("route_e64", T=500, d=128, f=128, E=64, k=8, R=8, bias_std=0.5, seed=3),
    inputs.LayerConfig("route_e256", T=100, d=128, f=128, E=256, k=16, R=8, renorm=1, seed=4),
]


@pytest.mark.parametrize("cfg", ROUTE_CASES, ids=[c.name for c in ROUTE_CASES])
def test_route_backward_matches_oracle(cfg):
    logits = inputs.make_logits(cfg)
    slot_of = np.random.default_rng(cfg.seed).permutation(cfg.E).astype(np.int32)
    T, E, k, R = cfg.T, cfg.E, cfg.k, cfg.R
    L, cap, tk = E // R, cfg.cap, T * k
    d_gate = torch.randn(tk, generator=torch.Generator().manual_seed(cfg.seed + 100))
    dev = lambda *s, dt=torch.int32: torch.empty(*s, dtype=dt, device=DEV)  # noqa: E731
    topk_idx, topk_w = dev(T, k), dev(T, k, dt=torch.float32)
    brim0, sfd_token, sfd_off = dev(R, T), dev(cap), dev(R + 1)
    brim1, epd_off, epd_sfd = dev(L, cap), dev(E + 1), dev(tk)
    epd_gate, c_t = dev(tk, dt=torch.float32), dev(1)
    ws = torch.empty(moe.moe_route_brim_workspace_size(T, E, R), dtype=torch.uint8, device=DEV)
    lg, so = logits.to(DEV), torch.from_numpy(slot_of).to(DEV)
    moe.moe_route_brim(lg, k, cfg.renorm, so, R, topk_idx, topk_w, brim0, sfd_token, sfd_off,
                       brim1, epd_off, epd_sfd, epd_gate, c_t, ws)
    d_logits = dev(T, E, dt=torch.float32)
    d_topk_w = dev(T, k, dt=torch.float32)
    moe.moe_route_backward(lg, k, cfg.renorm, topk_idx, so, R, brim0, brim1, d_gate.to(DEV),
                           d_logits, d_topk_w)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    idx, w = oracle_route(logits, k, cfg.renorm)
    b = oracle.brim(idx, w, slot_of, E, R)
    p = _brim_row_of(b, slot_of, E, R, T, k, idx)
    dw = d_gate.double().numpy()[p]
    assert np.array_equal(d_topk_w.cpu().numpy(), d_gate.numpy()[p])
    ref = oracle.route_backward(to_oracle(logits), idx, dw, cfg.renorm)
    assert rowwise_rel_err(d_logits.cpu().numpy(), ref) <= 1e-4


LAYER_CASES = [
    inputs.CONFIGS["tiny"],
    inputs.CONFIGS["tiny"].with_(name="tiny_renorm", renorm=1, seed=7),
    inputs.LayerConfig("shared_l1", T=300, d=256, f=192, E=4, k=2, R=4, S=1, fs=128, seed=8),
    inputs.LayerConfig("ragged_pair", T=777, d=256, f=256, E=16, k=4, R=4, seed=9),
]


def _layer_oracle(cfg, inp, dy, tokens=None, experts=None):
    idx, w = oracle_route(inp["logits"], cfg.k, cfg.renorm)
    shared = None
    if cfg.S:
        shared = (to_oracle(inp["sg"]), to_oracle(inp["su"]), to_oracle(inp["sd"]))
    g = oracle.dense_layer_backward(to_oracle(inp["x"]), idx, w, to_oracle(inp["wg"]),
                                    to_oracle(inp["wu"]), to_oracle(inp["wd"]),
                                    dy.float().double().numpy(), shared=shared, tokens=tokens,
                                    experts=experts, shared_grads=cfg.S > 0 and tokens is None)
    # d_logits needs the gate gradients of every token of the rows asked for
    sel = slice(None) if tokens is None else tokens
    g["dlogits"] = oracle.route_backward(to_oracle(inp["logits"])[sel], idx[sel], g["dw"],
                                         cfg.renorm)
    return idx, w, g


def _check_weight_grads(layer, grads, g, experts, cfg):
    slot_of = layer.slot_of.cpu().numpy()
    dwg, dwu = unpack_gate_up(grads["dw_gu"].float().cpu())
    dwd = grads["dw_dn"].float().cpu()
    for n, e in enumerate(experts):
        q = slot_of[e]
        assert normwise_err(dwg[q].numpy(), g["dwg"][n]) <= GRAD_RTOL, e
        assert normwise_err(dwu[q].numpy(), g["dwu"][n]) <= GRAD_RTOL, e
        assert normwise_err(dwd[q].numpy(), g["dwd"][n]) <= GRAD_RTOL, e


@pytest.mark.parametrize("cfg", LAYER_CASES, ids=[c.name for c in LAYER_CASES])
def test_layer_backward_matches_oracle(cfg):
    inp = inputs.make_inputs(cfg)
    slot_of = torch.from_numpy(np.random.default_rng(cfg.seed + 1).permutation(cfg.E)
                               .astype(np.int32))
    layer = make_layer(cfg, inp, slot_of=slot_of)
    logits, x = inp["logits"].to(DEV), inp["x"].to(DEV)
    y = layer.forward_train(logits, x).clone()
    dy = _bf16(torch.randn(cfg.T, cfg.d, generator=torch.Generator().manual_seed(cfg.seed + 2)))
    grads = layer.backward(dy.to(DEV))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    idx, w, g = _layer_oracle(cfg, inp, dy, experts=np.arange(cfg.E))
    shared = None
    if cfg.S:
        shared = (to_oracle(inp["sg"]), to_oracle(inp["su"]), to_oracle(inp["sd"]))
    y_ref = oracle.dense_layer(to_oracle(inp["x"]), idx, w, to_oracle(inp["wg"]),
                               to_oracle(inp["wu"]), to_oracle(inp["wd"]), shared=shared)
    assert rowwise_rel_err(y.float().cpu().numpy(), y_ref) <= OUT_RTOL
    assert rowwise_rel_err(grads["dx"].float().cpu().numpy(), g["dx"]) <= GRAD_RTOL
    assert gate_grad_err(grads["d_topk_w"].cpu().numpy(), g["dw"], g["dw_abs"]) <= GRAD_RTOL
    assert dlogits_err(grads["d_logits"].cpu().numpy(), g["dlogits"], inp["logits"].numpy(), idx,
                       g["dw_abs"], cfg.renorm) <= GRAD_RTOL
    _check_weight_grads(layer, grads, g, range(cfg.E), cfg)
    if cfg.S:
        sgr, sur = unpack_gate_up(grads["dsw_gu"].float().cpu()[0])
        F = cfg.S * cfg.fs
        for s in range(cfg.S):
            cols = slice(s * cfg.fs, (s + 1) * cfg.fs)
            assert normwise_err(sgr[cols].numpy(), g["dsg"][s]) <= GRAD_RTOL
            assert normwise_err(sur[cols].numpy(), g["dsu"][s]) <= GRAD_RTOL
            assert normwise_err(grads["dsw_dn"].float().cpu()[0][:, cols].numpy(),
                                g["dsd"][s]) <= GRAD_RTOL
        assert sgr.shape[0] == F


def test_layer_backward_twice_is_bitwise_equal():
    cfg = LAYER_CASES[3]
    inp = inputs.make_inputs(cfg)
    layer = make_layer(cfg, inp)
    logits, x = inp["logits"].to(DEV), inp["x"].to(DEV)
    layer.forward_train(logits, x)
    dy = _bf16(torch.randn(cfg.T, cfg.d, generator=torch.Generator().manual_seed(3))).to(DEV)
    a = {k: v.clone() for k, v in layer.backward(dy).items()}
    b = layer.backward(dy)
    torch.cuda.synchronize()
    for key in a:
        assert torch.equal(a[key], b[key]), key


FULL = [inputs.CONFIGS["olmoe"], inputs.CONFIGS["dsv2lite"]]


@pytest.mark.parametrize("cfg", FULL, ids=[c.name for c in FULL])
def test_layer_backward_full_size_sampled(cfg):
    """Full-size layer; dx / d_logits checked on sampled tokens, weight gradients
    on two experts (the most and the least loaded)."""
    inp = inputs.make_inputs(cfg)
    layer = make_layer(cfg, inp)
    logits, x = inp["logits"].to(DEV), inp["x"].to(DEV)
    layer.forward_train(logits, x)
    dy = _bf16(torch.randn(cfg.T, cfg.d, generator=torch.Generator().manual_seed(5)))
    grads = layer.backward(dy.to(DEV))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    tokens = np.sort(np.random.default_rng(0).choice(cfg.T, size=48, replace=False)).astype(np.int32)
    idx, _ = oracle_route(inp["logits"], cfg.k, cfg.renorm)
    load = np.bincount(idx.reshape(-1), minlength=cfg.E)
    experts = [int(load.argmax()), int(load.argmin())]
    _, _, g = _layer_oracle(cfg, inp, dy, tokens=tokens, experts=experts)
    assert rowwise_rel_err(grads["dx"].float().cpu().numpy()[tokens], g["dx"]) <= GRAD_RTOL
    assert gate_grad_err(grads["d_topk_w"].cpu().numpy()[tokens], g["dw"],
                         g["dw_abs"]) <= GRAD_RTOL
    assert dlogits_err(grads["d_logits"].cpu().numpy()[tokens], g["dlogits"],
                       inp["logits"].numpy()[tokens], idx[tokens], g["dw_abs"],
                       cfg.renorm) <= GRAD_RTOL
    _check_weight_grads(layer, grads, g, experts, cfg)


SKIP_FIRST_LOAD = 1


@pytest.mark.parametrize("variant", [FORCE_SINGLE, 0, FORCE_PAIR],
                         ids=["single", "pair", "pair_wgrad"])
def test_backward_bounded_wait_expires_and_context_survives(variant):
    """A stage that is never loaded makes the backward GEMMs' waits expire:
    MOE_ERR_TIMEOUT comes back through the device flag, and the next call on the
    same context gives the correct gradients."""
    sizes, d, f = [300, 0, 212], 256, 256
    off, x, wg, wu, wd, scale, dout = _ffn_problem(sizes, d, f, seed=21)
    G, rows = len(sizes), int(sum(sizes))
    w_gu = torch.empty(G, 2 * f, d, dtype=torch.bfloat16, device=DEV)
    w_dn = torch.empty(G, d, f, dtype=torch.bfloat16, device=DEV)
    moe.moe_prepare_weights(wg.to(DEV), wu.to(DEV), wd.to(DEV), None, w_gu, w_dn)
    z = torch.empty(rows, 2 * f, dtype=torch.bfloat16, device=DEV)
    h = torch.empty(rows, f, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    dx = torch.empty_like(out)
    drs = torch.empty(rows, dtype=torch.float32, device=DEV)
    dw_gu = torch.empty(G, 2 * f, d, device=DEV)
    dw_dn = torch.empty(G, d, f, device=DEV)
    ws = torch.empty(moe.moe_expert_ffn_backward_workspace_size(rows, f), dtype=torch.uint8,
                     device=DEV)
    offd, xd, sd, dyd = off.to(DEV), x.to(DEV), scale.to(DEV), dout.to(DEV)
    moe.moe_expert_ffn_train(xd, offd, w_gu, w_dn, f, sd, z, h, out)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    try:
        moe.moe_set_debug(SKIP_FIRST_LOAD | variant, 200.0)
        moe.moe_expert_ffn_backward(dyd, xd, z, offd, w_gu, w_dn, f, sd, dx, drs, dw_gu, dw_dn, ws)
        status = moe.moe_get_device_status()
    finally:
        moe.moe_set_debug(0, 4000.0)
    assert status == moe.MOE_ERR_TIMEOUT
    moe.moe_set_debug(variant, 4000.0)
    try:
        moe.moe_expert_ffn_backward(dyd, xd, z, offd, w_gu, w_dn, f, sd, dx, drs, dw_gu, dw_dn, ws)
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == moe.MOE_OK
    finally:
        moe.moe_set_debug(0, 4000.0)
    _, g = _ffn_oracle(off, x, wg, wu, wd, scale, dout)
    assert rowwise_rel_err(dx.float().cpu().numpy(), g["dx"]) <= GRAD_RTOL
    dwg, _ = unpack_gate_up(dw_gu.cpu())
    assert normwise_err(dwg[0].numpy(), g["dwg"][0]) <= GRAD_RTOL
    assert normwise_err(dw_dn[2].cpu().numpy(), g["dwd"][2]) <= GRAD_RTOL


def test_empty_batch_zeroes_weight_gradients():
    """T = 0: no rows at all; the weight gradients are zero (accumulate = 0) or
    left as they are (accumulate = 1)."""
    cfg = inputs.LayerConfig("empty", T=0, d=128, f=128, E=4, k=2, R=2, S=1, fs=128)
    full = cfg.with_(T=16)
    inp = inputs.make_inputs(full)
    layer = make_layer(cfg, inp)
    logits = torch.empty(0, cfg.E, device=DEV)
    x = torch.empty(0, cfg.d, dtype=torch.bfloat16, device=DEV)
    layer.forward_train(logits, x)
    grads = layer.backward(torch.empty(0, cfg.d, dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    for key in ("dw_gu", "dw_dn", "dsw_gu", "dsw_dn"):
        assert not grads[key].any(), key
    for key in ("dw_gu", "dw_dn"):
        grads[key].fill_(3.0)
    layer.backward(torch.empty(0, cfg.d, dtype=torch.bfloat16, device=DEV), grads=grads,
                   accumulate=True)
    torch.cuda.synchronize()
    assert bool((grads["dw_gu"] == 3.0).all()) and bool((grads["dw_dn"] == 3.0).all())

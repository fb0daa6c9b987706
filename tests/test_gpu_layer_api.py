"""The whole-layer entry points and the bounded-wait error path, on the GPU."""
import numpy as np
import pytest
import torch

import oracle
import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs
from helpers import OUT_RTOL, oracle_route, rowwise_rel_err, to_oracle
from test_gpu_parity import make_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    inputs.CONFIGS["tiny"],
    inputs.LayerConfig("shared", T=777, d=384, f=256, E=8, k=2, R=2, S=2, fs=128, seed=6),
    inputs.LayerConfig("l1", T=600, d=256, f=256, E=8, k=2, R=8, renorm=1, seed=14),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_layer_forward_equals_the_steps(cfg):
    """moe_layer_forward (one call) gives the same bits as the step-by-step calls."""
    inp = inputs.make_inputs(cfg)
    layer = make_layer(cfg, inp)
    logits, x = inp["logits"].to(DEV), inp["x"].to(DEV)
    y_steps = layer.forward(logits, x).clone()
    hist_steps = layer.hist.clone()
    ct_steps, pr_steps = layer.c_t.clone(), layer.per_rank.clone()
    layer.hist.zero_()
    y_fused = torch.empty_like(y_steps)
    layer.forward_fused(logits, x, y=y_fused)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert torch.equal(y_fused, y_steps)
    assert torch.equal(layer.c_t, ct_steps) and torch.equal(layer.per_rank, pr_steps)
    assert torch.equal(layer.hist, hist_steps)


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_layer_forward_host_buffers(cfg):
    """moe_layer_forward_host: host logits/x in, host y out, against the oracle."""
    inp = inputs.make_inputs(cfg)
    layer = make_layer(cfg, inp)
    h_logits = inp["logits"].contiguous().pin_memory()
    h_x = inp["x"].contiguous().pin_memory()
    h_y = torch.empty_like(h_x).pin_memory()
    layer.forward_host(h_logits, h_x, h_y)
    assert moe.moe_get_device_status() == moe.MOE_OK
    y_dev = layer.forward(h_logits.to(DEV), h_x.to(DEV)).cpu()
    assert torch.equal(h_y, y_dev)
    idx, w = oracle_route(inp["logits"], cfg.k, cfg.renorm)
    shared = None
    if cfg.S:
        shared = (to_oracle(inp["sg"]), to_oracle(inp["su"]), to_oracle(inp["sd"]))
    y_ref = oracle.dense_layer(to_oracle(inp["x"]), idx, w, to_oracle(inp["wg"]),
                               to_oracle(inp["wu"]), to_oracle(inp["wd"]), shared=shared)
    assert rowwise_rel_err(h_y.float().numpy(), y_ref) <= OUT_RTOL


def test_layer_forward_rejects_bad_arguments():
    cfg = inputs.CONFIGS["tiny"]
    inp = inputs.make_inputs(cfg)
    layer = make_layer(cfg, inp)
    small = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_layer_forward(inp["logits"].to(DEV), inp["x"].to(DEV), cfg.k, cfg.R, 0,
                              layer.slot_of, layer.w_gu, layer.w_dn, cfg.f, layer.y, small)
    assert e.value.code == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_layer_workspace_size(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, 3, 0, 0,
                                        moe.MOE_BF16, 0) == 0  # R does not divide E


# library debug bits (test only): 1 = the GEMM producer skips its first load,
# 2 / 4 = force the single-CTA / CTA-pair GEMM
SKIP_FIRST_LOAD, FORCE_SINGLE, FORCE_PAIR = 1, 2, 4


@pytest.mark.parametrize("variant", [FORCE_SINGLE, FORCE_PAIR], ids=["single", "pair"])
def test_bounded_wait_expires_and_context_survives(variant):
    """A stage that is never loaded makes the MMA issuer's wait expire: the kernel
    returns MOE_ERR_TIMEOUT through the device flag instead of hanging, and the
    next call on the same context computes correct results."""
    cfg = inputs.LayerConfig("timeout", T=512, d=256, f=256, E=4, k=1, R=2, seed=31)
    inp = inputs.make_inputs(cfg)
    layer = make_layer(cfg, inp)
    logits, x = inp["logits"].to(DEV), inp["x"].to(DEV)
    layer.route(logits)
    layer.build_brims()
    layer.dispatch(x)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    try:
        moe.moe_set_debug(SKIP_FIRST_LOAD | variant, 200.0)
        layer.experts()
        status = moe.moe_get_device_status()
    finally:
        moe.moe_set_debug(0, 4000.0)
    assert status == moe.MOE_ERR_TIMEOUT
    # the context is still usable and the same call now succeeds
    moe.moe_set_debug(variant, 4000.0)
    try:
        layer.experts()
        layer.combine()
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == moe.MOE_OK
    finally:
        moe.moe_set_debug(0, 4000.0)
    idx, w = oracle_route(inp["logits"], cfg.k, cfg.renorm)
    y_ref = oracle.dense_layer(to_oracle(inp["x"]), idx, w, to_oracle(inp["wg"]),
                               to_oracle(inp["wu"]), to_oracle(inp["wd"]))
    assert rowwise_rel_err(layer.y.float().cpu().numpy(), y_ref) <= OUT_RTOL


def test_layer_forward_host_async_two_batches_in_flight():
    """moe_layer_forward_host_async on two streams with their own workspaces:
    two different batches in flight give the same bits as one at a time."""
    cfg = inputs.LayerConfig("async", T=900, d=256, f=256, E=8, k=2, R=4, S=1, fs=128, seed=41)
    inp_a = inputs.make_inputs(cfg)
    inp_b = inputs.make_inputs(cfg, seed=42, weights=False)
    layer = make_layer(cfg, inp_a)
    hosts = []
    for inp in (inp_a, inp_b):
        hosts.append((inp["logits"].contiguous().pin_memory(), inp["x"].contiguous().pin_memory()))
    ref = []
    for h_l, h_x in hosts:
        h_y = torch.empty_like(h_x).pin_memory()
        layer.forward_host(h_l, h_x, h_y)
        ref.append(h_y.clone())
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [layer.host_workspace(), layer.host_workspace()]
    outs = [torch.empty_like(hosts[0][1]).pin_memory() for _ in range(2)]
    for rep in range(3):
        for i, (h_l, h_x) in enumerate(hosts):
            streams[i].synchronize()
            layer.forward_host(h_l, h_x, outs[i], stream=streams[i], ws=wss[i], asynchronous=True)
        for s in streams:
            s.synchronize()
        assert moe.moe_get_device_status() == moe.MOE_OK
        for i in range(2):
            assert torch.equal(outs[i], ref[i]), (rep, i)

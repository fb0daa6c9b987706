"""The copy-engine (TMA bulk copy) movers against the register movers.

moe_dispatch_gather and the combine entry points have two implementations:
warps moving 16-byte vectors through registers, and lane 0 of each warp
driving cp.async.bulk copies through shared-memory staging (debug flag 16,
kDebugBulkMovers).  Both must produce the same bits: the dispatch copies rows,
and the combine sums the same fp32 values in the same order.  Checked on the
layer's SFD / EPD rows, return rows and output, on small and full-size
workloads, on the expert-parallel combine modes, and against the oracle.
"""
import numpy as np
import pytest
import torch

import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs
from test_gpu_parity import make_layer, run_and_check_small

pytestmark = pytest.mark.gpu
DEV = "cuda"
BULK = 16


@pytest.fixture
def bulk_movers():
    moe.moe_set_debug(BULK, 4000.0)
    yield
    moe.moe_set_debug(0, 4000.0)


def _layer_outputs(cfg, flags, prune_m=0, slot_of=None, seed=None):
    moe.moe_set_debug(flags, 4000.0)
    try:
        inp = inputs.make_inputs(cfg, seed=seed)
        layer = make_layer(cfg, inp, slot_of=slot_of, prune_m=prune_m)
        layer.forward(inp["logits"].to(DEV), inp["x"].to(DEV))
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == moe.MOE_OK
        c_t = int(layer.c_t.item())
        n_epd = int(layer.epd_off[-1].item())
        out = dict(x_sfd=layer.x_sfd[:c_t].clone(), y_sfd=layer.y_sfd[:c_t].clone(),
                   y=layer.y.clone())
        if layer.x_epd is not None:
            out["x_epd"] = layer.x_epd[:n_epd].clone()
        return out
    finally:
        moe.moe_set_debug(0, 4000.0)


CASES = [
    inputs.CONFIGS["tiny"],
    inputs.CONFIGS["tiny"].with_(dtype="f32", renorm=1, seed=3),
    inputs.LayerConfig("edge1", T=1, d=128, f=128, E=8, k=2, R=4, seed=1),
    inputs.LayerConfig("k16", T=100, d=128, f=128, E=256, k=16, R=8, seed=2),
    inputs.LayerConfig("r64", T=513, d=128, f=128, E=64, k=8, R=64, seed=4),
    inputs.LayerConfig("wide", T=300, d=2048 + 64, f=128, E=16, k=4, R=4, seed=5),
    inputs.LayerConfig("l1", T=700, d=256, f=128, E=8, k=2, R=8, renorm=1, seed=6),
    inputs.LayerConfig("shared", T=600, d=384, f=128, E=16, k=6, R=8, S=2, fs=128, seed=7),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name + "_" + c.dtype for c in CASES])
def test_bulk_movers_bit_equal_to_register_movers(cfg):
    a = _layer_outputs(cfg, 0)
    b = _layer_outputs(cfg, BULK)
    assert a.keys() == b.keys()
    for key in a:
        assert torch.equal(a[key], b[key]), key


def test_bulk_movers_pruned_routing():
    cfg = inputs.LayerConfig("pruned", T=900, d=256, f=128, E=32, k=6, R=8, seed=8)
    a = _layer_outputs(cfg, 0, prune_m=2)
    b = _layer_outputs(cfg, BULK, prune_m=2)
    for key in a:
        assert torch.equal(a[key], b[key]), key


def test_bulk_movers_full_size_corr_prefill():
    cfg = inputs.CONFIGS["corr_prefill"]
    a = _layer_outputs(cfg, 0)
    b = _layer_outputs(cfg, BULK)
    for key in a:
        assert torch.equal(a[key], b[key]), key


def test_bulk_movers_against_the_oracle(bulk_movers):
    run_and_check_small(inputs.LayerConfig("bulkorc", T=777, d=192, f=128, E=16, k=4, R=4,
                                           seed=9))


def test_bulk_movers_expert_parallel(bulk_movers):
    from test_gpu_ep import _check
    _check(inputs.LayerConfig("ep_bulk", T=700, d=128, f=128, E=16, k=4, R=4), [300, 0, 255, 145],
           seed=10)

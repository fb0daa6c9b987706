"""The swapped-operand expert GEMM (ffn_gemm_swap.cuh) against the oracle.

The kernel puts the weights on the MMA's M side (256 rows per CTA pair) and a
group's rows on its N side (the tile's rows rounded up to 16), so that a short
group is padded to 16 rows instead of 256.  Debug flag 64 forces it wherever it
applies (bf16, the inference epilogues, N a multiple of 256).  Checked: ragged and
skewed groups, empty groups, groups of one and of a few rows (N = 16, 32, ...),
exact multiples of 256, shared experts (one tall group), the expert-parallel
destination's local groups, and the OLMoE-shaped layer at full size against the
row-major kernels' output and the oracle on sampled tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs
from expert_warp_top_b200.layer import MoELayer
from helpers import OUT_RTOL, oracle_route, rowwise_rel_err, to_oracle
from test_gpu_parity import run_and_check_small

pytestmark = pytest.mark.gpu
DEV = "cuda"
FORCE_SWAP = 64


@pytest.fixture
def swap():
    moe.moe_set_debug(FORCE_SWAP, 4000.0)
    yield
    moe.moe_set_debug(0, 4000.0)


CASES = [
    inputs.LayerConfig("swap_small", T=1500, d=256, f=256, E=8, k=2, R=4, seed=31),
    inputs.LayerConfig("swap_skew", T=2000, d=512, f=384, E=16, k=4, R=4, bias_std=1.5, seed=32),
    inputs.LayerConfig("swap_tiny_groups", T=40, d=256, f=128, E=16, k=4, R=4, seed=33),
    inputs.LayerConfig("swap_one_row", T=1, d=256, f=128, E=8, k=2, R=4, seed=34),
    inputs.LayerConfig("swap_exact", T=1024, d=256, f=128, E=4, k=1, R=4, seed=35),
    inputs.LayerConfig("swap_shared", T=600, d=512, f=256, E=16, k=6, R=8, S=2, fs=128, seed=36),
    inputs.LayerConfig("swap_renorm", T=900, d=256, f=256, E=8, k=2, R=8, renorm=1, seed=37),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_swap_gemm_matches_oracle(cfg, swap):
    run_and_check_small(cfg)


def test_swap_gemm_expert_parallel(swap):
    from test_gpu_ep import _check
    _check(inputs.LayerConfig("ep_swap", T=900, d=256, f=128, E=16, k=4, R=4), [300, 0, 455, 145],
           seed=38)


def test_swap_gemm_full_size_olmoe():
    cfg = inputs.CONFIGS["olmoe"]
    inp = inputs.make_inputs(cfg, device=DEV)
    layer = MoELayer(T=cfg.T, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k, R=cfg.R, renorm=cfg.renorm,
                     dtype=torch.bfloat16, device=DEV, wg=inp["wg"], wu=inp["wu"], wd=inp["wd"])
    y_rows = layer.forward(inp["logits"], inp["x"]).clone()
    moe.moe_set_debug(FORCE_SWAP, 4000.0)
    try:
        y_swap = layer.forward(inp["logits"], inp["x"]).clone()
        torch.cuda.synchronize()
    finally:
        moe.moe_set_debug(0, 4000.0)
    assert moe.moe_get_device_status() == moe.MOE_OK
    # against the row-major kernels' output: same products, other summation hardware
    assert rowwise_rel_err(y_swap.float().cpu().numpy(), y_rows.float().cpu().numpy()) <= 1e-2
    # against the oracle on sampled tokens
    rng = np.random.default_rng(3)
    tokens = np.sort(rng.choice(cfg.T, size=64, replace=False)).astype(np.int32)
    idx_ref, w_ref = oracle_route(inp["logits"].cpu(), cfg.k, cfg.renorm)
    used = np.unique(idx_ref[tokens])
    remap = -np.ones(cfg.E, np.int32)
    remap[used] = np.arange(len(used), dtype=np.int32)
    sel = torch.from_numpy(used).long().to(DEV)
    wg, wu, wd = (to_oracle(inp[key][sel]) for key in ("wg", "wu", "wd"))
    x_s = to_oracle(inp["x"][torch.from_numpy(tokens).long().to(DEV)])
    y_ref = oracle.dense_layer(x_s, remap[idx_ref[tokens]], w_ref[tokens], wg, wu, wd)
    y_gpu = y_swap[torch.from_numpy(tokens).long().to(DEV)].float().cpu().numpy()
    assert rowwise_rel_err(y_gpu, y_ref) <= OUT_RTOL

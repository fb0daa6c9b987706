"""The expert GEMM on 256 x 512 CTA-pair tiles (one accumulator filling TMEM's
512 columns, two N = 256 MMAs per K step, the weight panel in two 256-column
halves) against the oracle.  Debug flag 256 forces it wherever N % 512 == 0
(bf16, the inference epilogues).  Checked on ragged and skewed groups, empty
and one-row groups, shared experts, renormalised routing, and the correlated
prefill layer at full size against the 256-wide tiles' output and the oracle.
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
FORCE_WIDE = 256


@pytest.fixture
def wide():
    moe.moe_set_debug(FORCE_WIDE, 4000.0)
    yield
    moe.moe_set_debug(0, 4000.0)


CASES = [
    inputs.LayerConfig("wide_small", T=1500, d=512, f=256, E=8, k=2, R=4, seed=41),
    inputs.LayerConfig("wide_skew", T=2500, d=512, f=512, E=16, k=4, R=4, bias_std=1.5, seed=42),
    inputs.LayerConfig("wide_tiny_groups", T=40, d=512, f=256, E=16, k=4, R=4, seed=43),
    inputs.LayerConfig("wide_one_row", T=1, d=512, f=256, E=8, k=2, R=4, seed=44),
    inputs.LayerConfig("wide_shared", T=700, d=1024, f=256, E=16, k=6, R=8, S=2, fs=128, seed=45),
    inputs.LayerConfig("wide_renorm", T=900, d=512, f=512, E=8, k=2, R=8, renorm=1, seed=46),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_wide_tiles_match_oracle(cfg, wide):
    run_and_check_small(cfg)


def test_wide_tiles_full_size_corr_prefill():
    cfg = inputs.CONFIGS["corr_prefill"]
    inp = inputs.make_inputs(cfg, device=DEV)
    layer = MoELayer(T=cfg.T, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k, R=cfg.R, renorm=cfg.renorm,
                     dtype=torch.bfloat16, device=DEV, wg=inp["wg"], wu=inp["wu"], wd=inp["wd"])
    moe.moe_set_debug(512, 4000.0)  # 256-wide tiles, whatever the default
    try:
        y_256 = layer.forward(inp["logits"], inp["x"]).clone()
        moe.moe_set_debug(FORCE_WIDE, 4000.0)
        y_512 = layer.forward(inp["logits"], inp["x"]).clone()
        torch.cuda.synchronize()
    finally:
        moe.moe_set_debug(0, 4000.0)
    assert moe.moe_get_device_status() == moe.MOE_OK
    # the same products and K order per output element: the same bits
    assert torch.equal(y_512, y_256)
    rng = np.random.default_rng(5)
    tokens = np.sort(rng.choice(cfg.T, size=32, replace=False)).astype(np.int32)
    idx_ref, w_ref = oracle_route(inp["logits"].cpu(), cfg.k, cfg.renorm)
    used = np.unique(idx_ref[tokens])
    remap = -np.ones(cfg.E, np.int32)
    remap[used] = np.arange(len(used), dtype=np.int32)
    sel = torch.from_numpy(used).long().to(DEV)
    wg, wu, wd = (to_oracle(inp[key][sel]) for key in ("wg", "wu", "wd"))
    x_s = to_oracle(inp["x"][torch.from_numpy(tokens).long().to(DEV)])
    y_ref = oracle.dense_layer(x_s, remap[idx_ref[tokens]], w_ref[tokens], wg, wu, wd)
    y_gpu = y_512[torch.from_numpy(tokens).long().to(DEV)].float().cpu().numpy()
    assert rowwise_rel_err(y_gpu, y_ref) <= OUT_RTOL

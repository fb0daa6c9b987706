"""The named workloads at full size, in the launch configuration the benchmark
times.  Every index, count, BRIM entry and C_T is checked in full against the
oracle; layer outputs are checked on a seeded sample of tokens, which is valid
because each token's output depends on that token alone."""
import numpy as np
import pytest
import torch

import oracle
import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs
from expert_warp_top_b200.layer import MoELayer
from helpers import OUT_RTOL, oracle_route, rowwise_rel_err, to_oracle
from test_gpu_parity import check_indices

pytestmark = pytest.mark.gpu
DEV = "cuda"

SAMPLE = {"olmoe": 96, "mixtral": 24, "dsv2lite": 64, "corr_decode": 64, "corr_prefill": 48}


def correlated_placement(cfg):
    """Placement from the co-activation histogram of a separate calibration batch."""
    calib = cfg.with_(T=32768, seed=1)
    logits = inputs.make_logits(calib, device=DEV)
    idx = torch.empty(calib.T, calib.k, dtype=torch.int32, device=DEV)
    w = torch.empty(calib.T, calib.k, dtype=torch.float32, device=DEV)
    moe.moe_route_topk(logits, calib.k, 0, idx, w)
    hist = torch.zeros(calib.E, calib.E, dtype=torch.int32, device=DEV)
    moe.moe_coact_histogram(idx, calib.E, hist, 0)
    torch.cuda.synchronize()
    h = hist.cpu().numpy().astype(np.uint32)
    # the histogram itself must match the oracle's
    idx_ref, _ = oracle_route(logits.cpu(), calib.k, 0)
    assert np.array_equal(h, oracle.coact_histogram(idx_ref, calib.E))
    return oracle.place_greedy(h, calib.R)


@pytest.mark.parametrize("name,placement", [
    ("olmoe", "contiguous"), ("mixtral", "contiguous"), ("dsv2lite", "contiguous"),
    ("corr_decode", "contiguous"), ("corr_decode", "histogram"),
    ("corr_prefill", "contiguous"), ("corr_prefill", "histogram"),
])
def test_full_size_layer(name, placement):
    """The layer as the benchmark runs it (epd_mode auto)."""
    cfg = inputs.CONFIGS[name]
    inp = inputs.make_inputs(cfg, device=DEV)
    slot_of = (np.arange(cfg.E, dtype=np.int32) if placement == "contiguous"
               else correlated_placement(cfg))
    kw = dict(wg=inp["wg"], wu=inp["wu"], wd=inp["wd"])
    if cfg.S:
        kw.update(sg=inp["sg"], su=inp["su"], sd=inp["sd"])
    layer = MoELayer(T=cfg.T, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k, R=cfg.R, renorm=cfg.renorm,
                     dtype=torch.bfloat16, S=cfg.S, fs=cfg.fs,
                     slot_of=torch.from_numpy(slot_of), device=DEV, **kw)
    layer.hist.zero_()
    y = layer.forward(inp["logits"], inp["x"])
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    idx_ref, w_ref = oracle_route(inp["logits"].cpu(), cfg.k, cfg.renorm)
    b = check_indices(layer, idx_ref, w_ref, cfg, slot_of)
    assert np.array_equal(layer.hist.cpu().numpy().astype(np.uint32),
                          oracle.coact_histogram(idx_ref, cfg.E))
    if placement == "histogram":
        # correlated placement must cut the dispatched rows well below contiguous placement
        _, c_contig, _ = oracle.count_dispatched(idx_ref, np.arange(cfg.E, dtype=np.int32),
                                                 cfg.E, cfg.R)
        assert b["c_t"] < 0.6 * c_contig
    # dispatch copies, checked on every SFD row of a sample of ranks' segments
    c_t = b["c_t"]
    rng = np.random.default_rng(0)
    rows = rng.choice(c_t, size=min(c_t, 512), replace=False)
    x_cpu = inp["x"][torch.from_numpy(b["sfd_token"][rows]).long().to(DEV)].cpu()
    assert torch.equal(layer.x_sfd[torch.from_numpy(rows).long().to(DEV)].cpu(), x_cpu)
    # outputs on sampled tokens against the dense definition
    n = min(SAMPLE[name], cfg.T)
    tokens = np.sort(rng.choice(cfg.T, size=n, replace=False)).astype(np.int32)
    x_s = to_oracle(inp["x"][torch.from_numpy(tokens).long().to(DEV)])
    used = np.unique(idx_ref[tokens])
    # only the experts the sampled tokens use travel to the host
    remap = -np.ones(cfg.E, np.int32)
    remap[used] = np.arange(len(used), dtype=np.int32)
    sel = torch.from_numpy(used).long().to(DEV)
    wg, wu, wd = (to_oracle(inp[key][sel]) for key in ("wg", "wu", "wd"))
    shared = None
    if cfg.S:
        shared = (to_oracle(inp["sg"]), to_oracle(inp["su"]), to_oracle(inp["sd"]))
    y_ref = oracle.dense_layer(x_s, remap[idx_ref[tokens]], w_ref[tokens], wg, wu, wd,
                               shared=shared)
    y_gpu = y[torch.from_numpy(tokens).long().to(DEV)].float().cpu().numpy()
    err = rowwise_rel_err(y_gpu, y_ref)
    assert err <= OUT_RTOL, err

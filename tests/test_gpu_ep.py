"""Real expert parallelism on the GPU: the data plane of R ranks.

This run has one GPU, so the R ranks' kernels run in one process on that GPU
and LoopbackExchange moves the segments between them (the copies stand for
the network).  Every device step is the library's: routing and BRIMs on each
rank's own tokens, the SFD rows, the routing lists restricted to each
destination (moe_ep_pack_routing), the destination's BRIM build over the rows
it received, its EPD rows and grouped GEMMs over its own L experts, the
pre-reduced return rows (moe_ep_return_rows) and the source's combine of the
returned rows (moe_ep_combine).  Checked:
  - the rows each rank receives are, bit for bit, its SFD segment of the
    one-GPU layer over the concatenated batch, with the token's routing
    restricted to that rank's experts;
  - every token's output matches the oracle within the per-row tolerance,
    and the one-GPU layer's output;
  - NCCL with one rank (DistExchange over a real process group);
  - the exchange over peer memory (PeerExchange: the movers write straight
    into the receiving ranks' buffers), bit for bit against the loopback.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs
from expert_warp_top_b200.ep import (DistExchange, EPRank, LoopbackExchange, PeerExchange,
                                     ep_forward)
from expert_warp_top_b200.layer import MoELayer
from helpers import OUT_RTOL, expert_at_slot, rowwise_rel_err, to_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ranks(cfg, Ts, slot_of, inp):
    R, L = cfg.R, cfg.E // cfg.R
    at = torch.from_numpy(expert_at_slot(slot_of.numpy()).astype(np.int64))
    ranks = []
    for r in range(R):
        mine = at[r * L:(r + 1) * L]  # the experts at this rank's slots, in slot order
        kw = {}
        if cfg.S:
            kw = dict(S=cfg.S, fs=cfg.fs, sg=inp["sg"].to(DEV), su=inp["su"].to(DEV),
                      sd=inp["sd"].to(DEV))
        ranks.append(EPRank(rank=r, R=R, T=Ts[r], d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k,
                            renorm=cfg.renorm, dtype=inputs.torch_dtype(cfg), slot_of=slot_of,
                            wg=inp["wg"][mine].to(DEV), wu=inp["wu"][mine].to(DEV),
                            wd=inp["wd"][mine].to(DEV), recv_cap=sum(Ts), device=DEV, **kw))
    return ranks


def _check(cfg, Ts, seed=0, starve=False, placement="random", exchange=LoopbackExchange):
    assert sum(Ts) == cfg.T
    R, L = cfg.R, cfg.E // cfg.R
    inp = inputs.make_inputs(cfg, seed=seed)
    if placement == "random":
        slot_of = torch.randperm(cfg.E, generator=torch.Generator().manual_seed(seed + 1))
    else:
        slot_of = torch.arange(cfg.E)
    slot_of = slot_of.to(torch.int32)
    logits = inp["logits"].clone()
    if starve:  # nobody picks the experts of the last rank
        logits[:, (slot_of // L) == R - 1] -= 100.0
    logits_d, x_d = logits.to(DEV), inp["x"].to(DEV)
    # the one-GPU layer over the whole batch
    kw = dict(wg=inp["wg"].to(DEV), wu=inp["wu"].to(DEV), wd=inp["wd"].to(DEV))
    if cfg.S:
        kw.update(sg=inp["sg"].to(DEV), su=inp["su"].to(DEV), sd=inp["sd"].to(DEV))
    one = MoELayer(T=cfg.T, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k, R=R, renorm=cfg.renorm,
                   dtype=inputs.torch_dtype(cfg), S=cfg.S, fs=cfg.fs, slot_of=slot_of, device=DEV,
                   **kw)
    y_one = one.forward(logits_d, x_d).clone()
    # the R ranks, exchanging through loopback copies
    ranks = _ranks(cfg, Ts, slot_of, inp)
    bounds = np.cumsum([0] + list(Ts))
    ys = ep_forward(ranks, exchange(R),
                    [logits_d[bounds[r]:bounds[r + 1]].contiguous() for r in range(R)],
                    [x_d[bounds[r]:bounds[r + 1]].contiguous() for r in range(R)])
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    c_t = int(one.c_t.item())
    sfd_off = one.sfd_off.cpu().numpy()
    sfd_token = one.sfd_token[:c_t].cpu().numpy()
    idx = one.topk_idx.cpu().numpy()
    w = one.topk_w.cpu().numpy()
    assert sum(int(r.c_t.item()) for r in ranks) == c_t
    for q, r in enumerate(ranks):
        lo, hi = int(sfd_off[q]), int(sfd_off[q + 1])
        assert r.n_recv == hi - lo
        assert torch.equal(r.x_recv[:hi - lo], one.x_sfd[lo:hi])
        toks = sfd_token[lo:hi]
        mine = (slot_of.numpy()[idx[toks]] // L) == q
        assert np.array_equal(r.idx_recv[:hi - lo].cpu().numpy(), np.where(mine, idx[toks], -1))
        assert np.array_equal(r.w_recv[:hi - lo].cpu().numpy(), np.where(mine, w[toks], 0.0))
    y = torch.cat([yy[:t] for yy, t in zip(ys, Ts)])
    # against the one-GPU layer: the same EPD rows, gates and sums
    assert rowwise_rel_err(y.float().cpu().numpy(), y_one.float().cpu().numpy()) <= 1e-2
    # against the oracle (dense definition, double)
    idx_o, w_o = oracle.route(to_oracle(logits), cfg.k, cfg.renorm)
    shared = (to_oracle(inp["sg"]), to_oracle(inp["su"]), to_oracle(inp["sd"])) if cfg.S else None
    y_ref = oracle.dense_layer(to_oracle(inp["x"]), idx_o, w_o, to_oracle(inp["wg"]),
                               to_oracle(inp["wu"]), to_oracle(inp["wd"]), shared=shared)
    assert rowwise_rel_err(y.float().cpu().numpy(), y_ref) <= OUT_RTOL
    return ranks, one


def test_ep_loopback_tiny():
    cfg = inputs.CONFIGS["tiny"]
    _check(cfg, [64, 64, 64, 64])


def test_ep_loopback_uneven_batches_empty_rank_and_starved_rank():
    cfg = inputs.LayerConfig("ep_small", T=700, d=128, f=128, E=16, k=4, R=4)
    _check(cfg, [300, 0, 255, 145], seed=2)
    ranks, _ = _check(cfg, [175, 175, 175, 175], seed=3, starve=True)
    assert ranks[3].n_recv == 0


def test_ep_loopback_shared_experts():
    cfg = inputs.LayerConfig("ep_shared", T=1024, d=256, f=128, E=16, k=3, R=8, S=2, fs=128)
    _check(cfg, [128] * 8, seed=4)


def test_ep_loopback_olmoe_shaped():
    """The OLMoE-shaped layer (T = 4096 split over 8 ranks of 512 tokens, E = 64,
    k = 8, contiguous placement): real tile sizes, ragged groups per rank."""
    cfg = inputs.CONFIGS["olmoe"]
    _check(cfg, [512] * 8, placement="contiguous")


def test_ep_nccl_one_rank():
    """DistExchange over a one-rank NCCL group: the all-gather and all-to-all-v
    calls themselves, on device buffers (all experts on the one rank)."""
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device(DEV, torch.cuda.current_device()))
    try:
        cfg = inputs.LayerConfig("ep_nccl", T=512, d=128, f=128, E=8, k=2, R=1)
        inp = inputs.make_inputs(cfg, seed=6)
        (r,) = _ranks(cfg, [cfg.T], torch.arange(cfg.E, dtype=torch.int32), inp)
        (y,) = ep_forward([r], DistExchange(), [inp["logits"].to(DEV)], [inp["x"].to(DEV)])
        torch.cuda.synchronize()
        assert r.n_recv == cfg.T
        idx_o, w_o = oracle.route(to_oracle(inp["logits"]), cfg.k, cfg.renorm)
        y_ref = oracle.dense_layer(to_oracle(inp["x"]), idx_o, w_o, to_oracle(inp["wg"]),
                                   to_oracle(inp["wu"]), to_oracle(inp["wd"]))
        assert rowwise_rel_err(y.float().cpu().numpy(), y_ref) <= OUT_RTOL
    finally:
        dist.destroy_process_group()


def test_bench_ep_mode_line():
    """`bench.py --ep` on the tiny workload (4 loopback ranks on the one GPU):
    one JSON line whose C_T is the counter's, whose rows between ranks are the
    off-diagonal pair counts, and whose phases add up to the step."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--ep", "--config", "tiny",
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    cfg = inputs.CONFIGS["tiny"]
    ep = line["ep"]
    assert ep["ranks"] == cfg.R and line["config"]["R"] == cfg.R
    assert ep["c_t"] == line["placement"]["c_t_contiguous"]
    assert 0 <= ep["rows_between_ranks"] <= ep["c_t"]
    assert ep["payload_bytes_each_way"] == ep["rows_between_ranks"] * cfg.d * 2
    assert abs(sum(ep["phase_ms"].values()) - line["ms_per_step"]) <= 0.05 * line["ms_per_step"]
    assert line["value"] > 0 and line["unit"] == "tokens/s"


@pytest.mark.parametrize("case", ["tiny", "uneven_starved", "shared", "olmoe"])
def test_ep_peer_exchange(case):
    """The same checks with the rows moved by moe_ep_send_peer / moe_ep_return_peer."""
    if case == "tiny":
        cfg = inputs.CONFIGS["tiny"]
        _check(cfg, [cfg.T // cfg.R] * cfg.R, exchange=PeerExchange)
    elif case == "uneven_starved":
        cfg = inputs.LayerConfig("ep_uneven", T=700, d=128, f=128, E=16, k=4, R=4, seed=3)
        _check(cfg, [300, 0, 250, 150], seed=3, starve=True, exchange=PeerExchange)
    elif case == "shared":
        cfg = inputs.LayerConfig("ep_shared", T=512, d=256, f=128, E=8, k=2, R=4, S=1, fs=128,
                                 seed=4)
        _check(cfg, [128] * 4, seed=4, exchange=PeerExchange)
    else:
        cfg = inputs.CONFIGS["olmoe"]
        _check(cfg, [512] * 8, placement="contiguous", exchange=PeerExchange)


def test_ep_peer_exchange_equals_loopback_bit_for_bit():
    """Every received row, routing list and gate, and every output, equal to
    the loopback exchange's (random placement, uneven batches)."""
    cfg = inputs.LayerConfig("ep_bits", T=1536, d=256, f=256, E=32, k=6, R=8, seed=9)
    Ts = [300, 100, 0, 256, 180, 300, 200, 200]
    ranks_l, _ = _check(cfg, Ts, seed=9)
    ranks_p, _ = _check(cfg, Ts, seed=9, exchange=PeerExchange)
    for a, b in zip(ranks_l, ranks_p):
        n = a.n_recv
        assert b.n_recv == n
        assert torch.equal(a.x_recv[:n], b.x_recv[:n])
        assert torch.equal(a.idx_recv[:n], b.idx_recv[:n])
        assert torch.equal(a.w_recv[:n], b.w_recv[:n])
        c_t = int(a.c_t.item())
        assert torch.equal(a.y_ret[:c_t], b.y_ret[:c_t])
        assert torch.equal(a.y[:a.T], b.y[:b.T])

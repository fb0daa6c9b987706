"""Real expert parallelism over gloo ranks on the host (world sizes 2 and 4).

Each process holds one rank: its own slice of the batch and the experts at
its slots.  ep_forward() runs the exchanges of the expert-parallel layer
(the all-gather of the per-destination row counts, the all-to-all-v of the
SFD rows, of their routing lists and of the return rows) over a gloo process
group; every local step is the CPU oracle's (tests/ep_oracle_rank.py), so
these tests check the exchange logic of the library against the one-process
oracle layer:
  - the rows a rank receives are exactly its SFD segment of the one-process
    layer over the concatenated batch (the Occult paper, Figure 2/4: the
    all-to-all payload), with the token's routing restricted to its experts;
  - every rank's C_T adds up to the one-process C_T;
  - the output of every token equals the one-process oracle layer's.
Uneven batches, a rank with no tokens and a rank whose experts nobody picks
are included.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(Ts, E, k, seed, starve_last_rank):
    """The full batch (concatenated in rank order), the weights and a placement."""
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from expert_warp_top_b200 import inputs
    from helpers import to_oracle
    R = len(Ts)
    cfg = inputs.LayerConfig("ep", T=sum(Ts), d=64, f=64, E=E, k=k, R=R, seed=seed)
    inp = inputs.make_inputs(cfg)
    slot_of = torch.randperm(E, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
    logits = inp["logits"].clone()
    if starve_last_rank:  # nobody picks the experts of rank R-1
        L = E // R
        on_last = (slot_of // L) == R - 1
        logits[:, on_last] -= 100.0
    return (cfg, logits.numpy(), to_oracle(inp["x"]), to_oracle(inp["wg"]), to_oracle(inp["wu"]),
            to_oracle(inp["wd"]), slot_of.numpy())


def _worker(rank, Ts, E, k, seed, starve, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from ep_oracle_rank import OracleEPRank
    from expert_warp_top_b200.ep import DistExchange, ep_forward
    world = len(Ts)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, logits, x, wg, wu, wd, slot_of = _problem(Ts, E, k, seed, starve)
        lo = sum(Ts[:rank])
        T = Ts[rank]
        r = OracleEPRank(rank=rank, R=world, T=T, d=cfg.d, f=cfg.f, E=E, k=k, renorm=0,
                         slot_of=slot_of, wg=wg, wu=wu, wd=wd, recv_cap=max(sum(Ts), 1))
        ex = DistExchange()
        (y,) = ep_forward([r], ex, [logits[lo:lo + T]], [x[lo:lo + T]])
        n = r.n_recv
        out[rank] = dict(x_recv=r.x_recv[:n].numpy().copy(), idx_recv=r.idx_recv[:n].numpy().copy(),
                         w_recv=r.w_recv[:n].numpy().copy(), c_t=r.b["c_t"], y=y.numpy().copy(),
                         y_recv=r.y_recv[:n].numpy().copy())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _run(Ts, E, k, seed, starve=False):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from ep_oracle_rank import _widen
    world, port = len(Ts), _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(Ts, E, k, seed, starve, port, out), nprocs=world, join=True)
        res = dict(out)
    cfg, logits, x, wg, wu, wd, slot_of = _problem(Ts, E, k, seed, starve)
    R, L = world, E // world
    idx, w = oracle.route(logits, k, 0)
    b = oracle.brim(idx, w, slot_of, E, R)
    _, y_ref = oracle.occult_layer(x, slot_of, E, R, k, b, wg, wu, wd)
    x_sfd = np.stack([_widen(r) for r in oracle.gather_rows(x, b["sfd_token"])]) if b["c_t"] \
        else np.zeros((0, cfg.d))
    assert sum(res[q]["c_t"] for q in range(R)) == b["c_t"]
    for q in range(R):
        lo, hi = int(b["sfd_off"][q]), int(b["sfd_off"][q + 1])
        got = res[q]
        assert got["x_recv"].shape[0] == hi - lo
        # the received rows are rank q's SFD segment of the one-process layer, bit for bit
        assert np.array_equal(got["x_recv"], x_sfd[lo:hi])
        # with each row, the token's experts on rank q (and their gates), the rest empty
        for i, s in enumerate(range(lo, hi)):
            t = int(b["sfd_token"][s])
            for j in range(k):
                e = int(idx[t, j])
                mine = slot_of[e] // L == q
                assert got["idx_recv"][i, j] == (e if mine else -1)
                assert got["w_recv"][i, j] == (w[t, j] if mine else 0.0)
    y = np.concatenate([res[q]["y"] for q in range(R)])
    assert y.shape == y_ref.shape
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)
    return res, b


def test_ep_two_gloo_ranks_match_the_one_process_layer():
    _run([48, 48], E=8, k=3, seed=3)


def test_ep_four_gloo_ranks_uneven_batches_and_an_empty_rank():
    res, b = _run([40, 0, 30, 26], E=8, k=3, seed=4)
    assert res[1]["y"].shape[0] == 0


def test_ep_four_gloo_ranks_one_rank_receives_nothing():
    res, b = _run([24, 24, 24, 24], E=16, k=4, seed=5, starve=True)
    assert res[3]["x_recv"].shape[0] == 0
    assert int(b["sfd_off"][4] - b["sfd_off"][3]) == 0

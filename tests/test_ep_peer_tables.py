"""The host side of the exchange over peer memory (PeerExchange): the row
offsets and segments it hands the peer movers.  Replaying the movers' writes
with those tables must give every rank exactly the rows, in exactly the order,
that the all-to-all-v exchange (LoopbackExchange) delivers, and give every
source its return rows at its own SFD positions."""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

from expert_warp_top_b200.ep import LoopbackExchange, PeerExchange, pair_counts


def _ranks(R, counts, n_cols=3):
    """R fake ranks: counts[s][q] rows from s to q; SFD rows tagged (s, q, i)."""
    ranks = []
    for s in range(R):
        rows = [(s, q, i) for q in range(R) for i in range(counts[s][q])]
        x_sfd = torch.tensor(rows, dtype=torch.int64).reshape(-1, n_cols)
        n_in = sum(counts[src][s] for src in range(R))
        off = [0]
        for q in range(R):
            off.append(off[-1] + counts[s][q])
        ranks.append(SimpleNamespace(
            x_sfd=x_sfd, sfd_off=torch.tensor(off, dtype=torch.int32),
            x_recv=torch.full((max(n_in, 1), n_cols), -1, dtype=torch.int64),
            idx_recv=torch.zeros(1, dtype=torch.int32), w_recv=torch.zeros(1),
            y_ret=torch.full((max(len(rows), 1), n_cols), -1, dtype=torch.int64)))
    return ranks


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_peer_tables_reproduce_the_all_to_all(seed):
    R = 5
    rng = np.random.default_rng(seed)
    counts = rng.integers(0, 7, size=(R, R)).tolist()
    counts[2] = [0] * R                      # a source that sends nothing
    for s in range(R):
        counts[s][3] = 0                     # a rank nobody sends to
    ranks = _ranks(R, counts)
    offs = [r.sfd_off.tolist() for r in ranks]
    assert pair_counts(offs, R) == counts

    # what the all-to-all-v delivers
    expect = [torch.full_like(r.x_recv, -1) for r in ranks]
    LoopbackExchange(R).rows([r.x_sfd for r in ranks], counts, expect,
                             [[counts[s][q] for s in range(R)] for q in range(R)])

    # the peer movers' writes, replayed from the tables
    for src, r in enumerate(ranks):
        t = PeerExchange.send_peers(ranks, counts, offs, src)
        for q in range(R):
            assert t.rows[q] == ranks[q].x_recv.data_ptr()
            for s in range(offs[src][q], offs[src][q + 1]):
                ranks[q].x_recv[t.row0[q] + s] = r.x_sfd[s]
    for q in range(R):
        n = sum(counts[s][q] for s in range(R))
        assert torch.equal(ranks[q].x_recv[:n], expect[q][:n])

    # return rows: destination dst's received row i goes back to its source's
    # SFD row for dst, which is where that source sent it from
    for dst, r in enumerate(ranks):
        t = PeerExchange.return_peers(ranks, counts, offs, dst)
        n = sum(counts[s][dst] for s in range(R))
        assert [t.seg[q] for q in range(R + 1)] == list(
            np.concatenate([[0], np.cumsum([counts[s][dst] for s in range(R)])]))
        for i in range(n):
            q = max(q for q in range(R) if t.seg[q] <= i)
            assert t.rows[q] == ranks[q].y_ret.data_ptr()
            ranks[q].y_ret[t.row0[q] + i] = r.x_recv[i]
    for s, r in enumerate(ranks):
        c_t = offs[s][R]
        assert torch.equal(r.y_ret[:c_t], r.x_sfd[:c_t])

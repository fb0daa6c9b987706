"""Real expert parallelism: the layer's experts spread over R ranks (one
process per GPU), with the tokens exchanged by all-to-all.

On one GPU the library simulates the R ranks: the SFD segments stand for the
rows an all-to-all would carry.  Here the ranks are real.  The Occult paper
(Abstract; Figure 2) sends each token to the devices holding its experts and
sums, on each device, the outputs of the token's co-located experts before a
single row goes back ("intra-collaboration"); "Expert Coupling in MoE
Pretraining" (Abstract) calls the same thing a dispatcher that sends each
token to each GPU once.  C_T, the SFD row count, is then the number of rows
that really cross the network in each direction.

Rank r holds the experts at slots r*L .. r*L+L-1 and its own batch of tokens.
One forward:

  1 source       routing and the BRIM build over the rank's own tokens; the
                 SFD rows (one per token and destination rank), and with each
                 row the token's top-k list restricted to the destination's
                 experts                     moe_route_brim, moe_dispatch_gather,
                                             moe_ep_pack_routing
  2 exchange     every rank's sfd_off (all-gather): the row count of every
                 (source, destination) pair, read on the host
  3 exchange     all-to-all-v of the SFD rows and of their routing lists
  4 destination  the BRIM build over the received rows (its BRIM_1 and EPD
                 groups), the EPD rows, the grouped GEMMs of its L experts,
                 one pre-reduced return row per received row
                                             moe_brim_build, moe_dispatch_gather,
                                             moe_expert_ffn, moe_ep_return_rows
  5 exchange     all-to-all-v of the return rows back to their sources
  6 source       every token sums its returned rows in ORI order, plus the
                 shared experts computed on the rank's own tokens
                                             moe_ep_combine

The rows a rank receives in step 3 come source by source in rank order, and
from each source in ascending token order: exactly that rank's SFD segment of
the one-GPU layer over all ranks' batches concatenated in rank order.

The exchanges go through an exchange object: DistExchange uses a
torch.distributed process group (NCCL between GPUs, gloo on the host);
LoopbackExchange moves the segments between R ranks held by one process (all
on one GPU), so the whole data plane of R ranks can run and be checked on a
single GPU.  PeerExchange takes no collective for the rows: steps 1 and 3
become one mover that writes each SFD row and its routing list straight into
the receiving rank's buffer (moe_ep_send_peer), and steps 4 and 5 one mover
that writes each pre-reduced return row straight into its source's buffer
(moe_ep_return_peer); only the row counts (step 2) are exchanged on the host.
It holds the R ranks in one process and addresses their buffers directly.  ep_forward() drives the six steps over the ranks a process
holds: one with DistExchange, all R with LoopbackExchange.  The rank objects
are EPRank (the CUDA kernels) or anything with the same steps and buffers.
"""
from __future__ import annotations

import torch

from . import _binding as B


# ---------------------------------------------------------------------------
class DistExchange:
    """The exchanges over a torch.distributed process group.  The process holds
    one rank (its rank in the group); tensors live where the backend wants
    them (CUDA for NCCL, host for gloo)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.R = dist.get_world_size(group)
        self.ranks = [dist.get_rank(group)]

    def gather_offsets(self, sfd_offs):
        """[R][R+1] host lists: every rank's sfd_off."""
        (mine,) = sfd_offs
        parts = [torch.empty_like(mine) for _ in range(self.R)]
        self.dist.all_gather(parts, mine, group=self.group)
        return torch.stack(parts).cpu().tolist()

    def rows(self, sends, send_splits, recvs, recv_splits):
        """Segment q of this rank's send buffer goes to rank q; the segment
        from rank s lands at segment s of the receive buffer."""
        ((send,), (ss,), (recv,), (rs,)) = (sends, send_splits, recvs, recv_splits)
        self.dist.all_to_all_single(recv[:sum(rs)], send[:sum(ss)], rs, ss, group=self.group)


class LoopbackExchange:
    """The same exchanges between R ranks held by one process: segment q of
    rank s's send buffer is copied to segment s of rank q's receive buffer.
    The copies stand for the network."""

    def __init__(self, R: int):
        self.R = R
        self.ranks = list(range(R))

    def gather_offsets(self, sfd_offs):
        return torch.stack(list(sfd_offs)).cpu().tolist()

    def rows(self, sends, send_splits, recvs, recv_splits):
        R = self.R
        for q in range(R):
            at = 0
            for s in range(R):
                n = send_splits[s][q]
                if n != recv_splits[q][s]:
                    raise RuntimeError("send and receive counts disagree")
                lo = sum(send_splits[s][:q])
                if n:
                    recvs[q][at:at + n].copy_(sends[s][lo:lo + n])
                at += n


class PeerExchange(LoopbackExchange):
    """The exchange over peer memory for R ranks held by one process: the
    movers write into the other ranks' buffers through a table of their
    device addresses (moe_ep_peers).  The ranks' kernels run on one stream
    in rank order, which orders every send before every read of it."""

    peer = True

    def barrier(self):
        pass

    @staticmethod
    def send_peers(ranks, counts, offs, src):
        """The table for source `src`: its rows for rank q start at row
        sum(counts[s][q] for s < src) of q's receive buffers, and its SFD
        segment for q starts at offs[src][q]."""
        R = len(ranks)
        row0 = [sum(counts[s][q] for s in range(src)) - offs[src][q] for q in range(R)]
        return B.ep_peers([r.x_recv.data_ptr() for r in ranks], row0,
                          idx=[r.idx_recv.data_ptr() for r in ranks],
                          w=[r.w_recv.data_ptr() for r in ranks])

    @staticmethod
    def return_peers(ranks, counts, offs, dst):
        """The table for destination `dst`: its received rows from source q
        are rows seg[q] .. seg[q+1]-1 (source-major), and q wants row i of
        them at its SFD row offs[q][dst] + (i - seg[q])."""
        R = len(ranks)
        seg = [0]
        for q in range(R):
            seg.append(seg[-1] + counts[q][dst])
        row0 = [offs[q][dst] - seg[q] for q in range(R)]
        return B.ep_peers([r.y_ret.data_ptr() for r in ranks], row0, seg=seg)


def pair_counts(offs, R):
    """rows[s][q]: rows rank s sends to rank q, from every rank's sfd_off."""
    return [[offs[s][q + 1] - offs[s][q] for q in range(R)] for s in range(R)]


def ep_forward(ranks, exchange, logits, xs, marks=None):
    """One forward of the expert-parallel layer over the ranks this process
    holds (ranks[i] is rank exchange.ranks[i]; logits[i], xs[i] its batch).
    Returns each rank's output y [T_r, d] (a view of its buffer) and keeps
    every intermediate in the rank objects.  `marks`, if given, is called with
    a phase name ("sent", "exchanged", "computed", "returned") as each phase
    ends (e.g. to record CUDA events), and the pair counts of the forward are
    kept in `ep_forward.counts`."""
    R = exchange.R
    mark = marks or (lambda name: None)
    if getattr(exchange, "peer", False):
        return _ep_forward_peer(ranks, exchange, logits, xs, mark)
    for r, lg, x in zip(ranks, logits, xs):
        r.send_phase(lg, x)
    mark("sent")
    counts = pair_counts(exchange.gather_offsets([r.sfd_off for r in ranks]), R)
    ep_forward.counts = counts
    send_splits = [counts[q] for q in exchange.ranks]
    recv_splits = [[counts[s][q] for s in range(R)] for q in exchange.ranks]
    for r, rs in zip(ranks, recv_splits):
        r.reserve_received(sum(rs))
    exchange.rows([r.x_sfd for r in ranks], send_splits, [r.x_recv for r in ranks], recv_splits)
    exchange.rows([r.idx_send for r in ranks], send_splits, [r.idx_recv for r in ranks],
                  recv_splits)
    exchange.rows([r.w_send for r in ranks], send_splits, [r.w_recv for r in ranks], recv_splits)
    mark("exchanged")
    for r, rs in zip(ranks, recv_splits):
        r.recv_phase(sum(rs))
    mark("computed")
    exchange.rows([r.y_recv for r in ranks], recv_splits, [r.y_ret for r in ranks], send_splits)
    mark("returned")
    for r in ranks:
        r.combine_phase()
    return [r.y for r in ranks]


def _ep_forward_peer(ranks, exchange, logits, xs, mark):
    """ep_forward over peer memory: the routing and BRIMs of every source,
    the row counts, then each source's send straight into the receivers'
    buffers, each destination's experts and its return rows straight into
    the sources' buffers, and the combine."""
    R = exchange.R
    for r, lg, x in zip(ranks, logits, xs):
        r.route_phase(lg, x)
    offs = exchange.gather_offsets([r.sfd_off for r in ranks])
    counts = pair_counts(offs, R)
    ep_forward.counts = counts
    for q, r in enumerate(ranks):
        r.reserve_received(sum(counts[s][q] for s in range(R)))
    exchange.barrier()  # every receive buffer is free
    for q, (r, x) in enumerate(zip(ranks, xs)):
        r.send_peer(x, exchange.send_peers(ranks, counts, offs, q))
    mark("sent")
    exchange.barrier()  # every row has landed
    mark("exchanged")
    for q, r in enumerate(ranks):
        r.compute_phase(sum(counts[s][q] for s in range(R)))
    mark("computed")
    for q, r in enumerate(ranks):
        r.return_peer(exchange.return_peers(ranks, counts, offs, q))
    exchange.barrier()  # every return row has landed
    mark("returned")
    for r in ranks:
        r.combine_phase()
    return [r.y for r in ranks]


# ---------------------------------------------------------------------------
class EPRank:
    """One rank of the expert-parallel layer on its GPU: its tokens' source
    side and its experts' destination side, as CUDA kernels.

    rank, R       this rank and the number of ranks (E % R == 0, L = E / R)
    T             this rank's tokens per forward
    recv_cap      most rows it may receive (default R * T: every rank's T
                  tokens at most once each)
    slot_of [E]   placement (rank of expert e = slot_of[e] // L)
    wg, wu [L,f,d], wd [L,d,f]  the weights of THIS rank's experts, in slot
                  order (local expert j = slot r*L + j)
    sg, su, sd    shared experts (computed on the rank's own tokens)
    """

    def __init__(self, *, rank, R, T, d, f, E, k, renorm=0, dtype=torch.bfloat16, slot_of=None,
                 wg=None, wu=None, wd=None, S=0, fs=0, sg=None, su=None, sd=None,
                 recv_cap=None, device="cuda"):
        if E % R:
            raise ValueError("R must divide E")
        self.rank, self.R, self.T, self.d, self.f, self.E, self.k = rank, R, T, d, f, E, k
        self.L = L = E // R
        self.renorm, self.dtype, self.S, self.fs = renorm, dtype, S, fs
        dev = self.device = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        act = dict(dtype=dtype, device=dev)
        if slot_of is None:
            slot_of = torch.arange(E, dtype=torch.int32)
        self.slot_of = slot_of.to(**i32).contiguous()
        self.cap = cap = max(T * min(k, R), 1)
        self.recv_cap = rc = max(R * T if recv_cap is None else recv_cap, 1)
        # source side: the rank's own tokens
        self.topk_idx = torch.empty(max(T, 1), k, **i32)
        self.topk_w = torch.empty(max(T, 1), k, **f32)
        self.brim0 = torch.empty(R, max(T, 1), **i32)
        self.sfd_token = torch.empty(cap, **i32)
        self.sfd_off = torch.empty(R + 1, **i32)
        self.brim1 = torch.empty(L, cap, **i32)
        self.epd_off = torch.empty(E + 1, **i32)
        self.epd_sfd = torch.empty(max(T * k, 1), **i32)
        self.epd_gate = torch.empty(max(T * k, 1), **f32)
        self.c_t = torch.empty(1, **i32)
        self.ws = torch.empty(max(B.moe_route_brim_workspace_size(T, E, R), 256),
                              dtype=torch.uint8, device=dev)
        self.x_sfd = torch.empty(cap, d, **act)
        self.idx_send = torch.empty(cap, k, **i32)
        self.w_send = torch.empty(cap, k, **f32)
        self.y_ret = torch.empty(cap, d, **act)
        self.y = torch.empty(max(T, 1), d, **act)
        # destination side: the rows it receives (local BRIM build over them)
        self.x_recv = torch.empty(rc, d, **act)
        self.idx_recv = torch.empty(rc, k, **i32)
        self.w_recv = torch.empty(rc, k, **f32)
        kr = min(k, R)
        self._l_brim0 = torch.empty(R * rc, **i32)
        self._l_sfd_token = torch.empty(rc * kr, **i32)
        self._l_sfd_off = torch.empty(R + 1, **i32)
        self._l_brim1 = torch.empty(L * rc * kr, **i32)
        self._l_epd_off = torch.empty(E + 1, **i32)
        self._l_epd_sfd = torch.empty(rc * k, **i32)
        self._l_epd_gate = torch.empty(rc * k, **f32)
        self._l_c_t = torch.empty(1, **i32)
        self._l_ws = torch.empty(max(B.moe_brim_workspace_size(rc, E, R), 256),
                                 dtype=torch.uint8, device=dev)
        # Buffers indexed by the local build's rows are sized by the bounds its
        # kernels check (EPD rows < n*k, SFD rows < n*min(k, R) for n received
        # rows), so even routing lists that name other ranks' experts cannot
        # send a write past them; valid lists use at most n*min(k, L) and n.
        m_cap = rc * k
        self.x_epd = torch.empty(m_cap, d, **act)
        self.o_epd = torch.empty(m_cap, d, **act)
        self.y_recv = torch.empty(rc * kr, d, **act)
        self.ffn_ws = torch.empty(max(B.moe_expert_ffn_workspace_size(m_cap, f, B.dtype_code(dtype)),
                                      256), dtype=torch.uint8, device=dev)
        self.n_recv = 0
        # this rank's experts, packed (slot order = local order)
        self.w_gu = torch.empty(L, 2 * f, d, **act)
        self.w_dn = torch.empty(L, d, f, **act)
        B.moe_prepare_weights(wg.to(**act).contiguous(), wu.to(**act).contiguous(),
                              wd.to(**act).contiguous(), None, self.w_gu, self.w_dn)
        self.shared_out = None
        if S > 0:
            F = S * fs
            self.sw_gu = torch.empty(1, 2 * F, d, **act)
            self.sw_dn = torch.empty(1, d, F, **act)
            B.moe_prepare_shared_weights(sg.to(**act).contiguous(), su.to(**act).contiguous(),
                                         sd.to(**act).contiguous(), self.sw_gu, self.sw_dn)
            self.shared_off = torch.tensor([0, T], **i32)
            self.shared_out = torch.empty(max(T, 1), d, **act)
            self.shared_ws = torch.empty(
                max(B.moe_expert_ffn_workspace_size(max(T, 1), F, B.dtype_code(dtype)), 256),
                dtype=torch.uint8, device=dev)

    # -- source side -------------------------------------------------------
    def route_phase(self, logits, x, stream=None):
        """Routing and the BRIM build over this rank's tokens, and its shared
        experts."""
        T, k, R = self.T, self.k, self.R
        if T == 0:
            B.moe_brim_build(self.topk_idx[:0], self.topk_w[:0], self.slot_of, self.E, R,
                             self.brim0, self.sfd_token, self.sfd_off, self.brim1, self.epd_off,
                             self.epd_sfd, self.epd_gate, self.c_t, self.ws, stream)
            return
        B.moe_route_brim(logits, k, self.renorm, self.slot_of, R, self.topk_idx, self.topk_w,
                         self.brim0, self.sfd_token, self.sfd_off, self.brim1, self.epd_off,
                         self.epd_sfd, self.epd_gate, self.c_t, self.ws, stream=stream)
        if self.S > 0:
            B.moe_expert_ffn(x, self.shared_off, self.sw_gu, self.sw_dn, self.S * self.fs, None,
                             B.MOE_FFN_SWIGLU, self.shared_out, self.shared_ws, stream)

    def send_phase(self, logits, x, stream=None):
        """route_phase, then the SFD rows and their routing lists in this
        rank's send buffers (for a collective)."""
        self.route_phase(logits, x, stream)
        if self.T == 0:
            return
        B.moe_dispatch_gather(x, self.k, self.R, self.L, self.brim0, self.brim1, self.x_sfd, None,
                              stream)
        B.moe_ep_pack_routing(self.topk_idx, self.topk_w, self.slot_of, self.E, self.R,
                              self.sfd_token, self.sfd_off, self.c_t, self.idx_send, self.w_send,
                              stream)

    def send_peer(self, x, peers, stream=None):
        """The SFD rows and their routing lists written straight into the
        receiving ranks' buffers (moe_ep_send_peer)."""
        if self.T == 0:
            return
        B.moe_ep_send_peer(x, self.topk_idx, self.topk_w, self.slot_of, self.R, self.L,
                           self.brim0, self.brim1, self.sfd_token, self.sfd_off, self.c_t, peers,
                           stream)

    # -- destination side ----------------------------------------------------
    def reserve_received(self, n):
        if n > self.recv_cap:
            raise RuntimeError(f"rank {self.rank} receives {n} rows, more than its "
                               f"capacity {self.recv_cap}")

    def local_state(self, n=None):
        """Views of the BRIM build over the n received rows."""
        n = self.n_recv if n is None else n
        R, L, k = self.R, self.L, self.k
        cap = max(n * min(k, R), 1)
        return dict(brim0=self._l_brim0[:R * max(n, 1)].view(R, max(n, 1)),
                    sfd_token=self._l_sfd_token[:cap], sfd_off=self._l_sfd_off,
                    brim1=self._l_brim1[:L * cap].view(L, cap), epd_off=self._l_epd_off,
                    epd_sfd=self._l_epd_sfd[:max(n * k, 1)],
                    epd_gate=self._l_epd_gate[:max(n * k, 1)], c_t=self._l_c_t)

    def recv_phase(self, n, stream=None):
        """compute_phase, then one pre-reduced return row per received row in
        this rank's return buffer (for a collective)."""
        self.compute_phase(n, stream)
        if n == 0:
            return
        s = self.local_state(n)
        B.moe_ep_return_rows(self.o_epd, n, self.k, self.R, self.L, s["brim0"], s["brim1"],
                             self.y_recv, stream)

    def return_peer(self, peers, stream=None):
        """The pre-reduced return rows written straight into their sources'
        buffers (moe_ep_return_peer)."""
        n = self.n_recv
        if n == 0:
            return
        s = self.local_state(n)
        B.moe_ep_return_peer(self.o_epd, n, self.k, self.R, self.L, s["brim0"], s["brim1"], peers,
                             stream)

    def compute_phase(self, n, stream=None):
        """The local BRIM build over the n received rows, their EPD rows and
        the grouped GEMMs of this rank's experts."""
        self.n_recv = n
        s = self.local_state(n)
        B.moe_brim_build(self.idx_recv[:n], self.w_recv[:n], self.slot_of, self.E, self.R,
                         s["brim0"], s["sfd_token"], s["sfd_off"], s["brim1"], s["epd_off"],
                         s["epd_sfd"], s["epd_gate"], s["c_t"], self._l_ws, stream)
        if n == 0:
            return
        B.moe_dispatch_gather(self.x_recv[:n], self.k, self.R, self.L, s["brim0"], s["brim1"],
                              None, self.x_epd, stream)
        lo = self.rank * self.L
        B.moe_expert_ffn(self.x_epd, s["epd_off"][lo:lo + self.L + 1], self.w_gu, self.w_dn,
                         self.f, s["epd_gate"], B.MOE_FFN_SWIGLU, self.o_epd, self.ffn_ws, stream,
                         m_cap=n * self.k)

    # -- source side, after the return exchange ------------------------------
    def combine_phase(self, stream=None):
        if self.T == 0:
            return
        B.moe_ep_combine(self.y_ret, self.T, self.k, self.R, self.brim0, self.shared_out, self.y,
                         stream)

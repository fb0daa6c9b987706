"""One rank of the expert-parallel layer computed by the CPU oracle (test
infrastructure): the same steps and buffers as expert_warp_top_b200.ep.EPRank,
with every step done in double precision by the oracle or by its plain
definition in numpy, so that ep_forward's exchanges can be run with gloo ranks
on the host and checked against the one-process oracle layer.

Rows travel as float64 (the bf16 inputs widened exactly), routing ids as
int32 and gate weights as float64.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


class OracleEPRank:
    def __init__(self, *, rank, R, T, d, f, E, k, renorm, slot_of, wg, wu, wd, recv_cap):
        """wg, wu, wd: oracle arrays of ALL E experts (expert-id order); the rank
        only ever uses the experts at its own slots."""
        self.rank, self.R, self.T, self.d, self.f, self.E, self.k = rank, R, T, d, f, E, k
        self.L = E // R
        self.renorm = renorm
        self.slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
        self.expert_at = np.empty(E, np.int32)
        self.expert_at[self.slot_of] = np.arange(E, dtype=np.int32)
        self.wg, self.wu, self.wd = wg, wu, wd
        cap = max(T * min(k, R), 1)
        f64 = dict(dtype=torch.float64)
        self.x_sfd = torch.zeros(cap, d, **f64)
        self.idx_send = torch.full((cap, k), -1, dtype=torch.int32)
        self.w_send = torch.zeros(cap, k, **f64)
        self.y_ret = torch.zeros(cap, d, **f64)
        self.x_recv = torch.zeros(recv_cap, d, **f64)
        self.idx_recv = torch.full((recv_cap, k), -1, dtype=torch.int32)
        self.w_recv = torch.zeros(recv_cap, k, **f64)
        self.y_recv = torch.zeros(recv_cap, d, **f64)
        self.recv_cap = recv_cap
        self.n_recv = 0

    # -- source side -------------------------------------------------------
    def send_phase(self, logits, x):
        """logits float32 [T, E]; x [T, d] as the oracle takes it (bf16 bits)."""
        T, k, R, L = self.T, self.k, self.R, self.L
        self.x = x
        if T == 0:
            self.idx = np.zeros((0, k), np.int32)
            self.w = np.zeros((0, k))
        else:
            self.idx, self.w = oracle.route(np.asarray(logits, np.float32), k, self.renorm)
        self.b = oracle.brim(self.idx, self.w, self.slot_of, self.E, R)
        self.sfd_off = torch.from_numpy(self.b["sfd_off"].astype(np.int64))
        c_t = self.b["c_t"]
        xw = oracle.gather_rows(x, self.b["sfd_token"]) if c_t else None
        for s in range(c_t):
            t = int(self.b["sfd_token"][s])
            q = int(np.searchsorted(self.b["sfd_off"], s, side="right")) - 1
            self.x_sfd[s] = torch.from_numpy(_widen(xw[s]))
            for j in range(k):
                e = int(self.idx[t, j])
                on_q = e >= 0 and self.slot_of[e] // L == q
                self.idx_send[s, j] = e if on_q else -1
                self.w_send[s, j] = float(self.w[t, j]) if on_q else 0.0

    # -- destination side ----------------------------------------------------
    def reserve_received(self, n):
        assert n <= self.recv_cap

    def recv_phase(self, n):
        self.n_recv = n
        k, R, L, d = self.k, self.R, self.L, self.d
        idx = self.idx_recv[:n].numpy()
        w = self.w_recv[:n].numpy()
        self.lb = lb = oracle.brim(idx, w, self.slot_of, self.E, R)
        cap = n * min(k, R)
        n_epd = int(lb["epd_off"][self.E])
        o = np.zeros((max(n_epd, 1), d))
        for p in range(n_epd):
            q = int(np.searchsorted(lb["epd_off"], p, side="right")) - 1
            e = int(self.expert_at[q])
            a = self.x_recv[int(lb["epd_sfd"][p])].numpy()
            o[p] = lb["epd_gate"][p] * oracle.expert_row(a, self.wg[e], self.wu[e], self.wd[e])
        for s in range(n):
            acc = np.zeros(d)
            for j in range(L):
                p = int(lb["brim1"][j, s]) if cap else -1
                if p >= 0:
                    acc += o[p]
            self.y_recv[s] = torch.from_numpy(acc)

    # -- source side, after the return exchange ------------------------------
    def combine_phase(self):
        T, d = self.T, self.d
        y = np.zeros((T, d))
        for t in range(T):
            for q in range(self.R):
                s = int(self.b["brim0"][q, t])
                if s >= 0:
                    y[t] += self.y_ret[s].numpy()
        self.y = torch.from_numpy(y)


def _widen(row):
    """bf16 bits (uint16) or float -> float64, exactly."""
    row = np.asarray(row)
    if row.dtype == np.uint16:
        return (row.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return row.astype(np.float64)

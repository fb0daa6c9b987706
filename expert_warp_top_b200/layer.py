"""One Occult-style MoE layer on one GPU: buffers plus the call sequence.

PyTorch only allocates device memory here; every step of the layer runs in
the CUDA library through the binding:

  route (top-k, softmax)        moe_route_topk
  BRIM_0 / BRIM_1 / C_T         moe_brim_build
  ORI -> SFD (-> EPD)           moe_dispatch_gather
  routed experts (grouped GEMM) moe_expert_ffn over the EPD groups

How the experts reach their EPD rows (epd_mode):
  "stored"  the dispatch writes the EPD rows; the GEMM reads them as tiles
  "direct"  one local expert per rank (L = 1): the EPD state is the SFD state
            row for row (same order, same groups), so the GEMM reads the SFD
            payload as it is and no EPD copy exists
  "gather"  the GEMM gathers each EPD row out of the SFD payload (TMA gather4
            by epd_sfd); measured slower on B200 than "stored", kept as an option
  "auto"    "direct" when L = 1, else "stored"
  shared experts                moe_expert_ffn over the ORI rows (one group)
  pre-reduce + combine          moe_combine_scatter
  dispatched-row counter        moe_count_dispatched_rows
  co-activation histogram       moe_coact_histogram (accumulating)

Training: forward_train() (moe_layer_forward_train) keeps the layer's state in
a training workspace and backward() (moe_layer_backward) returns the gradients
of x, of the router logits and of the packed routed and shared weights.
"""
from __future__ import annotations

import torch

from . import _binding as B


class MoELayer:
    def __init__(self, *, T, d, f, E, k, R, renorm=0, dtype=torch.bfloat16, S=0, fs=0,
                 slot_of=None, wg=None, wu=None, wd=None, sg=None, su=None, sd=None,
                 ffn_kind=B.MOE_FFN_SWIGLU, device="cuda", stream=None, epd_mode="auto",
                 prune_m=0):
        if E % R:
            raise ValueError("R must divide E")
        self.T, self.d, self.f, self.E, self.k, self.R = T, d, f, E, k, R
        self.L = E // R
        self.renorm, self.dtype, self.S, self.fs = renorm, dtype, S, fs
        self.ffn_kind = ffn_kind
        self.prune_m = prune_m  # > 0: routing-score-based collaboration pruning
        if epd_mode == "auto":
            epd_mode = "direct" if E // R == 1 else "stored"
        if epd_mode not in ("stored", "direct", "gather"):
            raise ValueError(f"unknown epd_mode {epd_mode!r}")
        if epd_mode == "direct" and E // R != 1:
            raise ValueError("epd_mode='direct' needs one expert per rank (L = 1)")
        if ffn_kind == B.MOE_FFN_IDENTITY and epd_mode == "gather":
            epd_mode = "stored"  # the identity expert works on rows in place
        self.epd_mode = epd_mode
        self.cap = T * min(k, R)
        self.tk = T * k
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        act = dict(dtype=dtype, device=dev)
        if slot_of is None:
            slot_of = torch.arange(E, dtype=torch.int32)
        self.slot_of = slot_of.to(**i32).contiguous()
        # routing and BRIM state
        self.topk_idx = torch.empty(T, k, **i32)
        self.topk_w = torch.empty(T, k, **f32)
        self.brim0 = torch.empty(R, T, **i32)
        self.sfd_token = torch.empty(max(self.cap, 1), **i32)
        self.sfd_off = torch.empty(R + 1, **i32)
        self.brim1 = torch.empty(self.L, max(self.cap, 1), **i32)
        self.epd_off = torch.empty(E + 1, **i32)
        self.epd_sfd = torch.empty(max(self.tk, 1), **i32)
        self.epd_gate = torch.empty(max(self.tk, 1), **f32)
        self.c_t = torch.empty(1, **i32)
        self.brim_ws = torch.empty(max(B.moe_brim_workspace_size(T, E, R),
                                       B.moe_route_brim_workspace_size(T, E, R), 256),
                                   dtype=torch.uint8, device=dev)
        # token states
        self.x_sfd = torch.empty(max(self.cap, 1), d, **act)
        self.x_epd = torch.empty(max(self.tk, 1), d, **act) if epd_mode == "stored" else None
        self.o_epd = torch.empty(max(self.tk, 1), d, **act)
        self.y_sfd = torch.empty(max(self.cap, 1), d, **act)
        self.y = torch.empty(T, d, **act)
        # statistics
        self.per_rank = torch.empty(R, **i32)
        self.total = torch.empty(1, dtype=torch.int64, device=dev)
        self.remote = torch.empty(1, dtype=torch.int64, device=dev)
        self.hist = torch.zeros(E, E, dtype=torch.int32, device=dev)
        # weights (packed once, in slot order)
        code = B.dtype_code(dtype)
        self.w_gu = self.w_dn = None
        if ffn_kind == B.MOE_FFN_SWIGLU:
            self.w_gu = torch.empty(E, 2 * f, d, **act)
            self.w_dn = torch.empty(E, d, f, **act)
            B.moe_prepare_weights(wg.to(**act).contiguous(), wu.to(**act).contiguous(),
                                  wd.to(**act).contiguous(), self.slot_of, self.w_gu, self.w_dn,
                                  stream)
        self.ffn_ws = torch.empty(max(B.moe_expert_ffn_workspace_size(max(self.tk, 1), f, code), 256),
                                  dtype=torch.uint8, device=dev)
        self.shared_out = None
        if S > 0:
            F = S * fs
            self.sw_gu = torch.empty(1, 2 * F, d, **act)
            self.sw_dn = torch.empty(1, d, F, **act)
            B.moe_prepare_shared_weights(sg.to(**act).contiguous(), su.to(**act).contiguous(),
                                         sd.to(**act).contiguous(), self.sw_gu, self.sw_dn, stream)
            self.shared_off = torch.tensor([0, T], **i32)
            self.shared_out = torch.empty(T, d, **act)
            self.shared_ws = torch.empty(max(B.moe_expert_ffn_workspace_size(max(T, 1), F, code), 256),
                                         dtype=torch.uint8, device=dev)

    # -- the steps ---------------------------------------------------------
    def route(self, logits, stream=None):
        B.moe_route_topk(logits, self.k, self.renorm, self.topk_idx, self.topk_w, stream)

    def build_brims(self, stream=None):
        B.moe_brim_build(self.topk_idx, self.topk_w, self.slot_of, self.E, self.R, self.brim0,
                         self.sfd_token, self.sfd_off, self.brim1, self.epd_off, self.epd_sfd,
                         self.epd_gate, self.c_t, self.brim_ws, stream)

    def route_brim(self, logits, stream=None):
        """Routing, BRIMs, counter and histogram in three launches (moe_route_brim)."""
        B.moe_route_brim(logits, self.k, self.renorm, self.slot_of, self.R, self.topk_idx,
                         self.topk_w, self.brim0, self.sfd_token, self.sfd_off, self.brim1,
                         self.epd_off, self.epd_sfd, self.epd_gate, self.c_t, self.brim_ws,
                         per_rank=self.per_rank, total=self.total, remote=self.remote,
                         hist=self.hist, hist_accumulate=1, prune_m=self.prune_m, stream=stream)

    def dispatch(self, x, stream=None):
        B.moe_dispatch_gather(x, self.k, self.R, self.L, self.brim0, self.brim1, self.x_sfd,
                              self.x_epd, stream)

    def experts(self, stream=None):
        m_cap = max(self.tk, 1)
        if self.epd_mode == "stored":
            B.moe_expert_ffn(self.x_epd, self.epd_off, self.w_gu, self.w_dn, self.f,
                             self.epd_gate, self.ffn_kind, self.o_epd, self.ffn_ws, stream)
        elif self.epd_mode == "direct":
            B.moe_expert_ffn(self.x_sfd, self.epd_off, self.w_gu, self.w_dn, self.f,
                             self.epd_gate, self.ffn_kind, self.o_epd, self.ffn_ws, stream,
                             m_cap=m_cap)
        else:
            B.moe_expert_ffn(self.x_sfd, self.epd_off, self.w_gu, self.w_dn, self.f,
                             self.epd_gate, self.ffn_kind, self.o_epd, self.ffn_ws, stream,
                             a_row_index=self.epd_sfd, m_cap=m_cap)

    def shared_experts(self, x, stream=None):
        if self.S > 0:
            B.moe_expert_ffn(x, self.shared_off, self.sw_gu, self.sw_dn, self.S * self.fs, None,
                             B.MOE_FFN_SWIGLU, self.shared_out, self.shared_ws, stream)

    def combine(self, stream=None):
        B.moe_combine_scatter(self.o_epd, self.T, self.k, self.R, self.L, self.brim0, self.brim1,
                              self.shared_out, self.y_sfd, self.y, stream)

    def statistics(self, stream=None):
        B.moe_count_dispatched_rows(self.topk_idx, self.slot_of, self.E, self.R, self.per_rank,
                                    self.total, self.remote, stream)
        B.moe_coact_histogram(self.topk_idx, self.E, self.hist, 1, stream)

    def forward(self, logits, x, stream=None, fused_index=True):
        """All steps of the layer on `stream`; returns y [T, d] (a view of self.y).

        fused_index: routing, BRIMs, counter and histogram through moe_route_brim
        (three launches); otherwise through the four separate entry points."""
        if fused_index:
            self.route_brim(logits, stream)
        else:
            self.route(logits, stream)
            if self.prune_m > 0:
                B.moe_prune_topk(self.topk_idx, self.topk_w, self.slot_of, self.E, self.R,
                                 self.prune_m, stream)
            self.build_brims(stream)
        self.dispatch(x, stream)
        self.experts(stream)
        self.shared_experts(x, stream)
        self.combine(stream)
        if not fused_index:
            self.statistics(stream)
        return self.y

    # -- the whole layer through one C call ---------------------------------
    def _layer_ws(self, host: bool):
        key = "_ws_host" if host else "_ws_dev"
        ws = getattr(self, key, None)
        if ws is None:
            n = B.moe_layer_workspace_size(self.T, self.d, self.f, self.E, self.k, self.R, self.S,
                                           self.fs, B.dtype_code(self.dtype), int(host))
            ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.y.device)
            setattr(self, key, ws)
        return ws

    def forward_fused(self, logits, x, y=None, stream=None):
        """All steps in one moe_layer_forward call (state in a layer workspace)."""
        y = self.y if y is None else y
        B.moe_layer_forward(logits, x, self.k, self.R, self.renorm, self.slot_of, self.w_gu,
                            self.w_dn, self.f, y, self._layer_ws(False),
                            sw_gu=getattr(self, "sw_gu", None), sw_dn=getattr(self, "sw_dn", None),
                            S=self.S, fs=self.fs, c_t=self.c_t, per_rank=self.per_rank,
                            total=self.total, remote=self.remote, hist=self.hist,
                            prune_m=self.prune_m, stream=stream)
        return y

    def forward_host(self, h_logits, h_x, h_y, stream=None, ws=None, asynchronous=False):
        """Host buffers in and out through moe_layer_forward_host (synchronises), or
        moe_layer_forward_host_async (asynchronous=True; pass a workspace per batch in
        flight, from host_workspace())."""
        B.moe_layer_forward_host(h_logits, h_x, self.k, self.R, self.renorm, self.slot_of,
                                 self.w_gu, self.w_dn, self.f, h_y,
                                 self._layer_ws(True) if ws is None else ws,
                                 sw_gu=getattr(self, "sw_gu", None),
                                 sw_dn=getattr(self, "sw_dn", None), S=self.S, fs=self.fs,
                                 prune_m=self.prune_m, stream=stream, asynchronous=asynchronous)
        return h_y

    def host_workspace(self):
        """A fresh workspace for moe_layer_forward_host(_async)."""
        n = B.moe_layer_workspace_size(self.T, self.d, self.f, self.E, self.k, self.R, self.S,
                                       self.fs, B.dtype_code(self.dtype), 1)
        return torch.empty(max(n, 256), dtype=torch.uint8, device=self.y.device)

    # -- training: forward that keeps state, and the backward ----------------
    def _train_ws(self):
        ws = getattr(self, "_ws_train", None)
        if ws is None:
            n = B.moe_layer_train_workspace_size(self.T, self.d, self.f, self.E, self.k, self.R,
                                                 self.S, self.fs)
            if n == 0:
                raise ValueError("this layer shape is not supported for training "
                                 "(bf16, d a multiple of 128, f of 64)")
            ws = torch.empty(n, dtype=torch.uint8, device=self.y.device)
            self._ws_train = ws
        return ws

    def forward_train(self, logits, x, y=None, stream=None):
        """The layer (moe_layer_forward_train), keeping what backward() needs."""
        y = self.y if y is None else y
        self._train_inputs = (logits, x)
        B.moe_layer_forward_train(logits, x, self.k, self.R, self.renorm, self.slot_of, self.w_gu,
                                  self.w_dn, self.f, y, self._train_ws(),
                                  sw_gu=getattr(self, "sw_gu", None),
                                  sw_dn=getattr(self, "sw_dn", None), S=self.S, fs=self.fs,
                                  stream=stream)
        return y

    def backward(self, dy, dw_dtype=torch.float32, grads=None, accumulate=False, stream=None):
        """Gradients of the last forward_train for the upstream gradient dy [T, d].

        Returns a dict: dx [T, d], d_logits [T, E] f32, d_topk_w [T, k] f32 (the
        gate weights' gradient), dw_gu [E, 2f, d] and
        dw_dn [E, d, f] in the packed slot-order layout of w_gu / w_dn (see
        unpack_gate_up), and with shared experts dsw_gu / dsw_dn.  `grads`
        (a dict from an earlier call) is reused, and with accumulate=True the
        weight gradients are added to it."""
        logits, x = self._train_inputs
        dev = self.y.device
        if grads is None:
            wd = dict(dtype=dw_dtype, device=dev)
            grads = dict(dx=torch.empty(self.T, self.d, dtype=self.dtype, device=dev),
                         d_logits=torch.empty(self.T, self.E, dtype=torch.float32, device=dev),
                         d_topk_w=torch.empty(self.T, self.k, dtype=torch.float32, device=dev),
                         dw_gu=torch.empty(self.E, 2 * self.f, self.d, **wd),
                         dw_dn=torch.empty(self.E, self.d, self.f, **wd))
            if self.S > 0:
                F = self.S * self.fs
                grads["dsw_gu"] = torch.empty(1, 2 * F, self.d, **wd)
                grads["dsw_dn"] = torch.empty(1, self.d, F, **wd)
        B.moe_layer_backward(logits, x, self.k, self.R, self.renorm, self.slot_of, self.w_gu,
                             self.w_dn, self.f, dy, grads["dx"], grads["d_logits"],
                             grads["dw_gu"], grads["dw_dn"], self._train_ws(),
                             sw_gu=getattr(self, "sw_gu", None), sw_dn=getattr(self, "sw_dn", None),
                             S=self.S, fs=self.fs, dsw_gu=grads.get("dsw_gu"),
                             dsw_dn=grads.get("dsw_dn"), accumulate=int(accumulate),
                             d_topk_w=grads.get("d_topk_w"), stream=stream)
        return grads


def unpack_gate_up(w_gu: torch.Tensor):
    """Packed [..., 2F, d] gate/up rows (64-row blocks interleaved, as
    moe_prepare_weights writes them and the backward returns their gradients)
    -> (gate [..., F, d], up [..., F, d])."""
    *lead, two_f, d = w_gu.shape
    blocks = w_gu.reshape(*lead, two_f // 128, 2, 64, d)
    gate = blocks[..., 0, :, :].reshape(*lead, two_f // 2, d)
    up = blocks[..., 1, :, :].reshape(*lead, two_f // 2, d)
    return gate, up

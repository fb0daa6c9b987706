"""ctypes binding of libmoe_occult.so -- argument marshalling only.

Every function here has the name of the C entry point it calls and the same
arguments, with torch tensors in place of device pointers.  The binding
checks dtypes, devices, shapes and contiguity, passes raw pointers and the
current CUDA stream, and raises on a non-zero status.  All arithmetic runs in
the CUDA kernels; there is no fallback: without the built library every call
raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libmoe_occult.so"
_lib = None

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_DEVICE_CHECK = -4
MOE_ERR_TIMEOUT = -5
MOE_F32, MOE_BF16 = 0, 1
MOE_FFN_SWIGLU, MOE_FFN_IDENTITY = 0, 1

# every symbol the header declares (checked by the ABI test)
EXPORTS = (
    "moe_abi_version", "moe_last_error", "moe_set_debug", "moe_get_device_status",
    "moe_route_topk", "moe_brim_workspace_size", "moe_brim_build", "moe_brim_build_noalloc",
    "moe_dispatch_gather",
    "moe_prepare_weights", "moe_prepare_shared_weights", "moe_expert_ffn_workspace_size",
    "moe_expert_ffn", "moe_combine_scatter", "moe_count_dispatched_rows", "moe_coact_histogram",
    "moe_layer_workspace_size", "moe_layer_forward", "moe_layer_forward_host",
    "moe_place_greedy", "moe_route_brim_workspace_size", "moe_route_brim", "moe_prune_topk",
    "moe_expert_ffn_train", "moe_expert_ffn_backward_workspace_size", "moe_expert_ffn_backward",
    "moe_route_backward", "moe_layer_train_workspace_size", "moe_layer_forward_train",
    "moe_layer_backward", "moe_interlayer_histogram", "moe_rank_affinity", "moe_predict_home",
    "moe_count_local", "moe_token_shuffle_workspace_size", "moe_token_shuffle",
    "moe_layer_forward_host_async", "moe_ep_pack_routing", "moe_ep_return_rows", "moe_ep_combine",
    "moe_ep_send_peer", "moe_ep_return_peer",
)


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


def lib_path() -> Path:
    return _LIB_PATH


def load():
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not _LIB_PATH.exists():
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m expert_warp_top_b200.build` "
                "(there is no CPU fallback)")
        lib = ctypes.CDLL(str(_LIB_PATH))
        lib.moe_last_error.restype = ctypes.c_char_p
        lib.moe_brim_workspace_size.restype = ctypes.c_size_t
        lib.moe_expert_ffn_workspace_size.restype = ctypes.c_size_t
        lib.moe_layer_workspace_size.restype = ctypes.c_size_t
        lib.moe_route_brim_workspace_size.restype = ctypes.c_size_t
        lib.moe_expert_ffn_backward_workspace_size.restype = ctypes.c_size_t
        lib.moe_layer_train_workspace_size.restype = ctypes.c_size_t
        lib.moe_token_shuffle_workspace_size.restype = ctypes.c_size_t
        lib.moe_set_debug.argtypes = [ctypes.c_int, ctypes.c_double]
        for name in EXPORTS:
            getattr(lib, name)
        _lib = lib
    return _lib


def _check(fn: str, rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(fn, rc, load().moe_last_error().decode(errors="replace"))


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None, dtype=None, name: str = "tensor") -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return MOE_BF16
    if t == torch.float32:
        return MOE_F32
    raise TypeError(f"unsupported activation dtype {t}")


_ACT = (torch.bfloat16, torch.float32)
I32, F32, I64, U32 = torch.int32, torch.float32, torch.int64, torch.uint32


# ---------------------------------------------------------------------------
def moe_abi_version() -> int:
    return int(load().moe_abi_version())


def moe_set_debug(flags: int, wait_limit_ms: float) -> None:
    _check("moe_set_debug", load().moe_set_debug(int(flags), float(wait_limit_ms)))


def moe_get_device_status(stream=None) -> int:
    """Synchronise, read and clear the device error flag; returns the status code."""
    return int(load().moe_get_device_status(_stream(stream)))


def moe_route_topk(logits, k, renorm, topk_idx, topk_w, stream=None):
    T, E = logits.shape
    _check("moe_route_topk", load().moe_route_topk(
        _ptr(logits, F32, "logits"), T, E, int(k), int(renorm),
        _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"), _stream(stream)))


def moe_brim_workspace_size(T, E, R) -> int:
    return int(load().moe_brim_workspace_size(int(T), int(E), int(R)))


def moe_brim_build(topk_idx, topk_w, slot_of, E, R, brim0, sfd_token, sfd_off, brim1, epd_off,
                   epd_sfd, epd_gate, c_t, ws, stream=None):
    T, k = topk_idx.shape
    _check("moe_brim_build", load().moe_brim_build(
        _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"), T, k,
        _ptr(slot_of, I32, "slot_of"), int(E), int(R),
        _ptr(brim0, I32, "brim0"), _ptr(sfd_token, I32, "sfd_token"), _ptr(sfd_off, I32, "sfd_off"),
        _ptr(brim1, I32, "brim1"), _ptr(epd_off, I32, "epd_off"), _ptr(epd_sfd, I32, "epd_sfd"),
        _ptr(epd_gate, F32, "epd_gate"), _ptr(c_t, I32, "c_t"),
        _ptr(ws, None, "ws"), ctypes.c_size_t(ws.numel() * ws.element_size()), _stream(stream)))


def moe_brim_build_noalloc(topk_idx, topk_w, slot_of, E, R, brim0, sfd_token, sfd_off, brim1,
                           epd_off, epd_sfd, epd_gate, c_t, stream=None):
    T, k = topk_idx.shape
    _check("moe_brim_build_noalloc", load().moe_brim_build_noalloc(
        _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"), T, k,
        _ptr(slot_of, I32, "slot_of"), int(E), int(R),
        _ptr(brim0, I32, "brim0"), _ptr(sfd_token, I32, "sfd_token"), _ptr(sfd_off, I32, "sfd_off"),
        _ptr(brim1, I32, "brim1"), _ptr(epd_off, I32, "epd_off"), _ptr(epd_sfd, I32, "epd_sfd"),
        _ptr(epd_gate, F32, "epd_gate"), _ptr(c_t, I32, "c_t"), _stream(stream)))


def moe_route_brim_workspace_size(T, E, R) -> int:
    return int(load().moe_route_brim_workspace_size(int(T), int(E), int(R)))


def moe_prune_topk(topk_idx, topk_w, slot_of, E, R, m, stream=None):
    T, k = topk_idx.shape
    _check("moe_prune_topk", load().moe_prune_topk(
        _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"), T, k,
        _ptr(slot_of, I32, "slot_of"), int(E), int(R), int(m), _stream(stream)))


def moe_route_brim(logits, k, renorm, slot_of, R, topk_idx, topk_w, brim0, sfd_token, sfd_off,
                   brim1, epd_off, epd_sfd, epd_gate, c_t, ws, per_rank=None, total=None,
                   remote=None, hist=None, hist_accumulate=0, prune_m=0, stream=None):
    T, E = logits.shape
    _check("moe_route_brim", load().moe_route_brim(
        _ptr(logits, F32, "logits"), T, E, int(k), int(renorm), _ptr(slot_of, I32, "slot_of"),
        int(R), int(prune_m), _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"),
        _ptr(brim0, I32, "brim0"), _ptr(sfd_token, I32, "sfd_token"), _ptr(sfd_off, I32, "sfd_off"),
        _ptr(brim1, I32, "brim1"), _ptr(epd_off, I32, "epd_off"), _ptr(epd_sfd, I32, "epd_sfd"),
        _ptr(epd_gate, F32, "epd_gate"), _ptr(c_t, I32, "c_t"),
        _ptr(per_rank, I32, "per_rank"), _ptr(total, I64, "total"), _ptr(remote, I64, "remote"),
        _ptr(hist, (U32, torch.int32), "hist"), int(hist_accumulate),
        _ptr(ws, None, "ws"), ctypes.c_size_t(ws.numel() * ws.element_size()), _stream(stream)))


def moe_dispatch_gather(x, k, R, L, brim0, brim1, x_sfd, x_epd, stream=None):
    T, d = x.shape
    _check("moe_dispatch_gather", load().moe_dispatch_gather(
        _ptr(x, _ACT, "x"), T, d, dtype_code(x.dtype), int(k), int(R), int(L),
        _ptr(brim0, I32, "brim0"), _ptr(brim1, I32, "brim1"),
        _ptr(x_sfd, x.dtype, "x_sfd"), _ptr(x_epd, x.dtype, "x_epd"), _stream(stream)))


def moe_prepare_weights(wg, wu, wd, slot_of, w_gu, w_dn, stream=None):
    E, f, d = wg.shape
    _check("moe_prepare_weights", load().moe_prepare_weights(
        _ptr(wg, _ACT, "wg"), _ptr(wu, wg.dtype, "wu"), _ptr(wd, wg.dtype, "wd"), E, d, f,
        dtype_code(wg.dtype), _ptr(slot_of, I32, "slot_of"),
        _ptr(w_gu, wg.dtype, "w_gu"), _ptr(w_dn, wg.dtype, "w_dn"), _stream(stream)))


def moe_prepare_shared_weights(sg, su, sd, w_gu, w_dn, stream=None):
    S, fs, d = sg.shape
    _check("moe_prepare_shared_weights", load().moe_prepare_shared_weights(
        _ptr(sg, _ACT, "sg"), _ptr(su, sg.dtype, "su"), _ptr(sd, sg.dtype, "sd"), S, d, fs,
        dtype_code(sg.dtype), _ptr(w_gu, sg.dtype, "w_gu"), _ptr(w_dn, sg.dtype, "w_dn"),
        _stream(stream)))


def moe_expert_ffn_workspace_size(m_cap, f, dtype_code_) -> int:
    return int(load().moe_expert_ffn_workspace_size(int(m_cap), int(f), int(dtype_code_)))


def moe_expert_ffn(a, group_off, w_gu, w_dn, f, row_scale, ffn_kind, out, ws, stream=None,
                   a_row_index=None, m_cap=None):
    """out = row_scale * FFN_g(rows) per group; rows are a[a_row_index[p]] when a
    row index is given (m_cap = its length), else a[p] (m_cap = rows of a)."""
    a_rows, d = a.shape
    if m_cap is None:
        m_cap = a_row_index.numel() if a_row_index is not None else a_rows
    G = group_off.numel() - 1
    _check("moe_expert_ffn", load().moe_expert_ffn(
        _ptr(a, _ACT, "a"), int(a_rows), _ptr(a_row_index, I32, "a_row_index"),
        _ptr(group_off, I32, "group_off"), G, int(m_cap),
        _ptr(w_gu, a.dtype, "w_gu"), _ptr(w_dn, a.dtype, "w_dn"), d, int(f), dtype_code(a.dtype),
        _ptr(row_scale, F32, "row_scale"), int(ffn_kind), _ptr(out, a.dtype, "out"),
        _ptr(ws, None, "ws"), ctypes.c_size_t(0 if ws is None else ws.numel() * ws.element_size()),
        _stream(stream)))


def moe_combine_scatter(o_epd, T, k, R, L, brim0, brim1, shared_out, y_sfd, y, stream=None):
    d = o_epd.shape[1]
    _check("moe_combine_scatter", load().moe_combine_scatter(
        _ptr(o_epd, _ACT, "o_epd"), int(T), d, dtype_code(o_epd.dtype), int(k), int(R), int(L),
        _ptr(brim0, I32, "brim0"), _ptr(brim1, I32, "brim1"),
        _ptr(shared_out, o_epd.dtype, "shared_out"), _ptr(y_sfd, o_epd.dtype, "y_sfd"),
        _ptr(y, o_epd.dtype, "y"), _stream(stream)))


def moe_ep_pack_routing(topk_idx, topk_w, slot_of, E, R, sfd_token, sfd_off, c_t, idx_send,
                        w_send, stream=None):
    T, k = topk_idx.shape
    _check("moe_ep_pack_routing", load().moe_ep_pack_routing(
        _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"), T, k,
        _ptr(slot_of, I32, "slot_of"), int(E), int(R), _ptr(sfd_token, I32, "sfd_token"),
        _ptr(sfd_off, I32, "sfd_off"), _ptr(c_t, I32, "c_t"), _ptr(idx_send, I32, "idx_send"),
        _ptr(w_send, F32, "w_send"), _stream(stream)))


def moe_ep_return_rows(o_epd, T, k, R, L, brim0, brim1, y_ret, stream=None):
    d = o_epd.shape[1]
    _check("moe_ep_return_rows", load().moe_ep_return_rows(
        _ptr(o_epd, _ACT, "o_epd"), int(T), d, dtype_code(o_epd.dtype), int(k), int(R), int(L),
        _ptr(brim0, I32, "brim0"), _ptr(brim1, I32, "brim1"), _ptr(y_ret, o_epd.dtype, "y_ret"),
        _stream(stream)))


def moe_ep_combine(y_ret, T, k, R, brim0, shared_out, y, stream=None):
    d = y_ret.shape[1]
    _check("moe_ep_combine", load().moe_ep_combine(
        _ptr(y_ret, _ACT, "y_ret"), int(T), d, dtype_code(y_ret.dtype), int(k), int(R),
        _ptr(brim0, I32, "brim0"), _ptr(shared_out, y_ret.dtype, "shared_out"),
        _ptr(y, y_ret.dtype, "y"), _stream(stream)))


MOE_EP_MAX_PEERS = 64


class EpPeers(ctypes.Structure):
    """moe_ep_peers: the buffers of the ranks a mover writes into, by device address."""
    _fields_ = [("rows", ctypes.c_void_p * MOE_EP_MAX_PEERS),
                ("idx", ctypes.c_void_p * MOE_EP_MAX_PEERS),
                ("w", ctypes.c_void_p * MOE_EP_MAX_PEERS),
                ("row0", ctypes.c_int64 * MOE_EP_MAX_PEERS),
                ("seg", ctypes.c_int32 * (MOE_EP_MAX_PEERS + 1))]


def ep_peers(rows, row0, idx=None, w=None, seg=None) -> EpPeers:
    """The table for R ranks: rows[q], idx[q], w[q] device addresses (int), row0[q]
    and seg[0..R] ints (see moe_ep_peers in the header)."""
    R = len(rows)
    if R > MOE_EP_MAX_PEERS or len(row0) != R:
        raise ValueError("one row buffer and one row0 per rank, at most MOE_EP_MAX_PEERS")
    p = EpPeers()
    for q in range(R):
        p.rows[q] = int(rows[q])
        p.row0[q] = int(row0[q])
        if idx is not None:
            p.idx[q] = int(idx[q])
            p.w[q] = int(w[q])
    if seg is not None:
        for q in range(R + 1):
            p.seg[q] = int(seg[q])
    return p


def moe_ep_send_peer(x, topk_idx, topk_w, slot_of, R, L, brim0, brim1, sfd_token, sfd_off, c_t,
                     peers: EpPeers, stream=None):
    T, d = x.shape
    k = topk_idx.shape[1]
    _check("moe_ep_send_peer", load().moe_ep_send_peer(
        _ptr(x, _ACT, "x"), T, d, dtype_code(x.dtype), int(k), int(R), int(L),
        _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"), _ptr(slot_of, I32, "slot_of"),
        _ptr(brim0, I32, "brim0"), _ptr(brim1, I32, "brim1"), _ptr(sfd_token, I32, "sfd_token"),
        _ptr(sfd_off, I32, "sfd_off"), _ptr(c_t, I32, "c_t"), ctypes.byref(peers),
        _stream(stream)))


def moe_ep_return_peer(o_epd, T, k, R, L, brim0, brim1, peers: EpPeers, stream=None):
    d = o_epd.shape[1]
    _check("moe_ep_return_peer", load().moe_ep_return_peer(
        _ptr(o_epd, _ACT, "o_epd"), int(T), d, dtype_code(o_epd.dtype), int(k), int(R), int(L),
        _ptr(brim0, I32, "brim0"), _ptr(brim1, I32, "brim1"), ctypes.byref(peers),
        _stream(stream)))


def moe_count_dispatched_rows(topk_idx, slot_of, E, R, per_rank, total, remote, stream=None):
    T, k = topk_idx.shape
    _check("moe_count_dispatched_rows", load().moe_count_dispatched_rows(
        _ptr(topk_idx, I32, "topk_idx"), T, k, _ptr(slot_of, I32, "slot_of"), int(E), int(R),
        _ptr(per_rank, I32, "per_rank"), _ptr(total, I64, "total"), _ptr(remote, I64, "remote"),
        _stream(stream)))


def moe_coact_histogram(topk_idx, E, hist, accumulate, stream=None):
    T, k = topk_idx.shape
    _check("moe_coact_histogram", load().moe_coact_histogram(
        _ptr(topk_idx, I32, "topk_idx"), T, k, int(E), _ptr(hist, (U32, torch.int32), "hist"),
        int(accumulate), _stream(stream)))


def _host_ptr(t: torch.Tensor, dtype, name: str) -> ctypes.c_void_p:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def moe_layer_workspace_size(T, d, f, E, k, R, S, fs, dtype_code_, host_staging) -> int:
    return int(load().moe_layer_workspace_size(int(T), int(d), int(f), int(E), int(k), int(R),
                                               int(S), int(fs), int(dtype_code_),
                                               int(host_staging)))


def moe_layer_forward(logits, x, k, R, renorm, slot_of, w_gu, w_dn, f, y, ws, sw_gu=None,
                      sw_dn=None, S=0, fs=0, c_t=None, per_rank=None, total=None, remote=None,
                      hist=None, prune_m=0, stream=None):
    T, E = logits.shape
    d = x.shape[1]
    _check("moe_layer_forward", load().moe_layer_forward(
        int(T), int(d), int(f), int(E), int(k), int(R), int(renorm), int(prune_m), int(S), int(fs),
        dtype_code(x.dtype), _ptr(logits, F32, "logits"), _ptr(x, _ACT, "x"),
        _ptr(slot_of, I32, "slot_of"), _ptr(w_gu, x.dtype, "w_gu"), _ptr(w_dn, x.dtype, "w_dn"),
        _ptr(sw_gu, x.dtype, "sw_gu"), _ptr(sw_dn, x.dtype, "sw_dn"), _ptr(y, x.dtype, "y"),
        _ptr(c_t, I32, "c_t"), _ptr(per_rank, I32, "per_rank"), _ptr(total, I64, "total"),
        _ptr(remote, I64, "remote"), _ptr(hist, (U32, torch.int32), "hist"),
        _ptr(ws, None, "ws"), ctypes.c_size_t(ws.numel() * ws.element_size()), _stream(stream)))


def moe_layer_forward_host(h_logits, h_x, k, R, renorm, slot_of, w_gu, w_dn, f, h_y, ws,
                           sw_gu=None, sw_dn=None, S=0, fs=0, prune_m=0, stream=None,
                           asynchronous=False):
    """The layer on host buffers: H2D copies, every step, D2H copy, then synchronise
    (asynchronous=True: moe_layer_forward_host_async, no synchronisation)."""
    T, E = h_logits.shape
    d = h_x.shape[1]
    name = "moe_layer_forward_host_async" if asynchronous else "moe_layer_forward_host"
    _check(name, getattr(load(), name)(
        int(T), int(d), int(f), int(E), int(k), int(R), int(renorm), int(prune_m), int(S), int(fs),
        dtype_code(h_x.dtype), _host_ptr(h_logits, F32, "h_logits"), _host_ptr(h_x, _ACT, "h_x"),
        _ptr(slot_of, I32, "slot_of"), _ptr(w_gu, h_x.dtype, "w_gu"),
        _ptr(w_dn, h_x.dtype, "w_dn"), _ptr(sw_gu, h_x.dtype, "sw_gu"),
        _ptr(sw_dn, h_x.dtype, "sw_dn"), _host_ptr(h_y, h_x.dtype, "h_y"),
        _ptr(ws, None, "ws"), ctypes.c_size_t(ws.numel() * ws.element_size()), _stream(stream)))


# ---------------------------------------------------------------------------
# training
BF16 = torch.bfloat16


def _nbytes(t) -> ctypes.c_size_t:
    return ctypes.c_size_t(0 if t is None else t.numel() * t.element_size())


def moe_expert_ffn_train(a, group_off, w_gu, w_dn, f, row_scale, z, h, out, m_cap=None,
                         stream=None):
    """out = row_scale * FFN_g(a rows); also keeps z (pre-activations) and h."""
    a_rows, d = a.shape
    m_cap = a_rows if m_cap is None else m_cap
    _check("moe_expert_ffn_train", load().moe_expert_ffn_train(
        _ptr(a, BF16, "a"), int(a_rows), _ptr(group_off, I32, "group_off"),
        group_off.numel() - 1, int(m_cap), _ptr(w_gu, BF16, "w_gu"), _ptr(w_dn, BF16, "w_dn"),
        int(d), int(f), _ptr(row_scale, F32, "row_scale"), _ptr(z, BF16, "z"), _ptr(h, BF16, "h"),
        _ptr(out, BF16, "out"), _stream(stream)))


def moe_expert_ffn_backward_workspace_size(m_cap: int, f: int) -> int:
    return int(load().moe_expert_ffn_backward_workspace_size(int(m_cap), int(f)))


def moe_expert_ffn_backward(dout, a, z, group_off, w_gu, w_dn, f, row_scale, dx, d_row_scale,
                            dw_gu, dw_dn, ws, accumulate=0, m_cap=None, stream=None):
    """Gradients of moe_expert_ffn_train: dx, d_row_scale, dw_gu, dw_dn (any may be None
    except dx); the weight gradients' dtype (float32 or bfloat16) is taken from them."""
    a_rows, d = a.shape
    m_cap = a_rows if m_cap is None else m_cap
    dw = dw_gu if dw_gu is not None else dw_dn
    dw_dtype = dtype_code(dw.dtype) if dw is not None else MOE_F32
    _check("moe_expert_ffn_backward", load().moe_expert_ffn_backward(
        _ptr(dout, BF16, "dout"), _ptr(a, BF16, "a"), int(a_rows), _ptr(z, BF16, "z"),
        _ptr(group_off, I32, "group_off"), group_off.numel() - 1, int(m_cap),
        _ptr(w_gu, BF16, "w_gu"), _ptr(w_dn, BF16, "w_dn"), int(d), int(f),
        _ptr(row_scale, F32, "row_scale"), _ptr(dx, BF16, "dx"),
        _ptr(d_row_scale, F32, "d_row_scale"), _ptr(dw_gu, _ACT, "dw_gu"),
        _ptr(dw_dn, _ACT, "dw_dn"), int(dw_dtype), int(accumulate), _ptr(ws, None, "ws"),
        _nbytes(ws), _stream(stream)))


def moe_route_backward(logits, k, renorm, topk_idx, slot_of, R, brim0, brim1, d_gate_epd,
                       d_logits, d_topk_w=None, stream=None):
    T, E = logits.shape
    _check("moe_route_backward", load().moe_route_backward(
        _ptr(logits, F32, "logits"), int(T), int(E), int(k), int(renorm),
        _ptr(topk_idx, I32, "topk_idx"), _ptr(slot_of, I32, "slot_of"), int(R),
        _ptr(brim0, I32, "brim0"), _ptr(brim1, I32, "brim1"), _ptr(d_gate_epd, F32, "d_gate_epd"),
        _ptr(d_logits, F32, "d_logits"), _ptr(d_topk_w, F32, "d_topk_w"), _stream(stream)))


def moe_layer_train_workspace_size(T, d, f, E, k, R, S=0, fs=0) -> int:
    return int(load().moe_layer_train_workspace_size(int(T), int(d), int(f), int(E), int(k),
                                                     int(R), int(S), int(fs)))


def moe_layer_forward_train(logits, x, k, R, renorm, slot_of, w_gu, w_dn, f, y, ws, sw_gu=None,
                            sw_dn=None, S=0, fs=0, stream=None):
    T, E = logits.shape
    d = x.shape[1]
    _check("moe_layer_forward_train", load().moe_layer_forward_train(
        int(T), int(d), int(f), int(E), int(k), int(R), int(renorm), int(S), int(fs),
        _ptr(logits, F32, "logits"), _ptr(x, BF16, "x"), _ptr(slot_of, I32, "slot_of"),
        _ptr(w_gu, BF16, "w_gu"), _ptr(w_dn, BF16, "w_dn"), _ptr(sw_gu, BF16, "sw_gu"),
        _ptr(sw_dn, BF16, "sw_dn"), _ptr(y, BF16, "y"), _ptr(ws, None, "ws"), _nbytes(ws),
        _stream(stream)))


def moe_layer_backward(logits, x, k, R, renorm, slot_of, w_gu, w_dn, f, dy, dx, d_logits,
                       dw_gu, dw_dn, ws, sw_gu=None, sw_dn=None, S=0, fs=0, dsw_gu=None,
                       dsw_dn=None, accumulate=0, d_topk_w=None, stream=None):
    T, E = logits.shape
    d = x.shape[1]
    dw_dtype = dtype_code(dw_gu.dtype if dw_gu is not None else
                          (dw_dn.dtype if dw_dn is not None else torch.float32))
    _check("moe_layer_backward", load().moe_layer_backward(
        int(T), int(d), int(f), int(E), int(k), int(R), int(renorm), int(S), int(fs),
        _ptr(logits, F32, "logits"), _ptr(x, BF16, "x"), _ptr(slot_of, I32, "slot_of"),
        _ptr(w_gu, BF16, "w_gu"), _ptr(w_dn, BF16, "w_dn"), _ptr(sw_gu, BF16, "sw_gu"),
        _ptr(sw_dn, BF16, "sw_dn"), _ptr(dy, BF16, "dy"), _ptr(dx, BF16, "dx"),
        _ptr(d_logits, F32, "d_logits"), _ptr(d_topk_w, F32, "d_topk_w"),
        _ptr(dw_gu, _ACT, "dw_gu"), _ptr(dw_dn, _ACT, "dw_dn"),
        _ptr(dsw_gu, _ACT, "dsw_gu"), _ptr(dsw_dn, _ACT, "dsw_dn"), int(dw_dtype),
        int(accumulate), _ptr(ws, None, "ws"), _nbytes(ws), _stream(stream)))


# ---------------------------------------------------------------------------
# token shuffling across layers
def moe_interlayer_histogram(idx_l, idx_next, E, hist, accumulate=0, stream=None):
    T, k = idx_l.shape
    _check("moe_interlayer_histogram", load().moe_interlayer_histogram(
        _ptr(idx_l, I32, "idx_l"), _ptr(idx_next, I32, "idx_next"), int(T), int(k), int(E),
        _ptr(hist, (U32, torch.int32), "hist"), int(accumulate), _stream(stream)))


def moe_rank_affinity(hist, slot_of_next, R, table, stream=None):
    E = hist.shape[0]
    _check("moe_rank_affinity", load().moe_rank_affinity(
        _ptr(hist, (U32, torch.int32), "hist"), int(E), _ptr(slot_of_next, I32, "slot_of_next"),
        int(R), _ptr(table, (U32, torch.int32), "table"), _stream(stream)))


def moe_predict_home(idx_l, table, home, stream=None):
    T, k = idx_l.shape
    E, R = table.shape
    _check("moe_predict_home", load().moe_predict_home(
        _ptr(idx_l, I32, "idx_l"), int(T), int(k), int(E), _ptr(table, (U32, torch.int32), "table"),
        int(R), _ptr(home, I32, "home"), _stream(stream)))


def moe_count_local(idx, slot_of, E, R, out, home=None, stream=None):
    T, k = idx.shape
    _check("moe_count_local", load().moe_count_local(
        _ptr(idx, I32, "idx"), int(T), int(k), _ptr(slot_of, I32, "slot_of"), int(E), int(R),
        _ptr(home, I32, "home"), _ptr(out, I64, "out"), _stream(stream)))


def moe_token_shuffle_workspace_size(T: int, R: int) -> int:
    return int(load().moe_token_shuffle_workspace_size(int(T), int(R)))


def moe_token_shuffle(home, R, perm, rank_off, ws, x=None, x_out=None, inv=None, stream=None):
    T = home.numel()
    d = x.shape[1] if x is not None else 0
    dt = dtype_code(x.dtype) if x is not None else MOE_BF16
    _check("moe_token_shuffle", load().moe_token_shuffle(
        _ptr(home, I32, "home"), int(T), int(R), _ptr(x, _ACT, "x"), int(d), int(dt),
        _ptr(x_out, _ACT, "x_out"), _ptr(perm, I32, "perm"), _ptr(rank_off, I32, "rank_off"),
        _ptr(inv, I32, "inv"), _ptr(ws, None, "ws"), _nbytes(ws), _stream(stream)))


def moe_place_greedy(hist, R) -> torch.Tensor:
    """Correlated placement (host): hist [E, E] (any integer tensor) -> slot_of int32 [E]."""
    h = hist.detach().to("cpu").to(torch.int64)
    if (h < 0).any() or (h > 0xFFFFFFFF).any():
        raise ValueError("histogram counts must fit in uint32")
    h32 = h.to(torch.int32).contiguous()  # same bits as uint32 for counts < 2^31
    if (h >= 2 ** 31).any():
        raise ValueError("histogram counts must be < 2^31")
    E = h.shape[0]
    slot_of = torch.empty(E, dtype=torch.int32)
    _check("moe_place_greedy", load().moe_place_greedy(
        ctypes.c_void_p(h32.data_ptr()), int(E), int(R), ctypes.c_void_p(slot_of.data_ptr())))
    return slot_of

"""CPU oracle for one Occult-style MoE layer -- TEST INFRASTRUCTURE ONLY.

The arithmetic lives in ``moe_oracle.c`` (plain C, every float in double
precision); this module only compiles it with gcc and marshals numpy arrays
into it.  Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline may import this package.  The product library
(``expert_warp_top_b200``) never imports it, and this package imports nothing
from the product: the two share no code.

Sources are cited in ``moe_oracle.c`` by page title and figure/section.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "moe_oracle.c"
_LIB = _HERE / "libmoe_oracle.so"

DT_F32, DT_BF16, DT_F64 = 0, 1, 2
KIND_SWIGLU, KIND_IDENTITY = 0, 1

_lib = None


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (OpenMP over independent tokens)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-fopenmp", "-fPIC", "-shared",
               str(_SRC), "-o", str(tmp), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(str(_LIB))
        _lib.oracle_expert_row.restype = None
        _lib.oracle_gather_rows.restype = None
        _lib.oracle_coact_histogram.restype = None
        _lib.oracle_set_num_threads.restype = None
        _lib.oracle_interlayer_histogram.restype = None
        _lib.oracle_predict_home.restype = None
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return ctypes.c_void_p(0)
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _dt(a: np.ndarray) -> int:
    """dtype code of an activation/weight array; bf16 travels as uint16 bits."""
    if a.dtype == np.float32:
        return DT_F32
    if a.dtype == np.uint16:
        return DT_BF16
    if a.dtype == np.float64:
        return DT_F64
    raise TypeError(f"unsupported oracle dtype {a.dtype}")


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def route(logits: np.ndarray, k: int, renorm: int):
    """Top-k expert ids (int32 [T,k], descending) and gate weights (f64 [T,k])."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    rc = lib().oracle_route(_p(logits), T, E, k, int(renorm), _p(idx), _p(w))
    if rc != 0:
        raise ValueError(f"oracle_route rejected the arguments ({rc})")
    return idx, w


def brim(idx: np.ndarray, w: np.ndarray, slot_of: np.ndarray, E: int, R: int):
    """BRIM_0, BRIM_1 and their inverses (see moe_oracle.c: oracle_brim)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
    T, k = idx.shape
    L = E // R
    cap = T * min(k, R)
    out = dict(
        brim0=np.empty((R, T), np.int32),
        sfd_token=np.full(max(cap, 1), -7, np.int32),
        sfd_off=np.empty(R + 1, np.int32),
        brim1=np.empty((L, cap), np.int32),
        epd_off=np.empty(E + 1, np.int32),
        epd_sfd=np.empty(T * k, np.int32),
        epd_gate=np.empty(T * k, np.float64),
    )
    c_t = ctypes.c_int32(0)
    rc = lib().oracle_brim(_p(idx), _p(w), T, k, _p(slot_of), E, R,
                           _p(out["brim0"]), _p(out["sfd_token"]), _p(out["sfd_off"]),
                           _p(out["brim1"]), _p(out["epd_off"]), _p(out["epd_sfd"]),
                           _p(out["epd_gate"]), ctypes.byref(c_t))
    if rc != 0:
        raise ValueError(f"oracle_brim rejected the arguments ({rc})")
    out["c_t"] = int(c_t.value)
    out["sfd_token"] = out["sfd_token"][: out["c_t"]]
    return out


def gather_rows(src: np.ndarray, index: np.ndarray) -> np.ndarray:
    """dst[i] = src[index[i]], byte for byte."""
    src = np.ascontiguousarray(src)
    index = np.ascontiguousarray(index, dtype=np.int32)
    dst = np.empty((len(index),) + src.shape[1:], src.dtype)
    row_bytes = src.strides[0] if src.ndim > 1 else src.itemsize
    lib().oracle_gather_rows(_p(src), ctypes.c_size_t(row_bytes), _p(index),
                             int(len(index)), _p(dst))
    return dst


def expert_row(a: np.ndarray, wg, wu, wd, kind: int = KIND_SWIGLU) -> np.ndarray:
    """One expert on one row: o = Wd (silu(Wg a) * (Wu a)), in double."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    d = a.shape[0]
    if kind == KIND_IDENTITY:
        f, wdt = 0, DT_F64
    else:
        wg = np.ascontiguousarray(wg); wu = np.ascontiguousarray(wu)
        wd = np.ascontiguousarray(wd)
        f, wdt = wg.shape[0], _dt(wg)
    o = np.empty(d, np.float64)
    lib().oracle_expert_row(int(kind), _p(a), _p(wg), _p(wu), _p(wd), wdt, d, f, _p(o))
    return o


def dense_layer(x, idx, w, wg, wu, wd, kind=KIND_SWIGLU, shared=None, tokens=None):
    """Y[t] = sum_j w[t,j] FFN_{idx[t,j]}(x[t]) + sum_s FFN_shared_s(x[t]).

    ``shared`` is None or (sg, su, sd) with shapes [S,fs,d], [S,fs,d], [S,d,fs].
    ``tokens`` restricts the output to those token rows (in that order).
    """
    x = np.ascontiguousarray(x)
    T, d = x.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    k = idx.shape[1]
    if kind == KIND_IDENTITY:
        E, f, wdt = int(idx.max()) + 1 if idx.size else 1, 0, DT_F64
        wg = wu = wd = None
    else:
        wg = np.ascontiguousarray(wg); wu = np.ascontiguousarray(wu)
        wd = np.ascontiguousarray(wd)
        E, f, wdt = wg.shape[0], wg.shape[1], _dt(wg)
    if shared is not None:
        sg, su, sd = (np.ascontiguousarray(a) for a in shared)
        S, fs = sg.shape[0], sg.shape[1]
        if kind == KIND_IDENTITY:
            wdt = _dt(sg)
    else:
        sg = su = sd = None
        S, fs = 0, 0
    if tokens is not None:
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        n = len(tokens)
    else:
        n = T
    y = np.empty((n, d), np.float64)
    rc = lib().oracle_dense_layer(_p(x), _dt(x), T, d, _p(idx), _p(w), k,
                                  _p(wg), _p(wu), _p(wd), wdt, E, f, int(kind),
                                  _p(sg), _p(su), _p(sd), S, fs,
                                  _p(tokens), n, _p(y))
    if rc != 0:
        raise ValueError(f"oracle_dense_layer failed ({rc})")
    return y


def occult_layer(x, slot_of, E, R, k, b, wg, wu, wd, kind=KIND_SWIGLU, shared=None):
    """The BRIM-guided layer (dispatch, experts, pre-reduce, combine) in double.

    ``b`` is the dict returned by :func:`brim`.  Returns (Y_sfd, Y).
    """
    x = np.ascontiguousarray(x)
    T, d = x.shape
    slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
    if kind == KIND_IDENTITY:
        f, wdt = 0, DT_F64
        wg = wu = wd = None
    else:
        wg = np.ascontiguousarray(wg); wu = np.ascontiguousarray(wu)
        wd = np.ascontiguousarray(wd)
        f, wdt = wg.shape[1], _dt(wg)
    if shared is not None:
        sg, su, sd = (np.ascontiguousarray(a) for a in shared)
        S, fs = sg.shape[0], sg.shape[1]
        if kind == KIND_IDENTITY:
            wdt = _dt(sg)
    else:
        sg = su = sd = None
        S, fs = 0, 0
    c_t = b["c_t"]
    sfd_token = np.ascontiguousarray(b["sfd_token"], dtype=np.int32)
    y_sfd = np.empty((max(c_t, 1), d), np.float64)
    y = np.empty((T, d), np.float64)
    rc = lib().oracle_occult_layer(
        _p(x), _dt(x), T, d, _p(slot_of), E, R, k,
        _p(b["brim0"]), _p(sfd_token), _p(b["brim1"]), _p(b["epd_off"]),
        _p(b["epd_sfd"]), _p(b["epd_gate"]), c_t,
        _p(wg), _p(wu), _p(wd), wdt, f, int(kind),
        _p(sg), _p(su), _p(sd), S, fs, _p(y_sfd), _p(y))
    if rc != 0:
        raise ValueError(f"oracle_occult_layer failed ({rc})")
    return y_sfd[:c_t], y


def prune(idx, w, slot_of, E, R, m):
    """Routing-score-based collaboration pruning (returns pruned copies)."""
    idx = np.array(idx, dtype=np.int32, order="C", copy=True)
    w = np.array(w, dtype=np.float64, order="C", copy=True)
    slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
    T, k = idx.shape
    rc = lib().oracle_prune(_p(idx), _p(w), T, k, _p(slot_of), E, R, int(m))
    if rc != 0:
        raise ValueError(f"oracle_prune failed ({rc})")
    return idx, w


def count_dispatched(idx, slot_of, E, R):
    """(per_rank int32 [R], total, remote) for one placement."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
    T, k = idx.shape
    per_rank = np.empty(R, np.int32)
    total = ctypes.c_int64(0)
    remote = ctypes.c_int64(0)
    rc = lib().oracle_count_dispatched(_p(idx), T, k, _p(slot_of), E, R, _p(per_rank),
                                       ctypes.byref(total), ctypes.byref(remote))
    if rc != 0:
        raise ValueError(f"oracle_count_dispatched failed ({rc})")
    return per_rank, int(total.value), int(remote.value)


def coact_histogram(idx, E, hist=None):
    """uint32 [E,E] co-selection counts; adds into ``hist`` when given."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    acc = hist is not None
    h = hist if acc else np.empty((E, E), np.uint32)
    lib().oracle_coact_histogram(_p(idx), T, k, E, _p(h), int(acc))
    return h


def place_greedy(hist, R):
    """Correlated placement from a co-activation histogram -> slot_of [E]."""
    hist = np.ascontiguousarray(hist, dtype=np.uint32)
    E = hist.shape[0]
    slot_of = np.empty(E, np.int32)
    rc = lib().oracle_place_greedy(_p(hist), E, R, _p(slot_of))
    if rc != 0:
        raise ValueError(f"oracle_place_greedy failed ({rc})")
    return slot_of


def dense_layer_backward(x, idx, w, wg, wu, wd, dy, kind=KIND_SWIGLU, shared=None,
                         tokens=None, experts=None, shared_grads=False):
    """Backward of :func:`dense_layer` for the upstream gradient ``dy`` [T,d].

    Returns a dict with ``dx`` [n,d], ``dw`` [n,k] (n = len(tokens) or T) and
    ``dw_abs`` [n,k] (the sum of |terms| of each dw: its condition magnitude),
    and, when ``experts`` lists expert ids, ``dwg``/``dwu`` [n_exp,f,d] and
    ``dwd`` [n_exp,d,f]; with ``shared_grads`` the shared experts' ``dsg``,
    ``dsu``, ``dsd``.  Everything in double.
    """
    x = np.ascontiguousarray(x)
    T, d = x.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    k = idx.shape[1]
    if kind == KIND_IDENTITY:
        E, f, wdt = int(idx.max()) + 1 if idx.size else 1, 0, DT_F64
        wg = wu = wd = None
    else:
        wg = np.ascontiguousarray(wg); wu = np.ascontiguousarray(wu)
        wd = np.ascontiguousarray(wd)
        E, f, wdt = wg.shape[0], wg.shape[1], _dt(wg)
    if shared is not None:
        sg, su, sd = (np.ascontiguousarray(a) for a in shared)
        S, fs = sg.shape[0], sg.shape[1]
        if kind == KIND_IDENTITY:
            wdt = _dt(sg)
    else:
        sg = su = sd = None
        S, fs = 0, 0
    if tokens is not None:
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        n = len(tokens)
    else:
        n = T
    out = dict(dx=np.empty((n, d)), dw=np.empty((n, k)), dw_abs=np.empty((n, k)))
    if experts is not None:
        experts = np.ascontiguousarray(experts, dtype=np.int32)
        ne = len(experts)
        out.update(dwg=np.empty((ne, f, d)), dwu=np.empty((ne, f, d)), dwd=np.empty((ne, d, f)))
    else:
        ne = 0
    if shared_grads and S:
        out.update(dsg=np.empty((S, fs, d)), dsu=np.empty((S, fs, d)), dsd=np.empty((S, d, fs)))
    rc = lib().oracle_dense_layer_backward(
        _p(x), _dt(x), T, d, _p(idx), _p(w), k, _p(wg), _p(wu), _p(wd), wdt, E, f, int(kind),
        _p(sg), _p(su), _p(sd), S, fs, _p(dy), _p(tokens), n, _p(out["dx"]), _p(out["dw"]),
        _p(out["dw_abs"]), _p(experts), ne, _p(out.get("dwg")), _p(out.get("dwu")), _p(out.get("dwd")),
        _p(out.get("dsg")), _p(out.get("dsu")), _p(out.get("dsd")))
    if rc != 0:
        raise ValueError(f"oracle_dense_layer_backward failed ({rc})")
    return out


def route_backward(logits, idx, dw, renorm: int):
    """Gradient of the logits [T,E] (double) from the gate-weight gradient dw [T,k]."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    dw = np.ascontiguousarray(dw, dtype=np.float64)
    k = idx.shape[1]
    dl = np.empty((T, E))
    rc = lib().oracle_route_backward(_p(logits), T, E, k, int(renorm), _p(idx), _p(dw), _p(dl))
    if rc != 0:
        raise ValueError(f"oracle_route_backward failed ({rc})")
    return dl


def interlayer_histogram(idx_a, idx_b, E, hist=None):
    """uint32 [E,E]: H[a][b] = #tokens with a in idx_a[t] and b in idx_b[t]."""
    idx_a = np.ascontiguousarray(idx_a, dtype=np.int32)
    idx_b = np.ascontiguousarray(idx_b, dtype=np.int32)
    T, k = idx_a.shape
    acc = hist is not None
    h = hist if acc else np.empty((E, E), np.uint32)
    lib().oracle_interlayer_histogram(_p(idx_a), _p(idx_b), T, k, E, _p(h), int(acc))
    return h


def rank_affinity(hist, slot_of_b, R):
    """uint64 [E,R]: A[a][r] = sum over experts b on rank r of hist[a][b]."""
    hist = np.ascontiguousarray(hist, dtype=np.uint32)
    E = hist.shape[0]
    slot_of_b = np.ascontiguousarray(slot_of_b, dtype=np.int32)
    A = np.empty((E, R), np.uint64)
    rc = lib().oracle_rank_affinity(_p(hist), E, _p(slot_of_b), int(R), _p(A))
    if rc != 0:
        raise ValueError(f"oracle_rank_affinity failed ({rc})")
    return A


def predict_home(idx_a, A):
    """int32 [T]: the rank maximising sum_j A[idx_a[t][j]] (ties -> lower rank)."""
    idx_a = np.ascontiguousarray(idx_a, dtype=np.int32)
    A = np.ascontiguousarray(A, dtype=np.uint64)
    T, k = idx_a.shape
    E, R = A.shape
    home = np.empty(T, np.int32)
    lib().oracle_predict_home(_p(idx_a), T, k, E, _p(A), R, _p(home))
    return home


def count_local(idx, slot_of, E, R, home=None):
    """(assignments on the token's home rank, all assignments)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
    T, k = idx.shape
    if home is not None:
        home = np.ascontiguousarray(home, dtype=np.int32)
    out = np.empty(2, np.int64)
    rc = lib().oracle_count_local(_p(idx), T, k, _p(slot_of), E, int(R), _p(home), _p(out))
    if rc != 0:
        raise ValueError(f"oracle_count_local failed ({rc})")
    return int(out[0]), int(out[1])

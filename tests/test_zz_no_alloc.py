"""moe_brim_build_noalloc: the BRIM build for callers that cannot allocate.

Some callers of this library may not call cudaMalloc: code running inside a
host framework that owns all device memory through its own pool, or code on
a latency-critical path where an allocation could synchronise the device.
They call moe_brim_build_noalloc, which keeps its scratch in a fixed array
inside the library instead of a caller-supplied workspace.

This test calls that entry point directly through the C ABI, twice in a row
on different problems (so the second call runs on scratch the first one
left behind). It checks every output against the workspace-taking
moe_brim_build, bit for bit, since all outputs are integers or copied gate
weights. This file is named to be collected last.
"""
import ctypes

import pytest
import torch

import expert_warp_top_b200 as moe
from expert_warp_top_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(T, E, k, R):
    L, cap = E // R, T * min(k, R)
    i32 = dict(dtype=torch.int32, device=DEV)
    return dict(brim0=torch.full((R, T), -9, **i32), sfd_token=torch.full((cap,), -9, **i32),
                sfd_off=torch.full((R + 1,), -9, **i32), brim1=torch.full((L, cap), -9, **i32),
                epd_off=torch.full((E + 1,), -9, **i32), epd_sfd=torch.full((T * k,), -9, **i32),
                epd_gate=torch.full((T * k,), -9.0, dtype=torch.float32, device=DEV),
                c_t=torch.full((1,), -9, **i32))


def _noalloc_call(lib, idx, w, slot_of, E, R, o):
    T, k = idx.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.moe_brim_build_noalloc(
        _p(idx), _p(w), T, k, _p(slot_of), E, R, _p(o["brim0"]), _p(o["sfd_token"]),
        _p(o["sfd_off"]), _p(o["brim1"]), _p(o["epd_off"]), _p(o["epd_sfd"]),
        _p(o["epd_gate"]), _p(o["c_t"]), stream)


def _reference(idx, w, slot_of, E, R):
    T, k = idx.shape
    o = _outputs(T, E, k, R)
    ws = torch.empty(moe.moe_brim_workspace_size(T, E, R), dtype=torch.uint8, device=DEV)
    moe.moe_brim_build(idx, w, slot_of, E, R, o["brim0"], o["sfd_token"], o["sfd_off"],
                       o["brim1"], o["epd_off"], o["epd_sfd"], o["epd_gate"], o["c_t"], ws)
    return o


def _same(a, b):
    c_t = int(b["c_t"].item())
    assert int(a["c_t"].item()) == c_t
    for key in ("brim0", "sfd_off", "epd_off", "epd_sfd", "epd_gate"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["sfd_token"][:c_t], b["sfd_token"][:c_t])
    assert torch.equal(a["brim1"][:, :c_t], b["brim1"][:, :c_t])


def test_noalloc_brim_build_matches_workspace_version_twice():
    lib = moe.load()
    problems = [
        inputs.LayerConfig("a", T=20000, d=64, f=64, E=64, k=6, R=8, seed=11),
        inputs.LayerConfig("b", T=777, d=64, f=64, E=8, k=2, R=4, seed=12),
    ]
    results = []
    for cfg in problems:  # two calls in a row: the second reuses the first one's scratch
        logits = inputs.make_logits(cfg, device=DEV)
        idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
        w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
        moe.moe_route_topk(logits, cfg.k, 0, idx, w)
        slot_of = torch.randperm(cfg.E, generator=torch.Generator().manual_seed(cfg.seed))
        slot_of = slot_of.to(torch.int32).to(DEV)
        o = _outputs(cfg.T, cfg.E, cfg.k, cfg.R)
        assert _noalloc_call(lib, idx, w, slot_of, cfg.E, cfg.R, o) == moe.MOE_OK, \
            lib.moe_last_error()
        results.append((o, idx, w, slot_of, cfg))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    for o, idx, w, slot_of, cfg in results:
        _same(o, _reference(idx, w, slot_of, cfg.E, cfg.R))
    torch.cuda.synchronize()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = moe.load()
    null = ctypes.c_void_p(0)
    # (ceil(T/32) + 1) * (R + E) > 262144 entries
    T, E, R = 32 * 5000, 64, 8
    rc = lib.moe_brim_build_noalloc(null, null, T, 6, ctypes.c_void_p(8), E, R, null, null,
                                    ctypes.c_void_p(8),
                                    null, ctypes.c_void_p(8), null, null, ctypes.c_void_p(8), null)
    assert rc == moe.MOE_ERR_UNSUPPORTED
    assert b"1 MiB" in lib.moe_last_error()


def test_noalloc_empty_batch_clears_offsets():
    """T = 0: no token is sent, so every offset and C_T is zero (the fixed
    scratch is not touched)."""
    lib = moe.load()
    E, R, k = 64, 8, 6
    i32 = dict(dtype=torch.int32, device=DEV)
    sfd_off = torch.full((R + 1,), -9, **i32)
    epd_off = torch.full((E + 1,), -9, **i32)
    c_t = torch.full((1,), -9, **i32)
    one = torch.zeros(1, **i32)
    onef = torch.zeros(1, dtype=torch.float32, device=DEV)
    slot_of = torch.arange(E, **i32)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.moe_brim_build_noalloc(_p(one), _p(onef), 0, k, _p(slot_of), E, R, _p(one), _p(one),
                                    _p(sfd_off), _p(one), _p(epd_off), _p(one), _p(onef), _p(c_t),
                                    stream)
    assert rc == moe.MOE_OK, lib.moe_last_error()
    torch.cuda.synchronize()
    assert int(sfd_off.abs().sum()) == 0 and int(epd_off.abs().sum()) == 0
    assert int(c_t.item()) == 0


def test_noalloc_at_the_exact_limit_and_one_tile_past_it():
    """The largest batch the fixed scratch holds for E = 64, R = 8:
    (ceil(T/32) + 1) * (R + E) <= 262144 gives T = 116448 (262080 entries).
    It must match the workspace version bit for bit; one 32-token tile more
    (262152 entries) must be refused."""
    lib = moe.load()
    E, R, k = 64, 8, 6
    T = 116448
    assert (-(-T // 32) + 1) * (R + E) <= 1 << 18 < (-(-(T + 32) // 32) + 1) * (R + E)
    cfg = inputs.LayerConfig("limit", T=T, d=64, f=64, E=E, k=k, R=R, seed=13)
    logits = inputs.make_logits(cfg, device=DEV)
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    moe.moe_route_topk(logits, k, 0, idx, w)
    slot_of = torch.randperm(E, generator=torch.Generator().manual_seed(13)).to(torch.int32).to(DEV)
    o = _outputs(T, E, k, R)
    assert _noalloc_call(lib, idx, w, slot_of, E, R, o) == moe.MOE_OK, lib.moe_last_error()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    _same(o, _reference(idx, w, slot_of, E, R))
    null = ctypes.c_void_p(0)
    rc = lib.moe_brim_build_noalloc(null, null, T + 32, k, ctypes.c_void_p(8), E, R, null, null,
                                    ctypes.c_void_p(8), null, ctypes.c_void_p(8), null, null,
                                    ctypes.c_void_p(8), null)
    assert rc == moe.MOE_ERR_UNSUPPORTED

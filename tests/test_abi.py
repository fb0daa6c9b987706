"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import re
from pathlib import Path

import pytest

import expert_warp_top_b200 as moe
from expert_warp_top_b200 import _binding as B

ROOT = Path(__file__).resolve().parents[1]


def header_functions():
    text = (ROOT / "include" / "moe_occult.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(moe_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    lib = moe.load()
    declared = header_functions()
    assert len(declared) >= 14
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(B.EXPORTS)
    assert moe.moe_abi_version() == 1


def test_workspace_queries():
    assert moe.moe_brim_workspace_size(4096, 64, 8) >= 4 * 16 * 72
    assert moe.moe_brim_workspace_size(-1, 64, 8) == 0
    assert moe.moe_expert_ffn_workspace_size(1000, 1024, B.MOE_BF16) >= 1000 * 1024 * 2
    assert moe.moe_expert_ffn_workspace_size(1000, 1024, B.MOE_F32) >= 1000 * 1024 * 4


NULL = ctypes.c_void_p(0)


@pytest.mark.parametrize("T,E,k,renorm,code", [
    (-1, 8, 2, 0, B.MOE_ERR_INVALID_ARG),
    (4, 8, 9, 0, B.MOE_ERR_UNSUPPORTED),      # k > E
    (4, 300, 2, 0, B.MOE_ERR_UNSUPPORTED),    # E > 256
    (4, 64, 17, 0, B.MOE_ERR_UNSUPPORTED),    # k > 16
    (4, 8, 2, 2, B.MOE_ERR_INVALID_ARG),      # renorm not 0/1
    (4, 8, 2, 0, B.MOE_ERR_INVALID_ARG),      # null pointers
])
def test_route_rejects_bad_arguments_on_host(T, E, k, renorm, code):
    lib = moe.load()
    assert lib.moe_route_topk(NULL, T, E, k, renorm, NULL, NULL, NULL) == code
    assert lib.moe_last_error()


def test_route_empty_is_a_no_op():
    assert moe.load().moe_route_topk(NULL, 0, 8, 2, 0, NULL, NULL, NULL) == B.MOE_OK


@pytest.mark.parametrize("E,k,R", [(8, 2, 3), (8, 2, 0), (8, 2, 16)])
def test_brim_rejects_bad_rank_counts(E, k, R):
    lib = moe.load()
    rc = lib.moe_brim_build(NULL, NULL, 16, k, NULL, E, R, NULL, NULL, NULL, NULL, NULL, NULL,
                            NULL, NULL, NULL, ctypes.c_size_t(0), NULL)
    assert rc == B.MOE_ERR_UNSUPPORTED


def test_ffn_rejects_bad_shapes():
    lib = moe.load()

    def ffn(G=1, a_rows=16, ridx=NULL, m_cap=16, d=128, f=128, dtype=B.MOE_BF16,
            kind=B.MOE_FFN_SWIGLU):
        return lib.moe_expert_ffn(NULL, a_rows, ridx, NULL, G, m_cap, NULL, NULL, d, f, dtype,
                                  NULL, kind, NULL, NULL, ctypes.c_size_t(0), NULL)

    assert ffn(d=96) == B.MOE_ERR_UNSUPPORTED            # d not a multiple of 64
    assert ffn(dtype=7) == B.MOE_ERR_INVALID_ARG          # unknown dtype
    assert ffn(kind=5) == B.MOE_ERR_INVALID_ARG           # unknown kind
    assert ffn(G=5000) == B.MOE_ERR_UNSUPPORTED           # too many groups
    assert ffn(a_rows=8, m_cap=16) == B.MOE_ERR_INVALID_ARG  # a too short without a row index
    assert ffn(m_cap=-1) == B.MOE_ERR_INVALID_ARG
    assert ffn() == B.MOE_ERR_INVALID_ARG                 # null pointers


def test_training_entries_reject_bad_arguments_on_host():
    lib = moe.load()

    def bwd(G=1, a_rows=16, m_cap=16, d=128, f=128, dw_dtype=B.MOE_F32, acc=0, rs=NULL,
            drs=NULL):
        return lib.moe_expert_ffn_backward(NULL, NULL, a_rows, NULL, NULL, G, m_cap, NULL, NULL,
                                           d, f, rs, NULL, drs, NULL, NULL, dw_dtype, acc, NULL,
                                           ctypes.c_size_t(0), NULL)

    assert bwd(d=64) == B.MOE_ERR_UNSUPPORTED         # training needs d % 128 == 0
    assert bwd(f=96) == B.MOE_ERR_UNSUPPORTED
    assert bwd(G=0) == B.MOE_ERR_UNSUPPORTED
    assert bwd(a_rows=8) == B.MOE_ERR_INVALID_ARG      # a shorter than m_cap
    assert bwd(dw_dtype=9) == B.MOE_ERR_INVALID_ARG
    assert bwd(acc=2) == B.MOE_ERR_INVALID_ARG
    assert bwd(drs=ctypes.c_void_p(16)) == B.MOE_ERR_INVALID_ARG  # d_row_scale without row_scale
    assert bwd() == B.MOE_ERR_INVALID_ARG              # null pointers
    assert lib.moe_expert_ffn_train(NULL, 16, NULL, 1, 16, NULL, NULL, 64, 128, NULL, NULL, NULL,
                                    NULL, NULL) == B.MOE_ERR_UNSUPPORTED
    assert lib.moe_expert_ffn_train(NULL, 16, NULL, 1, 16, NULL, NULL, 128, 128, NULL, NULL, NULL,
                                    NULL, NULL) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_route_backward(NULL, 16, 8, 2, 3, NULL, NULL, 4, NULL, NULL, NULL, NULL, NULL,
                                  NULL) == B.MOE_ERR_INVALID_ARG   # renorm must be 0 or 1
    assert lib.moe_route_backward(NULL, 16, 8, 2, 0, NULL, NULL, 3, NULL, NULL, NULL, NULL, NULL,
                                  NULL) == B.MOE_ERR_UNSUPPORTED   # R does not divide E
    assert lib.moe_route_backward(NULL, 0, 8, 2, 0, NULL, NULL, 4, NULL, NULL, NULL, NULL, NULL,
                                  NULL) == B.MOE_OK                # empty batch: nothing to do
    assert moe.moe_layer_train_workspace_size(256, 64, 256, 8, 2, 4) == 0  # d % 128 != 0
    assert moe.moe_layer_train_workspace_size(256, 128, 256, 8, 2, 3) == 0  # R does not divide E
    ws = moe.moe_layer_train_workspace_size(256, 128, 256, 8, 2, 4)
    assert ws > 256 * 2 * (2 * 256 + 256) * 2               # holds z and h of every row
    assert moe.moe_expert_ffn_backward_workspace_size(1000, 1024) >= 1000 * 3 * 1024 * 2


def test_movers_reject_bad_shapes():
    lib = moe.load()
    assert lib.moe_dispatch_gather(NULL, 16, 100, B.MOE_BF16, 2, 4, 2, NULL, NULL, NULL, NULL,
                                   NULL) == B.MOE_ERR_UNSUPPORTED
    assert lib.moe_combine_scatter(NULL, 16, 128, B.MOE_BF16, 2, 4, 2, NULL, NULL, NULL, NULL,
                                   NULL, NULL) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_set_debug(0, ctypes.c_double(-1.0)) == B.MOE_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        moe.moe_route_topk(torch.zeros(4, 8), 2, 0, torch.zeros(4, 2, dtype=torch.int32),
                           torch.zeros(4, 2))


def test_place_greedy_matches_oracle():
    """The library's host-side placement against the oracle's, bit for bit."""
    import numpy as np
    import torch
    import oracle
    from expert_warp_top_b200 import inputs
    rng = np.random.default_rng(0)
    for E, R in [(8, 2), (64, 8), (16, 16), (32, 1), (256, 8)]:
        h = rng.integers(0, 50, size=(E, E)).astype(np.uint32)
        h = (h + h.T).astype(np.uint32)
        got = moe.moe_place_greedy(torch.from_numpy(h.astype(np.int64)), R).numpy()
        assert np.array_equal(got, oracle.place_greedy(h, R)), (E, R)
    # ties everywhere: a constant histogram
    h = np.full((16, 16), 7, np.uint32)
    assert np.array_equal(moe.moe_place_greedy(torch.from_numpy(h.astype(np.int64)), 4).numpy(),
                          oracle.place_greedy(h, 4))
    # the planted-group workload
    cfg = inputs.CONFIGS["corr_prefill"].with_(T=4096, seed=1)
    idx, _ = oracle.route(inputs.make_logits(cfg).numpy(), cfg.k, 0)
    h = oracle.coact_histogram(idx, cfg.E)
    assert np.array_equal(moe.moe_place_greedy(torch.from_numpy(h.astype(np.int64)), cfg.R).numpy(),
                          oracle.place_greedy(h, cfg.R))

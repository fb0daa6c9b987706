"""Pins for the oracle's backward pass (no GPU).

The backward is tied to the oracle's forward, which other pins fix, by
central finite differences on small inputs in double precision.  It is also
tied to the closed form of the identity expert.  Any dropped term, wrong sign,
transposed weight or swapped gate/up factor in the derivative fails one of
these tests.
"""
import numpy as np
import pytest

import oracle

H = 1e-6  # central-difference step for double inputs


def _problem(seed, T=5, d=6, f=5, E=4, k=2, S=1, fs=3):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, d))
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 0.9, size=(T, k))
    wg = rng.normal(scale=0.7, size=(E, f, d))
    wu = rng.normal(scale=0.7, size=(E, f, d))
    wd = rng.normal(scale=0.7, size=(E, d, f))
    shared = tuple(rng.normal(scale=0.7, size=s) for s in [(S, fs, d), (S, fs, d), (S, d, fs)])
    dy = rng.normal(size=(T, d))
    return x, idx, w, wg, wu, wd, shared, dy


def _loss(x, idx, w, wg, wu, wd, shared, dy):
    y = oracle.dense_layer(x, idx, w, wg, wu, wd, shared=shared)
    return float(np.sum(y * dy))


def _fd(fun, arr):
    """Central differences of fun() with respect to every entry of arr (in place)."""
    g = np.empty_like(arr)
    flat, gf = arr.reshape(-1), g.reshape(-1)
    for i in range(flat.size):
        v = flat[i]
        flat[i] = v + H
        lp = fun()
        flat[i] = v - H
        lm = fun()
        flat[i] = v
        gf[i] = (lp - lm) / (2 * H)
    return g


def _close(a, b, rtol=1e-6):
    scale = max(np.abs(b).max(), 1e-12)
    assert np.abs(a - b).max() <= rtol * scale, np.abs(a - b).max() / scale


@pytest.mark.parametrize("seed", [0, 1])
def test_layer_backward_equals_finite_differences(seed):
    x, idx, w, wg, wu, wd, shared, dy = _problem(seed)
    E = wg.shape[0]
    got = oracle.dense_layer_backward(x, idx, w, wg, wu, wd, dy, shared=shared,
                                      experts=np.arange(E), shared_grads=True)
    fun = lambda: _loss(x, idx, w, wg, wu, wd, shared, dy)  # noqa: E731
    _close(got["dx"], _fd(fun, x))
    _close(got["dw"], _fd(fun, w))
    assert (got["dw_abs"] >= np.abs(got["dw"]) * (1 - 1e-12)).all()
    assert (got["dw_abs"] > np.abs(got["dw"]) * 1.01).any()  # some terms cancel
    _close(got["dwg"], _fd(fun, wg))
    _close(got["dwu"], _fd(fun, wu))
    _close(got["dwd"], _fd(fun, wd))
    _close(got["dsg"], _fd(fun, shared[0]))
    _close(got["dsu"], _fd(fun, shared[1]))
    _close(got["dsd"], _fd(fun, shared[2]))


def test_expert_subset_and_token_subset_select_rows():
    x, idx, w, wg, wu, wd, shared, dy = _problem(3, T=7)
    full = oracle.dense_layer_backward(x, idx, w, wg, wu, wd, dy, shared=shared,
                                       experts=np.arange(4))
    sub = oracle.dense_layer_backward(x, idx, w, wg, wu, wd, dy, shared=shared,
                                      tokens=[6, 2], experts=[3, 1])
    assert np.array_equal(sub["dx"], full["dx"][[6, 2]])
    assert np.array_equal(sub["dw"], full["dw"][[6, 2]])
    assert np.array_equal(sub["dwg"], full["dwg"][[3, 1]])
    assert np.array_equal(sub["dwd"], full["dwd"][[3, 1]])


def test_unrouted_expert_has_zero_gradient_and_empty_slot_passes_none():
    x, idx, w, wg, wu, wd, shared, dy = _problem(4)
    idx[:, :] = np.where(idx == 3, 0, idx)   # nobody picks expert 3 ...
    idx[:, 1] = np.where(idx[:, 1] == idx[:, 0], 1 + (idx[:, 0] % 2), idx[:, 1])
    idx[2, 1] = -1                            # ... and token 2 has an empty slot
    got = oracle.dense_layer_backward(x, idx, w, wg, wu, wd, dy, experts=[3])
    assert not got["dwg"].any() and not got["dwu"].any() and not got["dwd"].any()
    assert got["dw"][2, 1] == 0.0
    # the token with the empty slot gets the gradient of its one expert only
    one = oracle.dense_layer_backward(x[2:3], idx[2:3, :1], w[2:3, :1], wg, wu, wd, dy[2:3])
    assert np.array_equal(got["dx"][2], one["dx"][0])


def test_identity_expert_closed_form():
    """kind IDENTITY: Y = (sum_j w_j) X, so dX = (sum_j w_j) dY and dw_j = <dY, X>."""
    x, idx, w, _, _, _, _, dy = _problem(5, T=9)
    got = oracle.dense_layer_backward(x, idx, w, None, None, None, dy, kind=oracle.KIND_IDENTITY)
    np.testing.assert_allclose(got["dx"], w.sum(1, keepdims=True) * dy, rtol=1e-14)
    np.testing.assert_allclose(got["dw"], np.repeat((dy * x).sum(1, keepdims=True), 2, 1),
                               rtol=1e-13)
    # the condition magnitude of dw_j: sum over c of |dY_c X_c|
    np.testing.assert_allclose(got["dw_abs"],
                               np.repeat(np.abs(dy * x).sum(1, keepdims=True), 2, 1), rtol=1e-13)


def _route_problem(seed, T=6, E=7):
    """fp32 logits on a 2^-8 grid with gaps of at least 2^-6 inside a row, so
    that a step of 2^-12 is exact in fp32 and never changes the selection."""
    rng = np.random.default_rng(seed)
    rows = []
    for _ in range(T):
        v = rng.permutation(E) * 0.25 + rng.integers(0, 8, size=E) / 256.0 - 1.0
        rows.append(v)
    return np.array(rows, dtype=np.float32)


@pytest.mark.parametrize("renorm", [0, 1])
def test_route_backward_equals_finite_differences(renorm):
    k = 3
    logits = _route_problem(7 + renorm)
    idx, _ = oracle.route(logits, k, renorm)
    dw = np.random.default_rng(2).normal(size=idx.shape)
    got = oracle.route_backward(logits, idx, dw, renorm)
    h = np.float32(2.0 ** -12)

    def loss(lg):
        i2, w2 = oracle.route(lg, k, renorm)
        assert np.array_equal(i2, idx)
        return float(np.sum(w2 * dw))

    fd = np.empty(logits.shape)
    for t in range(logits.shape[0]):
        for e in range(logits.shape[1]):
            lp = logits.copy(); lp[t, e] += h
            lm = logits.copy(); lm[t, e] -= h
            fd[t, e] = (loss(lp) - loss(lm)) / (2 * float(h))
    _close(got, fd, rtol=1e-5)
    if renorm:  # only the selected logits move the renormalised gates
        mask = np.zeros_like(got, dtype=bool)
        np.put_along_axis(mask, idx.astype(np.int64), True, axis=1)
        assert not got[~mask].any()
    # softmax invariance: adding a constant to a row changes nothing
    np.testing.assert_allclose(got.sum(1), 0.0, atol=1e-12)

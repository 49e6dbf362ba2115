"""Pins of the oracle's backward pass of gated block-sparse prefill (CPU).

The analytic gradients of ``oracle.backward.backward`` are checked against
central finite differences of ``oracle.backward.forward_fixed`` (the forward
with the kept lists held fixed, every score recomputed from Q and K), against
torch autograd of dense softmax attention where the sparse path reduces to it,
and against two invariants of softmax gradients."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob

F = oracle


def _problem(seed, B=1, Hq=2, Hkv=1, N=20, d=4, block=4, top_k=2, flags=None, sigma=1.5):
    rng = np.random.default_rng(seed)
    Q = rng.normal(0, sigma, (B, Hq, N, d))
    K = rng.normal(0, sigma, (B, Hkv, N, d))
    V = rng.normal(0, 1, (B, Hkv, N, d))
    dO = rng.normal(0, 1, (B, Hq, N, d))
    flags = (F.SINK | F.LOCAL | F.GATE | F.CAUSAL) if flags is None else flags
    sel = oracle.prefill(Q, K, V, block, top_k, flags, round_mode=oracle.ROUND_NONE, threads=1)
    lists = ob.lists_from_selection(sel)
    return Q, K, V, dO, flags, lists


def _loss(Q, K, V, dO, block, flags, lists, **kw):
    O, _ = ob.forward_fixed(Q, K, V, block, flags, lists, **kw)
    return float((O * dO).sum())


def _fd(fun, X, h=1e-6):
    g = np.zeros_like(X)
    it = np.nditer(X, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        x0 = X[i]
        X[i] = x0 + h
        fp = fun()
        X[i] = x0 - h
        fm = fun()
        X[i] = x0
        g[i] = (fp - fm) / (2 * h)
    return g


def _close(a, b, tol=1e-6):
    scale = max(1.0, np.abs(b).max())
    assert np.abs(a - b).max() <= tol * scale, (np.abs(a - b).max(), scale)


@pytest.mark.parametrize("seed,kw", [
    (0, {}),
    (1, dict(N=23, block=4, top_k=3)),             # ragged last block
    (2, dict(Hq=4, Hkv=2, N=16, block=4, top_k=1)),
    (3, dict(B=2, N=12, block=4, top_k=2)),
])
def test_gradients_match_finite_differences(seed, kw):
    block = kw.get("block", 4)
    Q, K, V, dO, flags, lists = _problem(seed, **kw)
    g = ob.backward(Q, K, V, dO, block, flags, lists)
    f = lambda: _loss(Q, K, V, dO, block, flags, lists)
    _close(g["dQ"], _fd(f, Q))
    _close(g["dK"], _fd(f, K))
    _close(g["dV"], _fd(f, V))


def test_score_gradient_matches_finite_differences():
    block = 4
    Q, K, V, dO, flags, lists = _problem(4, N=24, top_k=3)
    # scores as free inputs: the recomputed ones, perturbed one entry at a time
    g0 = ob.backward(Q, K, V, dO, block, flags, lists, selector=False)
    base = {}
    for u, idx in lists.items():
        b, gg, j = u
        rows, _, qbar, L, _ = ob._unit_pieces(np.asarray(Q, float), np.asarray(K, float), b, gg, j, block, 2)
        base[u] = (1 / np.sqrt(Q.shape[3])) * (L[idx] @ qbar)
    g = ob.backward(Q, K, V, dO, block, flags, lists, score_override=base)
    checked = 0
    for u, sc in base.items():
        sc = np.array(sc)
        def f():
            over = dict(base)
            over[u] = sc
            return _loss(Q, K, V, dO, block, flags, lists, score_override=over)
        fd = _fd(f, sc)
        _close(g["dscore"][u], fd)
        checked += int(np.abs(fd).max() > 1e-8)
        # the attention-only gradients do not depend on how the scores were given
        np.testing.assert_allclose(g["dscore"][u], g0["dscore"][u], rtol=1e-10, atol=1e-12)
    assert checked > 0


def test_dense_case_matches_torch_autograd():
    """All blocks kept, no causal mask, no gate: plain softmax attention."""
    rng = np.random.default_rng(7)
    B, Hq, Hkv, N, d, block = 1, 2, 2, 16, 8, 4
    Q, K, V, dO = (rng.normal(0, 1, s) for s in ((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d), (B, Hq, N, d)))
    nb = N // block
    lists = {(0, g, j): np.arange(nb) for g in range(Hkv) for j in range(nb)}
    g = ob.backward(Q, K, V, dO, block, 0, lists, selector=False)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    P = torch.softmax(tq @ tk.transpose(-1, -2) / np.sqrt(d), dim=-1)
    (P @ tv * torch.tensor(dO)).sum().backward()
    np.testing.assert_allclose(g["dQ"], tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dK"], tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dV"], tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_softmax_gradient_invariants():
    block = 4
    Q, K, V, dO, flags, lists = _problem(5, N=28, top_k=3)
    g = ob.backward(Q, K, V, dO, block, flags, lists, selector=False)
    # each row's dZ sums to zero, so the gate gradients of a unit do too
    for u, dg in g["dgate"].items():
        assert abs(dg.sum()) <= 1e-10 * max(1.0, np.abs(dg).max())
    # sum over keys of dV = sum of dO over the rows (every row sees its own key)
    np.testing.assert_allclose(g["dV"].sum(axis=2)[:, 0], dO.sum(axis=2).reshape(1, 2, -1).sum(axis=1),
                               rtol=1e-10, atol=1e-10)
    # the local block's score gradient balances the gated entries' ones
    for u, ds in g["dscore"].items():
        assert abs(ds.sum()) <= 1e-10 * max(1.0, np.abs(ds).max())

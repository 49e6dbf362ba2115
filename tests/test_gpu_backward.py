"""Backward of the gated block-sparse prefill through the C ABI, against the
oracle's fp64 backward (``oracle.backward``, pinned by finite differences in
test_oracle_backward.py) on the oracle's own lists and landmarks.

Tolerances: D = rowsum(dO * O) uses the forward's O rounded to the input
dtype (2^-9 relative in bf16), and the tensor-core path (bf16, d = 128)
rounds P and dS to bf16 before its products (2^-9 relative per term, summed
in fp32); gradients are checked to 1.5e-2 of their largest magnitude in bf16
(fp32 inputs, on the CUDA cores: 2e-3)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
import oracle
from oracle import backward as ob
from block_sparse_long_landmark_b200 import inputs
from _util import f64, oracle_sel_tensors, round_mode

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS
TOL = {"bf16": 1.5e-2, "fp32": 2e-3}

CASES = {
    "gated_b64_g4": W["gated_prefill_32k"].scaled(N=512, Hq=8, Hkv=2, top_k=3),
    "gated_b64_ragged": W["gated_prefill_32k"].scaled(N=300, Hq=4, Hkv=2, top_k=2),
    "gated_b128": W["long_prefill_256k"].scaled(N=640, Hq=4, Hkv=2, top_k=2),
    "gated_fp32_d64": W["gated_prefill_32k"].scaled(N=256, Hq=4, Hkv=2, d=64, dtype="fp32", top_k=3, sigma=1.0),
    "gated_batch2": W["gated_prefill_32k"].scaled(B=2, N=256, Hq=4, Hkv=1, top_k=2),
    # 128 tiles per kv-head: the sink tile is kept by more than 64 units, so its
    # dK, dV come from two work items summed in order
    "gated_b64_split": W["gated_prefill_32k"].scaled(N=8192, Hq=8, Hkv=2, top_k=8, n_plants=4),
}


def _close(got, ref, tol, what):
    scale = max(np.abs(ref).max(), 1e-6)
    err = np.abs(got - ref).max()
    assert err <= tol * scale, f"{what}: max err {err:.3g} vs {tol} x {scale:.3g}"


def _run(wl, flags=None):
    flags = wl.flags if flags is None else flags
    p = sa.params_for(wl)
    p.flags = flags
    Q, K, V = inputs.make_prefill(wl, device="cuda")
    ref = oracle.prefill(f64(Q), f64(K), f64(V), wl.block, wl.top_k, flags, round_mode=round_mode(wl.dtype))
    sel = oracle_sel_tensors(ref)
    ws = sa.workspace(p)
    L = sa.landmarks(p, K)
    O, lse = sa.prefill(p, Q, K, V, *sel, ws)
    g = torch.Generator().manual_seed(11)
    dO = torch.randn(Q.shape, generator=g, dtype=torch.float32).to(device="cuda", dtype=Q.dtype)
    dQ, dK, dV, dscore = sa.prefill_backward(p, Q, K, V, O, lse, dO, *sel, ws)
    attn_only = dQ.clone(), dK.clone()
    sa.select_backward(p, Q, L, sel[0], dscore, sel[2], dQ, dK, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    lists = ob.lists_from_selection(ref)
    want = ob.backward(f64(Q), f64(K), f64(V), f64(dO), wl.block, flags, lists, L=ref["L"])
    want_attn = ob.backward(f64(Q), f64(K), f64(V), f64(dO), wl.block, flags, lists, L=ref["L"], selector=False)
    return dict(dQ=dQ, dK=dK, dV=dV, dscore=dscore, attn=attn_only), want, want_attn, ref


@pytest.mark.parametrize("case", sorted(CASES))
def test_backward_matches_oracle(case):
    wl = CASES[case]
    tol = TOL[wl.dtype]
    got, want, want_attn, ref = _run(wl)
    _close(f64(got["dV"]), want["dV"], tol, "dV")
    _close(f64(got["attn"][0]), want_attn["dQ"], tol, "dQ (attention)")
    _close(f64(got["attn"][1]), want_attn["dK"], tol, "dK (attention)")
    _close(f64(got["dQ"]), want["dQ"], tol, "dQ (with selector)")
    _close(f64(got["dK"]), want["dK"], tol, "dK (with selector)")
    ds = f64(got["dscore"])
    cnt = ref["count"]
    allref = np.concatenate([v for v in want["dscore"].values()])
    scale = max(np.abs(allref).max(), 1e-6)
    for (b, g, j), v in want["dscore"].items():
        c = int(cnt[b, g, j])
        assert np.abs(ds[b, g, j, :c] - v).max() <= tol * scale, (b, g, j)
        assert np.all(ds[b, g, j, c:] == 0)
    # the gate gradients move the scores: something must be non-zero
    assert scale > 1e-6


def test_plain_mode_has_no_score_gradient():
    wl = CASES["gated_b64_g4"]
    flags = wl.flags & ~sa.SA_GATE
    got, want, _, _ = _run(wl, flags)
    assert torch.count_nonzero(got["dscore"]).item() == 0
    _close(f64(got["dQ"]), want["dQ"], TOL[wl.dtype], "dQ")
    _close(f64(got["dK"]), want["dK"], TOL[wl.dtype], "dK")
    _close(f64(got["dV"]), want["dV"], TOL[wl.dtype], "dV")


def _grads(wl, monkeypatch=None, path=None):
    if monkeypatch is not None:
        if path:
            monkeypatch.setenv("SPARSE_ATTN_BACKWARD_PATH", path)
        else:
            monkeypatch.delenv("SPARSE_ATTN_BACKWARD_PATH", raising=False)
    p = sa.params_for(wl)
    Q, K, V = inputs.make_prefill(wl, device="cuda")
    ws = sa.workspace(p)
    L = sa.landmarks(p, K)
    sel = sa.select(p, Q, L, ws)
    O, lse = sa.prefill(p, Q, K, V, *sel, ws)
    g = torch.Generator(device="cuda").manual_seed(5)
    dO = torch.randn(Q.shape, generator=g, device="cuda").to(Q.dtype)
    out = sa.prefill_backward(p, Q, K, V, O, lse, dO, *sel, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    return [t.clone() for t in out]


def test_backward_is_deterministic():
    """No atomics on the tensor-core path: two runs agree bit for bit."""
    wl = CASES["gated_b64_split"]
    a = _grads(wl)
    b = _grads(wl)
    for x, y, what in zip(a, b, ("dQ", "dK", "dV", "dscore")):
        assert torch.equal(x, y), what


@pytest.mark.parametrize("case", ["gated_b64_g4", "gated_b128", "gated_b64_split"])
def test_tensor_core_backward_matches_cuda_core(case, monkeypatch):
    wl = CASES[case]
    tc = _grads(wl, monkeypatch, None)
    cc = _grads(wl, monkeypatch, "simt")
    for x, y, what in zip(tc, cc, ("dQ", "dK", "dV", "dscore")):
        scale = max(y.abs().max().item(), 1e-6)
        assert (x - y).abs().max().item() <= TOL["bf16"] * scale, what

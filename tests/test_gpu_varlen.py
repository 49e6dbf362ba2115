"""Ragged decode batches and incremental landmarks, through the C ABI:
sequence b holds seq_len[b] keys of a cache allocated for N, and landmarks
are refreshed only for the blocks an append touched.  Checked against the
CPU oracle run on each sequence's own keys."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
import oracle
from block_sparse_long_landmark_b200 import inputs
from _util import GAP, LSE_TOL, O_TOL, f64, round_mode

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS

CASES = {
    "gated_bf16": W["gated_decode_128k"].scaled(B=6, N=8192, n_plants=8),
    "hier_bf16": W["hils_decode_1m"].scaled(B=5, N=6000, top_k=12, n_plants=8),
    "gated_fp32_d64": W["gated_decode_128k"].scaled(B=4, N=3000, d=64, dtype="fp32", Hq=8, Hkv=4, top_k=6,
                                                    n_plants=3, sigma=1.0),
}


def _lengths(wl, seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(wl.block + 1, wl.N + 1, size=wl.B)
    lens[0] = wl.N            # full
    lens[-1] = wl.block * 3 + 1   # a one-key local block
    return lens


def _run(wl, lens):
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = sa.workspace(p)
    L = torch.zeros(wl.B, wl.Hkv, wl.nb, wl.d, dtype=K.dtype, device="cuda")
    sa.landmarks_update(p, K, L, seq_len=sl)
    sel = sa.select_decode_varlen(p, q, L, sl, ws)
    o, lse = sa.decode_varlen(p, q, K, V, sl, *sel, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    return q, K, V, L, sel, o, lse


@pytest.mark.parametrize("case", sorted(CASES))
def test_varlen_decode_matches_oracle_per_sequence(case):
    wl = CASES[case]
    lens = _lengths(wl, 3)
    q, K, V, L, (idx, sc, cnt), o, lse = _run(wl, lens)
    gi, gs, gc = idx.cpu().numpy(), sc.cpu().numpy(), cnt.cpu().numpy()
    G = wl.Hq // wl.Hkv
    exact = checked = 0
    for b, n in enumerate(lens):
        ref = oracle.decode(f64(q[b:b + 1]), f64(K[b:b + 1, :, :n]), f64(V[b:b + 1, :, :n]), wl.block, wl.top_k,
                            wl.flags, round_mode=round_mode(wl.dtype))
        nbb = (n + wl.block - 1) // wl.block
        Lb = f64(L[b, :, :nbb])
        assert np.all(np.abs(Lb - ref["L"][0]) <= np.maximum(np.abs(ref["L"][0]), 1e-30) * 2.0 ** -7 + 1e-6)
        for g in range(wl.Hkv):
            checked += 1
            c = int(ref["count"][0, g])
            assert gc[b, g] == c
            if not np.array_equal(gi[b, g, :c], ref["idx"][0, g, :c]):
                assert ref["rel_gap"][0, g] <= GAP
                continue
            exact += 1
            assert np.all(np.abs(gs[b, g, :c] - ref["sc"][0, g, :c]) <= 1e-5 + 1e-4 * np.abs(ref["sc"][0, g, :c]))
            hs = slice(g * G, (g + 1) * G)
            assert np.abs(f64(o[b, hs]) - ref["O"][0, hs]).max() <= O_TOL[wl.dtype]
            assert np.abs(f64(lse[b, hs]) - ref["LSE"][0, hs]).max() <= LSE_TOL
    assert exact >= 0.9 * checked


def test_full_lengths_give_the_plain_path_bit_for_bit():
    wl = CASES["gated_bf16"]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    ws = sa.workspace(p)
    L = sa.landmarks(p, K)
    sel = sa.select_decode(p, q, L, ws)
    o, lse = sa.decode(p, q, K, V, *sel, ws)
    sl = torch.full((wl.B,), wl.N, dtype=torch.int32, device="cuda")
    L2 = torch.zeros_like(L)
    sa.landmarks_update(p, K, L2, seq_len=sl)
    sel2 = sa.select_decode_varlen(p, q, L2, sl, ws)
    o2, lse2 = sa.decode_varlen(p, q, K, V, sl, *sel2, ws)
    torch.cuda.synchronize()
    assert torch.equal(L, L2)
    for x, y in zip(sel, sel2):
        assert torch.equal(x, y)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_landmarks_update_refreshes_only_the_appended_blocks():
    wl = W["gated_decode_128k"].scaled(B=3, N=4096)
    p = sa.params_for(wl)
    _, K, _ = inputs.make_decode(wl, device="cuda")
    n0 = torch.tensor([1000, 64, 4000], dtype=torch.int32, device="cuda")
    n1 = torch.tensor([1500, 700, 4096], dtype=torch.int32, device="cuda")
    L = torch.zeros(wl.B, wl.Hkv, wl.nb, wl.d, dtype=K.dtype, device="cuda")
    sa.landmarks_update(p, K, L, seq_len=n0)
    fb = (n0 // wl.block).to(torch.int32)
    sentinel = L.clone()
    for b in range(wl.B):
        sentinel[b, :, :int(fb[b])] = 7.0          # blocks that must stay untouched
    L_upd = sentinel.clone()
    sa.landmarks_update(p, K, L_upd, seq_len=n1, first_block=fb)
    L_ref = torch.zeros_like(L)
    sa.landmarks_update(p, K, L_ref, seq_len=n1)
    torch.cuda.synchronize()
    for b in range(wl.B):
        f, e = int(fb[b]), (int(n1[b]) + wl.block - 1) // wl.block
        assert torch.all(L_upd[b, :, :f] == 7.0)
        assert torch.equal(L_upd[b, :, f:e], L_ref[b, :, f:e])
    # the refreshed partial block averages only the keys that exist
    kb = f64(K[0, 0, 1472:1500])
    assert np.allclose(f64(L_upd[0, 0, 1500 // 64]), kb.mean(axis=0), atol=2e-2)

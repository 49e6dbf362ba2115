"""Decode selection: the warp-per-chunk kernel (select_decode.cu) against the
CTA-per-chunk kernel (select.cu, forced with SPARSE_ATTN_SELECT_PATH=chunked)
and against the oracle.  Both kernels score in fp32 with the same operation
order, so the kept lists, counts and scores must be identical; the oracle
check uses the shared tolerance rules (exact lists wherever the K-th gap
exceeds 1e-3)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
import oracle
from block_sparse_long_landmark_b200 import inputs
from _util import compare_lists, f64, round_mode

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS
CASES = {
    # one CTA per unit (4 warp chunks)
    "gated_64k": (W["gated_decode_128k"].scaled(B=4, N=65536), None),
    # two CTAs per unit: cross-CTA merge, hierarchical flags
    "hier_256k": (W["hils_decode_1m"].scaled(B=2, N=262144, n_plants=32), None),
    # ragged lengths, some below one chunk
    "varlen": (W["gated_decode_128k"].scaled(B=6, N=40000), [40000, 17, 300, 9000, 25000, 16385]),
    # one list per query head
    "perqhead": (W["gated_decode_128k_perqhead"].scaled(B=2, N=32768), None),
    # fp32 with d = 64 (8 lanes per landmark row), block 32
    "fp32_d64": (W["gated_decode_128k"].scaled(B=2, N=20000, d=64, dtype="fp32", block=32, top_k=40,
                                                sigma=1.0), None),
    # bf16, d = 64, top-K above a chunk's warp slots (k = 200)
    "bf16_d64_k200": (W["gated_decode_128k"].scaled(B=1, N=131072, d=64, top_k=200), None),
}


def _run(wl, lens, monkeypatch, chunked):
    if chunked:
        monkeypatch.setenv("SPARSE_ATTN_SELECT_PATH", "chunked")
    else:
        monkeypatch.delenv("SPARSE_ATTN_SELECT_PATH", raising=False)
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    ws = sa.workspace(p)
    if lens is None:
        L = sa.landmarks(p, K)
        sel = sa.select_decode(p, q, L, ws)
    else:
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        L = torch.zeros(wl.B, wl.Hkv, wl.nb, wl.d, dtype=K.dtype, device="cuda")
        sa.landmarks_update(p, K, L, seq_len=sl)
        sel = sa.select_decode_varlen(p, q, L, sl, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    return q, K, sel


@pytest.mark.parametrize("case", sorted(CASES))
def test_warp_selection_equals_chunked_selection(case, monkeypatch):
    wl, lens = CASES[case]
    _, _, new = _run(wl, lens, monkeypatch, False)
    _, _, old = _run(wl, lens, monkeypatch, True)
    for a, b, what in zip(new, old, ("idx", "score", "count")):
        assert torch.equal(a, b), what


def test_warp_selection_matches_oracle(monkeypatch):
    wl, _ = CASES["hier_256k"]
    q, K, sel = _run(wl, None, monkeypatch, False)
    K0 = f64(K[:1])                     # sequence 0 only (the value cache is not needed for the lists)
    ref = oracle.decode(f64(q[:1]), K0, K0, wl.block, wl.top_k, wl.flags, round_mode=round_mode(wl.dtype),
                        units=[(0, g) for g in range(wl.Hkv)])
    units = [(0, g) for g in range(wl.Hkv)]
    n, exact, _ = compare_lists(ref, *sel, units=units)
    assert exact >= n - 1

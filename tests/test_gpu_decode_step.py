"""sparse_attn_decode_step: the selection and the decode of one step in one
call, with the decode's work for each (batch, selection head) starting as
soon as the selection publishes that list.  The step must give exactly what
the two separate calls give (same kernels, same arithmetic), on full and
ragged batches, for steps repeated on one workspace, and on shapes whose
kernels do not overlap; one case is checked against the oracle as well."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
import oracle
from block_sparse_long_landmark_b200 import inputs
from _util import LSE_TOL, O_TOL, compare_lists, f64, round_mode

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS

CASES = {
    # bf16, d 128, block 64: the overlapped path
    "gated_8k": W["gated_decode_128k"].scaled(B=4, N=8192),
    "gated_wide": W["gated_decode_128k"].scaled(B=64, N=4096),
    "gated_big_k": W["gated_decode_128k"].scaled(B=2, N=65536, top_k=200, n_plants=16),
    "hier_16k": W["hils_decode_1m"].scaled(B=2, N=16384, top_k=16, n_plants=16),
    # several selection CTAs per unit (the unit's last CTA merges, then publishes)
    "hier_long": W["hils_decode_1m"].scaled(B=2, N=262144, top_k=64, n_plants=16),
    "per_qhead": W["gated_decode_128k"].scaled(B=2, N=8192, per_qhead=True),
    # no overlap: the CUDA-core decode
    "fp32_d64": W["gated_decode_128k"].scaled(B=2, N=4096, d=64, dtype="fp32", Hq=8, Hkv=8, top_k=6,
                                              n_plants=3, sigma=1.0),
}


def _separate(p, q, L, K, V, seq_len=None):
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    if seq_len is None:
        sel = sa.select_decode(p, q, L, ws)
        o, lse = sa.decode(p, q, K, V, *sel, ws)
    else:
        sel = sa.select_decode_varlen(p, q, L, seq_len, ws)
        o, lse = sa.decode_varlen(p, q, K, V, seq_len, *sel, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    return sel, o, lse


def _same(a, b):
    (s1, o1, l1), (s2, o2, l2) = a, b
    for x, y in zip(s1, s2):
        assert torch.equal(x, y)
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)


@pytest.mark.parametrize("case", sorted(CASES))
def test_step_equals_the_two_calls(case):
    wl = CASES[case]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    L = sa.landmarks(p, K)
    ref = _separate(p, q, L, K, V)
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    sel, (o, lse) = sa.decode_step(p, q, L, K, V, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    _same(ref, (sel, o, lse))


@pytest.mark.parametrize("case", ["gated_wide", "hier_long"])
def test_steps_repeated_on_one_workspace(case):
    """Each step publishes its lists under a new number, so a later step never
    reads an earlier step's lists: alternate two queries over one workspace."""
    wl = CASES[case]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    q2 = inputs.make_decode(wl.scaled(seed=wl.seed + 3), device="cuda")[0]
    L = sa.landmarks(p, K)
    refs = [_separate(p, q, L, K, V), _separate(p, q2, L, K, V)]
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    for step in range(5):
        qs = q if step % 2 == 0 else q2
        sel, (o, lse) = sa.decode_step(p, qs, L, K, V, ws)
        torch.cuda.synchronize()
        assert sa.check_status(ws) == 0
        _same(refs[step % 2], (sel, o, lse))


def test_step_on_a_ragged_batch():
    wl = W["hils_decode_1m"].scaled(B=5, N=40000, top_k=12, n_plants=8)
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    lens = np.random.default_rng(4).integers(wl.block + 1, wl.N + 1, size=wl.B)
    lens[0] = wl.N
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    L = torch.zeros(wl.B, wl.Hkv, wl.nb, wl.d, dtype=K.dtype, device="cuda")
    sa.landmarks_update(p, K, L, seq_len=sl)
    ref = _separate(p, q, L, K, V, seq_len=sl)
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    sel, (o, lse) = sa.decode_step(p, q, L, K, V, ws, seq_len=sl)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    _same(ref, (sel, o, lse))


def test_step_matches_the_oracle():
    wl = CASES["gated_8k"]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    L = sa.landmarks(p, K)
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    (idx, sc, cnt), (o, lse) = sa.decode_step(p, q, L, K, V, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    ref = oracle.decode(f64(q), f64(K), f64(V), wl.block, wl.top_k, wl.flags, round_mode=round_mode(wl.dtype))
    n, exact, mask = compare_lists(ref, idx, sc, cnt)
    assert exact >= 0.5 * n
    rows = np.repeat(mask, wl.Hq // wl.Hkv, axis=1)      # units whose lists agree
    Og, lg, Or, lr = f64(o)[rows], f64(lse)[rows], ref["O"][rows], ref["LSE"][rows]
    assert np.abs(Og - Or).max() <= O_TOL[wl.dtype]
    assert np.abs(lg - lr).max() <= LSE_TOL

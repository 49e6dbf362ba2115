"""Full-size parity: the benchmark workloads at their real sizes, in the
launch configuration the benchmark times, checked against the CPU oracle on
sampled units (the oracle computes each sampled unit from scratch: landmarks
of its kv-head, selection, attention).

Samples: gated_prefill_32k -- every unit; gated_decode_128k -- 8 of the 64
sequences, all kv-heads; long_prefill_256k -- all kv-heads of 24 random tiles
plus every 64th tile of kv-head 0; hils_decode_1m -- 2 of the 8 sequences.
The decodes run as one decode-step call (selection and decode overlapped),
as the benchmark times them."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
import oracle
from block_sparse_long_landmark_b200 import inputs
from _util import GAP, LSE_TOL, O_TOL, f64, round_mode, run_prefill

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS


def _check_unit_lists(gi, gs, gc, ri, rs, rc, gap):
    assert gc == rc
    same = np.array_equal(gi[:rc], ri[:rc])
    if not same:
        assert gap <= GAP, (gi[:rc], ri[:rc], gap)
    else:
        assert np.all(np.abs(gs[:rc] - rs[:rc]) <= 1e-5 + 1e-4 * np.abs(rs[:rc]))
    return same


def _prefill_sampled(wl, tiles_by_group):
    p = sa.params_for(wl)
    Q, K, V = inputs.make_prefill(wl, device="cuda")
    _, (idx, sc, cnt), O, lse = run_prefill(p, Q, K, V)
    G = wl.Hq // wl.Hkv
    gi, gs, gc = idx.cpu().numpy(), sc.cpu().numpy(), cnt.cpu().numpy()
    checked = exact = 0
    max_err = max_lerr = 0.0
    for g, tiles in tiles_by_group.items():
        # the kv-head as a problem of its own: B=1, its G query heads, 1 kv-head
        Qg = f64(Q[:, g * G:(g + 1) * G])
        Kg, Vg = f64(K[:, g:g + 1]), f64(V[:, g:g + 1])
        ref = oracle.prefill(Qg, Kg, Vg, wl.block, wl.top_k, wl.flags, round_mode=round_mode(wl.dtype),
                             units=[(0, 0, j) for j in tiles])
        Og = f64(O[0, g * G:(g + 1) * G])
        lg = f64(lse[0, g * G:(g + 1) * G])
        for j in tiles:
            checked += 1
            same = _check_unit_lists(gi[0, g, j], gs[0, g, j], gc[0, g, j], ref["idx"][0, 0, j],
                                     ref["sc"][0, 0, j], ref["count"][0, 0, j], ref["rel_gap"][0, 0, j])
            if not same:
                continue
            exact += 1
            rows = slice(j * wl.block, min(wl.N, (j + 1) * wl.block))
            err = np.abs(Og[:, rows] - ref["O"][0, :, rows]).max()
            lerr = np.abs(lg[:, rows] - ref["LSE"][0, :, rows]).max()
            max_err, max_lerr = max(max_err, err), max(max_lerr, lerr)
    assert max_err <= O_TOL[wl.dtype] and max_lerr <= LSE_TOL, (max_err, max_lerr)
    assert exact >= 0.9 * checked
    return checked, exact, max_err, max_lerr


def test_gated_prefill_32k_every_unit():
    wl = W["gated_prefill_32k"]
    _prefill_sampled(wl, {g: list(range(wl.nb)) for g in range(wl.Hkv)})


def test_long_prefill_256k_sampled():
    wl = W["long_prefill_256k"]
    rng = np.random.default_rng(5)
    tiles = sorted(rng.choice(wl.nb, size=24, replace=False).tolist())
    groups = {g: list(tiles) for g in range(wl.Hkv)}
    groups[0] = sorted(set(groups[0]) | set(range(0, wl.nb, 64)) | {wl.nb - 1})
    _prefill_sampled(wl, groups)


def _decode_sampled(wl, seqs):
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    # the configuration the benchmark times: one decode-step call
    L = sa.landmarks(p, K)
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    (idx, sc, cnt), (o, lse) = sa.decode_step(p, q, L, K, V, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    gi, gs, gc = idx.cpu().numpy(), sc.cpu().numpy(), cnt.cpu().numpy()
    G = wl.Hq // wl.Hkv
    checked = exact = 0
    for b in seqs:
        ref = oracle.decode(f64(q[b:b + 1]), f64(K[b:b + 1]), f64(V[b:b + 1]), wl.block, wl.top_k, wl.flags,
                            round_mode=round_mode(wl.dtype))
        ob, lb = f64(o[b]), f64(lse[b])
        for g in range(wl.Hkv):
            checked += 1
            same = _check_unit_lists(gi[b, g], gs[b, g], gc[b, g], ref["idx"][0, g], ref["sc"][0, g],
                                     ref["count"][0, g], ref["rel_gap"][0, g])
            if not same:
                continue
            exact += 1
            hs = slice(g * G, (g + 1) * G)
            assert np.abs(ob[hs] - ref["O"][0, hs]).max() <= O_TOL[wl.dtype]
            assert np.abs(lb[hs] - ref["LSE"][0, hs]).max() <= LSE_TOL
    assert exact >= 0.9 * checked


def test_gated_decode_128k_sampled():
    _decode_sampled(W["gated_decode_128k"], seqs=[0, 9, 18, 27, 36, 45, 54, 63])


def test_hils_decode_1m_sampled():
    _decode_sampled(W["hils_decode_1m"], seqs=[0, 7])

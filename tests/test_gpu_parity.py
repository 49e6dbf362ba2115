"""GPU parity: every step of the CUDA path, called through the C ABI, against
the CPU oracle on the same seeded inputs (small and ragged problems here;
full-size sampled checks live in test_gpu_fullsize.py)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
import oracle
from block_sparse_long_landmark_b200 import inputs
from _util import (GAP, LSE_TOL, O_TOL, compare_lists, f64, oracle_sel_tensors, round_mode, run_decode,
                   run_prefill)

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS

PREFILL_CASES = {
    "tiny_fp32": W["tiny_fp32_prefill"],
    "tiny_fp32_ragged": W["tiny_fp32_prefill"].scaled(N=1000),
    "gqa_bf16_4k": W["gated_prefill_32k"].scaled(N=4096),
    "gqa_bf16_ragged": W["gated_prefill_32k"].scaled(N=2000, Hq=8, Hkv=2),
    "gqa_bf16_block128": W["long_prefill_256k"].scaled(N=8192, Hq=8, Hkv=2),
    "fp32_d128_gqa": W["gated_prefill_32k"].scaled(N=1536, Hq=4, Hkv=2, dtype="fp32", sigma=1.0),
}


def _prefill_inputs(wl):
    Q, K, V = inputs.make_prefill(wl, device="cuda")
    return Q, K, V


def _oracle_prefill(wl, Q, K, V, flags=None, top_k=None, sel_override=None):
    return oracle.prefill(f64(Q), f64(K), f64(V), wl.block, wl.top_k if top_k is None else top_k,
                          wl.flags if flags is None else flags, round_mode=round_mode(wl.dtype),
                          sel_override=sel_override)


def _check_outputs(wl, ref, O, lse, row_mask=None):
    Og, lg = f64(O), f64(lse)
    Or, lr = ref["O"], ref["LSE"]
    if row_mask is not None:
        Og, lg, Or, lr = Og[row_mask], lg[row_mask], Or[row_mask], lr[row_mask]
    err = np.abs(Og - Or).max() if Og.size else 0.0
    assert err <= O_TOL[wl.dtype], f"max |O - O_ref| = {err}"
    fin = np.isfinite(lr)
    assert np.array_equal(fin, np.isfinite(lg))
    lerr = np.abs(lg[fin] - lr[fin]).max() if fin.any() else 0.0
    assert lerr <= LSE_TOL, f"max |lse - lse_ref| = {lerr}"
    return err, lerr


@pytest.mark.parametrize("case", sorted(PREFILL_CASES))
def test_landmarks(case):
    wl = PREFILL_CASES[case]
    p = sa.params_for(wl)
    _, K, _ = _prefill_inputs(wl)
    L = f64(sa.landmarks(p, K))
    Kh = f64(K)
    for b in range(wl.B):
        for g in range(wl.Hkv):
            ref = oracle.landmarks(Kh[b, g], wl.block, round_mode(wl.dtype))
            if wl.dtype == "fp32":
                assert np.abs(L[b, g] - ref).max() <= 1e-6
            else:
                # fp32 sum vs exact mean: at most one bf16 step apart, and rarely
                ulp = np.maximum(np.abs(ref), 1e-30) * 2.0 ** -7
                diff = np.abs(L[b, g] - ref)
                assert np.all(diff <= ulp)
                assert np.mean(diff > 0) < 1e-3


@pytest.mark.parametrize("case", sorted(PREFILL_CASES))
def test_prefill_end_to_end(case):
    wl = PREFILL_CASES[case]
    p = sa.params_for(wl)
    Q, K, V = _prefill_inputs(wl)
    L, (idx, sc, cnt), O, lse = run_prefill(p, Q, K, V)
    ref = _oracle_prefill(wl, Q, K, V)
    n, exact, mask = compare_lists(ref, idx, sc, cnt)
    assert exact >= 0.9 * n
    # rows of units whose lists agree: element-wise comparison
    G = wl.Hq // wl.Hkv
    rows = np.zeros((wl.B, wl.Hq, wl.N), dtype=bool)
    for b, g, j in zip(*np.nonzero(mask)):
        rows[b, g * G:(g + 1) * G, j * wl.block:(j + 1) * wl.block] = True
    _check_outputs(wl, ref, O, lse, rows)


@pytest.mark.parametrize("case", sorted(PREFILL_CASES))
def test_prefill_on_oracle_lists(case):
    """The attention step alone: GPU prefill fed with the oracle's lists."""
    wl = PREFILL_CASES[case]
    p = sa.params_for(wl)
    Q, K, V = _prefill_inputs(wl)
    ref = _oracle_prefill(wl, Q, K, V)
    _, _, O, lse = run_prefill(p, Q, K, V, sel=oracle_sel_tensors(ref))
    _check_outputs(wl, ref, O, lse)


FLAG_CASES = [
    ("no_sink", inputs.F_LOCAL | inputs.F_GATE | inputs.F_CAUSAL, 4),
    ("no_gate", inputs.F_SINK | inputs.F_LOCAL | inputs.F_CAUSAL, 4),
    ("keep_all", inputs.F_SINK | inputs.F_LOCAL | inputs.F_CAUSAL, 64),
    ("top0", inputs.F_SINK | inputs.F_LOCAL | inputs.F_GATE | inputs.F_CAUSAL, 0),
    ("empty_tile0", inputs.F_CAUSAL, 3),
    ("sink_only", inputs.F_SINK | inputs.F_CAUSAL, 2),
    ("not_causal", inputs.F_SINK | inputs.F_LOCAL | inputs.F_GATE, 3),
    ("hier", inputs.F_SINK | inputs.F_LOCAL | inputs.F_HIER | inputs.F_CAUSAL, 3),
    ("per_qhead", inputs.F_SINK | inputs.F_LOCAL | inputs.F_GATE | inputs.F_CAUSAL | inputs.F_PER_QHEAD, 3),
]


FLAG_SHAPES = {
    "fp32_g2": dict(Hq=4, Hkv=2, block=64, dtype="fp32"),
    "bf16_g1": dict(Hq=2, Hkv=2, block=64, dtype="bf16"),       # CUDA-core kernel (odd group)
    "bf16_g4": dict(Hq=8, Hkv=2, block=64, dtype="bf16"),       # tensor-core kernel (block 64)
    "bf16_g2_b128": dict(Hq=4, Hkv=2, block=128, dtype="bf16"),  # tensor-core kernel (block 128)
}


@pytest.mark.parametrize("name,flags,top_k", FLAG_CASES)
@pytest.mark.parametrize("shape", sorted(FLAG_SHAPES))
def test_prefill_flags(name, flags, top_k, shape):
    wl = W["gated_prefill_32k"].scaled(N=1000, top_k=top_k, n_plants=2, **FLAG_SHAPES[shape])
    p = sa.params_for(wl, flags=flags)
    Q, K, V = _prefill_inputs(wl)
    L, (idx, sc, cnt), O, lse = run_prefill(p, Q, K, V)
    ref = _oracle_prefill(wl, Q, K, V, flags=flags)
    n, exact, mask = compare_lists(ref, idx, sc, cnt)
    per_q = bool(flags & inputs.F_PER_QHEAD)
    G = wl.Hq // wl.Hkv
    rows = np.zeros((wl.B, wl.Hq, wl.N), dtype=bool)
    for b, s_, j in zip(*np.nonzero(mask)):
        hs = slice(s_, s_ + 1) if per_q else slice(s_ * G, (s_ + 1) * G)
        rows[b, hs, j * wl.block:(j + 1) * wl.block] = True
    _check_outputs(wl, ref, O, lse, rows)
    if name == "empty_tile0":
        assert np.all(f64(O)[:, :, :wl.block] == 0) and np.all(np.isneginf(f64(lse)[:, :, :wl.block]))


DECODE_CASES = {
    "gated_8k": W["gated_decode_128k"].scaled(B=4, N=8192),
    "gated_ragged": W["gated_decode_128k"].scaled(B=3, N=5000, top_k=8, n_plants=4),
    "hier_16k": W["hils_decode_1m"].scaled(B=2, N=16384, top_k=16, n_plants=16),
    "hier_ragged": W["hils_decode_1m"].scaled(B=2, N=3001, top_k=5, n_plants=3),
    "gated_fp32_d64": W["gated_decode_128k"].scaled(B=2, N=4096, d=64, dtype="fp32", Hq=8, Hkv=8, top_k=6,
                                                    n_plants=3, sigma=1.0),
    "gated_big_k": W["gated_decode_128k"].scaled(B=2, N=65536, top_k=200, n_plants=16),
    # many units: 12 kept blocks per CTA, so every ring stage is reused several times
    "gated_wide": W["gated_decode_128k"].scaled(B=64, N=4096),
}


def _oracle_decode(wl, q, K, V, flags=None, sel_override=None):
    return oracle.decode(f64(q), f64(K), f64(V), wl.block, wl.top_k, wl.flags if flags is None else flags,
                         round_mode=round_mode(wl.dtype), sel_override=sel_override)


@pytest.mark.parametrize("case", sorted(DECODE_CASES))
def test_decode_end_to_end(case):
    wl = DECODE_CASES[case]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    L, (idx, sc, cnt), o, lse = run_decode(p, q, K, V)
    ref = _oracle_decode(wl, q, K, V)
    n, exact, mask = compare_lists(ref, idx, sc, cnt)
    G = wl.Hq // wl.Hkv
    rows = np.repeat(mask, G, axis=1)
    _check_outputs(wl, ref, o, lse, rows)
    assert exact >= 0.5 * n


@pytest.mark.parametrize("case", sorted(DECODE_CASES))
def test_decode_on_oracle_lists(case):
    wl = DECODE_CASES[case]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    ref = _oracle_decode(wl, q, K, V)
    _, _, o, lse = run_decode(p, q, K, V, sel=oracle_sel_tensors(ref))
    _check_outputs(wl, ref, o, lse)


@pytest.mark.parametrize("case", ["gated_8k", "gated_ragged", "hier_16k", "hier_ragged", "gated_big_k",
                                  "gated_wide"])
def test_decode_mma_matches_cuda_core(case, monkeypatch):
    """The tensor-core decode (TMA ring + mma.sync) against the CUDA-core decode
    on the oracle's lists."""
    wl = DECODE_CASES[case]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    ref = _oracle_decode(wl, q, K, V)
    sel = oracle_sel_tensors(ref)
    _, _, o, lse = run_decode(p, q, K, V, sel=sel)
    monkeypatch.setenv("SPARSE_ATTN_DECODE_PATH", "simt")
    _, _, o2, lse2 = run_decode(p, q, K, V, sel=sel)
    assert (o.float() - o2.float()).abs().max().item() <= 2e-2
    assert (lse - lse2).abs().max().item() <= 1e-3


@pytest.mark.parametrize("case", ["gated_wide", "hier_16k", "gated_ragged"])
def test_decode_steps_reuse_one_workspace(case):
    """Decode steps on one workspace with alternating queries: the kernel
    counts each unit's partial records in the workspace and the CTA that
    completes a unit merges it, returning the counter to zero, so every step
    must give the oracle's output for its own query (a counter left behind
    would merge a later step's unit early or never)."""
    wl = DECODE_CASES[case]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    q2 = inputs.make_decode(wl.scaled(seed=wl.seed + 7), device="cuda")[0]
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    L = sa.landmarks(p, K)
    refs = {}
    for step in range(4):
        qs = q if step % 2 == 0 else q2
        key = step % 2
        if key not in refs:
            refs[key] = _oracle_decode(wl, qs, K, V)
        sel = oracle_sel_tensors(refs[key])
        o, lse = sa.decode(p, qs, K, V, *sel, ws)
        torch.cuda.synchronize()
        assert sa.check_status(ws) == 0
        _check_outputs(wl, refs[key], o, lse)


@pytest.mark.parametrize("flags", [inputs.F_SINK | inputs.F_LOCAL | inputs.F_CAUSAL,
                                   inputs.F_LOCAL | inputs.F_GATE | inputs.F_CAUSAL,
                                   inputs.F_SINK | inputs.F_LOCAL | inputs.F_GATE | inputs.F_PER_QHEAD,
                                   inputs.F_SINK | inputs.F_HIER | inputs.F_PER_QHEAD])
def test_decode_flags(flags):
    wl = W["gated_decode_128k"].scaled(B=2, N=3000, top_k=5, n_plants=3)
    p = sa.params_for(wl, flags=flags)
    q, K, V = inputs.make_decode(wl, device="cuda")
    _, (idx, sc, cnt), o, lse = run_decode(p, q, K, V)
    ref = _oracle_decode(wl, q, K, V, flags=flags)
    n, exact, mask = compare_lists(ref, idx, sc, cnt)
    G = 1 if flags & inputs.F_PER_QHEAD else wl.Hq // wl.Hkv
    _check_outputs(wl, ref, o, lse, np.repeat(mask, G, axis=1))


TC_CASES = {
    "b64_g4": W["gated_prefill_32k"].scaled(N=4096),
    "b64_g8": W["gated_prefill_32k"].scaled(N=3000, Hq=16, Hkv=2),
    "b128_g4": W["long_prefill_256k"].scaled(N=8192, Hq=8, Hkv=2),
    "b128_ragged": W["long_prefill_256k"].scaled(N=5000, Hq=4, Hkv=2, top_k=5),
    "b64_g2": W["gated_prefill_32k"].scaled(N=3000, Hq=4, Hkv=2),
    "b64_hier": W["gated_prefill_32k"].scaled(N=4096, Hq=8, Hkv=2, hier=True),
    "b64_hier_ragged": W["gated_prefill_32k"].scaled(N=3001, Hq=4, Hkv=2, hier=True, top_k=7),
    "b128_g1": W["long_prefill_256k"].scaled(N=4096, Hq=2, Hkv=2),
    "b64_big_k": W["gated_prefill_32k"].scaled(N=8192, Hq=8, Hkv=2, top_k=100),
    "b64_odd_k": W["gated_prefill_32k"].scaled(N=4096, Hq=8, Hkv=2, top_k=7),
    "b64_g4_ragged": W["gated_prefill_32k"].scaled(N=3001, Hq=8, Hkv=2, top_k=6),
    "b64_g4_batch2": W["gated_prefill_32k"].scaled(B=2, N=2048, Hq=8, Hkv=2, top_k=9),
    "b128_g2_batch3": W["long_prefill_256k"].scaled(B=3, N=3000, Hq=4, Hkv=2, top_k=4),
    "b128_hier": W["long_prefill_256k"].scaled(N=4000, Hq=4, Hkv=2, top_k=5, hier=True),
    "b64_hier_batch2": W["gated_prefill_32k"].scaled(B=2, N=2500, Hq=8, Hkv=2, top_k=6, hier=True),
}


def _tc1_kernel(wl):
    """1 when the two-CTA kernel takes the shape (128-row tiles; hierarchical
    only at block 64), else 0 (CUDA cores)."""
    G = wl.Hq // wl.Hkv
    return 1 if (G * wl.block) % 128 == 0 and (not wl.hier or wl.block == 64) else 0


def _expected_kernel(wl):
    """2 = persistent kernel (256-row units), else what the two-CTA kernel takes."""
    G = wl.Hq // wl.Hkv
    return 2 if (G * wl.block) % 256 == 0 else _tc1_kernel(wl)


@pytest.mark.parametrize("case", sorted(TC_CASES))
def test_tensor_core_prefill_matches_oracle_and_cuda_core(case, monkeypatch):
    """The tensor-core kernel on the oracle's lists, against the oracle and
    against the CUDA-core kernel on the same lists."""
    wl = TC_CASES[case]
    p = sa.params_for(wl)
    kern = _expected_kernel(wl)
    assert sa.sparse_attn_prefill_kernel(p) == kern
    Q, K, V = _prefill_inputs(wl)
    ref = _oracle_prefill(wl, Q, K, V)
    sel = oracle_sel_tensors(ref)
    _, _, O, lse = run_prefill(p, Q, K, V, sel=sel)
    _check_outputs(wl, ref, O, lse)
    if kern == 2:
        # the persistent kernel agrees with the next path on the same lists
        monkeypatch.setenv("SPARSE_ATTN_PREFILL_PATH", "tc1")
        assert sa.sparse_attn_prefill_kernel(p) == _tc1_kernel(wl)
        _, _, O1, lse1 = run_prefill(p, Q, K, V, sel=sel)
        _check_outputs(wl, ref, O1, lse1)
        assert (O.float() - O1.float()).abs().max().item() <= 2e-2
        assert (lse - lse1).abs().max().item() <= 1e-3
    monkeypatch.setenv("SPARSE_ATTN_PREFILL_PATH", "simt")
    assert sa.sparse_attn_prefill_kernel(p) == 0
    _, _, O2, lse2 = run_prefill(p, Q, K, V, sel=sel)
    assert (O.float() - O2.float()).abs().max().item() <= 2e-2
    assert (lse - lse2).abs().max().item() <= 1e-3


def test_prefill_selection_in_chunks_with_merge():
    """More than 8192 candidate blocks: prefill selection splits every tile's
    candidates into chunks and merges the chunks' top-K lists."""
    wl = W["tiny_fp32_prefill"].scaled(N=140000, Hq=1, Hkv=1, block=16, top_k=4, n_plants=2)
    p = sa.params_for(wl)
    assert sa.sparse_attn_workspace_size(p, sa.SA_OP_SELECT) > 256     # the chunked path
    Q, K, V = _prefill_inputs(wl)
    L, (idx, sc, cnt), O, lse = run_prefill(p, Q, K, V)
    units = [(0, 0, j) for j in list(range(0, 40)) + list(range(8180, 8200)) + list(range(wl.nb - 40, wl.nb))]
    ref = oracle.prefill(f64(Q), f64(K), f64(V), wl.block, wl.top_k, wl.flags, round_mode=oracle.ROUND_FP32,
                         units=units)
    n, exact, mask = compare_lists(ref, idx, sc, cnt, units=units)
    assert exact >= 0.9 * n


def test_selection_is_deterministic():
    wl = W["gated_prefill_32k"].scaled(N=4096)
    p = sa.params_for(wl)
    Q, K, _ = _prefill_inputs(wl)
    ws = sa.workspace(p)
    L = sa.landmarks(p, K)
    a = [t.clone() for t in sa.select(p, Q, L, ws)]
    b = sa.select(p, Q, L, ws)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    wd = W["hils_decode_1m"].scaled(B=2, N=65536)
    pd = sa.params_for(wd)
    q, Kd, _ = inputs.make_decode(wd, device="cuda")
    wsd = sa.workspace(pd)
    Ld = sa.landmarks(pd, Kd)
    a = [t.clone() for t in sa.select_decode(pd, q, Ld, wsd)]
    b = sa.select_decode(pd, q, Ld, wsd)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bad_list_entry_sets_status_and_is_skipped():
    wl = W["gated_prefill_32k"].scaled(N=1024, Hq=4, Hkv=2)
    p = sa.params_for(wl)
    Q, K, V = _prefill_inputs(wl)
    ws = sa.workspace(p)
    L = sa.landmarks(p, K)
    idx, sc, cnt = sa.select(p, Q, L, ws)
    idx[0, 0, 5, 1] = 10_000          # beyond the tile's own block
    sa.prefill(p, Q, K, V, idx, sc, cnt, ws)
    with pytest.raises(sa.SparseAttnError) as ei:
        sa.check_status(ws)
    assert ei.value.code == sa.SA_ERR_DEVICE
    assert sa.check_status(ws) == 0   # cleared


def test_nan_score_sets_status():
    wl = W["gated_prefill_32k"].scaled(N=1024, Hq=4, Hkv=2)
    p = sa.params_for(wl)
    Q, K, V = _prefill_inputs(wl)
    Q[0, 0, 300, 5] = float("nan")
    ws = sa.workspace(p)
    L = sa.landmarks(p, K)
    sa.select(p, Q, L, ws)
    rc, detail = sa.sparse_attn_check_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == sa.SA_ERR_DEVICE and detail & 2


PERQ_TC_CASES = {
    # four query heads of a group share a 256-row unit: the union of their four lists
    "b64_g4": W["gated_prefill_32k_perqhead"].scaled(N=4096, Hq=8, Hkv=2),
    # two heads of a block-128 tile, ragged end
    "b128_g2_ragged": W["long_prefill_256k"].scaled(N=3000, Hq=4, Hkv=2, per_qhead=True),
    # plain (no gate) mode, batch 2
    "b64_plain_batch2": W["gated_prefill_32k_perqhead"].scaled(B=2, N=2048, Hq=8, Hkv=2),
}


@pytest.mark.parametrize("case", sorted(PERQ_TC_CASES))
def test_per_qhead_prefill_on_tensor_cores(case, monkeypatch):
    """One list per query head on the persistent tensor-core kernel: each unit
    reads the union of its heads' lists and masks, per row, the blocks its
    head did not keep.  Against the oracle (its own lists) and against the
    CUDA-core kernel on the same lists."""
    wl = PERQ_TC_CASES[case]
    flags = wl.flags & ~inputs.F_GATE if "plain" in case else wl.flags
    p = sa.params_for(wl, flags=flags)
    assert sa.sparse_attn_prefill_kernel(p) == 2
    Q, K, V = _prefill_inputs(wl)
    ref = _oracle_prefill(wl, Q, K, V, flags=flags)
    sel = oracle_sel_tensors(ref)
    _, _, O, lse = run_prefill(p, Q, K, V, sel=sel)
    _check_outputs(wl, ref, O, lse)
    monkeypatch.setenv("SPARSE_ATTN_PREFILL_PATH", "simt")
    assert sa.sparse_attn_prefill_kernel(p) == 0
    _, _, O2, lse2 = run_prefill(p, Q, K, V, sel=sel)
    assert (O.float() - O2.float()).abs().max().item() <= 2e-2
    assert (lse - lse2).abs().max().item() <= 1e-3

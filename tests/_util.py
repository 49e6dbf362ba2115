"""Shared helpers of the GPU parity tests (CUDA path vs the CPU oracle)."""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_long_landmark_b200 as sa
import oracle

# Tolerances: outputs max-abs 2e-2 (bf16) / 1e-4 (fp32); LSE 1e-3;
# indices exact wherever the K-th / (K+1)-th relative score gap exceeds 1e-3.
O_TOL = {"bf16": 2e-2, "fp32": 1e-4}
LSE_TOL = 1e-3
GAP = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def round_mode(dtype: str) -> int:
    return oracle.ROUND_BF16 if dtype == "bf16" else oracle.ROUND_FP32


def run_prefill(p, Q, K, V, sel=None):
    """GPU landmarks -> select -> prefill.  ``sel`` = (idx, sc, cnt) overrides selection."""
    ws = sa.workspace(p, ops=sa.FORWARD_OPS)
    L = sa.landmarks(p, K)
    if sel is None:
        sel = sa.select(p, Q, L, ws)
    O, lse = sa.prefill(p, Q, K, V, *sel, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    return L, sel, O, lse


def run_decode(p, q, K, V, sel=None):
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    L = sa.landmarks(p, K)
    if sel is None:
        sel = sa.select_decode(p, q, L, ws)
    o, lse = sa.decode(p, q, K, V, *sel, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    return L, sel, o, lse


def oracle_sel_tensors(ref, device="cuda"):
    """The oracle's lists as the ABI's tensors (oracle -> GPU direction only)."""
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).to(device)
    sc = torch.from_numpy(ref["sc"].astype(np.float32)).to(device)
    cnt = torch.from_numpy(ref["count"].astype(np.int32)).to(device)
    return idx, sc, cnt


def compare_lists(ref, idx, sc, cnt, units=None):
    """Checks the GPU lists against the oracle's.

    Returns (n_units_checked, n_exact, matched_mask) where matched_mask marks
    units whose kept lists are identical.  Every unit must agree on its count;
    its list must be identical unless the oracle's relative gap at the K-th
    score is at most GAP (a near-tie: both answers are correct)."""
    gi, gs, gc = (t.cpu().numpy() for t in (idx, sc, cnt))
    ri, rs, rc, gap = ref["idx"], ref["sc"], ref["count"], ref["rel_gap"]
    mask = np.zeros(rc.shape, dtype=bool)
    n = exact = 0
    it = units if units is not None else list(np.ndindex(rc.shape))
    for u in it:
        u = tuple(u)
        n += 1
        assert gc[u] == rc[u], f"count differs at unit {u}: gpu {gc[u]} oracle {rc[u]}"
        c = int(rc[u])
        same = np.array_equal(gi[u][:c], ri[u][:c])
        if not same:
            assert gap[u] <= GAP, f"selection differs at unit {u} with gap {gap[u]}: {gi[u][:c]} vs {ri[u][:c]}"
        else:
            exact += 1
            assert np.all(gi[u][c:] == -1)
            err = np.abs(gs[u][:c] - rs[u][:c])
            assert np.all(err <= 1e-5 + 1e-4 * np.abs(rs[u][:c])), (u, gs[u][:c], rs[u][:c])
        mask[u] = same
    return n, exact, mask

"""Bounded waits of the persistent tensor-core prefill run out cleanly.

Every mbarrier wait in the kernel gives up after a time limit: the CTA then
records status bit 4, lets the copies it issued land, frees its tensor
memory and exits, so the context stays usable.  The test hook
SPARSE_ATTN_TEST_STALL=<t> makes each CTA skip the K load of its key tile t
(nothing is put in flight for it) and lowers the limit to 1 ms; the MMA
warp's wait for that tile then runs out.  The next call on the same stream,
without the hook, must run normally and match the oracle."""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
import oracle
from block_sparse_long_landmark_b200 import inputs
from _util import LSE_TOL, O_TOL, compare_lists, f64, round_mode

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("stall", [0, 1, 3])
def test_prefill_wait_expiry_reports_and_the_next_call_recovers(monkeypatch, stall):
    wl = inputs.WORKLOADS["gated_prefill_32k"].scaled(N=4096, Hq=8, Hkv=2)
    p = sa.params_for(wl)
    assert sa.sparse_attn_prefill_kernel(p) == 2
    Q, K, V = inputs.make_prefill(wl, device="cuda")
    ws = sa.workspace(p)
    L = sa.landmarks(p, K)
    sel = sa.select(p, Q, L, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    stream = torch.cuda.current_stream().cuda_stream

    monkeypatch.setenv("SPARSE_ATTN_TEST_STALL", str(stall))
    t0 = time.perf_counter()
    sa.prefill(p, Q, K, V, *sel, ws)            # launches normally; the waits expire on the device
    rc, detail = sa.sparse_attn_check_status(ws.data_ptr(), stream)
    dt = time.perf_counter() - t0
    assert rc == sa.SA_ERR_DEVICE and detail & 4, (rc, detail)
    assert dt < 1.0, dt                          # 1 ms limits, not the default 2 s ones
    monkeypatch.delenv("SPARSE_ATTN_TEST_STALL")

    # the status word was cleared by the read; a normal call on the same stream runs through
    O, lse = sa.prefill(p, Q, K, V, *sel, ws)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    ref = oracle.prefill(f64(Q), f64(K), f64(V), wl.block, wl.top_k, wl.flags, round_mode=round_mode(wl.dtype))
    _, _, mask = compare_lists(ref, *sel)
    G = wl.Hq // wl.Hkv
    rows = np.repeat(np.repeat(mask, G, axis=1), wl.block, axis=2)[:, :, :wl.N]
    assert np.abs(f64(O) - ref["O"])[rows].max() <= O_TOL[wl.dtype]
    assert np.abs(f64(lse) - ref["LSE"])[rows].max() <= LSE_TOL

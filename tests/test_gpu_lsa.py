"""Flat clustered index (sparse_attn_lsa_build / sparse_attn_lsa_decode)
through the C ABI, against ``oracle.lsa`` on the same seeded inputs.

The clustering and the cluster choice run in fp64 on both sides (the
decisions are a chain of exact comparisons), so cluster membership must match
exactly and the centres to 1e-12; attention runs in fp32 on the GPU, checked
to the decode tolerances (O 2e-2 bf16 / 1e-4 fp32, LSE 1e-3)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
from oracle import lsa

pytestmark = pytest.mark.gpu

CASES = {
    "fp32_d64_ragged": dict(B=1, Hq=4, Hkv=2, d=64, N=1000, pool=4, seg=16, clusters=4, top=3, sink=8, window=32,
                            dtype="fp32", seed=1),
    "bf16_d128_batch2": dict(B=2, Hq=8, Hkv=2, d=128, N=4096, pool=4, seg=32, clusters=8, top=6, sink=16, window=64,
                             dtype="bf16", seed=2),
    "bf16_seg64_tail": dict(B=1, Hq=4, Hkv=1, d=128, N=64 * 4 * 5 + 37, pool=4, seg=64, clusters=16, top=5, sink=4,
                            window=40, dtype="bf16", seed=3),
    "bf16_pool1_everything": dict(B=1, Hq=2, Hkv=1, d=64, N=300, pool=1, seg=20, clusters=5, top=1000, sink=0,
                                  window=0, dtype="bf16", seed=4),
    # many centre chunks (merge across 6 chunk CTAs), eight query heads per kv-head, overlapping sink and window
    "bf16_many_chunks_g8": dict(B=1, Hq=16, Hkv=2, d=128, N=6144, pool=2, seg=32, clusters=16, top=40, sink=40,
                                window=300, dtype="bf16", seed=5),
    "fp32_g16_two_passes": dict(B=1, Hq=16, Hkv=1, d=64, N=2048, pool=4, seg=16, clusters=4, top=7, sink=3,
                                window=2100, dtype="fp32", seed=6),
    "bf16_no_clusters": dict(B=1, Hq=4, Hkv=2, d=128, N=100, pool=4, seg=32, clusters=4, top=8, sink=5,
                             window=20, dtype="bf16", seed=7),
    # more than 16 centre chunks: the block radix merge (every score passed: 18 chunks; each
    # chunk's best passed: 36 chunks); 2..16 chunks take the ordered lists and binary searches
    "bf16_radix_merge_all": dict(B=1, Hq=4, Hkv=1, d=64, N=4608, pool=1, seg=32, clusters=16, top=24, sink=8,
                                 window=64, dtype="bf16", seed=8),
    "bf16_radix_merge_best": dict(B=1, Hq=4, Hkv=1, d=64, N=9216, pool=1, seg=32, clusters=16, top=24, sink=8,
                                  window=64, dtype="bf16", seed=9),
}


def _inputs(c):
    g = torch.Generator().manual_seed(c["seed"])
    td = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
    q = torch.randn(c["B"], c["Hq"], c["d"], generator=g).to(td)
    K = torch.randn(c["B"], c["Hkv"], c["N"], c["d"], generator=g).to(td)
    V = torch.randn(c["B"], c["Hkv"], c["N"], c["d"], generator=g).to(td)
    return q, K, V


@pytest.mark.parametrize("case", sorted(CASES))
def test_flat_index_matches_oracle(case):
    c = CASES[case]
    p = sa.make_lsa_params(c["B"], c["Hq"], c["Hkv"], c["d"], c["N"], c["pool"], c["seg"], c["clusters"], c["top"],
                           c["sink"], c["window"], c["dtype"])
    q, K, V = _inputs(c)
    qd, Kd, Vd = q.cuda(), K.cuda(), V.cuda()
    index = sa.lsa_build(p, Kd)
    ws = sa.lsa_workspace(p)
    kept = torch.full((c["B"], c["Hkv"]), -1, dtype=torch.int32, device="cuda")
    o, lse = sa.lsa_decode(p, qd, Kd, Vd, index, ws, kept=kept)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    o2, lse2 = sa.lsa_decode(p, qd, Kd, Vd, index, ws)        # a second call: counters were reset
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    C = sa.sparse_attn_lsa_clusters(p)
    centres, members, sizes = (x.cpu().numpy() for x in index)
    q64, K64, V64 = (x.double().numpy() for x in (q, K, V))
    for b in range(c["B"]):
        for g in range(c["Hkv"]):
            ref = lsa.build_index(K64[b, g], c["pool"], c["seg"], c["clusters"])
            assert ref["centres"].shape[0] == C
            for cl in range(C):
                items = sorted({int(t) // c["pool"] for t in ref["positions"][cl]})
                assert list(members[b, g, cl, :sizes[b, g, cl]]) == items, (b, g, cl)
                assert np.all(members[b, g, cl, sizes[b, g, cl]:] == -1)
            if C:
                np.testing.assert_allclose(centres[b, g, :C], ref["centres"], rtol=1e-12, atol=1e-12)
    want = lsa.decode(q64, K64, V64, c["pool"], c["seg"], c["clusters"], c["top"], c["sink"], c["window"],
                      scale=float(np.float32(1.0 / np.sqrt(c["d"]))))
    for b in range(c["B"]):
        for g in range(c["Hkv"]):
            assert int(kept[b, g]) == len(want["kept"][(b, g)][1]), (b, g)
    tol = 2e-2 if c["dtype"] == "bf16" else 1e-4
    assert np.abs(o.float().cpu().numpy() - want["O"]).max() <= tol
    assert np.abs(lse.cpu().numpy() - want["LSE"]).max() <= 1e-3

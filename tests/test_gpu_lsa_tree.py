"""Tree over the flat clustered index (sparse_attn_lsa_tree_build /
sparse_attn_lsa_tree_decode) through the C ABI, against ``oracle.lsa``'s
``build_tree`` / ``tree_select`` on the same seeded inputs.

The tree's merges and the beam search are chains of fp64 comparisons on both
sides: the children of every node must match exactly, the node centres to
1e-10, the number of centres compared and of key positions kept exactly;
attention runs in fp32 (O 2e-2 bf16 / 1e-4 fp32, LSE 1e-3).  At a size the
oracle's tree is too slow for, a beam as wide as every level must give the
flat scan's choice (the property the oracle's own pin states)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
from oracle import lsa

pytestmark = pytest.mark.gpu

CASES = {
    # 128 leaves per head, fan-out 4: levels of 128, 32, 8, 2 nodes
    "fp32_d64_fan4": dict(B=1, Hq=4, Hkv=2, d=64, N=2048, pool=2, seg=16, clusters=2, top=6, sink=8, window=32,
                          dtype="fp32", fanout=4, beam=3, seed=11),
    # two sequences, fan-out 8 (128, 16, 2), bf16
    "bf16_d128_fan8": dict(B=2, Hq=8, Hkv=1, d=128, N=4096, pool=4, seg=16, clusters=2, top=9, sink=16, window=64,
                           dtype="bf16", fanout=8, beam=2, seed=12),
    # a ragged tail outside the complete segments, fan-out 3, a beam of 1
    "bf16_tail_fan3": dict(B=1, Hq=2, Hkv=1, d=128, N=1900, pool=2, seg=16, clusters=3, top=4, sink=4, window=50,
                           dtype="bf16", fanout=3, beam=1, seed=13),
}


def _inputs(c):
    g = torch.Generator().manual_seed(c["seed"])
    td = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
    q = torch.randn(c["B"], c["Hq"], c["d"], generator=g).to(td)
    K = torch.randn(c["B"], c["Hkv"], c["N"], c["d"], generator=g).to(td)
    V = torch.randn(c["B"], c["Hkv"], c["N"], c["d"], generator=g).to(td)
    return q, K, V


def _params(c):
    return sa.make_lsa_params(c["B"], c["Hq"], c["Hkv"], c["d"], c["N"], c["pool"], c["seg"], c["clusters"],
                              c["top"], c["sink"], c["window"], c["dtype"])


@pytest.mark.parametrize("case", sorted(CASES))
def test_tree_matches_oracle(case):
    c = CASES[case]
    p = _params(c)
    q, K, V = _inputs(c)
    qd, Kd, Vd = q.cuda(), K.cuda(), V.cuda()
    index = sa.lsa_build(p, Kd)
    tree, ws = sa.lsa_tree_build(p, c["fanout"], index)
    kept = torch.full((c["B"], c["Hkv"]), -1, dtype=torch.int32, device="cuda")
    comp = torch.full((c["B"], c["Hkv"]), -1, dtype=torch.int32, device="cuda")
    o, lse = sa.lsa_tree_decode(p, c["fanout"], c["beam"], qd, Kd, Vd, index, tree, ws, kept=kept, compared=comp)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0
    lv_gpu = sa.lsa_tree_levels(p, c["fanout"], tree)
    q64, K64, V64 = (x.double().numpy() for x in (q, K, V))
    G = c["Hq"] // c["Hkv"]
    scale = float(np.float32(1.0 / np.sqrt(c["d"])))
    O = np.zeros((c["B"], c["Hq"], c["d"]))
    L = np.zeros((c["B"], c["Hq"]))
    for b in range(c["B"]):
        for g in range(c["Hkv"]):
            idx = lsa.build_index(K64[b, g], c["pool"], c["seg"], c["clusters"])
            levels = lsa.build_tree(idx, c["fanout"])
            assert len(levels) == len(lv_gpu)
            np.testing.assert_array_equal(lv_gpu[0]["mass"][b, g].cpu().numpy(), levels[0]["mass"])
            for lvn in range(1, len(levels)):
                ref = levels[lvn]
                gl = lv_gpu[lvn]
                first = gl["first"][b, g].cpu().numpy()
                ch = gl["children"][b, g].cpu().numpy()
                got = [list(ch[first[i]:first[i + 1]]) for i in range(len(ref["children"]))]
                assert got == [list(map(int, k)) for k in ref["children"]], (b, g, lvn)
                np.testing.assert_array_equal(gl["mass"][b, g].cpu().numpy(), ref["mass"])
                np.testing.assert_allclose(gl["centres"][b, g].cpu().numpy(), ref["centres"], rtol=1e-10,
                                           atol=1e-12)
            qbar = q64[b, g * G:(g + 1) * G].mean(axis=0)
            leaves, compared = lsa.tree_select(levels, qbar, c["beam"], c["top"], scale)
            pos = lsa.kept_positions(idx, leaves, c["N"], c["N"] - 1, c["sink"], c["window"])
            assert int(comp[b, g]) == compared
            assert int(kept[b, g]) == len(pos)
            for h in range(g * G, (g + 1) * G):
                O[b, h], L[b, h] = lsa.attend(q64[b, h], K64[b, g], V64[b, g], pos, scale)
    tol = 2e-2 if c["dtype"] == "bf16" else 1e-4
    assert np.abs(o.float().cpu().numpy() - O).max() <= tol
    assert np.abs(lse.cpu().numpy() - L).max() <= 1e-3


def test_full_beam_tree_is_the_flat_scan():
    """2048 leaves per head (fan-out 4: six levels): a beam as wide as the leaf
    set must keep exactly the flat decode's clusters (same kept positions,
    same outputs), while a narrow beam compares far fewer centres."""
    c = dict(B=1, Hq=8, Hkv=2, d=128, N=32768, pool=4, seg=64, clusters=16, top=32, sink=64, window=512,
             dtype="bf16", seed=14)
    p = _params(c)
    q, K, V = (x.cuda() for x in _inputs(c))
    index = sa.lsa_build(p, K)
    tree, ws = sa.lsa_tree_build(p, 4, index)
    flat_ws = sa.lsa_workspace(p)
    kf = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    of, lf = sa.lsa_decode(p, q, K, V, index, flat_ws, kept=kf)
    kt = torch.zeros_like(kf)
    ct = torch.zeros_like(kf)
    ot, lt = sa.lsa_tree_decode(p, 4, 4096, q, K, V, index, tree, ws, kept=kt, compared=ct)
    torch.cuda.synchronize()
    assert sa.check_status(ws) == 0 and sa.check_status(flat_ws) == 0
    assert torch.equal(kf, kt)
    assert (ot.float() - of.float()).abs().max().item() <= 1e-2
    assert (lt - lf).abs().max().item() <= 1e-4
    kn = torch.zeros_like(kf)
    cn = torch.zeros_like(kf)
    sa.lsa_tree_decode(p, 4, 8, q, K, V, index, tree, ws, kept=kn, compared=cn)
    torch.cuda.synchronize()
    assert int(cn.max()) < 2048 // 4

"""sparse_attn_decode_static: decode for callers that cannot allocate device
memory (custom-allocator callbacks, servers whose pool owns all device memory,
plugins given only one call's tensors).  Its scratch is a static array inside
the library; the results must match sparse_attn_decode's, call after call.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test."""
import numpy as np
import pytest
import torch

import block_sparse_long_landmark_b200 as sa
from block_sparse_long_landmark_b200 import inputs

pytestmark = pytest.mark.gpu

O_TOL = {"bf16": 2e-2, "fp32": 1e-4}
LSE_TOL = 1e-3

CASES = {
    # many units, one split each
    "gated": inputs.WORKLOADS["gated_decode_128k"].scaled(B=8, N=16384),
    # few units: split partials live in the static scratch
    "hier_split": inputs.WORKLOADS["hils_decode_1m"].scaled(B=2, N=65536, top_k=32, n_plants=16),
    "fp32_split": inputs.WORKLOADS["gated_decode_128k"].scaled(B=1, N=8192, d=64, Hq=4, Hkv=2, dtype="fp32",
                                                             top_k=20, n_plants=4, sigma=1.0),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_static_decode_matches_workspace_decode(case):
    wl = CASES[case]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")
    ws = sa.workspace(p)
    L = sa.landmarks(p, K)
    sel = sa.select_decode(p, q, L, ws)
    o_ref, lse_ref = sa.decode(p, q, K, V, *sel, ws)
    torch.cuda.synchronize()
    for _ in range(2):          # two calls in a row share the static scratch
        o, lse = sa.decode_static(p, q, K, V, *sel)
        torch.cuda.synchronize()
        assert (o.float() - o_ref.float()).abs().max().item() <= O_TOL[wl.dtype]
        fin = torch.isfinite(lse_ref)
        assert torch.equal(fin, torch.isfinite(lse))
        assert (lse[fin] - lse_ref[fin]).abs().max().item() <= LSE_TOL


def test_static_decode_matches_the_oracle():
    """The same entry point against the CPU oracle on the oracle's own lists."""
    import oracle
    wl = CASES["gated"]
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device="cuda")

    def f64(t):
        return t.float().cpu().numpy().astype(np.float64)

    ref = oracle.decode(f64(q), f64(K), f64(V), wl.block, wl.top_k, wl.flags, round_mode=oracle.ROUND_BF16)
    sel = (torch.from_numpy(ref["idx"].astype(np.int32)).cuda(), torch.from_numpy(ref["sc"].astype(np.float32)).cuda(),
           torch.from_numpy(ref["count"].astype(np.int32)).cuda())
    for _ in range(2):
        o, lse = sa.decode_static(p, q, K, V, *sel)
        torch.cuda.synchronize()
        assert np.abs(f64(o) - ref["O"]).max() <= O_TOL[wl.dtype]
        assert np.abs(f64(lse) - ref["LSE"]).max() <= LSE_TOL


def test_static_decode_rejects_problems_beyond_the_scratch():
    # 74 units of 16 query heads each, split in 4: 2.46 MB of partials > 2 MiB
    wl = inputs.WORKLOADS["gated_decode_128k"].scaled(B=74, Hq=16, Hkv=1)
    p = sa.params_for(wl)
    assert sa.sparse_attn_workspace_size(p, sa.SA_OP_DECODE) > (2 << 20)
    fake = 256
    rc = sa.sparse_attn_decode_static(p, fake, fake, fake, fake, fake, fake, fake, fake, None)
    assert rc == sa.SA_ERR_WORKSPACE

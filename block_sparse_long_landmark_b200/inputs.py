"""Seeded synthetic workloads for selector-driven block-sparse attention.

This module only draws inputs.  It holds none of the method's arithmetic (no
pooling, scoring, selection or attention), so both the CUDA path and the CPU
oracle can be fed from it.

Inputs follow the long-context workloads the pages discuss (32K to 1M tokens
of context; the Latent Sparse Attention post's section "Ускорение видно на
слое, но дерево пока требует проверки" measures single layers at up to 10M
tokens).  The pages' quality benchmarks (RULER, PaperTrail) are not used:
seeded Gaussian Q/K/V with planted relevant blocks stand in for them.

Plant recipe.  A plant ties one query tile (prefill) or one decode query to
one earlier key block of the same kv-head group: a random unit direction u is
drawn per (batch, kv-head, tile); every query of every head of that group in
that tile gets ``+beta * u`` and every key of the planted block gets
``+alpha * u``.  The planted block then scores well above the noise for that
tile, which gives the top-K selection clear margins.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

F_SINK, F_LOCAL, F_GATE, F_HIER, F_CAUSAL, F_PER_QHEAD = 1, 2, 4, 8, 16, 32


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int               # sequence length (prefill) or context length incl. the query (decode)
    block: int
    top_k: int
    dtype: str           # "bf16" or "fp32"
    hier: bool
    sigma: float         # std of the Gaussian entries
    seed: int
    plant: str           # "per_tile", "every_4096", "per_seq"
    n_plants: int
    alpha: float = 0.5   # key shift along the planted direction
    beta: float | None = None   # query shift; None -> sigma
    per_qhead: bool = False     # one selection list per query head instead of per kv-head

    @property
    def flags(self) -> int:
        f = F_SINK | F_LOCAL | F_CAUSAL | (F_PER_QHEAD if self.per_qhead else 0)
        return f | (F_HIER if self.hier else F_GATE)

    @property
    def nb(self) -> int:
        return (self.N + self.block - 1) // self.block

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # B1 H2 (no GQA) d64 N1024 block 64, top-4 + sink + local, fp32.
    "tiny_fp32_prefill": Workload("tiny_fp32_prefill", "prefill", 1, 2, 2, 64, 1024, 64, 4, "fp32", False,
                                  1.0, 0, "per_tile", 2),
    # B1 Hq32 Hkv8 d128 N32768 block 64 top-16, bf16.
    "gated_prefill_32k": Workload("gated_prefill_32k", "prefill", 1, 32, 8, 128, 32768, 64, 16, "bf16", False,
                                  0.5, 1, "per_tile", 8),
    # 64 sequences x one query at context 131072, block 64 top-32, bf16 cache.
    "gated_decode_128k": Workload("gated_decode_128k", "decode", 64, 32, 8, 128, 131072, 64, 32, "bf16", False,
                                  0.5, 2, "per_seq", 16),
    # B1 N262144 block 128 top-16, bf16.
    "long_prefill_256k": Workload("long_prefill_256k", "prefill", 1, 32, 8, 128, 262144, 128, 16, "bf16", False,
                                  0.5, 3, "every_4096", 4),
    # the 32K prefill in hierarchical mode (per-block softmax, retrieval-score weights).
    "hils_prefill_32k": Workload("hils_prefill_32k", "prefill", 1, 32, 8, 128, 32768, 64, 16, "bf16", True,
                                 0.5, 5, "per_tile", 8),
    # 8 sequences x one query at context 1048576, block 64 top-64, hierarchical.
    "hils_decode_1m": Workload("hils_decode_1m", "decode", 8, 32, 8, 128, 1048576, 64, 64, "bf16", True,
                               0.5, 4, "per_seq", 64),
}
# the same workloads with one list per query head (each head selects its own blocks)
WORKLOADS["gated_prefill_32k_perqhead"] = WORKLOADS["gated_prefill_32k"].scaled(
    name="gated_prefill_32k_perqhead", per_qhead=True)
WORKLOADS["gated_decode_128k_perqhead"] = WORKLOADS["gated_decode_128k"].scaled(
    name="gated_decode_128k_perqhead", per_qhead=True)


def _randn(shape, gen, device, dtype, sigma, chunk=1 << 28):
    """Gaussian tensor, generated in chunks straight into the target dtype."""
    out = torch.empty(shape, device=device, dtype=dtype)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk):
        e = min(flat.numel(), s + chunk)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32).mul_(sigma).to(dtype)
    return out


def _unit_dirs(n, d, gen_cpu):
    u = torch.randn(n, d, generator=gen_cpu, dtype=torch.float64)
    return (u / u.norm(dim=1, keepdim=True)).float()


def _plan_prefill(wl: Workload, gen_cpu):
    """List of (b, g, tile, block) plants and the per-(b, g, tile) direction table."""
    nt = wl.nb
    plants = []
    if wl.plant == "per_tile":
        for b in range(wl.B):
            for g in range(wl.Hkv):
                for j in range(wl.n_plants + 1, nt):
                    perm = torch.randperm(j - 1, generator=gen_cpu)[:wl.n_plants] + 1
                    plants += [(b, g, j, int(x)) for x in perm]
    elif wl.plant == "every_4096":
        step = max(1, 4096 // wl.block)
        for b in range(wl.B):
            for g in range(wl.Hkv):
                for blk in range(step, nt - 1, step):
                    later = torch.randperm(nt - 1 - blk, generator=gen_cpu)[:wl.n_plants] + blk + 1
                    plants += [(b, g, int(j), blk) for j in later]
    else:
        raise ValueError(wl.plant)
    dirs = _unit_dirs(wl.B * wl.Hkv * nt, wl.d, gen_cpu).view(wl.B, wl.Hkv, nt, wl.d)
    return plants, dirs


def _add_to_blocks(K, block_vec, wl: Workload):
    """K [B,Hkv,N,d] += block_vec [B,Hkv,nb_full,d] broadcast over each full block."""
    nbf = wl.N // wl.block
    if nbf == 0:
        return
    Kv = K.view(wl.B * wl.Hkv, wl.N, wl.d)[:, :nbf * wl.block].view(wl.B * wl.Hkv, nbf, wl.block, wl.d)
    step = max(1, (1 << 26) // (wl.B * wl.Hkv * wl.block * wl.d))   # bound the fp32 temporary
    bv = block_vec.view(wl.B * wl.Hkv, nbf, 1, wl.d)
    for s in range(0, nbf, step):
        e = min(nbf, s + step)
        Kv[:, s:e] = (Kv[:, s:e].float() + bv[:, s:e]).to(K.dtype)


def make_prefill(wl: Workload, device="cpu"):
    """Q [B,Hq,N,d], K, V [B,Hkv,N,d] with the workload's plants."""
    assert wl.kind == "prefill"
    dt = wl.torch_dtype
    gen = torch.Generator(device=device).manual_seed(wl.seed)
    gen_cpu = torch.Generator().manual_seed(wl.seed + 7919)
    Q = _randn((wl.B, wl.Hq, wl.N, wl.d), gen, device, dt, wl.sigma)
    K = _randn((wl.B, wl.Hkv, wl.N, wl.d), gen, device, dt, wl.sigma)
    V = _randn((wl.B, wl.Hkv, wl.N, wl.d), gen, device, dt, wl.sigma)
    plants, dirs = _plan_prefill(wl, gen_cpu)
    if not plants:
        return Q, K, V
    beta = wl.sigma if wl.beta is None else wl.beta
    G = wl.Hq // wl.Hkv
    nt = wl.nb
    planted_tile = torch.zeros(wl.B, wl.Hkv, nt, dtype=torch.bool)
    block_vec = torch.zeros(wl.B, wl.Hkv, max(wl.N // wl.block, 1), wl.d)
    for (b, g, j, blk) in plants:
        planted_tile[b, g, j] = True
        block_vec[b, g, blk] += wl.alpha * dirs[b, g, j]
    qshift = (beta * dirs * planted_tile[..., None]).to(device)        # [B,Hkv,nt,d]
    nfull = wl.N // wl.block
    Qv = Q.view(wl.B, wl.Hkv, G, wl.N, wl.d)
    for g0 in range(G):
        for b in range(wl.B):
            main = Qv[b, :, g0, :nfull * wl.block].view(wl.Hkv, nfull, wl.block, wl.d)
            main.copy_((main.float() + qshift[b, :, :nfull, None, :]).to(dt))
            if nfull < nt:
                tail = Qv[b, :, g0, nfull * wl.block:]
                tail.copy_((tail.float() + qshift[b, :, nfull, None, :]).to(dt))
    _add_to_blocks(K, block_vec.to(device), wl)
    return Q, K, V


def make_decode(wl: Workload, device="cpu"):
    """q [B,Hq,d] (the query at position N-1) and the cache K, V [B,Hkv,N,d]."""
    assert wl.kind == "decode"
    dt = wl.torch_dtype
    gen = torch.Generator(device=device).manual_seed(wl.seed)
    gen_cpu = torch.Generator().manual_seed(wl.seed + 7919)
    q = _randn((wl.B, wl.Hq, wl.d), gen, device, dt, wl.sigma)
    K = _randn((wl.B, wl.Hkv, wl.N, wl.d), gen, device, dt, wl.sigma)
    V = _randn((wl.B, wl.Hkv, wl.N, wl.d), gen, device, dt, wl.sigma)
    local = (wl.N - 1) // wl.block
    ncand = local - 1
    n = min(wl.n_plants, max(ncand, 0))
    if n == 0:
        return q, K, V
    beta = wl.sigma if wl.beta is None else wl.beta
    G = wl.Hq // wl.Hkv
    dirs = _unit_dirs(wl.B * wl.Hkv, wl.d, gen_cpu).view(wl.B, wl.Hkv, wl.d)
    block_vec = torch.zeros(wl.B, wl.Hkv, max(wl.N // wl.block, 1), wl.d)
    for b in range(wl.B):
        for g in range(wl.Hkv):
            blocks = torch.randperm(ncand, generator=gen_cpu)[:n] + 1
            block_vec[b, g, blocks] += wl.alpha * dirs[b, g]
    qv = q.view(wl.B, wl.Hkv, G, wl.d)
    qv.copy_((qv.float() + beta * dirs.to(device)[:, :, None, :]).to(dt))
    _add_to_blocks(K, block_vec.to(device), wl)
    return q, K, V

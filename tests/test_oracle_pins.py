"""Pins for the CPU oracle: checks against what the definitions and the
mathematics fix, independent of the oracle's own code paths.

* rounding to bfloat16 -- torch's fp32->bf16 conversion, hand-made ties;
* log-sigmoid gate -- log_sigmoid(x) - log_sigmoid(-x) = x, <= 0, closed form;
* landmarks / pooled query -- constant blocks, arithmetic progressions,
  linearity, ragged tails;
* selection -- brute-force enumeration of K-subsets on tiny inputs, ties,
  one-hot closed form of the scores, always-kept sink and local blocks;
* attention -- reductions to torch's float64 scaled_dot_product_attention
  (dense causal attention when every candidate is kept; a uniform -ln 2 gate
  as an additive mask; hierarchical mode with one kept block; equal retrieval
  scores give the uniform mean of per-block outputs), empty kept sets.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import CAUSAL, GATE, HIER, LOCAL, PER_QHEAD, SINK


def sdpa(q, k, v, mask=None, causal=False, scale=None):
    """torch float64 attention on CPU. q [..., m, d], k/v [..., n, d]."""
    tq, tk, tv = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    m = None if mask is None else torch.as_tensor(mask, dtype=torch.float64)
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, is_causal=causal,
                                                           scale=scale)
    return out.numpy()


def lse_ref(q, k, scale, mask=None):
    logits = torch.as_tensor(q) @ torch.as_tensor(k).transpose(-1, -2) * scale
    if mask is not None:
        logits = logits + torch.as_tensor(mask)
    return torch.logsumexp(logits, dim=-1).numpy()


def expand_kv(K, G):
    return np.repeat(K, G, axis=1)


# ----------------------------------------------------------------------------
# rounding and gate
# ----------------------------------------------------------------------------

def test_round_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-40, 40, 20000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    got = np.array([oracle.round_bf16(float(v)) for v in x])
    assert np.array_equal(got, ref)


def test_round_bf16_ties_and_double_only_inputs():
    assert oracle.round_bf16(1 + 2 ** -8) == 1.0                 # tie -> even
    assert oracle.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6     # tie -> even (up)
    assert oracle.round_bf16(-(1 + 2 ** -8)) == -1.0
    # just above the tie, below fp32 resolution: a detour through fp32 would tie
    assert oracle.round_bf16(1 + 2 ** -8 + 2 ** -30) == 1 + 2 ** -7
    assert oracle.round_bf16(0.0) == 0.0


def test_log_sigmoid_identities():
    for x in np.linspace(-60, 60, 2401):
        a, b = oracle.log_sigmoid(x), oracle.log_sigmoid(-x)
        assert a <= 0.0
        assert abs((a - b) - x) <= 1e-12 * max(1.0, abs(x))
    assert oracle.log_sigmoid(0.0) == -math.log(2.0)
    for x in (-3.0, -0.5, 0.7, 4.0):
        assert abs(oracle.log_sigmoid(x) - math.log(1.0 / (1.0 + math.exp(-x)))) < 1e-14
    assert oracle.log_sigmoid(800.0) <= 0.0 and oracle.log_sigmoid(800.0) > -1e-300
    assert abs(oracle.log_sigmoid(-800.0) + 800.0) < 1e-9


# ----------------------------------------------------------------------------
# landmarks and pooled queries
# ----------------------------------------------------------------------------

def test_landmarks_constant_blocks_ragged_tail():
    rng = np.random.default_rng(2)
    n, d, bs = 150, 8, 32            # 5 blocks, the last one holds 22 keys
    vals = rng.integers(-8, 8, size=(5, d)).astype(np.float64) / 4
    k = np.repeat(vals, bs, axis=0)[:n]
    assert np.array_equal(oracle.landmarks(k, bs), vals)


def test_landmarks_arithmetic_progression():
    n, d, bs = 150, 3, 32
    t = np.arange(n, dtype=np.float64)
    k = np.stack([t, 2 * t + 1, -t], axis=1)
    L = oracle.landmarks(k, bs)
    for b in range(5):
        t0, t1 = b * bs, min(n, (b + 1) * bs)
        mid = (t0 + t1 - 1) / 2
        assert np.array_equal(L[b], [mid, 2 * mid + 1, -mid])


def test_landmarks_linear_and_permutation_invariant():
    rng = np.random.default_rng(3)
    n, d, bs = 256, 16, 64
    k1, k2 = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    L12 = oracle.landmarks(k1 + k2, bs)
    assert np.allclose(L12, oracle.landmarks(k1, bs) + oracle.landmarks(k2, bs), atol=1e-14)
    perm = np.concatenate([b * bs + rng.permutation(bs) for b in range(n // bs)])
    assert np.allclose(oracle.landmarks(k1[perm], bs), oracle.landmarks(k1, bs), atol=1e-14)


def test_landmarks_rounding_modes():
    x = 1 + 2 ** -8 + 2 ** -30          # exact mean of equal keys
    k = np.full((32, 2), x)
    assert oracle.landmarks(k, 32, oracle.ROUND_NONE)[0, 0] == x
    assert oracle.landmarks(k, 32, oracle.ROUND_BF16)[0, 0] == 1 + 2 ** -7
    assert oracle.landmarks(k, 32, oracle.ROUND_FP32)[0, 0] == float(np.float32(x))


def test_pool_queries_closed_form_and_clip():
    heads, n, d = 3, 10, 4
    h = np.arange(heads)[:, None, None]
    r = np.arange(n)[None, :, None]
    c = np.arange(d)[None, None, :]
    q = (h * 100 + r + c * 0.5).astype(np.float64)
    assert np.allclose(oracle.pool_queries(q, 2, 4), 100 + 3.5 + np.arange(d) * 0.5, atol=1e-13)
    assert np.allclose(oracle.pool_queries(q, 8, 5), 100 + 8.5 + np.arange(d) * 0.5, atol=1e-13)


# ----------------------------------------------------------------------------
# selection
# ----------------------------------------------------------------------------

def test_scores_one_hot_closed_form():
    rng = np.random.default_rng(4)
    d, nb = 8, 9
    lmk = rng.standard_normal((nb, d))
    qbar = np.zeros(d)
    qbar[5] = 1.75
    scale = 0.125
    sel = oracle.select(qbar, lmk, nb - 1, 3, SINK | LOCAL, scale)
    assert np.array_equal(sel["scores"], scale * (1.75 * lmk[:, 5]))


def _brute_force_kept(s, local, top_k, flags):
    first = 1 if flags & SINK else 0
    cand = list(range(first, local))
    keys = np.float32(s)
    kk = min(top_k, len(cand))
    best, best_sum = (), None
    for sub in itertools.combinations(cand, kk):
        tot = sum(float(keys[b]) for b in sub)
        if best_sum is None or tot > best_sum or (tot == best_sum and sub < best):
            best, best_sum = sub, tot
    kept = set(best)
    if flags & SINK:
        kept.add(0)
    if flags & LOCAL:
        kept.add(local)
    return sorted(kept), set(best)


@pytest.mark.parametrize("seed", range(40))
def test_selection_equals_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(1, 13))
    d = 8
    local = int(rng.integers(0, nb))
    top_k = int(rng.integers(0, 5))
    flags = int(rng.choice([0, SINK, LOCAL, SINK | LOCAL])) | int(rng.choice([0, GATE]))
    qbar = rng.standard_normal(d)
    lmk = rng.standard_normal((nb, d))
    scale = 1 / math.sqrt(d)
    sel = oracle.select(qbar, lmk, local, top_k, flags, scale)
    s = sel["scores"]
    kept, chosen = _brute_force_kept(s, local, top_k, flags)
    c = sel["count"]
    assert c == len(kept)
    assert list(sel["idx"][:c]) == kept
    for i, b in enumerate(kept):
        assert sel["sc"][i] == s[b]
        if (flags & GATE) and b in chosen:
            x = s[b] - s[local]
            assert abs(sel["gate"][i] - math.log(1 / (1 + math.exp(-x)))) < 1e-12
        else:
            assert sel["gate"][i] == 0.0
    # gap over the fp32 decision keys
    first = 1 if flags & SINK else 0
    keys = np.sort(np.float32(s[first:local]).astype(np.float64))[::-1]
    if top_k > 0 and len(keys) > top_k:
        a, b = keys[top_k - 1], keys[top_k]
        assert sel["rel_gap"] == pytest.approx((a - b) / max(abs(a), 1e-30), rel=1e-12, abs=0)
    else:
        assert sel["rel_gap"] == math.inf


def test_selection_ties_prefer_lower_index():
    d = 4
    lmk = np.full((8, d), -1.0)
    lmk[[2, 4, 6]] = 1.0        # three equal best candidates
    qbar = np.ones(d)
    sel = oracle.select(qbar, lmk, 7, 2, SINK | LOCAL, 0.5)
    assert list(sel["idx"][:sel["count"]]) == [0, 2, 4, 7]
    assert sel["rel_gap"] == 0.0


def test_selection_forced_blocks_and_small_candidate_sets():
    rng = np.random.default_rng(5)
    lmk = rng.standard_normal((6, 4))
    q = rng.standard_normal(4)
    assert list(oracle.select(q, lmk, 0, 4, SINK | LOCAL, 1.0)["idx"][:1]) == [0]
    assert oracle.select(q, lmk, 0, 4, SINK | LOCAL, 1.0)["count"] == 1
    assert oracle.select(q, lmk, 0, 4, 0, 1.0)["count"] == 0
    sel = oracle.select(q, lmk, 3, 8, SINK | LOCAL, 1.0)   # fewer candidates than K
    assert list(sel["idx"][:sel["count"]]) == [0, 1, 2, 3]
    sel = oracle.select(q, lmk, 5, 0, SINK | LOCAL, 1.0)
    assert list(sel["idx"][:sel["count"]]) == [0, 5]


# ----------------------------------------------------------------------------
# attention reductions
# ----------------------------------------------------------------------------

SHAPES = [
    (1, 2, 2, 96, 16, 16),     # B, Hq, Hkv, N, d, block
    (2, 4, 2, 200, 8, 32),     # GQA 2:1, ragged tail
    (1, 6, 3, 64, 16, 64),     # a single block
    (1, 3, 1, 130, 8, 16),     # GQA 3:1, 2-key tail
]


def _rand_qkv(seed, B, Hq, Hkv, N, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, Hq, N, d)), rng.standard_normal((B, Hkv, N, d)),
            rng.standard_normal((B, Hkv, N, d)))


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("sink", [True, False])
def test_prefill_keep_all_is_dense_causal_attention(shape, sink):
    B, Hq, Hkv, N, d, bs = shape
    Q, K, V = _rand_qkv(7, B, Hq, Hkv, N, d)
    nb = (N + bs - 1) // bs
    flags = (SINK if sink else 0) | LOCAL | CAUSAL
    out = oracle.prefill(Q, K, V, bs, nb, flags, round_mode=oracle.ROUND_NONE, threads=1)
    G = Hq // Hkv
    ref = sdpa(Q, expand_kv(K, G), expand_kv(V, G), causal=True)
    assert np.abs(out["O"] - ref).max() <= 1e-12
    causal = np.triu(np.full((N, N), -np.inf), 1)
    lref = lse_ref(Q, expand_kv(K, G), 1 / math.sqrt(d), causal)
    assert np.abs(out["LSE"] - lref).max() <= 1e-12


@pytest.mark.parametrize("shape", SHAPES[:2])
def test_prefill_per_qhead_keep_all_is_dense(shape):
    B, Hq, Hkv, N, d, bs = shape
    Q, K, V = _rand_qkv(8, B, Hq, Hkv, N, d)
    nb = (N + bs - 1) // bs
    out = oracle.prefill(Q, K, V, bs, nb, SINK | LOCAL | CAUSAL | PER_QHEAD, round_mode=oracle.ROUND_NONE)
    G = Hq // Hkv
    ref = sdpa(Q, expand_kv(K, G), expand_kv(V, G), causal=True)
    assert np.abs(out["O"] - ref).max() <= 1e-12
    assert out["idx"].shape[1] == Hq


def _identical_block_keys(rng, B, Hkv, nb, bs, d):
    base = rng.standard_normal((B, Hkv, bs, d))
    return np.tile(base, (1, 1, nb, 1))


def test_prefill_uniform_gate_is_minus_ln2_mask():
    B, Hq, Hkv, d, bs, nb = 1, 4, 2, 8, 16, 6
    N = nb * bs
    rng = np.random.default_rng(9)
    Q = rng.standard_normal((B, Hq, N, d))
    K = _identical_block_keys(rng, B, Hkv, nb, bs, d)
    V = rng.standard_normal((B, Hkv, N, d))
    flags = SINK | LOCAL | GATE | CAUSAL
    out = oracle.prefill(Q, K, V, bs, nb, flags, round_mode=oracle.ROUND_NONE)
    # every landmark is the same, so every selected block gets log_sigmoid(0)
    mask = np.full((N, N), -np.inf)
    for i in range(N):
        j = i // bs
        for t in range(i + 1):
            b = t // bs
            mask[i, t] = 0.0 if b in (0, j) else -math.log(2.0)
    G = Hq // Hkv
    ref = sdpa(Q, expand_kv(K, G), expand_kv(V, G), mask=mask)
    assert np.abs(out["O"] - ref).max() <= 1e-12
    lref = lse_ref(Q, expand_kv(K, G), 1 / math.sqrt(d), mask)
    assert np.abs(out["LSE"] - lref).max() <= 1e-12


def test_prefill_gate_as_additive_mask_random_scores():
    B, Hq, Hkv, N, d, bs = 1, 4, 2, 112, 8, 16
    Q, K, V = _rand_qkv(10, B, Hq, Hkv, N, d)
    nb = N // bs
    flags = SINK | LOCAL | GATE | CAUSAL
    out = oracle.prefill(Q, K, V, bs, nb, flags, round_mode=oracle.ROUND_NONE)
    G = Hq // Hkv
    scale = 1 / math.sqrt(d)
    for g in range(Hkv):
        Lg = K[0, g].reshape(nb, bs, d).mean(axis=1)
        for j in range(nb):
            qbar = Q[0, g * G:(g + 1) * G, j * bs:(j + 1) * bs].reshape(-1, d).mean(axis=0)
            s = scale * (Lg @ qbar)
            gate_of = {b: (0.0 if b in (0, j) else math.log(1 / (1 + math.exp(-(s[b] - s[j])))))
                       for b in range(j + 1)}
            rows = slice(j * bs, (j + 1) * bs)
            mask = np.full((bs, N), -np.inf)
            for r in range(bs):
                i = j * bs + r
                for t in range(i + 1):
                    mask[r, t] = gate_of[t // bs]
            for h in range(g * G, (g + 1) * G):
                ref = sdpa(Q[0, h, rows], K[0, g], V[0, g], mask=mask)
                assert np.abs(out["O"][0, h, rows] - ref).max() <= 1e-11


def test_prefill_empty_kept_set():
    B, Hq, Hkv, N, d, bs = 1, 2, 1, 64, 8, 16
    Q, K, V = _rand_qkv(11, B, Hq, Hkv, N, d)
    out = oracle.prefill(Q, K, V, bs, 2, CAUSAL | GATE)
    assert np.all(out["O"][0, :, :bs] == 0.0)
    assert np.all(out["LSE"][0, :, :bs] == -np.inf)
    assert np.all(out["count"][0, :, 0] == 0)
    assert np.all(np.isfinite(out["LSE"][0, :, bs:]))


def test_hier_single_kept_block_is_plain_attention():
    B, Hq, Hkv, N, d, bs = 1, 4, 2, 96, 8, 16
    Q, K, V = _rand_qkv(12, B, Hq, Hkv, N, d)
    out = oracle.prefill(Q, K, V, bs, 1, HIER | CAUSAL, round_mode=oracle.ROUND_NONE)
    G = Hq // Hkv
    for g in range(Hkv):
        assert out["count"][0, g, 0] == 0
        for j in range(1, N // bs):
            assert out["count"][0, g, j] == 1
            b = int(out["idx"][0, g, j, 0])
            assert 0 <= b < j
            rows = slice(j * bs, (j + 1) * bs)
            keys = slice(b * bs, (b + 1) * bs)
            for h in range(g * G, (g + 1) * G):
                ref = sdpa(Q[0, h, rows], K[0, g, keys], V[0, g, keys])
                assert np.abs(out["O"][0, h, rows] - ref).max() <= 1e-12
                assert np.allclose(out["LSE"][0, h, rows], out["sc"][0, g, j, 0], rtol=0, atol=1e-15)
    assert np.all(out["O"][0, :, :bs] == 0.0)


def test_hier_sink_only_gives_attention_over_block0():
    B, Hq, Hkv, N, d, bs = 1, 2, 2, 64, 8, 16
    Q, K, V = _rand_qkv(13, B, Hq, Hkv, N, d)
    out = oracle.prefill(Q, K, V, bs, 0, HIER | SINK | CAUSAL, round_mode=oracle.ROUND_NONE)
    for h in range(Hq):
        ref0 = sdpa(Q[0, h, :bs], K[0, h, :bs], V[0, h, :bs], causal=True)
        assert np.abs(out["O"][0, h, :bs] - ref0).max() <= 1e-12
        ref = sdpa(Q[0, h, bs:], K[0, h, :bs], V[0, h, :bs])
        assert np.abs(out["O"][0, h, bs:] - ref).max() <= 1e-12


def test_hier_equal_scores_give_uniform_mean():
    B, Hq, Hkv, d, bs, nb = 1, 2, 1, 8, 16, 5
    N = nb * bs
    rng = np.random.default_rng(14)
    Q = rng.standard_normal((B, Hq, N, d))
    K = _identical_block_keys(rng, B, Hkv, nb, bs, d)
    V = rng.standard_normal((B, Hkv, N, d))
    out = oracle.prefill(Q, K, V, bs, nb, HIER | SINK | LOCAL | CAUSAL, round_mode=oracle.ROUND_NONE)
    for j in range(nb):
        rows = slice(j * bs, (j + 1) * bs)
        for h in range(Hq):
            parts = []
            for b in range(j + 1):
                keys = slice(b * bs, (b + 1) * bs)
                parts.append(sdpa(Q[0, h, rows], K[0, 0, keys], V[0, 0, keys], causal=(b == j)))
            ref = np.mean(parts, axis=0)
            assert np.abs(out["O"][0, h, rows] - ref).max() <= 1e-12
            s0 = out["sc"][0, 0, j, 0]
            assert np.allclose(out["LSE"][0, h, rows], s0 + math.log(j + 1), atol=1e-12, rtol=0)


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("N", [64, 100, 129])
def test_decode_keep_all_is_dense_attention(N):
    B, Hq, Hkv, d, bs = 2, 4, 2, 8, 16
    rng = np.random.default_rng(15)
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    nb = (N + bs - 1) // bs
    out = oracle.decode(q, K, V, bs, nb, SINK | LOCAL | CAUSAL | GATE * 0, round_mode=oracle.ROUND_NONE)
    G = Hq // Hkv
    ref = sdpa(q[:, :, None, :], expand_kv(K, G), expand_kv(V, G))[:, :, 0]
    assert np.abs(out["O"] - ref).max() <= 1e-12
    lref = lse_ref(q[:, :, None, :], expand_kv(K, G), 1 / math.sqrt(d))[:, :, 0]
    assert np.abs(out["LSE"] - lref).max() <= 1e-12
    assert np.all(out["idx"][:, :, 0] == 0)
    assert np.all(out["count"] == nb)


def test_decode_hier_single_block_and_local_partial():
    B, Hq, Hkv, d, bs, N = 1, 2, 1, 8, 16, 71       # local block 4 holds 7 keys
    rng = np.random.default_rng(16)
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    out = oracle.decode(q, K, V, bs, 0, HIER | LOCAL | CAUSAL, round_mode=oracle.ROUND_NONE)
    assert list(out["idx"][0, 0, :1]) == [4]
    for h in range(Hq):
        ref = sdpa(q[0, h][None], K[0, 0, 64:], V[0, 0, 64:])[0]
        assert np.abs(out["O"][0, h] - ref).max() <= 1e-12
    # its landmark averages only the 7 keys that exist
    assert np.allclose(out["L"][0, 0, 4], K[0, 0, 64:].mean(axis=0), atol=1e-14, rtol=0)


# ----------------------------------------------------------------------------
# hierarchical weighting with unequal retrieval scores
# ----------------------------------------------------------------------------

def _hier_closed_form(q_rows, K, V, bs, kept, scores, local, qpos):
    """HiLS combination written out with torch float64: every kept block is
    attended on its own (causal inside the local block), and the per-block
    outputs are mixed with softmax(scores); LSE = logsumexp(scores)."""
    s = torch.as_tensor(np.asarray(scores, dtype=np.float64))
    w = torch.softmax(s, dim=0).numpy()
    out = np.zeros_like(q_rows)
    for wb, b in zip(w, kept):
        t0, t1 = b * bs, min((b + 1) * bs, K.shape[0])
        mask = None
        if b == local:
            pos = np.arange(t0, t1)
            mask = np.where(pos[None, :] <= np.asarray(qpos)[:, None], 0.0, -np.inf)
        out += wb * sdpa(q_rows, K[t0:t1], V[t0:t1], mask=mask)
    return out, float(torch.logsumexp(s, dim=0))


def _fixed_list(kept, scores, top_k):
    cap = top_k + 2
    idx = np.full(cap, -1, dtype=np.int32)
    sc = np.zeros(cap)
    idx[:len(kept)] = kept
    sc[:len(kept)] = scores
    return {"idx": idx, "sc": sc, "gate": np.zeros(cap), "count": len(kept), "rel_gap": np.inf}


@pytest.mark.parametrize("scores", [[0.3, -1.2, 2.0], [0.5, 1.5, 3.0], [-4.0, 0.0, -0.5]])
def test_hier_unequal_scores_mix_by_softmax_prefill(scores):
    B, Hq, Hkv, d, bs, N = 1, 2, 1, 8, 16, 80
    j, kept = 4, [0, 2, 4]
    Q, K, V = _rand_qkv(31, B, Hq, Hkv, N, d)
    out = oracle.prefill(Q, K, V, bs, 1, HIER | SINK | LOCAL | CAUSAL, round_mode=oracle.ROUND_NONE,
                         units=[(0, 0, j)], sel_override=lambda b, s, jj: _fixed_list(kept, scores, 1))
    rows = slice(j * bs, (j + 1) * bs)
    qpos = np.arange(j * bs, (j + 1) * bs)
    for h in range(Hq):
        ref, lse = _hier_closed_form(Q[0, h, rows], K[0, 0], V[0, 0], bs, kept, scores, j, qpos)
        assert np.abs(out["O"][0, h, rows] - ref).max() <= 1e-12
        assert np.abs(out["LSE"][0, h, rows] - lse).max() <= 1e-12
    if min(scores) > 0:
        # the linear reading w_b = s_b / sum(s) gives a clearly different output here
        lin = np.asarray(scores) / np.sum(scores)
        parts = []
        for b in kept:
            t0 = b * bs
            mask = None if b != j else np.where(np.arange(t0, t0 + bs)[None, :] <= qpos[:, None], 0.0, -np.inf)
            parts.append(sdpa(Q[0, 0, rows], K[0, 0, t0:t0 + bs], V[0, 0, t0:t0 + bs], mask=mask))
        alt = sum(wb * p for wb, p in zip(lin, parts))
        assert np.abs(out["O"][0, 0, rows] - alt).max() > 1e-2


def test_hier_unequal_scores_mix_by_softmax_decode():
    B, Hq, Hkv, d, bs, N = 1, 4, 2, 8, 16, 75          # local block 4 holds 11 keys
    kept, scores = [0, 1, 3, 4], [1.1, -0.7, 2.4, 0.2]
    rng = np.random.default_rng(32)
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    out = oracle.decode(q, K, V, bs, 2, HIER | SINK | LOCAL | CAUSAL, round_mode=oracle.ROUND_NONE,
                        sel_override=lambda b, s: _fixed_list(kept, scores, 2))
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G
        ref, lse = _hier_closed_form(q[0, h][None], K[0, g], V[0, g], bs, kept, scores, 4, [N - 1])
        assert np.abs(out["O"][0, h] - ref[0]).max() <= 1e-12
        assert abs(out["LSE"][0, h] - lse) <= 1e-12


def test_hier_own_selection_mixes_by_softmax_of_reported_scores():
    """With the oracle's own lists (random scores, every tile), the output is
    the softmax(sc)-weighted sum of per-block attention."""
    B, Hq, Hkv, d, bs, N = 1, 2, 1, 8, 16, 112
    Q, K, V = _rand_qkv(33, B, Hq, Hkv, N, d)
    out = oracle.prefill(Q, K, V, bs, 3, HIER | SINK | LOCAL | CAUSAL, round_mode=oracle.ROUND_NONE)
    for j in range(N // bs):
        c = int(out["count"][0, 0, j])
        kept = [int(x) for x in out["idx"][0, 0, j, :c]]
        scores = out["sc"][0, 0, j, :c]
        assert len(set(np.round(scores, 12))) == c or c <= 1
        rows = slice(j * bs, (j + 1) * bs)
        qpos = np.arange(j * bs, (j + 1) * bs)
        for h in range(Hq):
            ref, lse = _hier_closed_form(Q[0, h, rows], K[0, 0], V[0, 0], bs, kept, scores, j, qpos)
            assert np.abs(out["O"][0, h, rows] - ref).max() <= 1e-12
            assert np.abs(out["LSE"][0, h, rows] - lse).max() <= 1e-12

"""Backward pass of gated block-sparse prefill -- TEST INFRASTRUCTURE (oracle).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU leg may
import this module; it shares no code with the CUDA library.  Plain numpy in
float64, one unit (batch, kv-head, query tile) at a time.

What is differentiated ([SAS] "Как это применить": the selector's scores enter
the attention as a gate inside the softmax, which is what lets its gradient
reach the selector; "Ключевые факты": the top-K choice itself is hard).  With
the kept lists held fixed:

  qbar   = mean of the unit's query rows (all heads of the kv-head group, all
           rows of the tile);
  L_b    = mean of the keys of block b (the landmarks; the forward may round
           them to the key precision -- the backward treats that rounding as
           the identity);
  s_c    = scale * <qbar, L_{idx_c}> for every list entry c; s_loc is the local
           block's entry (the list's last one);
  g_c    = log_sigmoid(s_c - s_loc) for selected entries, 0 for the forced sink
           and local blocks;
  z_it   = scale * <q_i, k_t> + g_c(t) over the visible keys of the list;
  O_i    = softmax(z_i) V.

Given dO, the gradients are the textbook softmax-attention ones,
  P = exp(z - lse),  D_i = <dO_i, O_i>,  dZ = P * (dO V^T - D),
  dQ = scale dZ K,   dK = scale dZ^T Q,  dV = P^T dO,
  dg_c = sum of dZ over the rows and the keys of entry c,
followed by the gate and the selector:
  ds_c += dg_c * sigmoid(-(s_c - s_loc)),   ds_loc -= dg_c * sigmoid(-(s_c - s_loc)),
  dqbar = scale * sum_c ds_c L_{idx_c},     dL_{idx_c} += scale * ds_c * qbar,
  dQ[rows of the unit] += dqbar / R,        dK[keys of block b] += dL_b / n_b.
Pinned by central finite differences of ``forward_fixed`` (tests).
"""
from __future__ import annotations

import numpy as np

from . import CAUSAL, GATE, HIER, LOCAL, PER_QHEAD, SINK, default_scale


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _log_sigmoid(x):
    return -np.logaddexp(0.0, -x)


def _block_rows(b: int, block: int, N: int):
    return b * block, min((b + 1) * block, N)


def _unit_pieces(Q, K, b, g, j, block, G, L=None):
    """Rows of a unit, their positions, its pooled query and the landmarks used."""
    N, d = Q.shape[2], Q.shape[3]
    r0, r1 = _block_rows(j, block, N)
    rows = Q[b, g * G:(g + 1) * G, r0:r1].reshape(-1, d)
    qpos = np.tile(np.arange(r0, r1), G)
    qbar = rows.mean(axis=0)
    if L is None:
        nb = (N + block - 1) // block
        L = np.stack([K[b, g, slice(*_block_rows(x, block, N))].mean(axis=0) for x in range(nb)])
    return rows, qpos, qbar, L, (r0, r1)


def _scores_and_gates(qbar, L, idx, j, flags, scale, sc=None):
    if sc is None:
        sc = scale * (L[idx] @ qbar)
        s_loc = scale * float(L[j] @ qbar)
    else:
        sc = np.asarray(sc, np.float64)
        s_loc = float(sc[idx == j][0]) if np.any(idx == j) else scale * float(L[j] @ qbar)
    forced = ((idx == 0) & bool(flags & SINK)) | ((idx == j) & bool(flags & LOCAL))
    gated = (~forced) & bool(flags & GATE)
    gate = np.where(gated, _log_sigmoid(sc - s_loc), 0.0)
    return sc, s_loc, gate, gated


def _keys_and_mask(idx, qpos, j, N, block, flags):
    """Concatenated key positions of the list, entry of each key, visibility [R, T]."""
    keys, ent = [], []
    for c, blk in enumerate(idx):
        t0, t1 = _block_rows(int(blk), block, N)
        keys.extend(range(t0, t1))
        ent.extend([c] * (t1 - t0))
    keys = np.asarray(keys, dtype=np.int64)
    ent = np.asarray(ent, dtype=np.int64)
    vis = np.ones((len(qpos), len(keys)), dtype=bool)
    if flags & CAUSAL:
        in_local = idx[ent] == j
        vis &= ~(in_local[None, :] & (keys[None, :] > qpos[:, None]))
    return keys, ent, vis


def _check(flags, lists):
    if flags & (HIER | PER_QHEAD):
        raise ValueError("backward covers gated (or plain) attention with per-kv-head lists")


def forward_fixed(Q, K, V, block: int, flags: int, lists: dict, scale: float | None = None, L=None,
                  score_override: dict | None = None):
    """Forward with the kept lists fixed: every score recomputed from Q and K.

    lists: {(b, g, j): ascending block ids}.  ``score_override``: optional
    {(b, g, j): per-entry scores} used instead of recomputing them (the local
    entry's score is then s_loc).  Returns O [B,Hq,N,d] and LSE [B,Hq,N]
    (rows of units not listed stay 0 / -inf)."""
    _check(flags, lists)
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    B, Hq, N, d = Q.shape
    G = Hq // K.shape[1]
    scale = default_scale(d) if scale is None else scale
    O = np.zeros_like(Q)
    LSE = np.full((B, Hq, N), -np.inf)
    for (b, g, j), idx in lists.items():
        idx = np.asarray(idx, dtype=np.int64)
        Lbg = None if L is None else np.asarray(L[b, g], np.float64)
        rows, qpos, qbar, Lbg, (r0, r1) = _unit_pieces(Q, K, b, g, j, block, G, Lbg)
        so = None if score_override is None else score_override[(b, g, j)]
        sc, s_loc, gate, _ = _scores_and_gates(qbar, Lbg, idx, j, flags, scale, so)
        keys, ent, vis = _keys_and_mask(idx, qpos, j, N, block, flags)
        z = scale * rows @ K[b, g, keys].T + gate[ent][None, :]
        z = np.where(vis, z, -np.inf)
        m = z.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.exp(z - m)
        den = e.sum(axis=1, keepdims=True)
        o = (e / np.where(den > 0, den, 1.0)) @ V[b, g, keys]
        lse = np.where(den[:, 0] > 0, m[:, 0] + np.log(np.where(den[:, 0] > 0, den[:, 0], 1.0)), -np.inf)
        O[b, g * G:(g + 1) * G, r0:r1] = o.reshape(G, r1 - r0, d)
        LSE[b, g * G:(g + 1) * G, r0:r1] = lse.reshape(G, r1 - r0)
    return O, LSE


def backward(Q, K, V, dO, block: int, flags: int, lists: dict, scale: float | None = None, L=None,
             selector: bool = True, score_override: dict | None = None):
    """Gradients of sum(O * dO) for ``forward_fixed``.

    Returns dict(dQ, dK, dV, dscore, dgate): dscore / dgate are {(b, g, j):
    per-entry arrays}.  ``selector=False`` stops at the scores (no pooled-query
    / landmark chain into dQ, dK); it is implied by ``score_override``."""
    selector = selector and score_override is None
    _check(flags, lists)
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    dO = np.asarray(dO, np.float64)
    B, Hq, N, d = Q.shape
    G = Hq // K.shape[1]
    scale = default_scale(d) if scale is None else scale
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dscore, dgate = {}, {}
    for (b, g, j), idx in lists.items():
        idx = np.asarray(idx, dtype=np.int64)
        Lbg = None if L is None else np.asarray(L[b, g], np.float64)
        rows, qpos, qbar, Lbg, (r0, r1) = _unit_pieces(Q, K, b, g, j, block, G, Lbg)
        so = None if score_override is None else score_override[(b, g, j)]
        sc, s_loc, gate, gated = _scores_and_gates(qbar, Lbg, idx, j, flags, scale, so)
        keys, ent, vis = _keys_and_mask(idx, qpos, j, N, block, flags)
        Kt, Vt = K[b, g, keys], V[b, g, keys]
        z = scale * rows @ Kt.T + gate[ent][None, :]
        z = np.where(vis, z, -np.inf)
        m = z.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.exp(z - m)
        den = e.sum(axis=1, keepdims=True)
        P = e / np.where(den > 0, den, 1.0)
        o = P @ Vt
        do = dO[b, g * G:(g + 1) * G, r0:r1].reshape(-1, d)
        D = (do * o).sum(axis=1, keepdims=True)
        dZ = P * (do @ Vt.T - D)
        dq = scale * dZ @ Kt
        np.add.at(dK[b, g], keys, scale * dZ.T @ rows)
        np.add.at(dV[b, g], keys, P.T @ do)
        dg = np.zeros(len(idx))
        np.add.at(dg, ent, dZ.sum(axis=0))
        ds = np.zeros(len(idx))
        w = np.where(gated, dg * _sigmoid(-(sc - s_loc)), 0.0)
        ds += w
        loc = np.nonzero(idx == j)[0]
        if len(loc):
            ds[loc[0]] -= w.sum()
        dgate[(b, g, j)] = dg
        dscore[(b, g, j)] = ds
        if selector:
            dqbar = scale * (ds @ Lbg[idx])
            dq = dq + dqbar[None, :] / rows.shape[0]
            for c, blk in enumerate(idx):
                t0, t1 = _block_rows(int(blk), block, N)
                dK[b, g, t0:t1] += scale * ds[c] * qbar[None, :] / (t1 - t0)
        dQ[b, g * G:(g + 1) * G, r0:r1] += dq.reshape(G, r1 - r0, d)
    return {"dQ": dQ, "dK": dK, "dV": dV, "dscore": dscore, "dgate": dgate}


def lists_from_selection(out: dict) -> dict:
    """{(b, g, j): kept block ids} from ``oracle.prefill``'s selection output."""
    res = {}
    idx, cnt = out["idx"], out["count"]
    B, H, nb = cnt.shape
    for b in range(B):
        for g in range(H):
            for j in range(nb):
                c = int(cnt[b, g, j])
                if c > 0:
                    res[(b, g, j)] = np.asarray(idx[b, g, j, :c], dtype=np.int64)
    return res

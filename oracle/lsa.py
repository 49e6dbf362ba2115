"""Flat clustered index of Latent Sparse Attention -- TEST INFRASTRUCTURE (oracle).

Only ``tests/`` (and the CPU legs of ``bench.py``) may import this module; it
shares no code with the CUDA library.  Plain numpy in float64.

What it computes (the Latent Sparse Attention post, section "Индекс перестаёт
перебирать весь контекст"), in the raw key space (the post's learned latent
projections need trained weights and are not modelled):

  1. items: the keys are pooled in groups of ``pool`` adjacent positions
     (mean of the group's keys);
  2. segments of ``seg`` consecutive items are clustered once they are
     complete -- their composition is frozen from then on -- by Ward's
     agglomerative method into ``clusters_per_seg`` clusters;
  3. the index keeps, per cluster, its centre (mean of its items) and the
     table of token positions of its items;
  4. a query is scored against every centre (the flat variant: all centres
     are scanned), scale * <q, centre>; the ``top_clusters`` best, by
     (score desc, cluster id asc), are expanded back to their positions;
  5. the first ``sink`` positions and the last ``window`` positions are always
     added; plain softmax attention over the union (causal: positions <= the
     query's).

Readings where the post is silent: items are means of ``pool`` keys (the tail
group may be shorter); Ward's merge order breaks ties by the lower cluster pair
(smallest first id, then second); a cluster's centre is the mean of its items;
positions of the incomplete last segment are reachable only through the
recent window.
"""
from __future__ import annotations

import numpy as np

from . import default_scale


def ward_merges(X: np.ndarray, n_clusters: int, weights=None) -> np.ndarray:
    """Ward's agglomerative clustering of the rows of X down to n_clusters.

    Returns labels [len(X)] in 0..n_clusters-1, numbered in order of each
    cluster's first item.  Every step merges the two clusters A, B with the
    smallest increase of the within-cluster sum of squares,
        |A| |B| / (|A| + |B|) * ||c_A - c_B||^2,
    ties to the pair with the lowest (first id, second id).  ``weights``: the
    mass of each row (default 1), so that rows standing for groups of points
    merge as those groups would; |A| is then the summed mass."""
    X = np.asarray(X, np.float64)
    n = X.shape[0]
    n_clusters = max(1, min(n_clusters, n))
    w = np.ones(n) if weights is None else np.asarray(weights, np.float64)
    members = {i: [i] for i in range(n)}
    cent = {i: X[i].copy() for i in range(n)}
    mass = {i: float(w[i]) for i in range(n)}
    while len(members) > n_clusters:
        ids = sorted(members)
        best = None
        for ai, a in enumerate(ids):
            for b in ids[ai + 1:]:
                na, nb = mass[a], mass[b]
                diff = cent[a] - cent[b]
                cost = na * nb / (na + nb) * float(diff @ diff)
                if best is None or cost < best[0]:
                    best = (cost, a, b)
        _, a, b = best
        na, nb = mass[a], mass[b]
        cent[a] = (na * cent[a] + nb * cent[b]) / (na + nb)
        mass[a] = na + nb
        members[a] = sorted(members[a] + members[b])
        del members[b], cent[b], mass[b]
    labels = np.empty(n, dtype=np.int64)
    for new, cid in enumerate(sorted(members, key=lambda c: members[c][0])):
        labels[members[cid]] = new
    return labels


def build_index(K: np.ndarray, pool: int, seg: int, clusters_per_seg: int) -> dict:
    """Index of one (batch, kv-head): K [n, d].

    Returns dict(centres [C, d], positions: list of position arrays, items
    [n_items, d], complete_segments)."""
    K = np.asarray(K, np.float64)
    n, d = K.shape
    n_items = (n + pool - 1) // pool
    items = np.stack([K[i * pool:min((i + 1) * pool, n)].mean(axis=0) for i in range(n_items)]) if n_items else \
        np.zeros((0, d))
    complete = n // (pool * seg)          # segments whose seg * pool keys all exist
    centres, positions = [], []
    for sg in range(complete):
        it = items[sg * seg:(sg + 1) * seg]
        lab = ward_merges(it, clusters_per_seg)
        for c in range(lab.max() + 1):
            mem = np.nonzero(lab == c)[0]
            centres.append(it[mem].mean(axis=0))
            pos = np.concatenate([np.arange((sg * seg + m) * pool, (sg * seg + m + 1) * pool) for m in mem])
            positions.append(pos)
    centres = np.stack(centres) if centres else np.zeros((0, d))
    return {"centres": centres, "positions": positions, "items": items, "complete_segments": complete}


def select_clusters(index: dict, q: np.ndarray, top_clusters: int, scale: float) -> np.ndarray:
    """Ids of the best clusters for query q (flat scan of every centre)."""
    C = index["centres"].shape[0]
    if C == 0 or top_clusters <= 0:
        return np.zeros(0, dtype=np.int64)
    s = scale * (index["centres"] @ np.asarray(q, np.float64))
    order = sorted(range(C), key=lambda c: (-s[c], c))
    return np.asarray(sorted(order[:top_clusters]), dtype=np.int64)


def kept_positions(index: dict, clusters, n: int, qpos: int, sink: int, window: int) -> np.ndarray:
    """Union of the clusters' positions, the first `sink` and the last `window`
    positions up to and including qpos, ascending."""
    keep = set()
    for c in clusters:
        keep.update(int(t) for t in index["positions"][c])
    keep.update(range(0, min(sink, n)))
    keep.update(range(max(0, qpos + 1 - window), qpos + 1))
    return np.asarray(sorted(t for t in keep if t <= qpos and t < n), dtype=np.int64)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, positions: np.ndarray, scale: float):
    """Plain softmax attention of one query over the given key positions."""
    q = np.asarray(q, np.float64)
    if len(positions) == 0:
        return np.zeros(V.shape[1]), -np.inf
    z = scale * (np.asarray(K, np.float64)[positions] @ q)
    m = z.max()
    e = np.exp(z - m)
    o = e @ np.asarray(V, np.float64)[positions] / e.sum()
    return o, m + np.log(e.sum())


def decode(q, K, V, pool: int, seg: int, clusters_per_seg: int, top_clusters: int, sink: int, window: int,
           scale: float | None = None) -> dict:
    """One query per (batch, head) at the last position, through the flat index.

    q [B, Hq, d], K, V [B, Hkv, n, d]; the kv-group's query heads share the
    index and are pooled (mean) to pick clusters."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    B, Hq, d = q.shape
    Hkv, n = K.shape[1], K.shape[2]
    G = Hq // Hkv
    scale = default_scale(d) if scale is None else scale
    O = np.zeros((B, Hq, d))
    LSE = np.zeros((B, Hq))
    kept = {}
    for b in range(B):
        for g in range(Hkv):
            idx = build_index(K[b, g], pool, seg, clusters_per_seg)
            qbar = q[b, g * G:(g + 1) * G].mean(axis=0)
            cl = select_clusters(idx, qbar, top_clusters, scale)
            pos = kept_positions(idx, cl, n, n - 1, sink, window)
            kept[(b, g)] = (cl, pos)
            for h in range(g * G, (g + 1) * G):
                O[b, h], LSE[b, h] = attend(q[b, h], K[b, g], V[b, g], pos, scale)
    return {"O": O, "LSE": LSE, "kept": kept}


# ---------------------------------------------------------------------------
# Tree variant (same section of the post: the clusters are combined into a
# hierarchy that a beam search walks, keeping a few good branches per level,
# so a query needs a number of comparisons that grows logarithmically).
# Reading: the flat index's clusters are the leaves; every level above is a
# Ward clustering of the level below, weighted by the items each node holds,
# into ceil(n / fanout) nodes; a node's centre is the mean of all its items.
# ---------------------------------------------------------------------------

def build_tree(index: dict, fanout: int) -> list:
    """Levels from the leaves up: level 0 = the flat clusters.  Each level is
    dict(centres, mass, children) with children = lists of ids one level down.
    A fan-out below 2 would never shrink a level: it is rejected."""
    if int(fanout) < 2:
        raise ValueError(f"fanout must be at least 2, got {fanout}")
    cent = np.asarray(index["centres"], np.float64)
    mass = np.asarray([len(p) for p in index["positions"]], np.float64)
    levels = [{"centres": cent, "mass": mass, "children": [[c] for c in range(len(cent))]}]
    while len(levels[-1]["centres"]) > fanout:
        below = levels[-1]
        n = len(below["centres"])
        lab = ward_merges(below["centres"], (n + fanout - 1) // fanout, weights=below["mass"])
        kids = [list(np.nonzero(lab == c)[0]) for c in range(lab.max() + 1)]
        m = np.asarray([below["mass"][k].sum() for k in kids])
        c = np.stack([(below["mass"][k][:, None] * below["centres"][k]).sum(axis=0) / below["mass"][k].sum()
                      for k in kids])
        levels.append({"centres": c, "mass": m, "children": kids})
    return levels


def tree_select(levels: list, q: np.ndarray, beam: int, top_clusters: int, scale: float):
    """Beam search from the top level down; returns (leaf ids ascending, number
    of centre comparisons).  At each level the `beam` best nodes by (score
    desc, id asc) are kept and expanded; at the leaves the `top_clusters`
    best of the reached ones are returned."""
    q = np.asarray(q, np.float64)
    if len(levels) == 0 or len(levels[0]["centres"]) == 0 or top_clusters <= 0:
        return np.zeros(0, dtype=np.int64), 0
    top = len(levels) - 1
    frontier = list(range(len(levels[top]["centres"])))
    compared = 0
    for lv in range(top, -1, -1):
        s = scale * (levels[lv]["centres"][frontier] @ q)
        compared += len(frontier)
        order = sorted(range(len(frontier)), key=lambda i: (-s[i], frontier[i]))
        keep = [frontier[i] for i in order[:(top_clusters if lv == 0 else beam)]]
        if lv == 0:
            return np.asarray(sorted(keep), dtype=np.int64), compared
        frontier = sorted(c for node in keep for c in levels[lv]["children"][node])
    return np.zeros(0, dtype=np.int64), compared

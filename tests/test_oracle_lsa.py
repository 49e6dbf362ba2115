"""Pins of the flat clustered-index oracle (``oracle.lsa``), CPU only.

Ward's method against scipy's hierarchical clustering; the one-item-per-
cluster index against the block selection of the main oracle (the landmark
scan is the index's block-contiguous special case); the index that keeps
everything against dense causal attention; and the position tables against
their definition."""
from __future__ import annotations

import numpy as np
import pytest
import torch
from scipy.cluster.hierarchy import fcluster, linkage

import oracle
from oracle import lsa


def _canon(labels):
    """Relabel a partition by order of first appearance."""
    out, seen = np.empty(len(labels), dtype=np.int64), {}
    for i, l in enumerate(labels):
        out[i] = seen.setdefault(int(l), len(seen))
    return out


@pytest.mark.parametrize("n,k,seed", [(12, 3, 0), (20, 5, 1), (33, 7, 2), (16, 1, 3), (9, 9, 4)])
def test_ward_matches_scipy(n, k, seed):
    X = np.random.default_rng(seed).normal(size=(n, 5))
    ours = lsa.ward_merges(X, k)
    ref = fcluster(linkage(X, method="ward"), t=k, criterion="maxclust")
    assert np.array_equal(_canon(ours), _canon(ref))
    assert len(np.unique(ours)) == k


def test_one_item_per_cluster_is_the_landmark_selection():
    rng = np.random.default_rng(5)
    n, d, pool, top = 96, 16, 4, 5
    K = rng.normal(size=(n, d))
    q = rng.normal(size=d)
    idx = lsa.build_index(K, pool, 1, 1)            # every item its own cluster
    assert idx["centres"].shape[0] == n // pool
    scale = oracle.default_scale(d)
    ours = lsa.select_clusters(idx, q, top, scale)
    sel = oracle.select(q, idx["items"], n // pool, top, 0, scale)   # candidates: every block before "local"
    assert np.array_equal(ours, np.asarray(sel["idx"][:sel["count"]]))
    for c in ours:
        assert np.array_equal(idx["positions"][c], np.arange(c * pool, (c + 1) * pool))


def test_keeping_everything_is_dense_attention():
    rng = np.random.default_rng(6)
    B, Hq, Hkv, n, d = 1, 4, 2, 70, 8
    q = rng.normal(size=(B, Hq, d))
    K = rng.normal(size=(B, Hkv, n, d))
    V = rng.normal(size=(B, Hkv, n, d))
    out = lsa.decode(q, K, V, pool=2, seg=8, clusters_per_seg=3, top_clusters=1000, sink=n, window=0)
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[:, :, None], torch.tensor(K).repeat_interleave(G, 1), torch.tensor(V).repeat_interleave(G, 1))
    np.testing.assert_allclose(out["O"], ref[:, :, 0].numpy(), rtol=1e-12, atol=1e-12)


def test_position_tables_partition_the_complete_segments():
    rng = np.random.default_rng(7)
    n, d, pool, seg, k = 203, 6, 3, 10, 4
    idx = lsa.build_index(rng.normal(size=(n, d)), pool, seg, k)
    complete = n // (pool * seg)
    assert idx["complete_segments"] == complete
    allpos = np.sort(np.concatenate(idx["positions"]))
    assert np.array_equal(allpos, np.arange(complete * seg * pool))
    assert idx["centres"].shape[0] == complete * k
    # each centre is the mean of its items
    for c, pos in enumerate(idx["positions"]):
        items = sorted({int(t) // pool for t in pos})
        np.testing.assert_allclose(idx["centres"][c], idx["items"][items].mean(axis=0), rtol=1e-12)


def test_kept_positions_add_sink_and_window_and_stay_causal():
    rng = np.random.default_rng(8)
    n, d = 64, 4
    idx = lsa.build_index(rng.normal(size=(n, d)), 2, 8, 2)
    pos = lsa.kept_positions(idx, [0], n, qpos=40, sink=3, window=5)
    assert {0, 1, 2, 36, 37, 38, 39, 40} <= set(pos.tolist())
    assert pos.max() <= 40 and np.all(np.diff(pos) > 0)
    assert set(idx["positions"][0].tolist()) & set(range(41)) <= set(pos.tolist())


def test_weighted_ward_equals_ward_on_the_repeated_points():
    """Rows of mass m merge as m copies of the row would (checked on the
    first merge, where the copies themselves merge at zero cost first)."""
    rng = np.random.default_rng(9)
    X = rng.normal(size=(7, 3))
    w = np.array([1, 3, 1, 2, 1, 1, 4])
    lab_w = lsa.ward_merges(X, 3, weights=w)
    rep = np.repeat(X, w, axis=0)
    lab_r = lsa.ward_merges(rep, 3)
    owner = np.repeat(np.arange(len(X)), w)
    # every group of copies ends in one cluster, and the partitions agree
    for i in range(len(X)):
        assert len(set(lab_r[owner == i])) == 1
    assert np.array_equal(_canon(lab_w), _canon(np.array([lab_r[owner == i][0] for i in range(len(X))])))


def test_tree_with_a_full_beam_is_the_flat_scan():
    rng = np.random.default_rng(10)
    n, d, pool, seg, k = 512, 8, 2, 16, 4
    K = rng.normal(size=(n, d))
    idx = lsa.build_index(K, pool, seg, k)
    levels = lsa.build_tree(idx, fanout=4)
    assert len(levels) >= 3
    scale = oracle.default_scale(d)
    for t in range(5):
        q = rng.normal(size=d)
        flat = lsa.select_clusters(idx, q, 6, scale)
        tree, comps = lsa.tree_select(levels, q, beam=10 ** 6, top_clusters=6, scale=scale)
        assert np.array_equal(tree, flat)


def test_tree_nodes_are_item_means_and_the_beam_bounds_the_work():
    rng = np.random.default_rng(11)
    n, d, pool, seg, k, fan, beam = 1024, 8, 2, 16, 4, 4, 3
    idx = lsa.build_index(rng.normal(size=(n, d)), pool, seg, k)
    levels = lsa.build_tree(idx, fanout=fan)
    # every parent's centre is the mean of the items below it
    def items_under(lv, node):
        if lv == 0:
            return sorted({int(t) // pool for t in idx["positions"][node]})
        return sorted(x for c in levels[lv]["children"][node] for x in items_under(lv - 1, c))
    for lv in range(1, len(levels)):
        for node in range(len(levels[lv]["centres"])):
            it = items_under(lv, node)
            np.testing.assert_allclose(levels[lv]["centres"][node], idx["items"][it].mean(axis=0), rtol=1e-10,
                                       atol=1e-12)
    leaves = len(levels[0]["centres"])
    _, comps = lsa.tree_select(levels, rng.normal(size=d), beam=beam, top_clusters=beam,
                               scale=oracle.default_scale(d))
    widest = max(len(ch) for lv in levels[1:] for ch in lv["children"])
    assert comps <= len(levels[-1]["centres"]) + (len(levels) - 1) * beam * widest
    assert comps < leaves


@pytest.mark.parametrize("fanout", [1, 0, -3])
def test_tree_rejects_a_fanout_that_cannot_shrink_a_level(fanout):
    rng = np.random.default_rng(5)
    idx = lsa.build_index(rng.standard_normal((256, 8)), 2, 16, 4)
    with pytest.raises(ValueError):
        lsa.build_tree(idx, fanout)

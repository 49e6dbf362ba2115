"""The C-ABI library loads without a GPU, exports every symbol the public
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import block_sparse_long_landmark_b200 as sa
from block_sparse_long_landmark_b200 import build as sabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    sabuild.build()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(sparse_attn_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert {"sparse_attn_select", "sparse_attn_prefill", "sparse_attn_decode", "sparse_attn_landmarks"} <= names
    lib = ctypes.CDLL(sa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(sa.EXPORTS) >= names


def test_the_address_checking_build_exports_the_same_symbols():
    from block_sparse_long_landmark_b200 import build
    path = build.build(bounds=True)
    lib = ctypes.CDLL(path)
    for n in declared_symbols():
        assert hasattr(lib, n), n


def test_version_and_strings():
    assert sa.sparse_attn_version() >= 100
    for code in (0, -1, -2, -3, -4, -5):
        assert isinstance(sa.sparse_attn_status_string(code), str)


def _p(**kw):
    base = dict(B=1, Hq=8, Hkv=2, d=128, N=4096, block=64, top_k=16,
                flags=sa.SA_SINK | sa.SA_LOCAL | sa.SA_GATE | sa.SA_CAUSAL, dtype="bf16")
    base.update(kw)
    return sa.make_params(**base)


def test_workspace_size_host_only():
    p = _p()
    for op in range(5):
        n = sa.sparse_attn_workspace_size(p, op)
        assert n >= 256 and n % 256 == 0
    pd = _p(B=8, N=1 << 20, top_k=64, flags=sa.SA_SINK | sa.SA_LOCAL | sa.SA_HIER | sa.SA_CAUSAL)
    assert sa.sparse_attn_workspace_size(pd, sa.SA_OP_DECODE) > 256
    assert sa.sparse_attn_workspace_size(pd, sa.SA_OP_SELECT_DECODE) > 256
    assert sa.sparse_attn_workspace_size(_p(Hq=7), 0) == 0       # invalid: no size


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=7), sa.SA_ERR_ARG),
    (dict(N=0), sa.SA_ERR_ARG),
    (dict(top_k=-1), sa.SA_ERR_ARG),
    (dict(top_k=1000), sa.SA_ERR_ARG),
    (dict(flags=1 << 10), sa.SA_ERR_ARG),
    (dict(dtype=7), sa.SA_ERR_ARG),
    (dict(d=96), sa.SA_ERR_UNSUPPORTED),
    (dict(block=48 + 1), sa.SA_ERR_UNSUPPORTED),
    (dict(flags=sa.SA_GATE | sa.SA_HIER | sa.SA_LOCAL), sa.SA_ERR_UNSUPPORTED),
    (dict(flags=sa.SA_GATE | sa.SA_SINK), sa.SA_ERR_UNSUPPORTED),
])
def test_bad_params_rejected_before_launch(kw, code):
    p = _p(**kw)
    fake = 256   # 16-byte aligned, never dereferenced: the checks fail first
    assert sa.sparse_attn_landmarks(p, fake, fake, None) == code
    assert sa.sparse_attn_select(p, fake, fake, fake, fake, fake, fake, 1 << 20, None) == code
    assert sa.sparse_attn_prefill(p, fake, fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None) == code
    assert sa.sparse_attn_decode(p, fake, fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None) == code


def test_null_misaligned_and_small_workspace_rejected():
    p = _p()
    a = 256
    assert sa.sparse_attn_landmarks(p, None, a, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_landmarks(p, a + 8, a, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_select(p, a, a, a, a, a, None, 1 << 20, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_select(p, a, a, a, a, a, a, 16, None) == sa.SA_ERR_WORKSPACE
    assert sa.sparse_attn_prefill(p, a, a, a, a, a, a, a, a, a, 16, None) == sa.SA_ERR_WORKSPACE
    assert sa.sparse_attn_decode(p, a, a, a, a, a, a, a, a, a, 16, None) == sa.SA_ERR_WORKSPACE
    assert sa.sparse_attn_check_status(None, None)[0] == sa.SA_ERR_ARG


def test_varlen_entry_points_need_lengths():
    p = _p()
    a = 256
    assert sa.sparse_attn_select_decode_varlen(p, a, a, None, a, a, a, a, 1 << 20, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_decode_varlen(p, a, a, a, None, a, a, a, a, a, a, 1 << 20, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_landmarks_update(p, None, a, None, None, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_landmarks_update(_p(Hq=7), a, a, None, None, None) == sa.SA_ERR_ARG


def test_decode_step_checks_arguments():
    """The one-call decode step refuses what either of its two halves refuses,
    and wants a workspace big enough for both of them; nothing is launched."""
    p = _p(B=2, N=8192)
    a = 256
    big = 1 << 30
    for kw, code in [(dict(Hq=7), sa.SA_ERR_ARG), (dict(d=96), sa.SA_ERR_UNSUPPORTED)]:
        assert sa.sparse_attn_decode_step(_p(**kw), a, a, a, a, None, a, a, a, a, a, a, big, None) == code
    for i in (0, 1, 2, 3, 5, 6, 7, 8, 9, 10):     # q L K V - idx score count o lse ws
        ptrs = [a] * 11
        ptrs[i] = None
        assert sa.sparse_attn_decode_step(p, *ptrs[:4], None, *ptrs[5:], big, None) == sa.SA_ERR_ARG, i
    assert sa.sparse_attn_decode_step(p, a + 8, a, a, a, None, a, a, a, a, a, a, big, None) == sa.SA_ERR_ARG
    need = max(sa.sparse_attn_workspace_size(p, sa.SA_OP_SELECT_DECODE),
               sa.sparse_attn_workspace_size(p, sa.SA_OP_DECODE))
    assert sa.sparse_attn_decode_step(p, a, a, a, a, None, a, a, a, a, a, a, need - 256, None) == \
        sa.SA_ERR_WORKSPACE


def test_backward_entry_points_check_arguments():
    """Every call below fails its host-side checks before any launch."""
    p = _p()
    a = 256
    ptrs = [a] * 14                                   # Q K V O lse dO idx score count dQ dK dV dscore ws
    hier = _p(flags=sa.SA_SINK | sa.SA_LOCAL | sa.SA_HIER | sa.SA_CAUSAL)
    assert sa.sparse_attn_prefill_backward(hier, *ptrs, 1 << 20, None) == sa.SA_ERR_UNSUPPORTED
    assert sa.sparse_attn_select_backward(hier, a, a, a, a, a, a, a, a, 1 << 20, None) == sa.SA_ERR_UNSUPPORTED
    nulls = list(ptrs)
    nulls[5] = None                                   # dO
    assert sa.sparse_attn_prefill_backward(p, *nulls, 1 << 20, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_prefill_backward(p, *ptrs, 16, None) == sa.SA_ERR_WORKSPACE
    assert sa.sparse_attn_select_backward(p, a, a, a, a, a, a, a, a, 16, None) == sa.SA_ERR_WORKSPACE
    assert sa.sparse_attn_select_backward(p, None, a, a, a, a, a, a, a, 1 << 20, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_workspace_size(p, sa.SA_OP_PREFILL_BACKWARD) > 256
    assert sa.sparse_attn_workspace_size(p, sa.SA_OP_SELECT_BACKWARD) > 256


def test_lsa_entry_points_check_arguments():
    """Host-side checks of the flat-index entry points; nothing is launched."""
    ok = sa.make_lsa_params(1, 4, 2, 128, 4096, 4, 32, 8, 6, 16, 64)
    assert sa.sparse_attn_lsa_clusters(ok) == (4096 // 128) * 8
    assert sa.sparse_attn_lsa_workspace_size(ok) > 256
    for bad, code in [
        (dict(Hq=5), sa.SA_ERR_ARG), (dict(pool=0), sa.SA_ERR_ARG), (dict(seg=1), sa.SA_ERR_ARG),
        (dict(clusters=40), sa.SA_ERR_ARG), (dict(top_clusters=-1), sa.SA_ERR_ARG), (dict(d=96), sa.SA_ERR_UNSUPPORTED),
        (dict(seg=65, clusters=4), sa.SA_ERR_UNSUPPORTED), (dict(N=(1 << 20) + 1), sa.SA_ERR_UNSUPPORTED),
    ]:
        kw = dict(B=1, Hq=4, Hkv=2, d=128, N=4096, pool=4, seg=32, clusters=8, top_clusters=6, sink=16, window=64)
        kw.update(bad)
        p = sa.make_lsa_params(**kw)
        assert sa.sparse_attn_lsa_clusters(p) == code, bad
        assert sa.sparse_attn_lsa_workspace_size(p) == 0
        assert sa.sparse_attn_lsa_build(p, 256, 256, 256, 256, None) == code
    a = 256
    assert sa.sparse_attn_lsa_build(ok, None, a, a, a, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_lsa_build(ok, a, None, a, a, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_lsa_decode(ok, a, a, a, a, a, a, a, a, None, a, 16, None) == sa.SA_ERR_WORKSPACE
    assert sa.sparse_attn_lsa_decode(ok, None, a, a, a, a, a, a, a, None, a, 1 << 20, None) == sa.SA_ERR_ARG
    # the chunk merge of the decode runs in one CTA: too many candidates are refused up front
    big = sa.make_lsa_params(1, 4, 2, 128, 1 << 20, 1, 64, 64, 4096, 16, 64)
    assert sa.sparse_attn_lsa_clusters(big) == (1 << 20)
    assert sa.sparse_attn_lsa_workspace_size(big) == 0
    assert sa.sparse_attn_lsa_decode(big, a, a, a, a, a, a, a, a, None, a, 1 << 30, None) == sa.SA_ERR_UNSUPPORTED


def test_lsa_tree_host_checks():
    """The tree entry points' host-side checks (no launch happens)."""
    p = sa.make_lsa_params(1, 4, 2, 128, 8192, 4, 32, 8, 6, 16, 64)      # 512 clusters per kv-head
    nbytes, levels = sa.sparse_attn_lsa_tree_size(p, 4)
    assert nbytes > 0 and levels == 5                                       # 512, 128, 32, 8, 2
    assert sa.sparse_attn_lsa_tree_size(p, 8)[1] == 3                       # 512, 64, 8
    assert sa.sparse_attn_lsa_tree_size(p, 1)[0] == 0                       # a fan-out below 2 is refused
    assert sa.sparse_attn_lsa_tree_size(p, 65)[0] == 0
    ws = sa.sparse_attn_lsa_tree_workspace_size(p, 4)
    assert ws > sa.sparse_attn_lsa_workspace_size(p)
    a = 256
    assert sa.sparse_attn_lsa_tree_build(p, 1, a, a, a, a, ws, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_lsa_tree_build(p, 4, None, a, a, a, ws, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_lsa_tree_build(p, 4, a, a, a, a, 16, None) == sa.SA_ERR_WORKSPACE
    assert sa.sparse_attn_lsa_tree_decode(p, 4, 0, a, a, a, a, a, a, a, a, a, None, None, a, ws, None) == sa.SA_ERR_ARG
    assert sa.sparse_attn_lsa_tree_decode(p, 4, 3, None, a, a, a, a, a, a, a, a, None, None, a, ws, None) == \
        sa.SA_ERR_ARG
    assert sa.sparse_attn_lsa_tree_decode(p, 4, 3, a, a, a, a, a, a, a, a, a, None, None, a, 16, None) == \
        sa.SA_ERR_WORKSPACE
    # more leaves than a tree supports
    big = sa.make_lsa_params(1, 4, 2, 128, 1 << 17, 1, 16, 8, 6, 16, 64)   # 65536 clusters
    assert sa.sparse_attn_lsa_tree_size(big, 4)[0] == 0
    assert sa.sparse_attn_lsa_tree_decode(big, 4, 3, a, a, a, a, a, a, a, a, a, None, None, a, 1 << 30, None) == \
        sa.SA_ERR_UNSUPPORTED

"""CPU oracle for selector-driven block-sparse attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library
and never imports it.  The forward path's arithmetic lives in ``oracle.c``
(plain C, every step in double); this module compiles it with gcc, loads it
with ctypes and walks the units of a problem in the order the method takes its
steps (the backward pass, ``backward.py``, and the flat clustered index,
``lsa.py``, are plain numpy in float64):

  1. landmarks  -- mean of each block's keys ([HiLS] opening section: chunk
                   summaries named landmarks; [LSA] "Индекс перестаёт
                   перебирать весь контекст": adjacent keys pooled before
                   scoring), rounded to the storage precision of the keys;
  2. pooled query of the unit (all query heads of one kv-head group and all
     queries of one tile; decode: the one query);
  3. scores of every block against it, hard top-K over the candidate blocks,
     plus the always-kept sink block 0 ([LSA], same section) and local block
     ([SAS] "Ключевые факты": the current block is always kept);
  4. attention over the kept blocks -- gated (log-sigmoid gate inside the
     softmax, [SAS] "Как это применить") or hierarchical (per-block softmax
     combined by the softmax of the retrieval scores, [HiLS] opening section).

Page names: [SAS] "Учёные научили трансформеры отбирать контекст напрямую, а не
через имитацию полного внимания"; [HiLS] "HiLS-Attention: иерархическое
разреженное внимание для сверхдлинного контекста в языковых моделях"; [LSA] the
Latent Sparse Attention post on rit.work.

Readings of what the pages leave open (tile-level shared lists per kv-head,
the gate on selected blocks only, s_local from the tile's own block,
hierarchical weights over all kept blocks) are implemented as stated.  Every
function is pinned to the mathematics of its reading (closed forms, brute
force on tiny inputs, library routines); the pages print no worked values that
could decide between readings.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

SINK, LOCAL, GATE, HIER, CAUSAL, PER_QHEAD = 1, 2, 4, 8, 16, 32

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")
_lock = threading.Lock()
_lib = None

ROUND_NONE, ROUND_BF16, ROUND_FP32 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c into a shared library next to it (gcc, -O2, IEEE)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
            "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int)
            lp = ctypes.POINTER(ctypes.c_long)
            lib.orc_round_bf16.argtypes = [ctypes.c_double]
            lib.orc_round_bf16.restype = ctypes.c_double
            lib.orc_log_sigmoid.argtypes = [ctypes.c_double]
            lib.orc_log_sigmoid.restype = ctypes.c_double
            lib.orc_landmarks.argtypes = [dp, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp]
            lib.orc_landmarks.restype = None
            lib.orc_pool_queries.argtypes = [dp, ctypes.c_int, ctypes.c_long, ctypes.c_int, ctypes.c_long,
                                             ctypes.c_int, dp]
            lib.orc_pool_queries.restype = None
            lib.orc_select.argtypes = [dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_double, ip, dp, dp, dp, dp]
            lib.orc_select.restype = ctypes.c_int
            att = [dp, ctypes.c_int, lp, dp, dp, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                   ip, dp, ctypes.c_int, ctypes.c_int, ctypes.c_double, dp, dp]
            lib.orc_attend_gated.argtypes = att
            lib.orc_attend_gated.restype = None
            lib.orc_attend_hier.argtypes = att
            lib.orc_attend_hier.restype = None
            _lib = lib
    return _lib


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------
# Single steps
# ----------------------------------------------------------------------------

def round_bf16(x: float) -> float:
    return _load().orc_round_bf16(float(x))


def log_sigmoid(x: float) -> float:
    return _load().orc_log_sigmoid(float(x))


def landmarks(k, block: int, round_mode: int = ROUND_NONE) -> np.ndarray:
    """Landmarks of one (batch, kv-head): k [n, d] -> [ceil(n/block), d]."""
    k = _f64(k)
    n, d = k.shape
    out = np.empty(((n + block - 1) // block, d), dtype=np.float64)
    _load().orc_landmarks(_dp(k), n, d, block, round_mode, _dp(out))
    return out


def pool_queries(q, row0: int, nrows: int) -> np.ndarray:
    """Mean over heads and rows [row0, row0+nrows) of q [heads, n, d]."""
    q = _f64(q)
    h, n, d = q.shape
    out = np.empty(d, dtype=np.float64)
    _load().orc_pool_queries(_dp(q), h, n, d, row0, nrows, _dp(out))
    return out


def select(qbar, lmk, local: int, top_k: int, flags: int, scale: float) -> dict:
    """Selection for one unit whose own block is ``local`` (see oracle.c)."""
    qbar = _f64(qbar)
    lmk = _f64(lmk)
    d = qbar.shape[0]
    cap = max(top_k, 0) + 2
    idx = np.full(cap, -1, dtype=np.int32)
    sc = np.zeros(cap)
    gate = np.zeros(cap)
    gap = np.zeros(1)
    s_all = np.zeros(local + 1)
    cnt = _load().orc_select(_dp(qbar), _dp(lmk), d, local, top_k, flags, scale,
                             idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), _dp(sc), _dp(gate),
                             _dp(gap), _dp(s_all))
    return {"count": cnt, "idx": idx, "sc": sc, "gate": gate, "rel_gap": float(gap[0]), "scores": s_all}


def attend(q_rows, qpos, k, v, block: int, local: int, sel: dict, flags: int, scale: float):
    """Attention of query rows that share one kept list; gated unless HIER."""
    q_rows = _f64(q_rows)
    k = _f64(k)
    v = _f64(v)
    nrows, d = q_rows.shape
    n = k.shape[0]
    qpos = np.ascontiguousarray(qpos, dtype=np.int64)
    idx = np.ascontiguousarray(sel["idx"], dtype=np.int32)
    cnt = int(sel["count"])
    o = np.zeros((nrows, d))
    lse = np.zeros(nrows)
    lib = _load()
    fn = lib.orc_attend_hier if flags & HIER else lib.orc_attend_gated
    extra = _f64(sel["sc"] if flags & HIER else sel["gate"])
    fn(_dp(q_rows), nrows, qpos.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), _dp(k), _dp(v), n, d, block,
       local, idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), _dp(extra), cnt, flags, scale, _dp(o),
       _dp(lse))
    return o, lse


# ----------------------------------------------------------------------------
# Whole problems (or sampled units of them)
# ----------------------------------------------------------------------------

def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def _pool(threads, fn, items):
    if threads is None:
        threads = os.cpu_count() or 1
    if threads <= 1 or len(items) <= 1:
        return [fn(x) for x in items]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, items))


def prefill(Q, K, V, block: int, top_k: int, flags: int, scale: float | None = None,
            round_mode: int = ROUND_BF16, units=None, threads=None, sel_override=None) -> dict:
    """Block-sparse prefill of Q [B,Hq,N,d] over K, V [B,Hkv,N,d].

    ``units``: iterable of (b, g, j) selection units to compute (default: all);
    a unit is (batch, kv-head, query tile) -- or (batch, q-head, tile) when
    PER_QHEAD is set.  Entries not computed are left NaN / -2.
    ``sel_override``: optional callable (b, g, j) -> dict(idx, count, sc, gate)
    used instead of the oracle's own selection (to check attention alone).
    Returns landmarks, selection lists and outputs."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    nb = (N + block - 1) // block
    scale = default_scale(d) if scale is None else scale
    per_q = bool(flags & PER_QHEAD)
    nsel_heads = Hq if per_q else Hkv
    cap = max(top_k, 0) + 2
    L = np.full((B, Hkv, nb, d), np.nan)
    out = {
        "L": L,
        "idx": np.full((B, nsel_heads, nb, cap), -2, dtype=np.int32),
        "sc": np.full((B, nsel_heads, nb, cap), np.nan),
        "gate": np.full((B, nsel_heads, nb, cap), np.nan),
        "count": np.full((B, nsel_heads, nb), -2, dtype=np.int32),
        "rel_gap": np.full((B, nsel_heads, nb), np.nan),
        "O": np.full((B, Hq, N, d), np.nan),
        "LSE": np.full((B, Hq, N), np.nan),
    }
    if units is None:
        units = [(b, s, j) for b in range(B) for s in range(nsel_heads) for j in range(nb)]
    units = list(units)
    need = sorted({(b, (s // G) if per_q else s) for (b, s, _) in units})

    def lmk_of(bg):
        b, g = bg
        L[b, g] = landmarks(K[b, g], block, round_mode)

    _pool(threads, lmk_of, need)

    def run(u):
        b, s, j = u
        g = s // G if per_q else s
        heads = range(s, s + 1) if per_q else range(g * G, (g + 1) * G)
        h0, h1 = heads[0], heads[-1] + 1
        qh = _f64(Q[b, h0:h1])
        if sel_override is not None:
            sel = sel_override(b, s, j)
        else:
            qbar = pool_queries(qh, j * block, block)
            sel = select(qbar, L[b, g], j, top_k, flags, scale)
        r0, r1 = j * block, min((j + 1) * block, N)
        rows = qh[:, r0:r1].reshape(-1, d)
        qpos = np.tile(np.arange(r0, r1), h1 - h0)
        o, lse = attend(rows, qpos, K[b, g], V[b, g], block, j, sel, flags, scale)
        return u, sel, o.reshape(h1 - h0, r1 - r0, d), lse.reshape(h1 - h0, r1 - r0)

    for (b, s, j), sel, o, lse in _pool(threads, run, units):
        c = int(sel["count"])
        out["count"][b, s, j] = c
        out["idx"][b, s, j] = -1
        out["idx"][b, s, j, :c] = np.asarray(sel["idx"])[:c]
        out["sc"][b, s, j] = 0.0
        out["sc"][b, s, j, :c] = np.asarray(sel["sc"])[:c]
        out["gate"][b, s, j] = 0.0
        out["gate"][b, s, j, :c] = np.asarray(sel["gate"])[:c]
        out["rel_gap"][b, s, j] = sel.get("rel_gap", np.nan)
        g = s // G if per_q else s
        h0 = s if per_q else g * G
        out["O"][b, h0:h0 + o.shape[0], j * block:j * block + o.shape[1]] = o
        out["LSE"][b, h0:h0 + o.shape[0], j * block:j * block + o.shape[1]] = lse
    return out


def decode(q, K, V, block: int, top_k: int, flags: int, scale: float | None = None,
           round_mode: int = ROUND_BF16, units=None, threads=None, sel_override=None,
           L=None) -> dict:
    """One decode step: the query q [B,Hq,d] at position N-1 over the cache
    K, V [B,Hkv,N,d] (which already holds the query's own key and value).
    ``units``: (b, g) pairs to compute -- (b, h) with PER_QHEAD.
    ``L``: optional landmarks [B,Hkv,nb,d] the oracle computed earlier."""
    q = _f64(q)
    K = _f64(K)
    V = _f64(V)
    B, Hq, d = q.shape
    Hkv, N = K.shape[1], K.shape[2]
    G = Hq // Hkv
    nb = (N + block - 1) // block
    local = (N - 1) // block
    scale = default_scale(d) if scale is None else scale
    per_q = bool(flags & PER_QHEAD)
    nsel_heads = Hq if per_q else Hkv
    cap = max(top_k, 0) + 2
    if L is None:
        L = np.full((B, Hkv, nb, d), np.nan)
        have = set()
    else:
        have = None
    out = {
        "L": L,
        "idx": np.full((B, nsel_heads, cap), -2, dtype=np.int32),
        "sc": np.full((B, nsel_heads, cap), np.nan),
        "gate": np.full((B, nsel_heads, cap), np.nan),
        "count": np.full((B, nsel_heads), -2, dtype=np.int32),
        "rel_gap": np.full((B, nsel_heads), np.nan),
        "O": np.full((B, Hq, d), np.nan),
        "LSE": np.full((B, Hq), np.nan),
    }
    if units is None:
        units = [(b, s) for b in range(B) for s in range(nsel_heads)]
    units = list(units)
    if have is not None:
        need = sorted({(b, (s // G) if per_q else s) for (b, s) in units})

        def lmk_of(bg):
            b, g = bg
            L[b, g] = landmarks(K[b, g], block, round_mode)

        _pool(threads, lmk_of, need)

    def run(u):
        b, s = u
        g = s // G if per_q else s
        h0, h1 = (s, s + 1) if per_q else (g * G, (g + 1) * G)
        qh = _f64(q[b, h0:h1]).reshape(h1 - h0, 1, d)
        if sel_override is not None:
            sel = sel_override(b, s)
        else:
            qbar = pool_queries(qh, 0, 1)
            sel = select(qbar, L[b, g], local, top_k, flags, scale)
        o, lse = attend(qh.reshape(h1 - h0, d), np.full(h1 - h0, N - 1), K[b, g], V[b, g], block, local, sel,
                        flags, scale)
        return u, sel, o, lse

    for (b, s), sel, o, lse in _pool(threads, run, units):
        c = int(sel["count"])
        out["count"][b, s] = c
        out["idx"][b, s] = -1
        out["idx"][b, s, :c] = np.asarray(sel["idx"])[:c]
        out["sc"][b, s] = 0.0
        out["sc"][b, s, :c] = np.asarray(sel["sc"])[:c]
        out["gate"][b, s] = 0.0
        out["gate"][b, s, :c] = np.asarray(sel["gate"])[:c]
        out["rel_gap"][b, s] = sel.get("rel_gap", np.nan)
        g = s // G if per_q else s
        h0 = s if per_q else g * G
        out["O"][b, h0:h0 + o.shape[0]] = o
        out["LSE"][b, h0:h0 + o.shape[0]] = lse
    return out

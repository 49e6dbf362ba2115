"""Selector-driven block-sparse attention for B200 (sm_100a).

Thin Python binding of ``libsparse_attn.so`` (C ABI in ``include/sparse_attn.h``):
argument marshalling only -- every step runs in the library's CUDA kernels.
PyTorch provides device memory and streams.  The functions ``sparse_attn_*``
mirror the C entry points one to one (pointers as ints, the stream as an int
handle); the lower-case helpers take torch tensors, allocate outputs and raise
``SparseAttnError`` on a non-zero return code.

The library must have been built (``python -m block_sparse_long_landmark_b200.build``);
there is no fallback of any kind when it is missing.
"""
from __future__ import annotations

import ctypes
import os
import threading

from .inputs import F_CAUSAL, F_GATE, F_HIER, F_LOCAL, F_PER_QHEAD, F_SINK  # noqa: F401

SA_SINK, SA_LOCAL, SA_GATE, SA_HIER, SA_CAUSAL, SA_SELECT_PER_QHEAD = 1, 2, 4, 8, 16, 32
SA_BF16, SA_FP32 = 0, 1
SA_OP_LANDMARKS, SA_OP_SELECT, SA_OP_SELECT_DECODE, SA_OP_PREFILL, SA_OP_DECODE = 0, 1, 2, 3, 4
SA_OP_PREFILL_BACKWARD, SA_OP_SELECT_BACKWARD = 5, 6
SA_OK, SA_ERR_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_LAUNCH, SA_ERR_DEVICE = 0, -1, -2, -3, -4, -5

# SPARSE_ATTN_LIB selects another build of the same library (for example the
# address-checking one, lib/libsparse_attn_bounds.so)
LIB_PATH = os.environ.get("SPARSE_ATTN_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib",
                                                               "libsparse_attn.so")

EXPORTS = (
    "sparse_attn_workspace_size", "sparse_attn_landmarks", "sparse_attn_select", "sparse_attn_select_decode",
    "sparse_attn_prefill", "sparse_attn_decode", "sparse_attn_check_status", "sparse_attn_status_string",
    "sparse_attn_version", "sparse_attn_launch_count", "sparse_attn_decode_static",
    "sparse_attn_prefill_kernel", "sparse_attn_last_cuda_error", "sparse_attn_cuda_error_string",
    "sparse_attn_landmarks_update", "sparse_attn_select_decode_varlen", "sparse_attn_decode_varlen",
    "sparse_attn_decode_step", "sparse_attn_prefill_backward", "sparse_attn_select_backward",
    "sparse_attn_lsa_clusters", "sparse_attn_lsa_workspace_size", "sparse_attn_lsa_build", "sparse_attn_lsa_decode",
    "sparse_attn_lsa_tree_size", "sparse_attn_lsa_tree_workspace_size", "sparse_attn_lsa_tree_build",
    "sparse_attn_lsa_tree_decode",
)


class sa_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("N", ctypes.c_int), ("block", ctypes.c_int), ("top_k", ctypes.c_int), ("flags", ctypes.c_int),
                ("dtype", ctypes.c_int), ("scale", ctypes.c_float)]

    def __repr__(self):
        return "sa_params(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class sa_lsa_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("N", ctypes.c_int), ("pool", ctypes.c_int), ("seg", ctypes.c_int), ("clusters", ctypes.c_int),
                ("top_clusters", ctypes.c_int), ("sink", ctypes.c_int), ("window", ctypes.c_int),
                ("dtype", ctypes.c_int), ("scale", ctypes.c_float)]


class SparseAttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what}: {sparse_attn_status_string(code)} (code {code})"
        if code == SA_ERR_LAUNCH:
            err = lib().sparse_attn_last_cuda_error()
            msg += f"; CUDA error {err}: {lib().sparse_attn_cuda_error_string(err).decode()}"
        super().__init__(msg)
        self.code = code


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it was not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m block_sparse_long_landmark_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P = ctypes.POINTER(sa_params)
            vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
            L.sparse_attn_workspace_size.argtypes = [P, i]
            L.sparse_attn_workspace_size.restype = sz
            L.sparse_attn_landmarks.argtypes = [P, vp, vp, vp]
            L.sparse_attn_select.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
            L.sparse_attn_select_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
            L.sparse_attn_prefill.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.sparse_attn_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.sparse_attn_check_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int)]
            L.sparse_attn_status_string.argtypes = [i]
            L.sparse_attn_status_string.restype = ctypes.c_char_p
            L.sparse_attn_version.argtypes = []
            for n in EXPORTS[1:7]:
                getattr(L, n).restype = i
            L.sparse_attn_version.restype = i
            L.sparse_attn_landmarks_update.argtypes = [P, vp, vp, vp, vp, vp]
            L.sparse_attn_landmarks_update.restype = i
            L.sparse_attn_select_decode_varlen.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.sparse_attn_select_decode_varlen.restype = i
            L.sparse_attn_decode_varlen.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.sparse_attn_decode_varlen.restype = i
            L.sparse_attn_decode_step.argtypes = [P] + [vp] * 10 + [vp, sz, vp]
            L.sparse_attn_decode_step.restype = i
            L.sparse_attn_last_cuda_error.argtypes = []
            L.sparse_attn_last_cuda_error.restype = i
            L.sparse_attn_cuda_error_string.argtypes = [i]
            L.sparse_attn_cuda_error_string.restype = ctypes.c_char_p
            L.sparse_attn_prefill_kernel.argtypes = [P]
            L.sparse_attn_prefill_kernel.restype = i
            L.sparse_attn_decode_static.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            L.sparse_attn_decode_static.restype = i
            L.sparse_attn_prefill_backward.argtypes = [P] + [vp] * 14 + [sz, vp]
            L.sparse_attn_prefill_backward.restype = i
            L.sparse_attn_select_backward.argtypes = [P] + [vp] * 8 + [sz, vp]
            L.sparse_attn_select_backward.restype = i
            LP = ctypes.POINTER(sa_lsa_params)
            L.sparse_attn_lsa_clusters.argtypes = [LP]
            L.sparse_attn_lsa_clusters.restype = i
            L.sparse_attn_lsa_workspace_size.argtypes = [LP]
            L.sparse_attn_lsa_workspace_size.restype = sz
            L.sparse_attn_lsa_build.argtypes = [LP, vp, vp, vp, vp, vp]
            L.sparse_attn_lsa_build.restype = i
            L.sparse_attn_lsa_decode.argtypes = [LP] + [vp] * 10 + [sz, vp]
            L.sparse_attn_lsa_decode.restype = i
            L.sparse_attn_lsa_tree_size.argtypes = [LP, i, ctypes.POINTER(ctypes.c_int)]
            L.sparse_attn_lsa_tree_size.restype = sz
            L.sparse_attn_lsa_tree_workspace_size.argtypes = [LP, i]
            L.sparse_attn_lsa_tree_workspace_size.restype = sz
            L.sparse_attn_lsa_tree_build.argtypes = [LP, i, vp, vp, vp, vp, sz, vp]
            L.sparse_attn_lsa_tree_build.restype = i
            L.sparse_attn_lsa_tree_decode.argtypes = [LP, i, i] + [vp] * 12 + [sz, vp]
            L.sparse_attn_lsa_tree_decode.restype = i
            L.sparse_attn_launch_count.argtypes = []
            L.sparse_attn_launch_count.restype = ctypes.c_ulonglong
            _lib = L
    return _lib


# ----------------------------------------------------------------------------
# The C entry points, one to one
# ----------------------------------------------------------------------------

def sparse_attn_workspace_size(p: sa_params, op: int) -> int:
    return int(lib().sparse_attn_workspace_size(ctypes.byref(p), op))


def sparse_attn_landmarks(p, K, L, stream) -> int:
    return lib().sparse_attn_landmarks(ctypes.byref(p), K, L, stream)


def sparse_attn_select(p, Q, L, idx, score, count, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_select(ctypes.byref(p), Q, L, idx, score, count, ws, ws_bytes, stream)


def sparse_attn_select_decode(p, q, L, idx, score, count, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_select_decode(ctypes.byref(p), q, L, idx, score, count, ws, ws_bytes, stream)


def sparse_attn_prefill(p, Q, K, V, idx, score, count, O, lse, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_prefill(ctypes.byref(p), Q, K, V, idx, score, count, O, lse, ws, ws_bytes, stream)


def sparse_attn_decode(p, q, K, V, idx, score, count, o, lse, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_decode(ctypes.byref(p), q, K, V, idx, score, count, o, lse, ws, ws_bytes, stream)


def sparse_attn_prefill_backward(p, Q, K, V, O, lse, dO, idx, score, count, dQ, dK, dV, dscore, ws, ws_bytes,
                                 stream) -> int:
    return lib().sparse_attn_prefill_backward(ctypes.byref(p), Q, K, V, O, lse, dO, idx, score, count, dQ, dK, dV,
                                              dscore, ws, ws_bytes, stream)


def sparse_attn_lsa_clusters(p: sa_lsa_params) -> int:
    return int(lib().sparse_attn_lsa_clusters(ctypes.byref(p)))


def sparse_attn_lsa_workspace_size(p: sa_lsa_params) -> int:
    return int(lib().sparse_attn_lsa_workspace_size(ctypes.byref(p)))


def sparse_attn_lsa_build(p, K, centres, members, sizes, stream) -> int:
    return lib().sparse_attn_lsa_build(ctypes.byref(p), K, centres, members, sizes, stream)


def sparse_attn_lsa_decode(p, q, K, V, centres, members, sizes, o, lse, kept, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_lsa_decode(ctypes.byref(p), q, K, V, centres, members, sizes, o, lse, kept, ws,
                                        ws_bytes, stream)


def sparse_attn_lsa_tree_size(p: sa_lsa_params, fanout: int):
    """(bytes of the tree buffer, levels incl. the leaves); bytes 0 = invalid."""
    lv = ctypes.c_int(0)
    n = int(lib().sparse_attn_lsa_tree_size(ctypes.byref(p), fanout, ctypes.byref(lv)))
    return n, lv.value


def sparse_attn_lsa_tree_workspace_size(p: sa_lsa_params, fanout: int) -> int:
    return int(lib().sparse_attn_lsa_tree_workspace_size(ctypes.byref(p), fanout))


def sparse_attn_lsa_tree_build(p, fanout, centres, sizes, tree, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_lsa_tree_build(ctypes.byref(p), fanout, centres, sizes, tree, ws, ws_bytes, stream)


def sparse_attn_lsa_tree_decode(p, fanout, beam, q, K, V, centres, members, sizes, tree, o, lse, kept, compared, ws,
                                ws_bytes, stream) -> int:
    return lib().sparse_attn_lsa_tree_decode(ctypes.byref(p), fanout, beam, q, K, V, centres, members, sizes, tree, o,
                                             lse, kept, compared, ws, ws_bytes, stream)


def sparse_attn_select_backward(p, Q, L, idx, dscore, count, dQ, dK, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_select_backward(ctypes.byref(p), Q, L, idx, dscore, count, dQ, dK, ws, ws_bytes,
                                             stream)


def sparse_attn_prefill_kernel(p) -> int:
    return lib().sparse_attn_prefill_kernel(ctypes.byref(p))


def sparse_attn_decode_static(p, q, K, V, idx, score, count, o, lse, stream) -> int:
    return lib().sparse_attn_decode_static(ctypes.byref(p), q, K, V, idx, score, count, o, lse, stream)


def sparse_attn_landmarks_update(p, K, L, seq_len, first_block, stream) -> int:
    return lib().sparse_attn_landmarks_update(ctypes.byref(p), K, L, seq_len, first_block, stream)


def sparse_attn_select_decode_varlen(p, q, L, seq_len, idx, score, count, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_select_decode_varlen(ctypes.byref(p), q, L, seq_len, idx, score, count, ws, ws_bytes,
                                                  stream)


def sparse_attn_decode_varlen(p, q, K, V, seq_len, idx, score, count, o, lse, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_decode_varlen(ctypes.byref(p), q, K, V, seq_len, idx, score, count, o, lse, ws,
                                           ws_bytes, stream)


def sparse_attn_decode_step(p, q, L, K, V, seq_len, idx, score, count, o, lse, ws, ws_bytes, stream) -> int:
    return lib().sparse_attn_decode_step(ctypes.byref(p), q, L, K, V, seq_len, idx, score, count, o, lse, ws,
                                         ws_bytes, stream)


def sparse_attn_check_status(ws, stream):
    detail = ctypes.c_int(0)
    rc = lib().sparse_attn_check_status(ws, stream, ctypes.byref(detail))
    return rc, detail.value


def sparse_attn_status_string(code: int) -> str:
    return lib().sparse_attn_status_string(code).decode()


def sparse_attn_version() -> int:
    return lib().sparse_attn_version()


def sparse_attn_launch_count() -> int:
    return int(lib().sparse_attn_launch_count())


# ----------------------------------------------------------------------------
# Tensor helpers
# ----------------------------------------------------------------------------

def make_params(B, Hq, Hkv, d, N, block, top_k, flags, dtype="bf16", scale=0.0) -> sa_params:
    dt = {"bf16": SA_BF16, "fp32": SA_FP32}[dtype] if isinstance(dtype, str) else int(dtype)
    return sa_params(B, Hq, Hkv, d, N, block, top_k, flags, dt, float(scale))


def params_for(wl, **over) -> sa_params:
    """Parameters of an ``inputs.Workload`` (fields overridable)."""
    kw = dict(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, N=wl.N, block=wl.block, top_k=wl.top_k, flags=wl.flags,
              dtype=wl.dtype)
    kw.update(over)
    return make_params(**kw)


def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check(rc: int, what: str):
    if rc != SA_OK:
        raise SparseAttnError(rc, what)


def _tdtype(p):
    torch = _torch()
    return torch.bfloat16 if p.dtype == SA_BF16 else torch.float32


def _hsel(p):
    return p.Hq if p.flags & SA_SELECT_PER_QHEAD else p.Hkv


DECODE_OPS = (SA_OP_LANDMARKS, SA_OP_SELECT_DECODE, SA_OP_DECODE)
FORWARD_OPS = (SA_OP_LANDMARKS, SA_OP_SELECT, SA_OP_SELECT_DECODE, SA_OP_PREFILL, SA_OP_DECODE)


def workspace(p: sa_params, device="cuda", ops=None):
    """A zero-filled workspace large enough for the operations `ops` of `p`
    (SA_OP_* codes; every operation when None).  The backward's workspace
    grows with B * Hq * N, so a decode-only caller passes DECODE_OPS."""
    torch = _torch()
    ops = range(7) if ops is None else ops
    n = max(sparse_attn_workspace_size(p, op) for op in ops)
    if n == 0:
        raise SparseAttnError(SA_ERR_ARG, "workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def landmarks(p, K, out=None, stream=None):
    torch = _torch()
    nb = (p.N + p.block - 1) // p.block
    L = out if out is not None else torch.empty(p.B, p.Hkv, nb, p.d, dtype=_tdtype(p), device=K.device)
    _check(sparse_attn_landmarks(p, _ptr(K), _ptr(L), _stream(stream)), "sparse_attn_landmarks")
    return L


def _sel_out(p, decode, device):
    torch = _torch()
    cap = p.top_k + 2
    lead = (p.B, _hsel(p)) if decode else (p.B, _hsel(p), (p.N + p.block - 1) // p.block)
    return (torch.empty(*lead, cap, dtype=torch.int32, device=device),
            torch.empty(*lead, cap, dtype=torch.float32, device=device),
            torch.empty(*lead, dtype=torch.int32, device=device))


def select(p, Q, L, ws, out=None, stream=None):
    idx, sc, cnt = out if out is not None else _sel_out(p, False, Q.device)
    _check(sparse_attn_select(p, _ptr(Q), _ptr(L), _ptr(idx), _ptr(sc), _ptr(cnt), _ptr(ws), ws.numel(),
                              _stream(stream)), "sparse_attn_select")
    return idx, sc, cnt


def select_decode(p, q, L, ws, out=None, stream=None):
    idx, sc, cnt = out if out is not None else _sel_out(p, True, q.device)
    _check(sparse_attn_select_decode(p, _ptr(q), _ptr(L), _ptr(idx), _ptr(sc), _ptr(cnt), _ptr(ws), ws.numel(),
                                     _stream(stream)), "sparse_attn_select_decode")
    return idx, sc, cnt


def prefill(p, Q, K, V, idx, sc, cnt, ws, out=None, stream=None):
    torch = _torch()
    if out is None:
        O = torch.empty_like(Q)
        lse = torch.empty(p.B, p.Hq, p.N, dtype=torch.float32, device=Q.device)
    else:
        O, lse = out
    _check(sparse_attn_prefill(p, _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(sc), _ptr(cnt), _ptr(O), _ptr(lse),
                               _ptr(ws), ws.numel(), _stream(stream)), "sparse_attn_prefill")
    return O, lse


def decode(p, q, K, V, idx, sc, cnt, ws, out=None, stream=None):
    torch = _torch()
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(p.B, p.Hq, dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(sparse_attn_decode(p, _ptr(q), _ptr(K), _ptr(V), _ptr(idx), _ptr(sc), _ptr(cnt), _ptr(o), _ptr(lse),
                              _ptr(ws), ws.numel(), _stream(stream)), "sparse_attn_decode")
    return o, lse


def prefill_backward(p, Q, K, V, O, lse, dO, idx, sc, cnt, ws, out=None, stream=None):
    """Gradients of the gated prefill: (dQ, dK, dV, dscore), all fp32."""
    torch = _torch()
    if out is None:
        f32 = dict(dtype=torch.float32, device=Q.device)
        dQ = torch.empty(Q.shape, **f32)
        dK = torch.empty(K.shape, **f32)
        dV = torch.empty(V.shape, **f32)
        dscore = torch.empty(sc.shape, **f32)
    else:
        dQ, dK, dV, dscore = out
    _check(sparse_attn_prefill_backward(p, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), _ptr(dO), _ptr(idx),
                                        _ptr(sc), _ptr(cnt), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dscore), _ptr(ws),
                                        ws.numel(), _stream(stream)), "sparse_attn_prefill_backward")
    return dQ, dK, dV, dscore


def select_backward(p, Q, L, idx, dscore, cnt, dQ, dK, ws, stream=None):
    """Adds the selector's gradient (through pooled query and landmarks) into dQ, dK."""
    _check(sparse_attn_select_backward(p, _ptr(Q), _ptr(L), _ptr(idx), _ptr(dscore), _ptr(cnt), _ptr(dQ), _ptr(dK),
                                       _ptr(ws), ws.numel(), _stream(stream)), "sparse_attn_select_backward")
    return dQ, dK


def make_lsa_params(B, Hq, Hkv, d, N, pool, seg, clusters, top_clusters, sink, window, dtype="bf16",
                    scale=0.0) -> sa_lsa_params:
    dt = {"bf16": SA_BF16, "fp32": SA_FP32}.get(dtype, dtype)
    return sa_lsa_params(B, Hq, Hkv, d, N, pool, seg, clusters, top_clusters, sink, window, dt, float(scale))


def lsa_build(p: sa_lsa_params, K, stream=None):
    """Flat clustered index of K: (centres fp64, members int32, sizes int32)."""
    torch = _torch()
    C = sparse_attn_lsa_clusters(p)
    if C < 0:
        raise SparseAttnError(C, "sparse_attn_lsa_clusters")
    n = max(C, 1)
    centres = torch.empty(p.B, p.Hkv, n, p.d, dtype=torch.float64, device=K.device)
    members = torch.empty(p.B, p.Hkv, n, p.seg, dtype=torch.int32, device=K.device)
    sizes = torch.empty(p.B, p.Hkv, n, dtype=torch.int32, device=K.device)
    _check(sparse_attn_lsa_build(p, _ptr(K), _ptr(centres), _ptr(members), _ptr(sizes), _stream(stream)),
           "sparse_attn_lsa_build")
    return centres, members, sizes


def lsa_workspace(p: sa_lsa_params, device="cuda"):
    torch = _torch()
    n = sparse_attn_lsa_workspace_size(p)
    if n == 0:
        raise SparseAttnError(SA_ERR_ARG, "sparse_attn_lsa_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def lsa_decode(p: sa_lsa_params, q, K, V, index, ws, out=None, kept=None, stream=None):
    """Decode through the flat index: (o, lse).  ``kept``: optional int32
    [B, Hkv] tensor that receives the number of key positions attended."""
    torch = _torch()
    centres, members, sizes = index
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(p.B, p.Hq, dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(sparse_attn_lsa_decode(p, _ptr(q), _ptr(K), _ptr(V), _ptr(centres), _ptr(members), _ptr(sizes), _ptr(o),
                                  _ptr(lse), _ptr(kept), _ptr(ws), ws.numel(), _stream(stream)),
           "sparse_attn_lsa_decode")
    return o, lse


def decode_static(p, q, K, V, idx, sc, cnt, out=None, stream=None):
    """sparse_attn_decode without a workspace: for callers that cannot
    allocate device memory (the library's own static scratch is used)."""
    torch = _torch()
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(p.B, p.Hq, dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(sparse_attn_decode_static(p, _ptr(q), _ptr(K), _ptr(V), _ptr(idx), _ptr(sc), _ptr(cnt), _ptr(o),
                                     _ptr(lse), _stream(stream)), "sparse_attn_decode_static")
    return o, lse


def landmarks_update(p, K, L, seq_len=None, first_block=None, stream=None):
    """Refresh the landmarks of blocks first_block[b] .. (for appends) over
    each sequence's own length; int32 device tensors or None."""
    _check(sparse_attn_landmarks_update(p, _ptr(K), _ptr(L), _ptr(seq_len), _ptr(first_block), _stream(stream)),
           "sparse_attn_landmarks_update")
    return L


def select_decode_varlen(p, q, L, seq_len, ws, out=None, stream=None):
    idx, sc, cnt = out if out is not None else _sel_out(p, True, q.device)
    _check(sparse_attn_select_decode_varlen(p, _ptr(q), _ptr(L), _ptr(seq_len), _ptr(idx), _ptr(sc), _ptr(cnt),
                                            _ptr(ws), ws.numel(), _stream(stream)), "sparse_attn_select_decode_varlen")
    return idx, sc, cnt


def decode_varlen(p, q, K, V, seq_len, idx, sc, cnt, ws, out=None, stream=None):
    torch = _torch()
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(p.B, p.Hq, dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(sparse_attn_decode_varlen(p, _ptr(q), _ptr(K), _ptr(V), _ptr(seq_len), _ptr(idx), _ptr(sc), _ptr(cnt),
                                     _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "sparse_attn_decode_varlen")
    return o, lse


def decode_step(p, q, L, K, V, ws, seq_len=None, sel=None, out=None, stream=None):
    """One decode step: the selection into `sel` (idx, score, count) and the
    decode into `out` (o, lse), the two launches overlapped when the kernels
    allow it.  `ws` must cover SA_OP_SELECT_DECODE and SA_OP_DECODE."""
    torch = _torch()
    idx, sc, cnt = sel if sel is not None else _sel_out(p, True, q.device)
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(p.B, p.Hq, dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    sl = _ptr(seq_len) if seq_len is not None else None
    _check(sparse_attn_decode_step(p, _ptr(q), _ptr(L), _ptr(K), _ptr(V), sl, _ptr(idx), _ptr(sc), _ptr(cnt),
                                   _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "sparse_attn_decode_step")
    return (idx, sc, cnt), (o, lse)


def check_status(ws, stream=None):
    """Raises SparseAttnError when the status word reports a device problem."""
    rc, detail = sparse_attn_check_status(_ptr(ws), _stream(stream))
    if rc != SA_OK:
        raise SparseAttnError(rc, f"device status bits {detail:#x}")
    return detail


def lsa_tree_build(p: sa_lsa_params, fanout: int, index, stream=None):
    """Tree over the flat index's clusters: (tree buffer uint8, workspace)."""
    torch = _torch()
    centres, members, sizes = index
    nbytes, _ = sparse_attn_lsa_tree_size(p, fanout)
    if nbytes == 0:
        raise SparseAttnError(SA_ERR_UNSUPPORTED, "sparse_attn_lsa_tree_size")
    tree = torch.zeros(nbytes, dtype=torch.uint8, device=centres.device)
    ws = torch.zeros(sparse_attn_lsa_tree_workspace_size(p, fanout), dtype=torch.uint8, device=centres.device)
    _check(sparse_attn_lsa_tree_build(p, fanout, _ptr(centres), _ptr(sizes), _ptr(tree), _ptr(ws), ws.numel(),
                                      _stream(stream)), "sparse_attn_lsa_tree_build")
    return tree, ws


def lsa_tree_decode(p: sa_lsa_params, fanout: int, beam: int, q, K, V, index, tree, ws, out=None, kept=None,
                    compared=None, stream=None):
    """Decode through the tree (beam search to the leaves): (o, lse)."""
    torch = _torch()
    centres, members, sizes = index
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(p.B, p.Hq, dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(sparse_attn_lsa_tree_decode(p, fanout, beam, _ptr(q), _ptr(K), _ptr(V), _ptr(centres), _ptr(members),
                                       _ptr(sizes), _ptr(tree), _ptr(o), _ptr(lse), _ptr(kept), _ptr(compared),
                                       _ptr(ws), ws.numel(), _stream(stream)), "sparse_attn_lsa_tree_decode")
    return o, lse


def lsa_tree_levels(p: sa_lsa_params, fanout: int, tree):
    """Views of a built tree buffer, following the layout the header documents:
    a list over levels of dict(mass [B,Hkv,n], and for levels >= 1 centres
    [B,Hkv,n,d], first [B,Hkv,n+1], children [B,Hkv,n_below])."""
    torch = _torch()
    C = sparse_attn_lsa_clusters(p)
    n = [C]
    while n[-1] > fanout:
        n.append((n[-1] + fanout - 1) // fanout)
    bgs = p.B * p.Hkv

    def al(x):
        return (x + 255) & ~255

    off, out = 0, []
    for lv, nl in enumerate(n):
        d = {"mass": tree[off:off + bgs * nl * 8].view(torch.float64).view(p.B, p.Hkv, nl)}
        off += al(bgs * nl * 8)
        if lv > 0:
            d["centres"] = tree[off:off + bgs * nl * p.d * 8].view(torch.float64).view(p.B, p.Hkv, nl, p.d)
            off += al(bgs * nl * p.d * 8)
            d["first"] = tree[off:off + bgs * (nl + 1) * 4].view(torch.int32).view(p.B, p.Hkv, nl + 1)
            off += al(bgs * (nl + 1) * 4)
            d["children"] = tree[off:off + bgs * n[lv - 1] * 4].view(torch.int32).view(p.B, p.Hkv, n[lv - 1])
            off += al(bgs * n[lv - 1] * 4)
        out.append(d)
    return out

"""kv_shared_b200 -- Python binding of libhs2, the B200 HySparse2 hybrid-block library.

Argument marshalling only: every function below forwards torch tensors (device
memory) and the current CUDA stream to the C ABI declared in include/hs2.h, with
the same names, and raises HS2Error on a non-OK status.  All computation runs in
the CUDA kernels of libhs2.so; there is no fallback.  Build the library with
``python -m kv_shared_b200.build`` (or ``__graft_entry__.build()``).
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs2.so")

HS2_F32, HS2_BF16, HS2_E4M3 = 0, 1, 2
HS2_OK, HS2_ERR_INVALID_ARG, HS2_ERR_UNSUPPORTED, HS2_ERR_WORKSPACE, HS2_ERR_CUDA, \
    HS2_ERR_TIMEOUT, HS2_ERR_INDEX = range(7)

EXPORTS = ("hs2_workspace_size", "hs2_workspace_init", "hs2_full_attn_select", "hs2_full_attn_launches",
           "hs2_topk_select",
           "hs2_sparse_attn", "hs2_sparse_attn_noalloc", "hs2_kv_bridge_proj", "hs2_kv_quantize_fp8", "hs2_last_status",
           "hs2_status_string")


class hs2_attn_desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("window", ctypes.c_int32), ("budget", ctypes.c_int32),
                ("q_dtype", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("idx_stride", ctypes.c_int32),
                ("kv_capacity", ctypes.c_int64), ("max_ctx", ctypes.c_int64)]


class HS2Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} ({status})")


_lib = None


def lib():
    """The loaded libhs2.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m kv_shared_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
        dp = ctypes.POINTER(hs2_attn_desc)
        L.hs2_workspace_size.argtypes = [dp, i32]
        L.hs2_workspace_size.restype = sz
        L.hs2_workspace_init.argtypes = [vp, vp]
        L.hs2_full_attn_select.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.hs2_full_attn_launches.argtypes = [dp]
        L.hs2_topk_select.argtypes = [dp, vp, i64, vp, i32, vp, vp, vp, sz, vp]
        L.hs2_sparse_attn.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.hs2_sparse_attn_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.hs2_kv_bridge_proj.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, i64, vp, vp, vp, vp, vp]
        L.hs2_kv_quantize_fp8.argtypes = [vp, i64, i32, vp, vp, vp]
        L.hs2_last_status.argtypes = [vp, vp]
        L.hs2_status_string.argtypes = [ctypes.c_int]
        L.hs2_status_string.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name not in ("hs2_workspace_size", "hs2_status_string"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, status):
    if status != HS2_OK:
        raise HS2Error(fn, status)


def status_string(status):
    return lib().hs2_status_string(int(status)).decode()


def make_desc(batch, n_q, heads, head_dim, window=128, budget=1024, q_dtype=HS2_BF16,
              kv_dtype=HS2_BF16, softmax_scale=0.0, idx_stride=None, kv_capacity=None, max_ctx=None):
    d = hs2_attn_desc()
    d.batch, d.n_q, d.heads, d.head_dim = batch, n_q, heads, head_dim
    d.window, d.budget, d.q_dtype, d.kv_dtype = window, budget, q_dtype, kv_dtype
    d.softmax_scale = softmax_scale
    d.idx_stride = window + budget if idx_stride is None else idx_stride
    d.max_ctx = max_ctx
    d.kv_capacity = max_ctx if kv_capacity is None else kv_capacity
    return d


# ------------------------------------------------------------------ C-ABI calls
def hs2_workspace_size(desc, scores_in_workspace=True):
    return int(lib().hs2_workspace_size(ctypes.byref(desc), int(bool(scores_in_workspace))))


def hs2_full_attn_launches(desc):
    """Kernels one hs2_full_attn_select call with `desc` enqueues (host query)."""
    return int(lib().hs2_full_attn_launches(ctypes.byref(desc)))


def hs2_workspace_init(workspace, stream=None):
    _check("hs2_workspace_init", lib().hs2_workspace_init(_p(workspace), _stream(stream)))


def hs2_full_attn_select(desc, q, k, v, k_scale, v_scale, q_pos0, o, lse, idx, cnt, scores,
                         workspace, stream=None):
    st = lib().hs2_full_attn_select(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(k_scale), _p(v_scale),
                                    _p(q_pos0), _p(o), _p(lse), _p(idx), _p(cnt), _p(scores),
                                    _p(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream))
    _check("hs2_full_attn_select", st)


def hs2_topk_select(desc, scores, score_row_stride, q_pos0, block_size, idx, cnt, workspace, stream=None):
    st = lib().hs2_topk_select(ctypes.byref(desc), _p(scores), int(score_row_stride), _p(q_pos0),
                               int(block_size), _p(idx), _p(cnt), _p(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check("hs2_topk_select", st)


def hs2_sparse_attn(desc, q, k, v, k_scale, v_scale, idx, cnt, o, lse, workspace, stream=None):
    st = lib().hs2_sparse_attn(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(k_scale), _p(v_scale),
                               _p(idx), _p(cnt), _p(o), _p(lse), _p(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check("hs2_sparse_attn", st)


def hs2_sparse_attn_noalloc(desc, q, k, v, k_scale, v_scale, idx, cnt, o, lse, stream=None):
    """hs2_sparse_attn without a workspace: for callers that cannot allocate device memory
    where they call us; scratch is a fixed array inside the library (see include/hs2.h)."""
    st = lib().hs2_sparse_attn_noalloc(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(k_scale), _p(v_scale),
                                       _p(idx), _p(cnt), _p(o), _p(lse), _stream(stream))
    _check("hs2_sparse_attn_noalloc", st)


def hs2_kv_bridge_proj(hidden, w_kv, batch, n, d_model, head_dim, pos0, kv_capacity, k, v,
                       kv_dtype=HS2_BF16, k_scale=None, v_scale=None, stream=None):
    st = lib().hs2_kv_bridge_proj(_p(hidden), _p(w_kv), batch, n, d_model, head_dim, _p(pos0),
                                  int(kv_dtype), int(kv_capacity), _p(k), _p(v), _p(k_scale), _p(v_scale),
                                  _stream(stream))
    _check("hs2_kv_bridge_proj", st)


def hs2_kv_quantize_fp8(src, rows, head_dim, codes, scales, stream=None):
    st = lib().hs2_kv_quantize_fp8(_p(src), int(rows), int(head_dim), _p(codes), _p(scales), _stream(stream))
    _check("hs2_kv_quantize_fp8", st)


def hs2_last_status(workspace, stream=None):
    """Waits for the stream and returns (and clears) the device status word."""
    return int(lib().hs2_last_status(_p(workspace), _stream(stream)))


# ------------------------------------------------------------------ allocation helpers (plumbing)
def alloc_workspace(desc, scores_in_workspace=True, device="cuda"):
    n = hs2_workspace_size(desc, scores_in_workspace)
    if n == 0:
        raise HS2Error("hs2_workspace_size", HS2_ERR_INVALID_ARG)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    hs2_workspace_init(ws)
    return ws


__all__ = ["hs2_attn_desc", "HS2Error", "make_desc", "lib", "status_string", "alloc_workspace",
           "HS2_F32", "HS2_BF16", "HS2_E4M3", "EXPORTS"] + list(EXPORTS)

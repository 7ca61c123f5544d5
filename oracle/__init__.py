"""CPU oracle for the HySparse2 hybrid-block hot path (ctypes binding of hs2_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with the
CUDA path and never imports the product package.

All floating-point routines take and return numpy float64 arrays; inputs are the
exact upcasts of the bytes the GPU path receives (bf16 -> fp64 and
e4m3 * scale -> fp64 are exact).  The arithmetic follows the definitions cited
in hs2_oracle.c:

  full_attn      causal MQA attention, LSE and head-summed key importance
                 (Lynxflow blog, "Two-Level KV Sharing", KV Reuse paragraph)
  select_*       window of the most recent W plus the K_sel best earlier
                 positions (Lynxflow blog, "Token-Level Sparse Selection";
                 MiMo-V3 news flash for the block-of-64 rule)
  sparse_attn    one softmax over the selected positions of the shared cache
                 (Agentik explainer, sections 2 and 3)
  bridge         K/V projection of hidden states (Lynxflow blog, KV Bridging)
  fp8_quantize   per-token e4m3 cache with an fp32 scale (AINews article, FP8
                 caches at one million tokens)
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_full_attn.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                       _f64p, _f64p, _f64p, _i64p, ctypes.c_double,
                                       _f64p, _f64p, ctypes.c_void_p, ctypes.c_int64]
        L.oracle_full_attn.restype = None
        L.oracle_select_tokens.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _f64p, _i32p]
        L.oracle_select_tokens.restype = ctypes.c_int
        L.oracle_select_blocks.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           _f64p, _i32p]
        L.oracle_select_blocks.restype = ctypes.c_int
        L.oracle_sparse_attn.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p, _f64p, _f64p,
                                         _i32p, _i32p, ctypes.c_int, ctypes.c_double, _f64p,
                                         ctypes.c_void_p]
        L.oracle_sparse_attn.restype = None
        L.oracle_bridge.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _f64p, _f64p,
                                    _f64p, _f64p]
        L.oracle_bridge.restype = None
        L.oracle_round_bf16_array.argtypes = [ctypes.c_int64, _f64p, _u16p]
        L.oracle_round_bf16_array.restype = None
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_fp8_quantize.argtypes = [ctypes.c_int64, ctypes.c_int, _f32p, _u8p, _f32p]
        L.oracle_fp8_quantize.restype = None
        L.oracle_fp8_dequantize.argtypes = [ctypes.c_int64, ctypes.c_int, _u8p, _f32p, _f64p]
        L.oracle_fp8_dequantize.restype = None
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- formats
def bf16_to_f64(bits):
    """Exact value of bfloat16 bit patterns (uint16 array) as float64."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x):
    """Nearest bfloat16 (ties to even) of float64 values, as uint16 bit patterns."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_round_bf16_array(x.size, x.reshape(-1), out.reshape(-1))
    return out


def e4m3_decode(codes):
    L = lib()
    table = np.array([L.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(y):
    L = lib()
    y = np.asarray(y, dtype=np.float32)
    return np.array([L.oracle_e4m3_encode(float(v)) for v in y.reshape(-1)],
                    dtype=np.uint8).reshape(y.shape)


def fp8_quantize(x):
    """Per-row e4m3 quantizer of an fp32 [n, D] array -> (codes uint8 [n, D], scales f32 [n])."""
    x = _c(x, np.float32)
    n, D = x.shape
    codes = np.empty((n, D), dtype=np.uint8)
    scales = np.empty(n, dtype=np.float32)
    lib().oracle_fp8_quantize(n, D, x, codes, scales)
    return codes, scales


def fp8_dequantize(codes, scales):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    n, D = codes.shape
    out = np.empty((n, D), dtype=np.float64)
    lib().oracle_fp8_dequantize(n, D, codes, scales, out)
    return out


# --------------------------------------------------------------------------- attention
def default_scale(D):
    return 1.0 / np.sqrt(D)


def full_attn(q, k, v, pos, scale=None, want_scores=True, score_len=None):
    """Causal MQA attention of one sequence.

    q [n_rows, H, D], k/v [n_keys, D], pos [n_rows] absolute positions.
    Returns (o [n_rows, H, D], lse [n_rows, H], scores [n_rows, score_len] or None).
    """
    q = _c(q, np.float64)
    k = _c(k, np.float64)
    v = _c(v, np.float64)
    pos = _c(pos, np.int64)
    n_rows, H, D = q.shape
    n_keys = k.shape[0]
    assert v.shape == k.shape and k.shape[1] == D and pos.shape == (n_rows,)
    assert n_rows == 0 or int(pos.max()) < n_keys
    scale = default_scale(D) if scale is None else float(scale)
    o = np.empty((n_rows, H, D), dtype=np.float64)
    lse = np.empty((n_rows, H), dtype=np.float64)
    scores = None
    ptr = None
    stride = 0
    if want_scores:
        stride = n_keys if score_len is None else int(score_len)
        scores = np.empty((n_rows, stride), dtype=np.float64)
        ptr = scores.ctypes.data_as(ctypes.c_void_p)
    lib().oracle_full_attn(n_rows, H, D, n_keys, q, k, v, pos, scale, o, lse, ptr, stride)
    return o, lse, scores


def select_tokens(score, p, W, K_sel):
    """Window [p-W+1, p] plus the K_sel best of [0, p-W] (score desc, index asc); ascending."""
    score = _c(score, np.float64)
    assert score.shape[0] >= max(p - W + 1, 0)
    out = np.empty(W + K_sel, dtype=np.int32)
    c = lib().oracle_select_tokens(int(p), int(W), int(K_sel), score, out)
    return out[:c].copy()


def select_blocks(score, p, W, K_sel, bs):
    """Window plus the floor(K_sel/bs) best bs-token blocks of [0, p-W] (max rule); ascending."""
    score = _c(score, np.float64)
    out = np.empty(W + (K_sel // bs + 1) * bs + 1, dtype=np.int32)
    c = lib().oracle_select_blocks(int(p), int(W), int(K_sel), int(bs), score, out)
    return out[:c].copy()


def select_rows(scores, pos, W, K_sel, block_size=1, cap=None):
    """Selection for every row: returns (idx [n_rows, cap] int32, -1 padded; cnt [n_rows] int32)."""
    scores = np.asarray(scores)
    n_rows = scores.shape[0]
    cap = W + K_sel if cap is None else cap
    idx = np.full((n_rows, cap), -1, dtype=np.int32)
    cnt = np.zeros(n_rows, dtype=np.int32)
    for r in range(n_rows):
        p = int(pos[r])
        if block_size == 1:
            sel = select_tokens(scores[r], p, W, K_sel)
        else:
            sel = select_blocks(scores[r], p, W, K_sel, block_size)
        assert sel.size <= cap
        idx[r, :sel.size] = sel
        cnt[r] = sel.size
    return idx, cnt


def sparse_attn(q, k, v, idx, cnt, scale=None, want_lse=False):
    """Attention of q [n_rows, H, D] over the selected rows idx[r, :cnt[r]] of k/v [n_keys, D]."""
    q = _c(q, np.float64)
    k = _c(k, np.float64)
    v = _c(v, np.float64)
    idx = _c(idx, np.int32)
    cnt = _c(cnt, np.int32)
    n_rows, H, D = q.shape
    if n_rows:
        assert int(idx[:, :1].min()) >= 0 or int(cnt.min()) == 0
        for r in range(n_rows):
            c = int(cnt[r])
            assert c <= idx.shape[1]
            if c:
                assert 0 <= int(idx[r, :c].min()) and int(idx[r, :c].max()) < k.shape[0]
    scale = default_scale(D) if scale is None else float(scale)
    o = np.empty((n_rows, H, D), dtype=np.float64)
    lse = np.empty((n_rows, H), dtype=np.float64) if want_lse else None
    lib().oracle_sparse_attn(n_rows, H, D, q, k, v, idx, cnt, idx.shape[1], scale, o,
                             lse.ctypes.data_as(ctypes.c_void_p) if want_lse else None)
    return (o, lse) if want_lse else o


def bridge(x, w, D):
    """KV bridging: x [n, dm] @ w [dm, 2D] -> (K [n, D], V [n, D]) exact fp64 products."""
    x = _c(x, np.float64)
    w = _c(w, np.float64)
    n, dm = x.shape
    assert w.shape == (dm, 2 * D)
    kk = np.empty((n, D), dtype=np.float64)
    vv = np.empty((n, D), dtype=np.float64)
    lib().oracle_bridge(n, dm, D, x, w, kk, vv)
    return kk, vv


def hybrid_block(q_full, q_sparse, k, v, pos, W, K_sel, block_size=1, scale=None,
                 score_len=None):
    """One hybrid block for one sequence: full attention with importance, selection,
    then every sparse layer of q_sparse (list of [n_rows, H, D]) over the same cache and
    indices.  Returns a dict of all intermediate results."""
    o_full, lse, scores = full_attn(q_full, k, v, pos, scale=scale, score_len=score_len)
    idx, cnt = select_rows(scores, pos, W, K_sel, block_size=block_size)
    outs = [sparse_attn(qs, k, v, idx, cnt, scale=scale) for qs in q_sparse]
    return {"o_full": o_full, "lse": lse, "scores": scores, "idx": idx, "cnt": cnt,
            "o_sparse": outs}


__all__ = ["bf16_to_f64", "round_bf16", "e4m3_decode", "e4m3_encode", "fp8_quantize",
           "fp8_dequantize", "full_attn", "select_tokens", "select_blocks", "select_rows",
           "sparse_attn", "bridge", "hybrid_block", "default_scale", "lib"]

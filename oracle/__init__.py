"""fp64 CPU oracle for MLA decode over a paged latent cache (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
this package imports nothing from the product: it shares no code with the CUDA
path.  Inputs are the raw bit patterns the GPU sees (bf16 as uint16, the FP8
cache as bytes), decoded exactly inside the C oracle.

Each wrapper names the C routine it calls; the passages each routine follows
are cited in ``mla_oracle.c``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_D = 576


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        f64p = ctypes.POINTER(ctypes.c_double)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_round_bf16.restype = ctypes.c_double
        L.oracle_round_bf16.argtypes = [ctypes.c_double]
        L.oracle_rmsnorm.restype = None
        L.oracle_rmsnorm.argtypes = [f64p, f64p, ctypes.c_int, ctypes.c_double, f64p]
        L.oracle_rope64.restype = None
        L.oracle_rope64.argtypes = [f64p, ctypes.c_double, ctypes.c_double, ctypes.c_int, f64p]
        L.oracle_decode_row656.restype = None
        L.oracle_decode_row656.argtypes = [u8p, f64p]
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [ctypes.c_int, f64p, f64p, ctypes.c_int, f64p, f64p]
        L.oracle_dense_decode.restype = ctypes.c_int
        L.oracle_dense_decode.argtypes = [
            u16p, u16p, ctypes.c_int, i32p, ctypes.c_int, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, i64p, ctypes.c_int64,
            i32p, i32p, f64p, f64p]
        L.oracle_fused_decode.restype = ctypes.c_int
        L.oracle_fused_decode.argtypes = [
            u16p, f64p, ctypes.c_double, ctypes.c_double, i32p, u16p, ctypes.c_int, i32p,
            ctypes.c_int, i32p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, i64p, ctypes.c_int64,
            u8p, f64p, f64p, f64p]
        L.oracle_sparse_decode.restype = ctypes.c_int
        L.oracle_sparse_decode.argtypes = [
            u16p, u8p, ctypes.c_int64, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, i64p, ctypes.c_int64, f64p, f64p]
        L.oracle_e8m0_decode.restype = ctypes.c_double
        L.oracle_e8m0_decode.argtypes = [ctypes.c_uint8]
        L.oracle_decode_row528.restype = None
        L.oracle_decode_row528.argtypes = [u8p, f64p]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_decode_row288.restype = None
        L.oracle_decode_row288.argtypes = [u8p, f64p]
        for fn in (L.oracle_sparse_decode_v41, L.oracle_sparse_decode_v41_fp4):
            fn.restype = ctypes.c_int
            fn.argtypes = [
                u16p, u8p, ctypes.c_int64, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, i64p, ctypes.c_int64, f64p, f64p]
        L.oracle_sparse_decode_v41.restype = ctypes.c_int
        L.oracle_sparse_decode_v41.argtypes = [
            u16p, u8p, ctypes.c_int64, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, i64p, ctypes.c_int64, f64p, f64p]
        L.oracle_fused_sparse_decode.restype = ctypes.c_int
        L.oracle_fused_sparse_decode.argtypes = [
            u16p, f64p, ctypes.c_double, ctypes.c_double, i32p, u8p, ctypes.c_int64, i32p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, i64p, ctypes.c_int64,
            u8p, f64p, f64p]
        L.oracle_sparse_prefill.restype = ctypes.c_int
        L.oracle_sparse_prefill.argtypes = [
            u16p, u16p, ctypes.c_int64, i32p, i32p, f64p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, i64p, ctypes.c_int64, f64p, f64p]
        _LIB = L
    return _LIB


# ------------------------------------------------------------------ helpers

def _np(x, dtype):
    """torch tensor / array -> C-contiguous numpy array of `dtype` (bit view
    for bf16 -> uint16)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                x = x.view(torch.int16).numpy().view(np.uint16)
            elif x.dtype == torch.float8_e4m3fn:
                x = x.view(torch.uint8).numpy()
            else:
                x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x), dtype=dtype) if np.asarray(x).dtype != dtype \
        else np.ascontiguousarray(x)


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


# --------------------------------------------------------------- formats

def e4m3_decode(codes):
    """oracle_e4m3_decode over an array of uint8 codes -> float64."""
    c = _np(codes, np.uint8)
    f = lib().oracle_e4m3_decode
    return np.array([f(int(v)) for v in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_encode(x):
    """oracle_e4m3_encode (RNE, saturating) over an array -> uint8 codes."""
    a = np.asarray(x, dtype=np.float64)
    f = lib().oracle_e4m3_encode
    return np.array([f(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def round_bf16(x):
    """oracle_round_bf16 (ties to even) over an array -> float64."""
    a = np.asarray(x, dtype=np.float64)
    f = lib().oracle_round_bf16
    return np.array([f(float(v)) for v in a.ravel()], dtype=np.float64).reshape(a.shape)


def decode_row656(row):
    """oracle_decode_row656: one 656-byte FP8 cache row -> float64[576]."""
    r = _np(row, np.uint8).ravel()
    assert r.size == 656
    out = np.zeros(_D, dtype=np.float64)
    lib().oracle_decode_row656(_ptr(r, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


def e8m0_decode(codes):
    """oracle_e8m0_decode over an array of uint8 exponent bytes -> float64."""
    c = _np(codes, np.uint8)
    f = lib().oracle_e8m0_decode
    return np.array([f(int(v)) for v in c.ravel()], dtype=np.float64).reshape(c.shape)


def decode_row528(row):
    """oracle_decode_row528: one 528-byte V4.1 FP8 cache row -> float64[512]."""
    r = _np(row, np.uint8).ravel()
    assert r.size == 528
    out = np.zeros(512, dtype=np.float64)
    lib().oracle_decode_row528(_ptr(r, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


def e2m1_decode(codes):
    """oracle_e2m1_decode over an array of 4-bit codes (0..15) -> float64."""
    c = _np(codes, np.uint8)
    f = lib().oracle_e2m1_decode
    return np.array([f(int(v)) for v in c.ravel()], dtype=np.float64).reshape(c.shape)


def decode_row288(row):
    """oracle_decode_row288: one 288-byte V4.1 FP4 cache row -> float64[512]."""
    r = _np(row, np.uint8).ravel()
    assert r.size == 288
    out = np.zeros(512, dtype=np.float64)
    lib().oracle_decode_row288(_ptr(r, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


def rmsnorm(x, g, eps):
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(g, dtype=np.float64)
    y = np.zeros_like(x)
    lib().oracle_rmsnorm(_ptr(x, ctypes.c_double), _ptr(g, ctypes.c_double), x.size, float(eps),
                         _ptr(y, ctypes.c_double))
    return y


def rope64(x, pos, base=10000.0, sign=+1):
    x = np.ascontiguousarray(x, dtype=np.float64)
    assert x.size == 64
    y = np.zeros_like(x)
    lib().oracle_rope64(_ptr(x, ctypes.c_double), float(pos), float(base), int(sign),
                        _ptr(y, ctypes.c_double))
    return y


def combine(lse_i, o_i):
    """oracle_combine: LSE-weighted merge of split partials of one row."""
    lse_i = np.ascontiguousarray(lse_i, dtype=np.float64)
    o_i = np.ascontiguousarray(o_i, dtype=np.float64)
    n, d_v = o_i.shape
    o = np.zeros(d_v, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    lib().oracle_combine(n, _ptr(lse_i, ctypes.c_double), _ptr(o_i, ctypes.c_double), d_v,
                         _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    return o, float(lse[0])


# -------------------------------------------------------------- decode paths

def dense_decode(q, kcache, block_table, cache_seqlens, d_v, softmax_scale, causal=True,
                 rows=None, token_lo=None, token_hi=None, allow_faults=False):
    """oracle_dense_decode.  q [b, s_q, h_q, 576] bf16; kcache [NB, page, 1, 576]
    bf16; block_table [b, max_pages] int32; cache_seqlens [b] int32.
    Returns (out fp64 [b, s_q, h_q, d_v] or [n_rows, d_v], lse fp64).
    A block id outside [0, NB) reads block 0 and a length above
    max_pages * page is cut there; such inputs raise ValueError unless
    allow_faults is set."""
    b, s_q, h_q, dq = q.shape
    assert dq == _D
    page = kcache.shape[1]
    qa = _np(q, np.uint16)
    ka = _np(kcache, np.uint16)
    bt = _np(block_table, np.int32)
    sl = _np(cache_seqlens, np.int32)
    max_pages = bt.shape[1]
    ra = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = b * s_q * h_q if ra is None else ra.size
    lo = None if token_lo is None else np.ascontiguousarray(token_lo, dtype=np.int32)
    hi = None if token_hi is None else np.ascontiguousarray(token_hi, dtype=np.int32)
    out = np.zeros((n, d_v), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = lib().oracle_dense_decode(
        _ptr(qa, ctypes.c_uint16), _ptr(ka, ctypes.c_uint16), kcache.shape[0],
        _ptr(bt, ctypes.c_int32), max_pages, _ptr(sl, ctypes.c_int32), b, s_q, h_q, d_v, page,
        float(softmax_scale), int(bool(causal)), _ptr(ra, ctypes.c_int64), n,
        _ptr(lo, ctypes.c_int32), _ptr(hi, ctypes.c_int32), _ptr(out, ctypes.c_double),
        _ptr(lse, ctypes.c_double))
    if rc != 0 and not allow_faults:
        raise ValueError("block id or sequence length out of range")
    if ra is None:
        return out.reshape(b, s_q, h_q, d_v), lse.reshape(b, s_q, h_q)
    return out, lse


def fused_decode(q_raw, gain, eps, rope_base, kcache, block_table, cache_seqlens, softmax_scale,
                 positions=None, rows=None, want_pre_cast=False, allow_faults=False):
    """oracle_fused_decode (s_q = 1, d_v = 576).
    Returns (codes uint8, scale fp64, lse fp64[, o_pre fp64]).  Out-of-range
    block ids and lengths as in dense_decode."""
    b, s_q, h_q, dq = q_raw.shape
    assert s_q == 1 and dq == _D
    page = kcache.shape[1]
    qa = _np(q_raw, np.uint16)
    g = np.ascontiguousarray(_np(gain, np.float32), dtype=np.float64)
    ka = _np(kcache, np.uint16)
    bt = _np(block_table, np.int32)
    sl = _np(cache_seqlens, np.int32)
    pos = None if positions is None else _np(positions, np.int32)
    ra = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = b * h_q if ra is None else ra.size
    codes = np.zeros((n, _D), dtype=np.uint8)
    scale = np.zeros(n, dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    pre = np.zeros((n, _D), dtype=np.float64) if want_pre_cast else None
    rc = lib().oracle_fused_decode(
        _ptr(qa, ctypes.c_uint16), _ptr(g, ctypes.c_double), float(eps), float(rope_base),
        _ptr(pos, ctypes.c_int32), _ptr(ka, ctypes.c_uint16), kcache.shape[0],
        _ptr(bt, ctypes.c_int32), bt.shape[1], _ptr(sl, ctypes.c_int32), b, h_q, page,
        float(softmax_scale), _ptr(ra, ctypes.c_int64), n, _ptr(codes, ctypes.c_uint8),
        _ptr(scale, ctypes.c_double), _ptr(lse, ctypes.c_double), _ptr(pre, ctypes.c_double))
    if rc != 0 and not allow_faults:
        raise ValueError("block id or sequence length out of range")
    if ra is None:
        codes = codes.reshape(b, 1, h_q, _D)
        scale = scale.reshape(b, 1, h_q)
        lse = lse.reshape(b, 1, h_q)
        if pre is not None:
            pre = pre.reshape(b, 1, h_q, _D)
    return (codes, scale, lse, pre) if want_pre_cast else (codes, scale, lse)


def sparse_decode(q, kcache656, indices, d_v, softmax_scale, rows=None, allow_faults=False):
    """oracle_sparse_decode.  q [b, s_q, h_q, 576] bf16; kcache656 [..., 656] uint8
    (flattened to slots); indices [b, s_q, topk] int32 (-1 = invalid)."""
    b, s_q, h_q, dq = q.shape
    assert dq == _D
    qa = _np(q, np.uint16)
    ca = _np(kcache656, np.uint8).reshape(-1, 656)
    ix = _np(indices, np.int32)
    topk = ix.shape[-1]
    ra = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = b * s_q * h_q if ra is None else ra.size
    out = np.zeros((n, d_v), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = lib().oracle_sparse_decode(
        _ptr(qa, ctypes.c_uint16), _ptr(ca, ctypes.c_uint8), ca.shape[0], _ptr(ix, ctypes.c_int32),
        b, s_q, h_q, topk, d_v, float(softmax_scale), _ptr(ra, ctypes.c_int64), n,
        _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0 and not allow_faults:
        raise ValueError("sparse index out of range")
    if ra is None:
        return out.reshape(b, s_q, h_q, d_v), lse.reshape(b, s_q, h_q)
    return out, lse


def sparse_decode_v41(q, kcache, indices, softmax_scale, rows=None, allow_faults=False):
    """oracle_sparse_decode_v41 (528-byte FP8 rows) or
    oracle_sparse_decode_v41_fp4 (288-byte FP4 rows), told apart by the bytes
    per row.  q [b, s_q, h_q, 512] bf16; kcache [..., 528 | 288] uint8
    (flattened to slots); indices [b, s_q, topk] int32 (-1 = invalid).
    Returns O [.., 512] (V = the whole latent) and LSE."""
    b, s_q, h_q, dq = q.shape
    assert dq == 512
    row = int(kcache.shape[-1])
    assert row in (528, 288)
    fn = lib().oracle_sparse_decode_v41 if row == 528 else lib().oracle_sparse_decode_v41_fp4
    qa = _np(q, np.uint16)
    ca = _np(kcache, np.uint8).reshape(-1, row)
    ix = _np(indices, np.int32)
    topk = ix.shape[-1]
    ra = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = b * s_q * h_q if ra is None else ra.size
    out = np.zeros((n, 512), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = fn(
        _ptr(qa, ctypes.c_uint16), _ptr(ca, ctypes.c_uint8), ca.shape[0], _ptr(ix, ctypes.c_int32),
        b, s_q, h_q, topk, float(softmax_scale), _ptr(ra, ctypes.c_int64), n,
        _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0 and not allow_faults:
        raise ValueError("sparse index out of range")
    if ra is None:
        return out.reshape(b, s_q, h_q, 512), lse.reshape(b, s_q, h_q)
    return out, lse


def fused_sparse_decode(q_raw, gain, eps, rope_base, positions, kcache656, indices,
                        softmax_scale, rows=None, allow_faults=False):
    """oracle_fused_sparse_decode: the fused steps over the valid slots of
    indices [b, 1, topk] in the 656-byte FP8 cache; positions [b] required.
    Returns (codes uint8, scale fp64, lse fp64)."""
    b, s_q, h_q, dq = q_raw.shape
    assert s_q == 1 and dq == _D
    qa = _np(q_raw, np.uint16)
    g = np.ascontiguousarray(_np(gain, np.float32), dtype=np.float64)
    pos = _np(positions, np.int32)
    ca = _np(kcache656, np.uint8).reshape(-1, 656)
    ix = _np(indices, np.int32)
    topk = ix.shape[-1]
    ra = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = b * h_q if ra is None else ra.size
    codes = np.zeros((n, _D), dtype=np.uint8)
    scale = np.zeros(n, dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = lib().oracle_fused_sparse_decode(
        _ptr(qa, ctypes.c_uint16), _ptr(g, ctypes.c_double), float(eps), float(rope_base),
        _ptr(pos, ctypes.c_int32), _ptr(ca, ctypes.c_uint8), ca.shape[0], _ptr(ix, ctypes.c_int32),
        b, h_q, topk, float(softmax_scale), _ptr(ra, ctypes.c_int64), n,
        _ptr(codes, ctypes.c_uint8), _ptr(scale, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0 and not allow_faults:
        raise ValueError("sparse index out of range")
    if ra is None:
        return codes.reshape(b, 1, h_q, _D), scale.reshape(b, 1, h_q), lse.reshape(b, 1, h_q)
    return codes, scale, lse


def sparse_prefill(q, kv, indices, softmax_scale, d_v=512, topk_length=None, attn_sink=None,
                   rows=None, allow_faults=False):
    """oracle_sparse_prefill.  q [s_q, h_q, 576] bf16; kv [s_kv, 576] bf16;
    indices [s_q, topk] int32 (-1 = invalid); topk_length [s_q] int32 or None;
    attn_sink [h_q] or None.  Returns O [s_q, h_q, d_v] and LSE [s_q, h_q]
    (or the sampled rows)."""
    s_q, h_q, dq = q.shape
    assert dq == _D
    qa = _np(q, np.uint16)
    ka = _np(kv, np.uint16).reshape(-1, _D)
    ix = _np(indices, np.int32).reshape(s_q, -1)
    topk = ix.shape[-1]
    tl = None if topk_length is None else _np(topk_length, np.int32)
    sk = None if attn_sink is None else np.ascontiguousarray(_np(attn_sink, np.float32),
                                                             dtype=np.float64)
    ra = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = s_q * h_q if ra is None else ra.size
    out = np.zeros((n, d_v), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = lib().oracle_sparse_prefill(
        _ptr(qa, ctypes.c_uint16), _ptr(ka, ctypes.c_uint16), ka.shape[0], _ptr(ix, ctypes.c_int32),
        _ptr(tl, ctypes.c_int32), _ptr(sk, ctypes.c_double), s_q, h_q, topk, d_v,
        float(softmax_scale), _ptr(ra, ctypes.c_int64), n, _ptr(out, ctypes.c_double),
        _ptr(lse, ctypes.c_double))
    if rc != 0 and not allow_faults:
        raise ValueError("sparse index out of range")
    if ra is None:
        return out.reshape(s_q, h_q, d_v), lse.reshape(s_q, h_q)
    return out, lse

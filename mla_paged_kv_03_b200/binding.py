"""ctypes binding of libmla_b200 (the C ABI in include/mla.h).

Argument marshalling only: every step of the decode path runs in the
library's CUDA kernels.  torch supplies device memory (outputs, workspace) and
the current CUDA stream.  There is no fallback: if the shared library is
missing or was built for another GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_CUDA = -3
MLA_ERR_TIMEOUT = -4

D_QK = 576
EXPORTED = [
    "mla_last_error", "mla_num_sms", "mla_num_sm_parts", "mla_metadata_size",
    "mla_get_metadata", "mla_get_metadata_host", "mla_workspace_size", "mla_fused_workspace_size",
    "mla_decode_fwd",
    "mla_fused_norm_rope_attn_rope_cast", "mla_sparse_workspace_size", "mla_sparse_decode",
    "mla_device_status", "mla_noalloc_scratch_bytes", "mla_decode_fwd_noalloc",
    "mla_set_kernel_events", "mla_sparse_v41_workspace_size", "mla_sparse_decode_v41",
    "mla_sparse_decode_v41_fp4", "mla_sparse_fused_workspace_size",
    "mla_sparse_fused_norm_rope_attn_rope_cast", "mla_sparse_prefill_workspace_size",
    "mla_sparse_prefill_fwd", "mla_set_slot_trace",
]


class MLAError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"libmla_b200 error {code}: {msg}")
        self.code = code


_lib = None


def lib():
    """Load libmla_b200.so (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mla_paged_kv_03_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                 ctypes.c_size_t)
        szp = ctypes.POINTER(ctypes.c_size_t)
        ip = ctypes.POINTER(ctypes.c_int)
        L.mla_last_error.restype = ctypes.c_char_p
        L.mla_last_error.argtypes = []
        L.mla_num_sms.argtypes = [i32, ip]
        L.mla_num_sm_parts.argtypes = [i32, i32, i32, ip]
        L.mla_metadata_size.argtypes = [i32, i32, szp, szp]
        L.mla_get_metadata.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
        L.mla_get_metadata_host.argtypes = [vp, i32, i32, i32, i32, vp, vp]
        L.mla_workspace_size.argtypes = [i32, i32, i32, i32, szp]
        L.mla_fused_workspace_size.argtypes = [i32, i32, i32, szp]
        L.mla_decode_fwd.argtypes = [vp, vp, vp, i32, i32, vp, i32, i32, i32, i32, i32, f32, i32,
                                     vp, vp, i32, vp, sz, vp, vp, vp]
        L.mla_fused_norm_rope_attn_rope_cast.argtypes = [
            vp, vp, f32, f32, vp, vp, vp, i32, i32, vp, i32, i32, f32, vp, vp, i32, vp, sz, vp,
            vp, vp, vp]
        L.mla_sparse_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, szp]
        L.mla_sparse_decode.argtypes = [vp, vp, i64, vp, i32, i32, i32, i32, i32, f32, i32, vp,
                                        sz, vp, vp, vp]
        L.mla_sparse_v41_workspace_size.argtypes = [i32, i32, i32, i32, i32, szp]
        L.mla_sparse_decode_v41.argtypes = [vp, vp, i64, vp, i32, i32, i32, i32, f32, i32, vp,
                                            sz, vp, vp, vp]
        L.mla_sparse_decode_v41_fp4.argtypes = L.mla_sparse_decode_v41.argtypes
        L.mla_sparse_fused_workspace_size.argtypes = [i32, i32, i32, i32, szp]
        L.mla_sparse_prefill_workspace_size.argtypes = [i32, i32, i32, i32, szp]
        L.mla_sparse_prefill_fwd.argtypes = [vp, vp, i64, vp, i32, vp, vp, i32, i32, i32, f32,
                                             i32, vp, sz, vp, vp, vp]
        L.mla_sparse_fused_norm_rope_attn_rope_cast.argtypes = [
            vp, vp, f32, f32, vp, vp, i64, vp, i32, i32, i32, f32, i32, vp, sz, vp, vp, vp, vp]
        L.mla_device_status.argtypes = [ip, i32]
        L.mla_noalloc_scratch_bytes.argtypes = []
        L.mla_set_kernel_events.argtypes = [vp, vp]
        L.mla_set_slot_trace.argtypes = [vp, i64]
        L.mla_decode_fwd_noalloc.argtypes = [vp, vp, vp, i32, i32, vp, i32, i32, i32, i32, i32,
                                             f32, i32, vp, vp, vp]
        for name in EXPORTED:
            if name not in ("mla_last_error", "mla_noalloc_scratch_bytes"):
                getattr(L, name).restype = ctypes.c_int
        L.mla_noalloc_scratch_bytes.restype = ctypes.c_size_t
        _lib = L
    return _lib


def _check(rc):
    if rc != MLA_OK:
        raise MLAError(rc, lib().mla_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require(cond, msg):
    if not cond:
        raise ValueError(msg)


# ---------------------------------------------------------------- scheduler

def mla_num_sms(device=None) -> int:
    """Streaming multiprocessors of `device` (default: the current device)."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    out = ctypes.c_int(0)
    _check(lib().mla_num_sms(dev.index if dev.index is not None else torch.cuda.current_device(),
                             ctypes.byref(out)))
    return int(out.value)


def mla_num_sm_parts(heads_per_kv: int, h_kv: int = 1, device=None) -> int:
    dev = torch.cuda.current_device() if device is None else torch.device(device).index or 0
    out = ctypes.c_int(0)
    _check(lib().mla_num_sm_parts(dev, int(heads_per_kv), int(h_kv), ctypes.byref(out)))
    return out.value


def mla_get_metadata_host(cache_seqlens, heads_per_kv: int, num_sm_parts: int, h_kv: int = 1):
    """Host planner: returns (metadata int32[num_sm_parts, 8], num_splits
    int32[batch + 1]) as CPU tensors."""
    sl = torch.as_tensor(cache_seqlens, dtype=torch.int32).contiguous().cpu()
    b = sl.numel()
    meta = torch.zeros((num_sm_parts, 8), dtype=torch.int32)
    ns = torch.zeros((b + 1,), dtype=torch.int32)
    _check(lib().mla_get_metadata_host(_ptr(sl), b, int(heads_per_kv), int(h_kv),
                                       int(num_sm_parts), _ptr(meta), _ptr(ns)))
    return meta, ns


def mla_get_metadata(cache_seqlens: torch.Tensor, heads_per_kv: int, h_kv: int = 1,
                     num_sm_parts: Optional[int] = None):
    """Device planner on the current stream: (metadata, num_splits, num_sm_parts)."""
    _require(cache_seqlens.is_cuda and cache_seqlens.dtype == torch.int32,
             "cache_seqlens must be a CUDA int32 tensor")
    sl = cache_seqlens.contiguous()
    if num_sm_parts is None:
        num_sm_parts = mla_num_sm_parts(heads_per_kv, h_kv, sl.device)
    b = sl.numel()
    meta = torch.empty((num_sm_parts, 8), dtype=torch.int32, device=sl.device)
    ns = torch.empty((b + 1,), dtype=torch.int32, device=sl.device)
    _check(lib().mla_get_metadata(_ptr(sl), b, int(heads_per_kv), int(h_kv), int(num_sm_parts),
                                  _ptr(meta), _ptr(ns), _stream(sl.device)))
    return meta, ns, num_sm_parts


def mla_workspace_size(batch, rows_per_kv, d_v, num_sm_parts) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().mla_workspace_size(int(batch), int(rows_per_kv), int(d_v), int(num_sm_parts),
                                    ctypes.byref(out)))
    return out.value


def mla_fused_workspace_size(batch, h_q, num_sm_parts) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().mla_fused_workspace_size(int(batch), int(h_q), int(num_sm_parts),
                                          ctypes.byref(out)))
    return out.value


def mla_sparse_workspace_size(batch, s_q, h_q, topk, d_v, num_sm_parts) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().mla_sparse_workspace_size(int(batch), int(s_q), int(h_q), int(topk), int(d_v),
                                           int(num_sm_parts), ctypes.byref(out)))
    return out.value


def mla_sparse_v41_workspace_size(batch, s_q, h_q, topk, num_sm_parts) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().mla_sparse_v41_workspace_size(int(batch), int(s_q), int(h_q), int(topk),
                                               int(num_sm_parts), ctypes.byref(out)))
    return int(out.value)


def mla_sparse_fused_workspace_size(batch, h_q, topk, num_sm_parts) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().mla_sparse_fused_workspace_size(int(batch), int(h_q), int(topk),
                                                 int(num_sm_parts), ctypes.byref(out)))
    return int(out.value)


def mla_sparse_prefill_workspace_size(s_q, h_q, topk, num_sm_parts) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().mla_sparse_prefill_workspace_size(int(s_q), int(h_q), int(topk),
                                                   int(num_sm_parts), ctypes.byref(out)))
    return int(out.value)


def _workspace(nbytes, device, workspace):
    if workspace is not None:
        _require(workspace.numel() * workspace.element_size() >= nbytes, "workspace too small")
        return workspace
    return torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ decode

def mla_decode_fwd(q: torch.Tensor, kcache: torch.Tensor, block_table: torch.Tensor,
                   cache_seqlens: torch.Tensor, d_v: int, metadata: torch.Tensor,
                   num_splits: torch.Tensor, num_sm_parts: int, causal: bool = True,
                   softmax_scale: Optional[float] = None, out=None, lse=None, workspace=None):
    """Dense paged decode.  q [b, s_q, h_q, 576] bf16, kcache [NB, 64, 1, 576]
    bf16, block_table [b, max_pages] int32, cache_seqlens [b] int32.
    Returns (out [b, s_q, h_q, d_v] bf16, lse [b, s_q, h_q] fp32)."""
    _require(q.dim() == 4 and q.shape[-1] == D_QK and q.dtype == torch.bfloat16,
             "q must be [b, s_q, h_q, 576] bf16")
    _require(kcache.dim() == 4 and kcache.shape[1] == 64 and kcache.shape[-1] == D_QK and
             kcache.dtype == torch.bfloat16, "kcache must be [NB, 64, h_kv, 576] bf16")
    b, s_q, h_q, _ = q.shape
    h_kv = kcache.shape[2]
    q = q.contiguous()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D_QK)
    if out is None:
        out = torch.empty((b, s_q, h_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((b, s_q, h_q), dtype=torch.float32, device=q.device)
    ws_bytes = mla_workspace_size(b, s_q * h_q, d_v, num_sm_parts)
    ws = _workspace(ws_bytes, q.device, workspace)
    bt = block_table.contiguous()
    _check(lib().mla_decode_fwd(
        _ptr(q), _ptr(kcache), _ptr(bt), bt.shape[1], kcache.shape[0], _ptr(cache_seqlens), b,
        s_q, h_q, h_kv, int(d_v), float(softmax_scale), int(bool(causal)), _ptr(metadata),
        _ptr(num_splits), int(num_sm_parts), _ptr(ws), ws.numel(), _ptr(out), _ptr(lse),
        _stream(q.device)))
    return out, lse


def mla_set_kernel_events(start: Optional[torch.cuda.Event], stop: Optional[torch.cuda.Event]):
    """Record `start` / `stop` around the attention kernel of the following
    decode calls of this thread (None, None clears)."""
    _check(lib().mla_set_kernel_events(
        None if start is None else ctypes.c_void_p(start.cuda_event),
        None if stop is None else ctypes.c_void_p(stop.cuda_event)))


def mla_set_slot_trace(trace: Optional[torch.Tensor]):
    """Debug slot trace of the following decode calls of this thread: an
    int32 device tensor the kernels write the physical slot of every cache row
    they read into (two planes; layout in include/mla.h), or None to stop."""
    if trace is None:
        _check(lib().mla_set_slot_trace(None, 0))
        return
    _require(trace.dtype == torch.int32 and trace.is_cuda and trace.is_contiguous(),
             "trace must be a contiguous int32 CUDA tensor")
    _check(lib().mla_set_slot_trace(_ptr(trace), trace.numel()))


def mla_noalloc_scratch_bytes() -> int:
    return int(lib().mla_noalloc_scratch_bytes())


def mla_decode_fwd_noalloc(q: torch.Tensor, kcache: torch.Tensor, block_table: torch.Tensor,
                           cache_seqlens: torch.Tensor, d_v: int, causal: bool = True,
                           softmax_scale: Optional[float] = None, out=None, lse=None):
    """Dense paged decode with the planner run inside the call and all scratch
    in the library's fixed device array (no workspace argument).  The output
    tensors are allocated here unless given; the C call itself allocates
    nothing.  Calls on one device share the scratch array: keep them ordered."""
    _require(q.dim() == 4 and q.shape[-1] == D_QK and q.dtype == torch.bfloat16,
             "q must be [b, s_q, h_q, 576] bf16")
    _require(kcache.dim() == 4 and kcache.shape[1] == 64 and kcache.shape[-1] == D_QK and
             kcache.dtype == torch.bfloat16, "kcache must be [NB, 64, h_kv, 576] bf16")
    b, s_q, h_q, _ = q.shape
    q = q.contiguous()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D_QK)
    if out is None:
        out = torch.empty((b, s_q, h_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((b, s_q, h_q), dtype=torch.float32, device=q.device)
    bt = block_table.contiguous()
    with torch.cuda.device(q.device):
        _check(lib().mla_decode_fwd_noalloc(
            _ptr(q), _ptr(kcache), _ptr(bt), bt.shape[1], kcache.shape[0], _ptr(cache_seqlens),
            b, s_q, h_q, kcache.shape[2], int(d_v), float(softmax_scale), int(bool(causal)),
            _ptr(out), _ptr(lse), _stream(q.device)))
    return out, lse


def mla_fused_norm_rope_attn_rope_cast(q_raw, norm_gain, eps, rope_base, kcache, block_table,
                                       cache_seqlens, metadata, num_splits, num_sm_parts,
                                       softmax_scale=None, positions=None, out=None,
                                       out_scale=None, lse=None, workspace=None):
    """Fused RMSNorm -> Q-RoPE -> attention -> conjugate O-RoPE -> E4M3 cast.
    Returns (codes uint8 [b, 1, h_q, 576], scale fp32 [b, 1, h_q], lse)."""
    _require(q_raw.dim() == 4 and q_raw.shape[1] == 1 and q_raw.shape[-1] == D_QK and
             q_raw.dtype == torch.bfloat16, "q_raw must be [b, 1, h_q, 576] bf16")
    b, _, h_q, _ = q_raw.shape
    q_raw = q_raw.contiguous()
    gain = norm_gain.to(torch.float32).contiguous()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D_QK)
    dev = q_raw.device
    if out is None:
        out = torch.empty((b, 1, h_q, D_QK), dtype=torch.uint8, device=dev)
    if out_scale is None:
        out_scale = torch.empty((b, 1, h_q), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((b, 1, h_q), dtype=torch.float32, device=dev)
    ws = _workspace(mla_fused_workspace_size(b, h_q, num_sm_parts), dev, workspace)
    bt = block_table.contiguous()
    pos = None if positions is None else positions.to(torch.int32).contiguous()
    _check(lib().mla_fused_norm_rope_attn_rope_cast(
        _ptr(q_raw), _ptr(gain), float(eps), float(rope_base), _ptr(pos), _ptr(kcache), _ptr(bt),
        bt.shape[1], kcache.shape[0], _ptr(cache_seqlens), b, h_q, float(softmax_scale),
        _ptr(metadata), _ptr(num_splits), int(num_sm_parts), _ptr(ws), ws.numel(), _ptr(out),
        _ptr(out_scale), _ptr(lse), _stream(dev)))
    return out, out_scale, lse


def mla_sparse_decode(q, kcache_fp8, indices, d_v=512, softmax_scale=None, num_sm_parts=None,
                      out=None, lse=None, workspace=None):
    """Token-level sparse decode over an FP8 latent cache whose format is told
    by its bytes per token, as the method's interface does:
      656 bytes  q [b, s_q, h_q, 576] bf16 (mla_sparse_decode)
      528 bytes  V4.1 FP8, q [b, s_q, h_q, 512] bf16, d_v = 512 (mla_sparse_decode_v41)
      288 bytes  V4.1 FP4, q as for 528 (mla_sparse_decode_v41_fp4)
    indices [b, s_q, topk] int32 physical slots (-1 = unused).  Returns
    (out [b, s_q, h_q, d_v] bf16, lse [b, s_q, h_q] fp32)."""
    _require(kcache_fp8.dtype == torch.uint8 and kcache_fp8.shape[-1] in (656, 528, 288),
             "kcache_fp8 must be uint8 [..., 656], [..., 528] or [..., 288]")
    row = int(kcache_fp8.shape[-1])
    width = D_QK if row == 656 else 512
    _require(q.dim() == 4 and q.shape[-1] == width and q.dtype == torch.bfloat16,
             f"q must be [b, s_q, h_q, {width}] bf16 for {row}-byte cache rows")
    _require(row == 656 or d_v == 512, "the V4.1 formats have d_v = 512")
    b, s_q, h_q, _ = q.shape
    q = q.contiguous()
    idx = indices.to(torch.int32).contiguous()
    topk = idx.shape[-1]
    num_slots = kcache_fp8.numel() // row
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(width)
    if num_sm_parts is None:
        num_sm_parts = mla_num_sm_parts(h_q, 1, q.device)
    dev = q.device
    if out is None:
        out = torch.empty((b, s_q, h_q, d_v), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((b, s_q, h_q), dtype=torch.float32, device=dev)
    if row == 656:
        ws = _workspace(mla_sparse_workspace_size(b, s_q, h_q, topk, d_v, num_sm_parts), dev,
                        workspace)
        _check(lib().mla_sparse_decode(
            _ptr(q), _ptr(kcache_fp8), num_slots, _ptr(idx), topk, b, s_q, h_q, int(d_v),
            float(softmax_scale), int(num_sm_parts), _ptr(ws), ws.numel(), _ptr(out), _ptr(lse),
            _stream(dev)))
    else:
        ws = _workspace(mla_sparse_v41_workspace_size(b, s_q, h_q, topk, num_sm_parts), dev,
                        workspace)
        fn = lib().mla_sparse_decode_v41 if row == 528 else lib().mla_sparse_decode_v41_fp4
        _check(fn(
            _ptr(q), _ptr(kcache_fp8), num_slots, _ptr(idx), topk, b, s_q, h_q,
            float(softmax_scale), int(num_sm_parts), _ptr(ws), ws.numel(), _ptr(out), _ptr(lse),
            _stream(dev)))
    return out, lse


MLA_DEVERR_TIMEOUT = 1
MLA_DEVERR_BAD_INDEX = 2


def device_status(reset: bool = True) -> int:
    """Device status word (0 = ok, else code << 16 | site; code 1 = a wait
    expired, 2 = an out-of-range block id, length or index); synchronises the
    device."""
    v = ctypes.c_int(0)
    rc = lib().mla_device_status(ctypes.byref(v), int(bool(reset)))
    if rc not in (MLA_OK, MLA_ERR_TIMEOUT):
        _check(rc)
    return v.value


def mla_sparse_fused_norm_rope_attn_rope_cast(q_raw, norm_gain, eps, rope_base, positions,
                                              kcache_fp8, indices, softmax_scale=None,
                                              num_sm_parts=None, out=None, out_scale=None,
                                              lse=None, workspace=None):
    """The fused decode in sparse mode over the 656-byte FP8 cache.
    q_raw [b, 1, h_q, 576] bf16; positions [b] int32 (required); indices
    [b, 1, topk] int32 physical slots (-1 = unused).  Returns (codes uint8
    [b, 1, h_q, 576], scale fp32 [b, 1, h_q], lse fp32 [b, 1, h_q])."""
    _require(q_raw.dim() == 4 and q_raw.shape[1] == 1 and q_raw.shape[-1] == D_QK and
             q_raw.dtype == torch.bfloat16, "q_raw must be [b, 1, h_q, 576] bf16")
    _require(kcache_fp8.dtype == torch.uint8 and kcache_fp8.shape[-1] == 656,
             "kcache_fp8 must be uint8 [..., 656]")
    _require(positions is not None, "positions are required in sparse mode")
    b, _, h_q, _ = q_raw.shape
    q_raw = q_raw.contiguous()
    gain = norm_gain.to(torch.float32).contiguous()
    pos = positions.to(torch.int32).contiguous()
    idx = indices.to(torch.int32).contiguous()
    topk = idx.shape[-1]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D_QK)
    if num_sm_parts is None:
        num_sm_parts = mla_num_sm_parts(h_q, 1, q_raw.device)
    dev = q_raw.device
    if out is None:
        out = torch.empty((b, 1, h_q, D_QK), dtype=torch.uint8, device=dev)
    if out_scale is None:
        out_scale = torch.empty((b, 1, h_q), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((b, 1, h_q), dtype=torch.float32, device=dev)
    ws = _workspace(mla_sparse_fused_workspace_size(b, h_q, topk, num_sm_parts), dev, workspace)
    _check(lib().mla_sparse_fused_norm_rope_attn_rope_cast(
        _ptr(q_raw), _ptr(gain), float(eps), float(rope_base), _ptr(pos), _ptr(kcache_fp8),
        kcache_fp8.numel() // 656, _ptr(idx), topk, b, h_q, float(softmax_scale),
        int(num_sm_parts), _ptr(ws), ws.numel(), _ptr(out), _ptr(out_scale), _ptr(lse),
        _stream(dev)))
    return out, out_scale, lse


def mla_sparse_prefill_fwd(q, kv, indices, softmax_scale=None, d_v=512, topk_length=None,
                           attn_sink=None, num_sm_parts=None, out=None, lse=None,
                           workspace=None):
    """Token-level sparse prefill (no batch dimension).  q [s_q, h_q, 576] bf16;
    kv [s_kv, 576] bf16 (or [s_kv, 1, 576]); indices [s_q, topk] (or
    [s_q, 1, topk]) int32 rows of kv (-1 = unused); topk_length [s_q] int32 or
    None; attn_sink [h_q] fp32 or None.  Returns (out [s_q, h_q, d_v] bf16,
    lse [s_q, h_q] fp32)."""
    _require(q.dim() == 3 and q.shape[-1] == D_QK and q.dtype == torch.bfloat16,
             "q must be [s_q, h_q, 576] bf16")
    _require(kv.dtype == torch.bfloat16 and kv.shape[-1] == D_QK, "kv must be [s_kv, 576] bf16")
    s_q, h_q, _ = q.shape
    q = q.contiguous()
    kv = kv.contiguous()
    idx = indices.to(torch.int32).contiguous().view(s_q, -1)
    topk = idx.shape[-1]
    tl = None if topk_length is None else topk_length.to(torch.int32).contiguous()
    sk = None if attn_sink is None else attn_sink.to(torch.float32).contiguous()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D_QK)
    if num_sm_parts is None:
        num_sm_parts = mla_num_sm_parts(h_q, 1, q.device)
    dev = q.device
    if out is None:
        out = torch.empty((s_q, h_q, d_v), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((s_q, h_q), dtype=torch.float32, device=dev)
    ws = _workspace(mla_sparse_prefill_workspace_size(s_q, h_q, topk, num_sm_parts), dev,
                    workspace)
    _check(lib().mla_sparse_prefill_fwd(
        _ptr(q), _ptr(kv), kv.numel() // D_QK, _ptr(idx), topk, _ptr(tl), _ptr(sk), s_q, h_q,
        int(d_v), float(softmax_scale), int(num_sm_parts), _ptr(ws), ws.numel(), _ptr(out),
        _ptr(lse), _stream(dev)))
    return out, lse

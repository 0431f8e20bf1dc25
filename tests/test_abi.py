"""The C-ABI library loads on a machine without a GPU, exports every symbol
that include/mla.h declares, and rejects bad arguments before launching."""
import ctypes
import os
import re

import pytest
import torch

from mla_paged_kv_03_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = declared_functions()
    assert len(names) >= 10
    L = B.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(B.EXPORTED)


def test_no_other_global_symbols_leak():
    out = os.popen(f"nm -D --defined-only {B.LIB_PATH}").read().split("\n")
    funcs = [l.split()[-1] for l in out if " T " in l]
    assert set(funcs) == set(declared_functions()), set(funcs) ^ set(declared_functions())


def call_decode(**over):
    args = dict(q=16, kc=16, bt=16, max_pages=4, num_blocks=8, sl=16, batch=2, s_q=1, h_q=16,
                h_kv=1, d_v=512, scale=0.04, causal=1, meta=16, ns=16, parts=4, ws=16,
                ws_bytes=1 << 30, out=16, lse=16)
    args.update(over)
    a = args
    return B.lib().mla_decode_fwd(a["q"], a["kc"], a["bt"], a["max_pages"], a["num_blocks"], a["sl"],
                                  a["batch"], a["s_q"], a["h_q"], a["h_kv"], a["d_v"], a["scale"],
                                  a["causal"], a["meta"], a["ns"], a["parts"], a["ws"],
                                  a["ws_bytes"], a["out"], a["lse"], None)


@pytest.mark.parametrize("over,code", [
    (dict(h_kv=2), B.MLA_ERR_UNSUPPORTED),
    (dict(d_v=256), B.MLA_ERR_INVALID_ARG),
    (dict(q=None), B.MLA_ERR_INVALID_ARG),
    (dict(q=18), B.MLA_ERR_INVALID_ARG),       # misaligned (not 16-byte)
    (dict(kc=24), B.MLA_ERR_INVALID_ARG),
    (dict(scale=0.0), B.MLA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.MLA_ERR_INVALID_ARG),
    (dict(parts=0), B.MLA_ERR_INVALID_ARG),
    (dict(s_q=0), B.MLA_ERR_INVALID_ARG),
    (dict(ws_bytes=10), B.MLA_ERR_INVALID_ARG),
    (dict(max_pages=0), B.MLA_ERR_INVALID_ARG),
    (dict(num_blocks=1 << 26), B.MLA_ERR_INVALID_ARG),
])
def test_decode_rejects_before_launch(over, code):
    assert call_decode(**over) == code
    assert B.lib().mla_last_error().decode() != ""


def test_decode_empty_batch_is_a_no_op():
    assert call_decode(batch=0) == B.MLA_OK


def test_sparse_and_fused_validation():
    L = B.lib()
    rc = L.mla_sparse_decode(16, 16, 100, 16, 2048, 2, 1, 128, 576, 0.04, 74, 256, 1 << 30, 16, 16,
                             None)
    assert rc == B.MLA_ERR_INVALID_ARG  # d_v must be 512
    rc = L.mla_sparse_decode(16, 16, 0, 16, 2048, 2, 1, 128, 512, 0.04, 74, 256, 1 << 30, 16, 16,
                             None)
    assert rc == B.MLA_ERR_INVALID_ARG  # num_slots
    rc = L.mla_sparse_decode_v41(16, 16, 100, 16, 0, 2, 1, 128, 0.04, 74, 256, 1 << 30, 16, 16,
                                 None)
    assert rc == B.MLA_ERR_INVALID_ARG  # topk must be >= 1
    rc = L.mla_sparse_decode_v41(16, 16, 100, 16, 2048, 2, 1, 128, 0.04, 74, 256, 1024, 16, 16,
                                 None)
    assert rc == B.MLA_ERR_INVALID_ARG  # workspace too small
    assert "workspace" in L.mla_last_error().decode()
    rc = L.mla_sparse_decode_v41(16, 16, 100, 16, 2048, 0, 1, 128, 0.04, 74, 256, 1 << 30, 16,
                                 16, None)
    assert rc == B.MLA_OK  # empty batch: nothing launched
    rc = L.mla_sparse_fused_norm_rope_attn_rope_cast(16, 16, 1e-6, 1e4, None, 16, 100, 16, 2048,
                                                     2, 64, 0.04, 74, 256, 1 << 30, 16, 16, 16,
                                                     None)
    assert rc == B.MLA_ERR_INVALID_ARG  # positions are required
    assert "positions" in L.mla_last_error().decode()
    rc = L.mla_sparse_fused_norm_rope_attn_rope_cast(16, 16, 1e-6, 1e4, 16, 16, 100, 16, 2048,
                                                     2, 64, 0.04, 74, 256, 4096, 16, 16, 16, None)
    assert rc == B.MLA_ERR_INVALID_ARG  # workspace too small
    rc = L.mla_sparse_prefill_fwd(16, 16, 100, 16, 64, None, None, 8, 128, 576, 0.04, 74, 256,
                                  1 << 30, 16, 16, None)
    assert rc == B.MLA_ERR_INVALID_ARG  # d_v must be 512
    rc = L.mla_sparse_prefill_fwd(16, 16, 100, 16, 64, None, None, 8, 128, 512, 0.04, 74, 256,
                                  1024, 16, 16, None)
    assert rc == B.MLA_ERR_INVALID_ARG  # workspace too small
    rc = L.mla_sparse_prefill_fwd(16, 16, 100, 16, 64, None, None, 0, 128, 512, 0.04, 74, 256,
                                  1 << 30, 16, 16, None)
    assert rc == B.MLA_OK  # no query token: nothing launched
    rc = L.mla_fused_norm_rope_attn_rope_cast(16, 16, -1.0, 1e4, None, 16, 16, 4, 8, 16, 2, 64,
                                              0.04, 16, 16, 4, 16, 1 << 30, 16, 16, 16, None)
    assert rc == B.MLA_ERR_INVALID_ARG  # eps < 0


def test_size_queries():
    m = ctypes.c_size_t()
    s = ctypes.c_size_t()
    assert B.lib().mla_metadata_size(10, 74, ctypes.byref(m), ctypes.byref(s)) == 0
    assert m.value == 74 * 8 * 4 and s.value == 11 * 4
    n = B.mla_workspace_size(64, 128, 512, 74)
    assert n >= (64 + 74) * 128 * 512 * 4
    assert B.mla_sparse_workspace_size(32, 1, 128, 2048, 512, 74) > n // 2
    assert B.mla_sparse_fused_workspace_size(32, 64, 2048, 148) >= 32 * 2048 * 576 * 2
    # the fused decode adds the prologue's query rows to the dense workspace
    assert (B.mla_fused_workspace_size(32, 64, 148) >=
            B.mla_workspace_size(32, 64, 576, 148) + 32 * 64 * 576 * 2)
    assert (B.mla_sparse_fused_workspace_size(32, 64, 2048, 148) >=
            B.mla_fused_workspace_size(32, 64, 148) + 32 * 2048 * 576 * 2)
    # prefill: partials only for tokens split over several parts (at most
    # 2 * parts of them), plus per-token tables of one pass of <= 8192 tokens and
    # the list of split tokens (one entry per part)
    n_pf = B.mla_sparse_prefill_workspace_size(4096, 128, 2048, 74)
    partials = 2 * 74 * 128 * (512 + 1) * 4
    assert partials <= n_pf < partials + 4096 * 12 + 74 * 36 + 6 * 256
    assert (B.mla_sparse_prefill_workspace_size(20000, 128, 2048, 74) ==
            B.mla_sparse_prefill_workspace_size(8192, 128, 2048, 74))
    # the V4.1 workspace adds the query widened to 576 dims
    assert (B.mla_sparse_v41_workspace_size(32, 1, 128, 2048, 74) >=
            B.mla_sparse_workspace_size(32, 1, 128, 2048, 512, 74) + 32 * 128 * 576 * 2)


# Every pointer argument of every compute entry point: set to NULL, the call
# must fail with MLA_ERR_INVALID_ARG before it launches anything.  Fake but
# aligned addresses fill the other slots (nothing dereferences them).
def _sparse(L, **o):
    a = dict(q=16, kc=16, ns=100, idx=16, topk=64, b=2, s_q=1, h_q=128, d_v=512, scale=0.04,
             parts=74, ws=256, wsb=1 << 30, out=16, lse=16)
    a.update(o)
    return L.mla_sparse_decode(a["q"], a["kc"], a["ns"], a["idx"], a["topk"], a["b"], a["s_q"],
                               a["h_q"], a["d_v"], a["scale"], a["parts"], a["ws"], a["wsb"],
                               a["out"], a["lse"], None)


def _v41(fn, L, **o):
    a = dict(q=16, kc=16, ns=100, idx=16, topk=64, b=2, s_q=1, h_q=128, scale=0.04, parts=74,
             ws=256, wsb=1 << 30, out=16, lse=16)
    a.update(o)
    return getattr(L, fn)(a["q"], a["kc"], a["ns"], a["idx"], a["topk"], a["b"], a["s_q"],
                          a["h_q"], a["scale"], a["parts"], a["ws"], a["wsb"], a["out"],
                          a["lse"], None)


def _fused(L, **o):
    a = dict(q=16, g=16, pos=None, kc=16, bt=16, sl=16, meta=16, ns=16, ws=16, out=16, sc=16,
             lse=16)
    a.update(o)
    return L.mla_fused_norm_rope_attn_rope_cast(a["q"], a["g"], 1e-6, 1e4, a["pos"], a["kc"],
                                                a["bt"], 4, 8, a["sl"], 2, 64, 0.04, a["meta"],
                                                a["ns"], 4, a["ws"], 1 << 30, a["out"], a["sc"],
                                                a["lse"], None)


def _fused_sparse(L, **o):
    a = dict(q=16, g=16, pos=16, kc=16, idx=16, ws=256, out=16, sc=16, lse=16)
    a.update(o)
    return L.mla_sparse_fused_norm_rope_attn_rope_cast(a["q"], a["g"], 1e-6, 1e4, a["pos"],
                                                       a["kc"], 100, a["idx"], 64, 2, 64, 0.04,
                                                       74, a["ws"], 1 << 30, a["out"], a["sc"],
                                                       a["lse"], None)


def _prefill(L, **o):
    a = dict(q=16, kv=16, idx=16, ws=256, out=16, lse=16)
    a.update(o)
    return L.mla_sparse_prefill_fwd(a["q"], a["kv"], 100, a["idx"], 64, None, None, 8, 128, 512,
                                    0.04, 74, a["ws"], 1 << 30, a["out"], a["lse"], None)


def _noalloc(L, **o):
    a = dict(q=16, kc=16, bt=16, sl=16, out=16, lse=16)
    a.update(o)
    return L.mla_decode_fwd_noalloc(a["q"], a["kc"], a["bt"], 4, 100, a["sl"], 2, 1, 16, 1, 512,
                                    0.04, 1, a["out"], a["lse"], None)


@pytest.mark.parametrize("call,pointer", [
    (lambda L, **o: _sparse(L, **o), p) for p in ("q", "kc", "idx", "ws", "out", "lse")
] + [
    (lambda L, **o: _noalloc(L, **o), p) for p in ("q", "kc", "bt", "sl", "out", "lse")
] + [
    (lambda L, **o: _v41("mla_sparse_decode_v41", L, **o), p)
    for p in ("q", "kc", "idx", "ws", "out", "lse")
] + [
    (lambda L, **o: _v41("mla_sparse_decode_v41_fp4", L, **o), p)
    for p in ("q", "kc", "idx", "ws", "out", "lse")
] + [
    (lambda L, **o: _fused(L, **o), p)
    for p in ("q", "g", "kc", "bt", "sl", "meta", "ns", "ws", "out", "sc", "lse")
] + [
    (lambda L, **o: _fused_sparse(L, **o), p)
    for p in ("q", "g", "pos", "kc", "idx", "ws", "out", "sc", "lse")
] + [
    (lambda L, **o: _prefill(L, **o), p) for p in ("q", "kv", "idx", "ws", "out", "lse")
])
def test_null_pointers_are_rejected_before_launch(call, pointer):
    L = B.lib()
    assert call(L, **{pointer: None}) == B.MLA_ERR_INVALID_ARG
    assert L.mla_last_error().decode() != ""


def test_slot_trace_too_small_is_rejected_before_launch():
    L = B.lib()
    assert L.mla_set_slot_trace(16, 200) == B.MLA_OK  # each call below needs >= 256
    try:
        assert call_decode() == B.MLA_ERR_INVALID_ARG
        assert "slot trace" in L.mla_last_error().decode()
        assert _sparse(L) == B.MLA_ERR_INVALID_ARG
        assert _prefill(L) == B.MLA_ERR_INVALID_ARG
    finally:
        assert L.mla_set_slot_trace(None, 0) == B.MLA_OK
    assert L.mla_set_slot_trace(18, 100) == B.MLA_ERR_INVALID_ARG  # misaligned


def test_max_pages_beyond_int32_tokens_is_rejected():
    assert call_decode(max_pages=1 << 25) == B.MLA_ERR_INVALID_ARG

"""Index and block-table handling on the GPU, bit for bit.

- Inputs that name nothing in the cache (a block id outside [0, num_blocks),
  a length above max_pages * 64, a sparse index outside [0, num_slots)) take
  the documented stand-in, set status code 2, and stop no kernel: the result
  matches the oracle's reading (dense) or the same call with those entries
  set to -1 (sparse) exactly, and a clean call that follows on the same
  stream, with the status not reset, is correct.
- The debug slot trace records the physical slot of every cache row each
  kernel read; it must equal what the block table (dense) or the indices
  (sparse) name.
Every path checks its indices before it loads, so no case here reads outside
its buffers.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_paged_kv_03_b200 import binding as B
from mla_paged_kv_03_b200 import workloads as W
from parity_util import assert_fp8_close, assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

BAD = B.MLA_DEVERR_BAD_INDEX

# (s_q, h_q, d_v): page kernel, 1-CTA kernel, CTA-pair kernel, 1-CTA with d_v 576
DENSE_SHAPES = [(2, 16, 512), (1, 64, 512), (1, 128, 512), (1, 16, 576)]


def status_code(reset):
    return B.device_status(reset=reset) >> 16


def dense_gpu(case, bt=None, sl=None):
    dev = torch.device("cuda")
    bt = (case.block_table if bt is None else bt).to(dev)
    sl = (case.cache_seqlens if sl is None else sl).to(dev)
    meta, ns, parts = B.mla_get_metadata(sl, case.s_q * case.h_q, 1)
    return B.mla_decode_fwd(case.q.to(dev), case.kcache.to(dev), bt, sl, case.d_v, meta, ns,
                            parts, causal=case.causal, softmax_scale=case.softmax_scale)


def dense_oracle(case, bt=None, sl=None):
    bt = case.block_table if bt is None else bt
    sl = case.cache_seqlens if sl is None else sl
    return oracle.dense_decode(case.q, case.kcache, bt, sl, case.d_v, case.softmax_scale,
                               causal=case.causal, allow_faults=True)


def assert_clean_call_after_fault(case):
    """A correct call right after a faulty one, status not reset in between."""
    out, lse = dense_gpu(case)
    torch.cuda.synchronize()
    ro, rl = dense_oracle(case)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    assert status_code(reset=True) == BAD  # sticky until reset
    assert B.device_status() == 0


@pytest.mark.parametrize("s_q,h_q,d_v", DENSE_SHAPES)
def test_dense_out_of_range_block_ids(s_q, h_q, d_v):
    B.device_status(reset=True)
    case = W.make_dense([700, 130, 64], s_q, h_q, seed=31, d_v=d_v, spare_blocks=2)
    nb = case.kcache.shape[0]
    bt = case.block_table.clone()
    bt[0, 3] = nb + 11
    bt[0, 10] = -5          # the last (partial) page of sequence 0
    bt[1, 0] = 1 << 30
    out, lse = dense_gpu(case, bt=bt)
    torch.cuda.synchronize()
    assert status_code(reset=False) == BAD
    ro, rl = dense_oracle(case, bt=bt)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    assert_clean_call_after_fault(case)


@pytest.mark.parametrize("s_q,h_q,d_v", DENSE_SHAPES)
def test_dense_length_beyond_the_block_table(s_q, h_q, d_v):
    B.device_status(reset=True)
    case = W.make_dense([700, 130], s_q, h_q, seed=32, d_v=d_v, spare_blocks=1)
    cap = case.block_table.shape[1] * 64
    sl = torch.tensor([cap + 300, cap + 77], dtype=torch.int32)
    bt = case.block_table.clone()
    bt[bt < 0] = 0  # the longer lengths reach entries the generator left unused
    out, lse = dense_gpu(case, bt=bt, sl=sl)
    torch.cuda.synchronize()
    assert status_code(reset=False) == BAD
    ro, rl = dense_oracle(case, bt=bt, sl=sl)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    assert_clean_call_after_fault(case)


def test_fused_out_of_range_block_id_and_length():
    B.device_status(reset=True)
    case = W.fused(seed=33, seqlens=[400, 129], h_q=64)
    dev = torch.device("cuda")
    nb = case.kcache.shape[0]
    bt = case.block_table.clone()
    bt[0, 2] = nb + 1
    cap = bt.shape[1] * 64
    sl = torch.tensor([400, cap + 5], dtype=torch.int32)
    bt[bt < 0] = 0
    meta, ns, parts = B.mla_get_metadata(sl.to(dev), case.h_q, 1)
    codes, scale, lse = B.mla_fused_norm_rope_attn_rope_cast(
        case.q_raw.to(dev), case.gain.to(dev), case.eps, case.rope_base, case.kcache.to(dev),
        bt.to(dev), sl.to(dev), meta, ns, parts, softmax_scale=case.softmax_scale)
    torch.cuda.synchronize()
    assert status_code(reset=True) == BAD
    rc, rs, rl = oracle.fused_decode(case.q_raw, case.gain, case.eps, case.rope_base, case.kcache,
                                     bt, sl, case.softmax_scale, allow_faults=True)
    assert_fp8_close(codes, scale, rc, rs)
    assert_lse_close(lse, rl)


# ------------------------------------------------------------------ sparse

def _poison(indices, num_slots):
    """Copies of `indices` with some valid entries moved out of range, and the
    same entries set to -1."""
    bad = indices.clone()
    minus = indices.clone()
    sel = torch.zeros_like(indices, dtype=torch.bool)
    sel[..., 7::13] = True
    sel &= indices >= 0
    bad[sel] = num_slots + torch.arange(int(sel.sum()), dtype=torch.int32) % 1000
    far = torch.zeros_like(sel)
    far[..., 11::29] = True
    far &= (indices >= 0) & ~sel
    bad[far] = 1 << 30
    minus[sel | far] = -1
    return bad, minus


def _sparse_call(kind, case, idx):
    dev = torch.device("cuda")
    if kind == "fused_sparse":
        return B.mla_sparse_fused_norm_rope_attn_rope_cast(
            case.q_raw.to(dev), case.gain.to(dev), case.eps, case.rope_base,
            case.positions.to(dev), case.kcache.to(dev), idx.to(dev), case.softmax_scale)
    if kind == "prefill":
        return B.mla_sparse_prefill_fwd(case.q.to(dev), case.kv.to(dev), idx.to(dev),
                                        case.softmax_scale,
                                        topk_length=case.topk_length.to(dev),
                                        attn_sink=case.attn_sink.to(dev))
    return B.mla_sparse_decode(case.q.to(dev), case.kcache.to(dev), idx.to(dev), case.d_v,
                               case.softmax_scale)


def _sparse_case(kind):
    kw = dict(seed=34, batch=2, h_q=64, seqlens=[3000, 900], topk=300)
    if kind == "656":
        return W.sparse(**kw)
    if kind == "528":
        return W.sparse_v41(**kw)
    if kind == "288":
        return W.sparse_v41_fp4(**kw)
    if kind == "fused_sparse":
        return W.fused_sparse(**kw)
    return W.sparse_prefill(seed=34, s_q=70, s_kv=600, h_q=64, topk=256)


def _num_rows(kind, case):
    return case.kv.shape[0] if kind == "prefill" else case.kcache.reshape(
        -1, case.kcache.shape[-1]).shape[0]


@pytest.mark.parametrize("kind", ["656", "528", "288", "fused_sparse", "prefill"])
def test_sparse_out_of_range_indices_equal_minus_one(kind):
    B.device_status(reset=True)
    case = _sparse_case(kind)
    bad, minus = _poison(case.indices, _num_rows(kind, case))
    got = _sparse_call(kind, case, bad)
    torch.cuda.synchronize()
    assert status_code(reset=False) == BAD
    ref = _sparse_call(kind, case, minus)
    clean = _sparse_call(kind, case, case.indices)  # after the fault, status not reset
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        assert torch.equal(g, r)
    assert status_code(reset=True) == BAD
    assert B.device_status() == 0
    # the clean call against the oracle
    if kind == "fused_sparse":
        rc, rs, rl = oracle.fused_sparse_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                                case.positions, case.kcache, case.indices,
                                                case.softmax_scale)
        assert_fp8_close(clean[0], clean[1], rc, rs)
        assert_lse_close(clean[2], rl)
        return
    if kind == "prefill":
        ro, rl = oracle.sparse_prefill(case.q, case.kv, case.indices, case.softmax_scale,
                                       topk_length=case.topk_length, attn_sink=case.attn_sink)
    elif kind == "656":
        ro, rl = oracle.sparse_decode(case.q, case.kcache, case.indices, case.d_v,
                                      case.softmax_scale)
    else:
        ro, rl = oracle.sparse_decode_v41(case.q, case.kcache, case.indices, case.softmax_scale)
    assert_out_close(clean[0], ro)
    assert_lse_close(clean[1], rl)


# -------------------------------------------------------------- slot trace

def _expected_dense_trace(bt, sl, nb):
    b, max_pages = bt.shape
    exp = torch.full((b, max_pages * 64), -2, dtype=torch.int32)
    for i in range(b):
        L = min(int(sl[i]), max_pages * 64)
        for p in range((L + 63) // 64):
            blk = int(bt[i, p])
            blk = blk if 0 <= blk < nb else 0
            exp[i, p * 64:(p + 1) * 64] = blk * 64 + torch.arange(64, dtype=torch.int32)
    return exp


def _traced(n_per_plane, fn):
    trace = torch.full((2 * n_per_plane,), -2, dtype=torch.int32, device="cuda")
    B.mla_set_slot_trace(trace)
    try:
        res = fn()
        torch.cuda.synchronize()
    finally:
        B.mla_set_slot_trace(None)
    return res, trace.cpu().view(2, -1)


@pytest.mark.parametrize("s_q,h_q,d_v", DENSE_SHAPES)
@pytest.mark.parametrize("parts", [None, 3])
def test_dense_slot_trace_matches_block_table(s_q, h_q, d_v, parts):
    B.device_status(reset=True)
    case = W.make_dense([1000, 64, 0, 333, 1], s_q, h_q, seed=35, d_v=d_v, spare_blocks=3)
    nb = case.kcache.shape[0]
    bt = case.block_table.clone()
    bt[3, 2] = nb + 4  # one out-of-range id: traced as block 0
    dev = torch.device("cuda")
    sl = case.cache_seqlens.to(dev)

    def call():
        meta, ns, p = B.mla_get_metadata(sl, s_q * h_q, 1, parts)
        return B.mla_decode_fwd(case.q.to(dev), case.kcache.to(dev), bt.to(dev), sl, d_v, meta,
                                ns, p, causal=case.causal, softmax_scale=case.softmax_scale)

    n = case.batch * bt.shape[1] * 64
    _, tr = _traced(n, call)
    exp = _expected_dense_trace(bt, case.cache_seqlens, nb).view(-1)
    assert torch.equal(tr[0], exp), "rows read as K"
    assert torch.equal(tr[1], exp), "rows read as V"
    assert status_code(reset=True) == BAD


def test_fused_slot_trace_matches_block_table():
    case = W.fused(seed=36, seqlens=[900, 65, 1], h_q=64)
    dev = torch.device("cuda")
    sl = case.cache_seqlens.to(dev)

    def call():
        meta, ns, p = B.mla_get_metadata(sl, case.h_q, 1)
        return B.mla_fused_norm_rope_attn_rope_cast(
            case.q_raw.to(dev), case.gain.to(dev), case.eps, case.rope_base, case.kcache.to(dev),
            case.block_table.to(dev), sl, meta, ns, p, softmax_scale=case.softmax_scale)

    n = case.batch * case.block_table.shape[1] * 64
    _, tr = _traced(n, call)
    exp = _expected_dense_trace(case.block_table, case.cache_seqlens,
                                case.kcache.shape[0]).view(-1)
    assert torch.equal(tr[0], exp) and torch.equal(tr[1], exp)
    assert B.device_status() == 0


@pytest.mark.parametrize("kind", ["656", "528", "288", "fused_sparse", "prefill"])
def test_sparse_slot_trace_matches_indices(kind):
    B.device_status(reset=True)
    case = _sparse_case(kind)
    rows = _num_rows(kind, case)
    bad, _ = _poison(case.indices, rows)
    idx = bad.reshape(-1, bad.shape[-1])
    n = idx.numel()
    _, tr = _traced(n, lambda: _sparse_call(kind, case, bad))
    valid = (idx >= 0) & (idx < rows)
    if kind == "prefill":
        valid &= torch.arange(idx.shape[1])[None, :] < case.topk_length[:, None]
    exp0 = torch.where(valid, idx, torch.full_like(idx, -1))
    if kind == "prefill":  # rows are read in place: plane 1 holds the entry's own position
        pos = torch.arange(idx.shape[1], dtype=torch.int32).expand_as(idx)
        exp1 = torch.where(valid, pos, torch.full_like(idx, -1))
    else:  # compacted in index order
        exp1 = torch.where(valid, valid.to(torch.int32).cumsum(1, dtype=torch.int32) - 1,
                           torch.full_like(idx, -1))
    assert torch.equal(tr[0].view_as(idx), exp0), "slot of each entry"
    assert torch.equal(tr[1].view_as(idx), exp1), "compacted row of each entry"
    assert status_code(reset=True) == BAD

"""GPU parity of the token-level sparse prefill (C ABI mla_sparse_prefill_fwd:
per-token top-k length, per-head attention sinks, one attention launch per
8192 query tokens) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from mla_paged_kv_03_b200 import binding as B
from mla_paged_kv_03_b200 import workloads as W
from parity_util import assert_lse_close, assert_out_close, full_size_rows

pytestmark = pytest.mark.gpu


def run_gpu(case, num_sm_parts=None, topk_length="case", attn_sink="case"):
    dev = torch.device("cuda")
    tl = case.topk_length if isinstance(topk_length, str) else topk_length
    sk = case.attn_sink if isinstance(attn_sink, str) else attn_sink
    out, lse = B.mla_sparse_prefill_fwd(
        case.q.to(dev), case.kv.to(dev), case.indices.to(dev), case.softmax_scale,
        topk_length=None if tl is None else tl.to(dev),
        attn_sink=None if sk is None else sk.to(dev), num_sm_parts=num_sm_parts)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    return out, lse, tl, sk


def check(case, num_sm_parts=None, topk_length="case", attn_sink="case", rows=None, gpu=None):
    out, lse, tl, sk = gpu if gpu is not None else run_gpu(case, num_sm_parts, topk_length,
                                                           attn_sink)
    ro, rl = oracle.sparse_prefill(case.q.cpu(), case.kv.cpu(), case.indices.cpu(),
                                   case.softmax_scale,
                                   topk_length=None if tl is None else tl.cpu(),
                                   attn_sink=None if sk is None else sk.cpu(), rows=rows)
    if rows is not None:
        t = torch.as_tensor(rows)
        out = out.reshape(-1, 512)[t]
        lse = lse.reshape(-1)[t]
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def small(seed=0, s_q=100, s_kv=100, h_q=128, topk=64, **kw):
    return W.sparse_prefill(seed=seed, s_q=s_q, s_kv=s_kv, h_q=h_q, topk=topk, **kw)


def test_prefill_lengths_and_sinks():
    case = small()
    assert int(case.topk_length.min()) < case.topk
    check(case)


def test_prefill_more_tokens_than_one_launch():
    """8200 tokens: two launches of the attention kernel (8192 and 8 tokens),
    checked on every head of the first tokens and of those around the seam."""
    dev = torch.device("cuda")
    case = W.sparse_prefill(seed=5, s_q=8200, s_kv=8200, h_q=16, topk=8, device=dev)
    gpu = run_gpu(case)
    toks = list(range(4)) + list(range(8186, 8200))
    rows = [t * case.h_q + h for t in toks for h in range(case.h_q)]
    check(case, rows=rows, gpu=gpu)


def test_prefill_without_lengths_or_sinks():
    case = small(seed=1, s_q=40, s_kv=300, topk=130)
    check(case, topk_length=None, attn_sink=None)


@pytest.mark.parametrize("h_q", [16, 64])
def test_prefill_head_counts(h_q):
    check(small(seed=2, h_q=h_q, topk=200, s_q=70, s_kv=500))


@pytest.mark.parametrize("parts", [1, 74])
def test_prefill_split_counts(parts):
    check(small(seed=3, s_q=36, s_kv=3000, topk=1000), num_sm_parts=parts)


def test_prefill_empty_tokens_take_the_sink():
    case = small(seed=4, s_q=40)
    tl = case.topk_length.clone()
    tl[3] = 0
    tl[35] = 0
    out, lse, _, _ = gpu = run_gpu(case, topk_length=tl)
    assert (out[3].float() == 0).all() and (out[35].float() == 0).all()
    assert torch.equal(lse[3].cpu(), case.attn_sink)
    check(case, topk_length=tl, gpu=gpu)


def test_prefill_full_size_sampled():
    dev = torch.device("cuda")
    case = W.sparse_prefill(seed=0, device=dev)
    gpu = run_gpu(case)
    rows = full_size_rows(case.h_q, case.topk_length.cpu().numpy(), 64, 9)
    check(case, rows=rows, gpu=gpu)

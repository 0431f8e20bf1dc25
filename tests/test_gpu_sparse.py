"""GPU parity of the token-level sparse decode over the 656-byte FP8 cache
(C ABI mla_sparse_decode) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from mla_paged_kv_03_b200 import binding as B
from mla_paged_kv_03_b200 import workloads as W
from parity_util import assert_lse_close, assert_out_close, full_size_rows

pytestmark = pytest.mark.gpu


def run_gpu(case, num_sm_parts=None, indices=None):
    dev = torch.device("cuda")
    idx = (case.indices if indices is None else indices).to(dev)
    out, lse = B.mla_sparse_decode(case.q.to(dev), case.kcache.to(dev), idx, case.d_v,
                                   case.softmax_scale, num_sm_parts)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    return out, lse


def check(case, num_sm_parts=None, indices=None, rows=None, gpu=None):
    out, lse = gpu if gpu is not None else run_gpu(case, num_sm_parts, indices)
    idx = case.indices if indices is None else indices
    ro, rl = oracle.sparse_decode(case.q.cpu(), case.kcache.cpu(), idx.cpu(), case.d_v,
                                  case.softmax_scale, rows=rows)
    if rows is not None:
        t = torch.as_tensor(rows)
        out = out.reshape(-1, case.d_v)[t]
        lse = lse.reshape(-1)[t]
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def small(seed=0, seqlens=(3000, 700), topk=300, h_q=128, s_q=1, invalid=0.05):
    return W.sparse(seed=seed, batch=len(seqlens), h_q=h_q, s_q=s_q, seqlens=list(seqlens),
                    topk=topk, invalid_frac=invalid)


def test_sparse_small():
    check(small())


@pytest.mark.parametrize("parts", [1, 3, 74])
def test_sparse_split_counts(parts):
    check(small(seed=1), num_sm_parts=parts)


@pytest.mark.parametrize("h_q,s_q", [(16, 1), (64, 2), (128, 2)])
def test_sparse_shapes(h_q, s_q):
    check(small(seed=2, h_q=h_q, s_q=s_q, topk=200))


def test_sparse_all_invalid_and_out_of_range():
    case = small(seed=3, topk=130)
    idx = case.indices.clone()
    idx[0] = -1                      # a query with no valid token
    check(case, indices=idx)


def test_sparse_full_size_sampled():
    dev = torch.device("cuda")
    case = W.sparse(seed=0, device=dev)
    gpu = run_gpu(case)
    valid = (case.indices.cpu() >= 0).sum(-1).reshape(-1).numpy()
    rows = full_size_rows(case.h_q, valid, 48, 5)
    check(case, rows=rows, gpu=gpu)

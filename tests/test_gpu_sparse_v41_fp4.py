"""GPU parity of the token-level sparse decode over the 288-byte V4.1 FP4 cache
(C ABI mla_sparse_decode_v41_fp4, reached through the binding's format
dispatch on the bytes per row) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from mla_paged_kv_03_b200 import workloads as W
from parity_util import full_size_rows
from test_gpu_sparse_v41 import check, run_gpu

pytestmark = pytest.mark.gpu


def small(seed=0, seqlens=(3000, 700), topk=300, h_q=128, s_q=1, invalid=0.05):
    return W.sparse_v41_fp4(seed=seed, batch=len(seqlens), h_q=h_q, s_q=s_q,
                            seqlens=list(seqlens), topk=topk, invalid_frac=invalid)


def test_sparse_v41_fp4_small():
    check(small())


@pytest.mark.parametrize("parts", [1, 74])
def test_sparse_v41_fp4_split_counts(parts):
    check(small(seed=1), num_sm_parts=parts)


@pytest.mark.parametrize("h_q,s_q", [(16, 1), (64, 2)])
def test_sparse_v41_fp4_shapes(h_q, s_q):
    check(small(seed=2, h_q=h_q, s_q=s_q, topk=200))


def test_sparse_v41_fp4_ragged_topk_and_empty_query():
    case = small(seed=3, topk=130)
    idx = case.indices.clone()
    idx[1] = -1
    check(case, indices=idx)


def test_sparse_v41_fp4_full_size_sampled():
    dev = torch.device("cuda")
    case = W.sparse_v41_fp4(seed=0, device=dev)
    gpu = run_gpu(case)
    valid = (case.indices.cpu() >= 0).sum(-1).reshape(-1).numpy()
    rows = full_size_rows(case.h_q, valid, 48, 7)
    check(case, rows=rows, gpu=gpu)

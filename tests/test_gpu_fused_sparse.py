"""GPU parity of the fused decode in sparse mode (C ABI
mla_sparse_fused_norm_rope_attn_rope_cast) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from mla_paged_kv_03_b200 import binding as B
from mla_paged_kv_03_b200 import workloads as W
from parity_util import assert_fp8_close, assert_lse_close, full_size_rows

pytestmark = pytest.mark.gpu


def run_gpu(case, num_sm_parts=None, indices=None):
    dev = torch.device("cuda")
    idx = (case.indices if indices is None else indices).to(dev)
    codes, scale, lse = B.mla_sparse_fused_norm_rope_attn_rope_cast(
        case.q_raw.to(dev), case.gain.to(dev), case.eps, case.rope_base, case.positions.to(dev),
        case.kcache.to(dev), idx, case.softmax_scale, num_sm_parts)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    return codes, scale, lse


def check(case, num_sm_parts=None, indices=None, rows=None, gpu=None):
    codes, scale, lse = gpu if gpu is not None else run_gpu(case, num_sm_parts, indices)
    idx = case.indices if indices is None else indices
    rc, rs, rl = oracle.fused_sparse_decode(case.q_raw.cpu(), case.gain.cpu(), case.eps,
                                            case.rope_base, case.positions.cpu(),
                                            case.kcache.cpu(), idx.cpu(), case.softmax_scale,
                                            rows=rows)
    if rows is not None:
        t = torch.as_tensor(rows)
        codes = codes.reshape(-1, 576)[t]
        scale = scale.reshape(-1)[t]
        lse = lse.reshape(-1)[t]
    assert_fp8_close(codes, scale, rc, rs)
    assert_lse_close(lse, rl)


def small(seed=0, seqlens=(3000, 700, 5000), topk=300, h_q=64):
    return W.fused_sparse(seed=seed, batch=len(seqlens), h_q=h_q, seqlens=list(seqlens),
                          topk=topk)


def test_fused_sparse_small():
    check(small())


@pytest.mark.parametrize("parts", [1, 4, 148])
def test_fused_sparse_split_counts(parts):
    check(small(seed=1), num_sm_parts=parts)


@pytest.mark.parametrize("h_q", [16, 128])
def test_fused_sparse_head_counts(h_q):
    check(small(seed=2, h_q=h_q, topk=200))


def test_fused_sparse_ragged_topk_and_empty_row():
    case = small(seed=3, topk=130)
    idx = case.indices.clone()
    idx[1] = -1  # sequence 1 has no valid slot
    gpu = run_gpu(case, indices=idx)
    codes, scale, lse = gpu
    # the empty rows: O = 0 (either sign of zero), scale 1, LSE = -inf
    assert ((codes[1].cpu() & 0x7F) == 0).all()
    assert (scale[1] == 1.0).all() and torch.isneginf(lse[1]).all()
    rows = np.array([r for r in range(case.batch * case.h_q) if r // case.h_q != 1])
    check(case, indices=idx, rows=rows, gpu=gpu)


def test_fused_sparse_full_size_sampled():
    dev = torch.device("cuda")
    case = W.fused_sparse(seed=0, device=dev)
    gpu = run_gpu(case)
    valid = (case.indices.cpu() >= 0).sum(-1).reshape(-1).numpy()
    rows = full_size_rows(case.h_q, valid, 48, 8)
    check(case, rows=rows, gpu=gpu)

"""GPU parity of the fused RMSNorm -> Q-RoPE -> attention -> conjugate O-RoPE
-> E4M3 cast decode (C ABI mla_fused_norm_rope_attn_rope_cast) against the
fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from mla_paged_kv_03_b200 import binding as B
from mla_paged_kv_03_b200 import workloads as W
from parity_util import assert_fp8_close, assert_lse_close, full_size_rows

pytestmark = pytest.mark.gpu


def run_gpu(case, num_sm_parts=None, positions=None):
    dev = torch.device("cuda")
    sl = case.cache_seqlens.to(dev)
    meta, ns, parts = B.mla_get_metadata(sl, case.h_q, 1, num_sm_parts)
    codes, scale, lse = B.mla_fused_norm_rope_attn_rope_cast(
        case.q_raw.to(dev), case.gain.to(dev), case.eps, case.rope_base, case.kcache.to(dev),
        case.block_table.to(dev), sl, meta, ns, parts, softmax_scale=case.softmax_scale,
        positions=None if positions is None else positions.to(dev))
    torch.cuda.synchronize()
    assert B.device_status() == 0
    return codes, scale, lse


def check(case, num_sm_parts=None, positions=None, rows=None, gpu=None):
    codes, scale, lse = gpu if gpu is not None else run_gpu(case, num_sm_parts, positions)
    cpu = dict(q_raw=case.q_raw.cpu(), gain=case.gain.cpu(), kcache=case.kcache.cpu(),
               block_table=case.block_table.cpu(), cache_seqlens=case.cache_seqlens.cpu())
    rc, rs, rl = oracle.fused_decode(cpu["q_raw"], cpu["gain"], case.eps, case.rope_base,
                                     cpu["kcache"], cpu["block_table"], cpu["cache_seqlens"],
                                     case.softmax_scale, positions=positions, rows=rows)
    if rows is not None:
        t = torch.as_tensor(rows)
        codes = codes.reshape(-1, 576)[t]
        scale = scale.reshape(-1)[t]
        lse = lse.reshape(-1)[t]
    assert_fp8_close(codes, scale, rc, rs)
    assert_lse_close(lse, rl)


def test_fused_small():
    check(W.fused(seed=0, seqlens=[1, 70, 300, 1025], h_q=64))


@pytest.mark.parametrize("parts", [1, 4, 148])
def test_fused_split_counts(parts):
    check(W.fused(seed=1, seqlens=[2048, 511], h_q=64), num_sm_parts=parts)


@pytest.mark.parametrize("h_q", [16, 128])
def test_fused_head_counts(h_q):
    check(W.fused(seed=2, seqlens=[400, 129], h_q=h_q))


def test_fused_explicit_positions():
    case = W.fused(seed=3, seqlens=[300, 90], h_q=64)
    check(case, positions=torch.tensor([5000, 17], dtype=torch.int32))


@pytest.mark.parametrize("batch", [1, 32])
def test_fused_full_size_sampled(batch):
    dev = torch.device("cuda")
    case = W.fused(seed=0, device=dev, batch=batch)
    gpu = run_gpu(case)
    rows = full_size_rows(case.h_q, case.cache_seqlens.cpu().numpy(), 48, batch)
    check(case, rows=rows, gpu=gpu)


@pytest.mark.parametrize("explicit_positions", [False, True])
def test_fused_prologue_rows_bit_exact(explicit_positions):
    """The prologue's normalised, rotated bf16 query rows, read back from the
    workspace (they follow the mla_workspace_size(batch, h_q, 576, parts)
    bytes of split partials), equal the oracle's RMSNorm -> RoPE -> bf16
    rounding bit for bit on every element of 512 rows."""
    dev = torch.device("cuda")
    batch = 8
    case = W.fused(seed=5, batch=batch)
    sl = case.cache_seqlens.to(dev)
    pos = (torch.randint(0, 1 << 20, (batch,), generator=torch.Generator().manual_seed(11),
                         dtype=torch.int32) if explicit_positions else None)
    meta, ns, parts = B.mla_get_metadata(sl, case.h_q, 1)
    ws = torch.zeros((B.mla_fused_workspace_size(batch, case.h_q, parts),), dtype=torch.uint8,
                     device=dev)
    B.mla_fused_norm_rope_attn_rope_cast(
        case.q_raw.to(dev), case.gain.to(dev), case.eps, case.rope_base, case.kcache.to(dev),
        case.block_table.to(dev), sl, meta, ns, parts, softmax_scale=case.softmax_scale,
        positions=None if pos is None else pos.to(dev), workspace=ws)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    rows = batch * case.h_q
    off = B.mla_workspace_size(batch, case.h_q, 576, parts)
    q_gpu = ws[off:off + rows * 576 * 2].view(torch.bfloat16).view(rows, 576).cpu().double().numpy()
    raw = case.q_raw.cpu().double().numpy().reshape(rows, 576)
    gain = case.gain.cpu().double().numpy()
    for r in range(rows):
        b = r // case.h_q
        p = int(pos[b]) if pos is not None else int(case.cache_seqlens[b]) - 1
        y = oracle.rmsnorm(raw[r], gain, case.eps)
        y[512:] = oracle.rope64(y[512:], p, case.rope_base, +1)
        np.testing.assert_array_equal(q_gpu[r], oracle.round_bf16(y), err_msg=f"row {r}")

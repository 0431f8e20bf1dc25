"""GPU parity of the dense paged decode (C ABI mla_decode_fwd) against the
fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from mla_paged_kv_03_b200 import binding as B
from mla_paged_kv_03_b200 import workloads as W
from parity_util import assert_lse_close, assert_out_close, full_size_rows

pytestmark = pytest.mark.gpu


def run_gpu(case, num_sm_parts=None):
    dev = torch.device("cuda")
    q = case.q.to(dev)
    kc = case.kcache.to(dev)
    bt = case.block_table.to(dev)
    sl = case.cache_seqlens.to(dev)
    meta, ns, parts = B.mla_get_metadata(sl, case.s_q * case.h_q, 1, num_sm_parts)
    out, lse = B.mla_decode_fwd(q, kc, bt, sl, case.d_v, meta, ns, parts, causal=case.causal,
                                softmax_scale=case.softmax_scale)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    return out, lse


def check_full(case, num_sm_parts=None):
    out, lse = run_gpu(case, num_sm_parts)
    ro, rl = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 case.d_v, case.softmax_scale, causal=case.causal)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("batch", [97, 2048, 2049, 5000])
def test_device_planner_matches_host_planner(batch):
    # 2048 is the largest batch the device planner deals in parallel; above it
    # one thread deals serially.
    rng = np.random.default_rng(batch)
    for parts in (1, 7, 74, 148):
        sl = rng.integers(0, 20000, size=batch).astype(np.int32)
        sl[:5] = [0, 1, 64, 65, 128]
        hm, hn = B.mla_get_metadata_host(sl, 16, parts)
        dm, dn, _ = B.mla_get_metadata(torch.tensor(sl, device="cuda"), 16, 1, parts)
        assert torch.equal(hm, dm.cpu()) and torch.equal(hn, dn.cpu())


def test_tiny_workload():
    check_full(W.tiny(seed=0))


@pytest.mark.parametrize("parts", [1, 3, 148])
def test_tiny_split_counts(parts):
    check_full(W.tiny(seed=1), num_sm_parts=parts)


@pytest.mark.parametrize("seqlens", [[1], [64], [65], [127, 128, 129], [0, 3, 0], [300, 1, 777]])
def test_edge_lengths(seqlens):
    check_full(W.make_dense(seqlens, 1, 16, seed=2, spare_blocks=2))


@pytest.mark.parametrize("s_q,h_q", [(2, 16), (1, 64), (1, 128), (2, 64), (3, 16), (1, 1)])
def test_row_shapes(s_q, h_q):
    check_full(W.make_dense([200, 513, 64], s_q, h_q, seed=3, spare_blocks=1))


def test_noncausal_and_dv576():
    c = W.make_dense([130, 9], 2, 16, seed=4, causal=False)
    check_full(c)
    c = W.make_dense([130, 9], 1, 16, seed=5, d_v=576)
    check_full(c)


@pytest.mark.parametrize("parts", [1, 5, 148])
def test_compute_bound_shape_reduced(parts):
    """h_q = 128 (two 64-row groups), several tiles and a ragged tail."""
    c = W.make_dense([1000, 333, 129], 1, 128, seed=6, q_std=0.5, k_std=0.5)
    check_full(c, num_sm_parts=parts)


def test_memory_bound_shape_reduced():
    """s_q = 2 causal pair, h_q = 16, lengths spanning several tiles."""
    sl = W.lengths_loguniform(6, 100, 2000, seed=7)
    check_full(W.make_dense(sl, 2, 16, seed=7))


def test_large_scores_trigger_rescale():
    """Growing scores along the sequence force the lazy reference-max update
    on many tiles."""
    c = W.make_dense([1500, 700], 1, 32, seed=8)
    L = 1500
    ramp = torch.linspace(0.2, 4.0, steps=c.kcache.shape[0] * 64).view(-1, 64, 1, 1)
    c.kcache = (c.kcache.float() * ramp).to(torch.bfloat16)
    c.q = (c.q.float() * 3.0).to(torch.bfloat16)
    check_full(c)


@pytest.mark.parametrize("name", ["compute", "memory"])
def test_full_size_sampled(name):
    """Full-size workloads in the benchmark's launch configuration, checked on
    sampled rows the oracle computes one by one."""
    dev = torch.device("cuda")
    case = W.WORKLOADS[name](seed=0, device=dev)
    out, lse = run_gpu(case)
    cpu = W.DenseCase(q=case.q.cpu(), kcache=case.kcache.cpu(), block_table=case.block_table.cpu(),
                      cache_seqlens=case.cache_seqlens.cpu(), s_q=case.s_q, h_q=case.h_q,
                      d_v=case.d_v, causal=case.causal, softmax_scale=case.softmax_scale)
    rows = full_size_rows(case.s_q * case.h_q, cpu.cache_seqlens.numpy(), 48, 0)
    ro, rl = oracle.dense_decode(cpu.q, cpu.kcache, cpu.block_table, cpu.cache_seqlens, cpu.d_v,
                                 cpu.softmax_scale, causal=cpu.causal, rows=rows)
    assert_out_close(out.reshape(-1, case.d_v)[torch.as_tensor(rows)], ro)
    assert_lse_close(lse.reshape(-1)[torch.as_tensor(rows)], rl)
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("h_q,d_v", [(128, 512), (64, 576), (16, 512)])
def test_buffers_aligned_to_16_bytes_only(h_q, d_v):
    """Workspace and output 16-byte aligned but not 32 (the ABI asks for 16):
    the kernels fall back from their 32-byte stores, and the results equal
    those of the call with 256-byte aligned buffers bit for bit."""
    dev = torch.device("cuda")
    case = W.make_dense(W.lengths_uniform(3, 1000, 3000, seed=11), 1, h_q, seed=11, d_v=d_v,
                        name="align16")
    q, kc = case.q.to(dev), case.kcache.to(dev)
    bt, sl = case.block_table.to(dev), case.cache_seqlens.to(dev)
    meta, ns, parts = B.mla_get_metadata(sl, h_q, 1)
    ref_out, ref_lse = B.mla_decode_fwd(q, kc, bt, sl, d_v, meta, ns, parts, causal=case.causal)
    nbytes = B.mla_workspace_size(3, h_q, d_v, parts)
    ws_raw = torch.empty((nbytes + 256,), dtype=torch.uint8, device=dev)
    ws = ws_raw[16:16 + nbytes]
    n_out = 3 * h_q * d_v
    out_raw = torch.empty((n_out + 64,), dtype=torch.bfloat16, device=dev)
    out = out_raw[8:8 + n_out].view(3, 1, h_q, d_v)
    assert ws.data_ptr() % 32 == 16 and out.data_ptr() % 32 == 16
    out, lse = B.mla_decode_fwd(q, kc, bt, sl, d_v, meta, ns, parts, causal=case.causal,
                                out=out, workspace=ws)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    assert int(ns[-1]) > 3  # some sequences were split: the partials went through ws

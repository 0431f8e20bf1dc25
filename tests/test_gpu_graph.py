"""A whole decode step (device planner, attention kernel, combine and, for
sparse, the FP8 gather) recorded as a CUDA graph through the Python binding:
a replay must reproduce the direct call bit for bit, and a replay after new
inputs are written into the same buffers must match the fp64 oracle on those
inputs."""
import pytest
import torch

import oracle
from mla_paged_kv_03_b200 import binding as B
from mla_paged_kv_03_b200 import workloads as W
from parity_util import assert_fp8_close, assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu


def capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def replay_matches_direct(fn, outs):
    fn()
    torch.cuda.synchronize()
    ref = [t.clone() for t in outs]
    g = capture(fn)
    for t in outs:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert B.device_status() == 0
    for a, b in zip(ref, outs):
        assert torch.equal(a, b)
    return g


def test_graph_dense_tiny_and_new_query():
    case = W.tiny(seed=3)
    dev = torch.device("cuda")
    q = case.q.to(dev)
    kc, bt, sl = case.kcache.to(dev), case.block_table.to(dev), case.cache_seqlens.to(dev)
    R = case.s_q * case.h_q
    parts = B.mla_num_sm_parts(R, 1, dev)
    out = torch.empty((case.batch, case.s_q, case.h_q, case.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((case.batch, case.s_q, case.h_q), dtype=torch.float32, device=dev)
    ws = torch.empty((B.mla_workspace_size(case.batch, R, case.d_v, parts),), dtype=torch.uint8,
                     device=dev)

    def step():
        m, n, _ = B.mla_get_metadata(sl, R, 1, parts)
        B.mla_decode_fwd(q, kc, bt, sl, case.d_v, m, n, parts, causal=case.causal,
                         softmax_scale=case.softmax_scale, out=out, lse=lse, workspace=ws)

    g = replay_matches_direct(step, [out, lse])
    gen = torch.Generator().manual_seed(11)
    q_new = (torch.randn(case.q.shape, generator=gen) * 0.5).to(torch.bfloat16)
    q.copy_(q_new.to(dev))
    g.replay()
    torch.cuda.synchronize()
    ro, rl = oracle.dense_decode(q_new, case.kcache, case.block_table, case.cache_seqlens,
                                 case.d_v, case.softmax_scale, causal=case.causal)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_graph_fused():
    case = W.fused(seed=4, seqlens=[1, 70, 300, 1025], h_q=64)
    dev = torch.device("cuda")
    q_raw, gain = case.q_raw.to(dev), case.gain.to(dev)
    kc, bt, sl = case.kcache.to(dev), case.block_table.to(dev), case.cache_seqlens.to(dev)
    b = case.batch
    parts = B.mla_num_sm_parts(case.h_q, 1, dev)
    codes = torch.empty((b, 1, case.h_q, 576), dtype=torch.uint8, device=dev)
    scale = torch.empty((b, 1, case.h_q), dtype=torch.float32, device=dev)
    lse = torch.empty((b, 1, case.h_q), dtype=torch.float32, device=dev)
    ws = torch.empty((B.mla_fused_workspace_size(b, case.h_q, parts),), dtype=torch.uint8, device=dev)

    def step():
        m, n, _ = B.mla_get_metadata(sl, case.h_q, 1, parts)
        B.mla_fused_norm_rope_attn_rope_cast(q_raw, gain, case.eps, case.rope_base, kc, bt, sl, m, n,
                                             parts, softmax_scale=case.softmax_scale, out=codes,
                                             out_scale=scale, lse=lse, workspace=ws)

    replay_matches_direct(step, [codes, scale, lse])
    rc, rs, rl = oracle.fused_decode(case.q_raw.cpu(), case.gain.cpu(), case.eps, case.rope_base,
                                     case.kcache.cpu(), case.block_table.cpu(),
                                     case.cache_seqlens.cpu(), case.softmax_scale)
    assert_fp8_close(codes, scale, rc, rs)
    assert_lse_close(lse, rl)


def test_graph_sparse():
    case = W.sparse(seed=5, batch=2, h_q=128, s_q=1, seqlens=[3000, 700], topk=300,
                    invalid_frac=0.05)
    dev = torch.device("cuda")
    q, kc, idx = case.q.to(dev), case.kcache.to(dev), case.indices.to(dev)
    parts = B.mla_num_sm_parts(case.s_q * case.h_q, 1, dev)
    out = torch.empty((case.batch, case.s_q, case.h_q, case.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((case.batch, case.s_q, case.h_q), dtype=torch.float32, device=dev)
    ws = torch.empty((B.mla_sparse_workspace_size(case.batch, case.s_q, case.h_q, case.topk,
                                                  case.d_v, parts),), dtype=torch.uint8, device=dev)

    def step():
        B.mla_sparse_decode(q, kc, idx, case.d_v, case.softmax_scale, parts, out=out, lse=lse,
                            workspace=ws)

    replay_matches_direct(step, [out, lse])
    ro, rl = oracle.sparse_decode(case.q.cpu(), case.kcache.cpu(), case.indices.cpu(), case.d_v,
                                  case.softmax_scale)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)

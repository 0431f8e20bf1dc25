"""Pins of the oracle's readings for inputs that name nothing in the cache.

- A block id outside [0, num_blocks) is read as block 0.
- A length above max_pages * 64 is read as max_pages * 64; the fused path's
  default query position still follows the length as given.
- A sparse index outside [0, num_slots) is read like -1.

Each reading is checked against torch SDPA (or the library chain of the fused
path) over rows gathered by torch indexing, not against the oracle itself, and
the oracle refuses such inputs unless allow_faults is set.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from mla_paged_kv_03_b200 import workloads as W
from test_oracle_pins import attention_rows, fused_library_reference, sparse_small


def sdpa_rows(q_rows, K, d_v, scale, vis):
    """SDPA (fp64) of query rows [n, 576] over K [L, 576] with row i seeing
    its first vis[i] tokens; LSE by torch.logsumexp."""
    L = K.shape[0]
    mask = torch.arange(L)[None, :] < torch.as_tensor(vis)[:, None]
    o = F.scaled_dot_product_attention(q_rows[None], K[None], K[None, :, :d_v],
                                       attn_mask=mask[None], scale=scale)[0]
    s = ((q_rows @ K.T) * scale).masked_fill(~mask, float("-inf"))
    return o.numpy(), torch.logsumexp(s, dim=-1).numpy()


def gather_k(kcache, blocks, L):
    """fp64 rows [L, 576] of the pages `blocks`, gathered by torch indexing."""
    return kcache[torch.as_tensor(blocks).long(), :, 0, :].reshape(-1, 576)[:L].to(torch.float64)


@pytest.mark.parametrize("bad", [-7, 1 << 20])
def test_out_of_range_block_id_reads_block_zero(bad):
    case = W.make_dense([200, 90], 2, 3, seed=21, spare_blocks=2)
    bt = case.block_table.clone()
    bt[0, 1] = bad          # a middle page of sequence 0
    bt[1, 1] = bad + 3      # the partial last page of sequence 1
    with pytest.raises(ValueError):
        oracle.dense_decode(case.q, case.kcache, bt, case.cache_seqlens, 512, case.softmax_scale)
    o, lse = oracle.dense_decode(case.q, case.kcache, bt, case.cache_seqlens, 512,
                                 case.softmax_scale, allow_faults=True)
    for b, L in enumerate([200, 90]):
        blocks = case.block_table[b, :(L + 63) // 64].clone()
        blocks[1] = 0
        K = gather_k(case.kcache, blocks, L)
        q = case.q[b].to(torch.float64).reshape(-1, 576)
        vis = [L - 2 + 1 + i for i in range(2) for _ in range(3)]
        ro, rl = sdpa_rows(q, K, 512, case.softmax_scale, vis)
        np.testing.assert_allclose(o[b].reshape(-1, 512), ro, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[b].reshape(-1), rl, rtol=1e-12, atol=1e-12)


def test_table_entries_past_the_length_are_not_read():
    """Entries beyond ceil(L / 64) may hold anything: no fault, same result."""
    case = W.make_dense([100, 30], 1, 2, seed=22, spare_blocks=1)
    bt = case.block_table.clone()
    bt[0, 2:] = 123456
    bt[1, 1:] = -99
    o1, l1 = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens, 512,
                                 case.softmax_scale)
    o2, l2 = oracle.dense_decode(case.q, case.kcache, bt, case.cache_seqlens, 512,
                                 case.softmax_scale)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("causal,s_q", [(True, 2), (False, 1)])
def test_length_beyond_table_is_cut_at_the_table(causal, s_q):
    case = W.make_dense([150, 64], s_q, 2, seed=23, causal=causal)
    max_pages = case.block_table.shape[1]
    cap = max_pages * 64
    sl = torch.tensor([cap + 41, 64], dtype=torch.int32)
    with pytest.raises(ValueError):
        oracle.dense_decode(case.q, case.kcache, case.block_table, sl, 512, case.softmax_scale,
                            causal=causal)
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, sl, 512,
                                 case.softmax_scale, causal=causal, allow_faults=True)
    blocks = case.block_table[0, :max_pages]
    assert (blocks >= 0).all()
    K = gather_k(case.kcache, blocks, cap)
    q = case.q[0].to(torch.float64).reshape(-1, 576)
    vis = [(cap - s_q + 1 + i) if causal else cap for i in range(s_q) for _ in range(2)]
    ro, rl = sdpa_rows(q, K, 512, case.softmax_scale, vis)
    np.testing.assert_allclose(o[0].reshape(-1, 512), ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse[0].reshape(-1), rl, rtol=1e-12, atol=1e-12)


def test_fused_length_beyond_table_keeps_the_raw_position():
    """The fused path attends over the tokens the table reaches, and rotates
    at position L - 1 of the length as given."""
    case = W.fused(seed=24, seqlens=[130, 70], h_q=2)
    max_pages = case.block_table.shape[1]
    cap = max_pages * 64
    raw = cap + 9
    pos = torch.tensor([raw - 1, 69], dtype=torch.int32)
    sl = torch.tensor([raw, 70], dtype=torch.int32)
    codes, sc, lse = oracle.fused_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                         case.kcache, case.block_table, sl, case.softmax_scale,
                                         allow_faults=True)
    # reference: the library chain over the capped length, at the raw position
    case.cache_seqlens = torch.tensor([cap, 70], dtype=torch.int32)
    c2, s2, l2 = oracle.fused_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                     case.kcache, case.block_table, case.cache_seqlens,
                                     case.softmax_scale, positions=pos)
    rc, rs, rl, _ = fused_library_reference(case, positions=pos.tolist())
    np.testing.assert_array_equal(codes.reshape(rc.shape), c2.reshape(rc.shape))
    assert (codes.reshape(rc.shape) == rc).mean() >= 0.999
    np.testing.assert_allclose(sc.reshape(rs.shape), rs, rtol=1e-12)
    np.testing.assert_allclose(lse.reshape(rl.shape), rl, rtol=1e-12, atol=1e-12)


def test_sparse_out_of_range_index_reads_like_minus_one():
    case = sparse_small(seed=25)
    num_slots = case.kcache.reshape(-1, 656).shape[0]
    ix = case.indices.clone()
    ix[..., 3::17] = num_slots + 5
    ix[..., 5::23] = 1 << 30
    with pytest.raises(ValueError):
        oracle.sparse_decode(case.q, case.kcache, ix, 512, case.softmax_scale)
    o, l = oracle.sparse_decode(case.q, case.kcache, ix, 512, case.softmax_scale, allow_faults=True)
    keep = (ix >= 0) & (ix < num_slots)
    # reference: SDPA over the torch-dequantised rows of the in-range entries
    rows = attention_rows(case.kcache)
    for b in range(case.batch):
        sel = ix[b, 0][keep[b, 0]].long()
        K = rows[sel]
        q = case.q[b, 0].to(torch.float64)
        ro, rl = sdpa_rows(q, K, 512, case.softmax_scale, [K.shape[0]] * q.shape[0])
        np.testing.assert_allclose(o[b, 0], ro, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(l[b, 0], rl, rtol=1e-12, atol=1e-12)

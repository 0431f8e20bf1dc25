"""Pins of the oracle's sparse prefill (no batch dimension, per-token top-k
length, per-head attention sink) against facts that do not come from the
oracle: torch SDPA over the gathered rows, the closed form of a sink logit
(O scaled by 1 / (1 + e^(sink - LSE)), LSE -> logaddexp(LSE, sink)), and
the equivalence of a top-k length with -1 padding."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
from mla_paged_kv_03_b200 import workloads as W


def sdpa_rows(case, lengths=None):
    """No-sink reference per (token, head) with torch SDPA (fp64)."""
    s_q, h = case.s_q, case.h_q
    K = case.kv.to(torch.float64)
    out = np.zeros((s_q, h, 512))
    lse = np.zeros((s_q, h))
    for t in range(s_q):
        idx = case.indices[t]
        n = case.topk if lengths is None else int(lengths[t])
        idx = idx[:n]
        sel = K[idx[idx >= 0].long()]
        q = case.q[t].to(torch.float64)
        if sel.shape[0] == 0:
            lse[t] = -np.inf
            continue
        out[t] = F.scaled_dot_product_attention(q[None], sel[None], sel[None, :, :512],
                                                scale=case.softmax_scale)[0].numpy()
        lse[t] = torch.logsumexp((q @ sel.T) * case.softmax_scale, dim=-1).numpy()
    return out, lse


def small(seed=0, **kw):
    args = dict(s_q=100, s_kv=100, h_q=3, topk=64)
    args.update(kw)
    return W.sparse_prefill(seed=seed, **args)


def test_prefill_without_sink_matches_sdpa():
    case = small(seed=1, with_length=False, with_sink=False)
    o, lse = oracle.sparse_prefill(case.q, case.kv, case.indices, case.softmax_scale)
    ro, rl = sdpa_rows(case)
    np.testing.assert_allclose(o, ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12)


def test_prefill_sink_closed_form():
    case = small(seed=2, with_length=False)
    o, lse = oracle.sparse_prefill(case.q, case.kv, case.indices, case.softmax_scale,
                                   attn_sink=case.attn_sink)
    ro, rl = sdpa_rows(case)
    sink = case.attn_sink.to(torch.float64).numpy()[None, :]
    want_lse = np.logaddexp(rl, sink)
    np.testing.assert_allclose(lse, want_lse, rtol=1e-12)
    np.testing.assert_allclose(o, ro / (1.0 + np.exp(sink - rl))[..., None], rtol=1e-10,
                               atol=1e-12)


def test_prefill_topk_length_equals_padding():
    case = small(seed=3)
    assert int(case.topk_length.min()) < case.topk  # early tokens see fewer rows
    o, lse = oracle.sparse_prefill(case.q, case.kv, case.indices, case.softmax_scale,
                                   topk_length=case.topk_length, attn_sink=case.attn_sink)
    ix = case.indices.clone()
    # scramble the entries past each length: the length must hide them
    for t in range(case.s_q):
        ix[t, int(case.topk_length[t]):] = t % 7
    o2, l2 = oracle.sparse_prefill(case.q, case.kv, ix, case.softmax_scale,
                                   topk_length=case.topk_length, attn_sink=case.attn_sink)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, l2)
    ro, rl = sdpa_rows(case, lengths=case.topk_length)
    sink = case.attn_sink.to(torch.float64).numpy()[None, :]
    np.testing.assert_allclose(lse, np.logaddexp(rl, sink), rtol=1e-12)


def test_prefill_empty_row_gives_zero_and_the_sink():
    case = small(seed=4, s_q=4, s_kv=50)
    lengths = case.topk_length.clone()
    lengths[1] = 0
    o, lse = oracle.sparse_prefill(case.q, case.kv, case.indices, case.softmax_scale,
                                   topk_length=lengths, attn_sink=case.attn_sink)
    assert (o[1] == 0).all()
    np.testing.assert_array_equal(lse[1], case.attn_sink.to(torch.float64).numpy())
    o2, l2 = oracle.sparse_prefill(case.q, case.kv, case.indices, case.softmax_scale,
                                   topk_length=lengths)
    assert (o2[1] == 0).all() and np.isneginf(l2[1]).all()


def test_prefill_generator_recipe():
    """Token t sits at position s_kv - s_q + t: its first topk_length[t] =
    min(topk, position + 1) entries are distinct rows at or before that
    position and the rest are -1; the draw is fixed by the seed."""
    case = W.sparse_prefill(seed=5, s_q=80, s_kv=120, h_q=2, topk=64)
    for t in range(case.s_q):
        pos = 120 - 80 + t
        n = int(case.topk_length[t])
        assert n == min(64, pos + 1)
        row = case.indices[t]
        assert (row[n:] == -1).all()
        valid = row[:n]
        assert (valid >= 0).all() and (valid <= pos).all()
        assert len(set(valid.tolist())) == n
    again = W.sparse_prefill(seed=5, s_q=80, s_kv=120, h_q=2, topk=64)
    assert torch.equal(case.indices, again.indices) and torch.equal(case.q, again.q)

"""Pins of the oracle's fused decode in sparse mode (the fused steps over the
valid slots of a 656-byte FP8 cache) against facts that do not come from the
oracle: the same step chain built from library routines (torch rms_norm,
complex rotation, SDPA over torch-dequantised rows rounded to bf16, the
float8_e4m3fn cast),
and its reduction to the dense fused oracle when the slots are a sequence's
tokens in order."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
from mla_paged_kv_03_b200 import workloads as W
from test_oracle_pins import attention_rows, dequant_cache_torch


def library_chain(case):
    b, _, h, _ = case.q_raw.shape
    theta_k = case.rope_base ** (-np.arange(32) * 2.0 / 64.0)
    K_all = attention_rows(case.kcache)
    codes = np.zeros((b, h, 576), dtype=np.uint8)
    scales = np.zeros((b, h))
    lses = np.zeros((b, h))
    for bi in range(b):
        pos = int(case.positions[bi])
        x = case.q_raw[bi, 0].to(torch.float64)
        y = F.rms_norm(x, (576,), weight=case.gain.to(torch.float64), eps=case.eps).numpy()
        z = (y[:, 512::2] + 1j * y[:, 513::2]) * np.exp(1j * pos * theta_k)
        y[:, 512::2], y[:, 513::2] = z.real, z.imag
        q = torch.tensor(y).to(torch.bfloat16).to(torch.float64)
        idx = case.indices[bi, 0]
        K = K_all[idx[idx >= 0].long()]
        o = F.scaled_dot_product_attention(q[None], K[None], K[None],
                                           scale=case.softmax_scale)[0].numpy()
        lses[bi] = torch.logsumexp((q @ K.T) * case.softmax_scale, dim=-1).numpy()
        w = (o[:, 512::2] + 1j * o[:, 513::2]) * np.exp(-1j * pos * theta_k)
        o[:, 512::2], o[:, 513::2] = w.real, w.imag
        amax = np.abs(o).max(axis=1)
        sc = np.where(amax > 0, amax / 448.0, 1.0)
        codes[bi] = torch.tensor((o / sc[:, None]).astype(np.float32)).to(
            torch.float8_e4m3fn).view(torch.uint8).numpy()
        scales[bi] = sc
    return codes, scales, lses


def test_fused_sparse_matches_library_chain():
    case = W.fused_sparse(seed=1, batch=3, h_q=4, seqlens=[300, 130, 70], topk=96)
    codes, sc, lse = oracle.fused_sparse_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                                case.positions, case.kcache, case.indices,
                                                case.softmax_scale)
    rc, rs, rl = library_chain(case)
    np.testing.assert_allclose(sc[:, 0], rs, rtol=1e-10)
    np.testing.assert_allclose(lse[:, 0], rl, rtol=1e-12, atol=1e-12)
    assert (codes[:, 0] == rc).mean() > 0.999


def test_fused_sparse_all_tokens_in_order_equals_dense_fused():
    """Slots = every token of a sequence in logical order: the fused sparse
    oracle equals the dense fused oracle over a bf16 cache holding the same
    (bf16-exact) values."""
    case = W.fused_sparse(seed=2, batch=1, h_q=3, seqlens=[100], topk=100, invalid_frac=0.0)
    L = 100
    t = torch.arange(L)
    phys = case.block_table[0].long()[t // 64] * 64 + t % 64
    idx = phys.to(torch.int32).view(1, 1, L)
    # rebuild the rows so that the dequantised values are exact in bf16: codes
    # with unit fp32 scales
    rows = case.kcache.view(-1, 656).clone()
    rows[:, 512:528] = torch.ones(rows.shape[0], 4).view(torch.uint8).view(-1, 16)
    codes, sc, lse = oracle.fused_sparse_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                                case.positions, rows, idx, case.softmax_scale)
    K = dequant_cache_torch(rows)[phys].to(torch.bfloat16)
    assert torch.equal(K.to(torch.float64), dequant_cache_torch(rows)[phys])
    kc = K.view(1, L, 1, 576)
    pad = torch.zeros(1, 128 - L, 1, 576, dtype=torch.bfloat16)
    kcache = torch.cat([kc, pad], dim=1).view(2, 64, 1, 576)
    bt = torch.tensor([[0, 1]], dtype=torch.int32)
    rc, rs, rl = oracle.fused_decode(case.q_raw, case.gain, case.eps, case.rope_base, kcache, bt,
                                     torch.tensor([L], dtype=torch.int32), case.softmax_scale,
                                     positions=case.positions)
    np.testing.assert_array_equal(codes, rc)
    np.testing.assert_array_equal(sc, rs)
    np.testing.assert_allclose(lse, rl, rtol=1e-13)


def test_fused_sparse_empty_row_and_invalid_slots():
    case = W.fused_sparse(seed=3, batch=2, h_q=2, seqlens=[200, 90], topk=64)
    ix = case.indices.clone()
    ix[0] = -1
    codes, sc, lse = oracle.fused_sparse_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                                case.positions, case.kcache, ix,
                                                case.softmax_scale)
    # an empty row: O = 0 (the conjugate rotation may leave -0, code 0x80),
    # scale 1, LSE = -inf
    assert ((codes[0] & 0x7F) == 0).all() and (sc[0] == 1.0).all() and np.isneginf(lse[0]).all()
    keep = ix[1, 0] >= 0
    ix2 = ix[1:, :, keep].contiguous()
    c2, s2, l2 = oracle.fused_sparse_decode(case.q_raw[1:], case.gain, case.eps, case.rope_base,
                                            case.positions[1:], case.kcache, ix2,
                                            case.softmax_scale)
    np.testing.assert_array_equal(codes[1:], c2)
    np.testing.assert_array_equal(lse[1:], l2)

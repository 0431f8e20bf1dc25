"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test checks the oracle against a closed form, an invariant, a library
routine on a special case (torch's SDPA / rms_norm / float8 cast, numpy's
complex exponential), or values fixed by the E4M3 format definition.  They are
chosen so that a plausible slip in the oracle (dropped term, wrong sign, wrong
index, transposed operand, wrong rounding) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from mla_paged_kv_03_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ helpers

def bf16_to_f64(t):
    return t.to(torch.float64)


def contiguous_k(case, b):
    """Latent rows of sequence b in logical order (library gather via torch
    indexing), fp64 [L, 576]."""
    L = int(case.cache_seqlens[b])
    pages = (L + 63) // 64
    blocks = case.block_table[b, :pages].long()
    rows = case.kcache[blocks, :, 0, :].reshape(-1, 576)[:L]
    return rows.to(torch.float64)


def sdpa_reference(case):
    """torch SDPA (fp64, CPU) per sequence with a bottom-right causal mask and
    torch.logsumexp of the scaled scores for the LSE."""
    outs, lses = [], []
    for b in range(case.batch):
        K = contiguous_k(case, b)
        L = K.shape[0]
        q = case.q[b].to(torch.float64).reshape(case.s_q * case.h_q, 576)
        qi = torch.arange(case.s_q).repeat_interleave(case.h_q)
        vis = (L - case.s_q + 1 + qi) if case.causal else torch.full_like(qi, L)
        mask = torch.arange(L)[None, :] < vis[:, None]
        o = F.scaled_dot_product_attention(q[None], K[None], K[None, :, :case.d_v],
                                           attn_mask=mask[None], scale=case.softmax_scale)[0]
        scores = (q @ K.T) * case.softmax_scale
        scores = scores.masked_fill(~mask, float("-inf"))
        lse = torch.logsumexp(scores, dim=-1)
        outs.append(o.reshape(case.s_q, case.h_q, case.d_v))
        lses.append(lse.reshape(case.s_q, case.h_q))
    return torch.stack(outs).numpy(), torch.stack(lses).numpy()


def small_dense(seqlens, s_q=1, h_q=4, seed=0, causal=True, d_v=512):
    return W.make_dense(seqlens, s_q, h_q, seed=seed, causal=causal, d_v=d_v, spare_blocks=2)


# ------------------------------------------------------------------- E4M3

def test_e4m3_golden_points():
    """Codes fixed by the OCP 8-bit floating point definition of E4M3."""
    path = os.path.join(GOLDEN, "e4m3_points.txt")
    vals, codes = [], []
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        v, c = line.split()
        vals.append(float.fromhex(v) if v.startswith(("0x", "-0x")) else float(v))
        codes.append(int(c, 16))
    assert len(vals) >= 10
    enc = oracle.e4m3_encode(np.array(vals))
    dec = oracle.e4m3_decode(np.array(codes, dtype=np.uint8))
    assert enc.tolist() == codes
    np.testing.assert_array_equal(dec, np.array(vals))


def test_e4m3_exhaustive_roundtrip():
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_decode(codes)
    nan = (codes & 0x7F) == 0x7F
    assert np.isnan(dec[nan]).all() and not np.isnan(dec[~nan]).any()
    enc = oracle.e4m3_encode(dec[~nan])
    assert (enc == codes[~nan]).all()


def test_e4m3_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = oracle.e4m3_decode(codes.numpy())
    np.testing.assert_array_equal(np.isnan(ref), np.isnan(ours))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ref[ok], ours[ok])


def test_e4m3_encode_matches_torch_rne():
    """Random fp32 values plus every midpoint between neighbouring codes and
    its two fp32 neighbours, within |x| <= 464 (torch does not saturate above
    the last rounding boundary; the oracle does)."""
    g = torch.Generator().manual_seed(1)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 200.0)])
    pos = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32)
    mids = (pos[:-1] + pos[1:]) / 2
    mids = torch.cat([mids, torch.tensor([464.0])])
    nb = torch.cat([mids, torch.nextafter(mids, torch.tensor(0.0)),
                    torch.nextafter(mids, torch.tensor(1e9))])
    x = torch.cat([x, nb, -nb]).clamp(-464.0, 464.0)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode(x.to(torch.float64).numpy())
    assert (ref == ours).all(), np.nonzero(ref != ours)[0][:10]


def test_round_bf16_matches_torch():
    g = torch.Generator().manual_seed(2)
    x = torch.randn(50000, generator=g, dtype=torch.float64) * 3.0
    # exact midpoints between neighbouring bf16 values exercise the ties
    b = x[:2000].to(torch.bfloat16).to(torch.float64)
    mid = b + (torch.nextafter(b.to(torch.bfloat16), torch.tensor(1e9, dtype=torch.bfloat16))
               .to(torch.float64) - b) / 2
    x = torch.cat([x, mid])
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x.numpy()), ref)


def test_e4m3_saturates():
    assert oracle.e4m3_encode(np.array([1e6, -1e6, 470.0, 448.0])).tolist() == \
        [0x7E, 0xFE, 0x7E, 0x7E]


# ------------------------------------------------------------------- RoPE

def test_rope_position_zero_is_identity():
    x = np.random.default_rng(0).standard_normal(64)
    np.testing.assert_array_equal(oracle.rope64(x, 0.0), x)


def test_rope_matches_complex_rotation():
    """Interleaved pairs as complex numbers times exp(i*pos*base^(-2k/64))."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal(64)
    for pos in (1.0, 17.0, 4095.0, 32767.0):
        z = x[0::2] + 1j * x[1::2]
        theta = pos * 10000.0 ** (-np.arange(32) * 2.0 / 64.0)
        w = z * np.exp(1j * theta)
        ref = np.empty(64)
        ref[0::2], ref[1::2] = w.real, w.imag
        np.testing.assert_allclose(oracle.rope64(x, pos), ref, rtol=0, atol=1e-10)
        wc = z * np.exp(-1j * theta)
        refc = np.empty(64)
        refc[0::2], refc[1::2] = wc.real, wc.imag
        np.testing.assert_allclose(oracle.rope64(x, pos, sign=-1), refc, rtol=0, atol=1e-10)


def test_rope_conjugate_inverts_and_composes():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(64)
    y = oracle.rope64(x, 1234.0)
    np.testing.assert_allclose(oracle.rope64(y, 1234.0, sign=-1), x, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y), np.linalg.norm(x), rtol=1e-13)
    np.testing.assert_allclose(oracle.rope64(oracle.rope64(x, 100.0), 23.0),
                               oracle.rope64(x, 123.0), atol=1e-11)


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_matches_torch_and_is_scale_invariant():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(576)
    g = 1.0 + 0.1 * rng.standard_normal(576)
    ref = F.rms_norm(torch.tensor(x), (576,), weight=torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, g, 1e-6), ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(oracle.rmsnorm(7.5 * x, g, 0.0), oracle.rmsnorm(x, g, 0.0),
                               rtol=1e-13)
    y = oracle.rmsnorm(x, np.ones(576), 0.0)
    assert abs(np.mean(y * y) - 1.0) < 1e-13


# ------------------------------------------------------------ dense decode

@pytest.mark.parametrize("seqlens,s_q,causal", [
    ([37, 200], 1, True),
    ([1, 64, 65, 130], 2, True),
    ([5, 129], 3, False),
])
def test_dense_matches_torch_sdpa(seqlens, s_q, causal):
    case = small_dense(seqlens, s_q=s_q, h_q=3, causal=causal)
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 case.d_v, case.softmax_scale, causal=causal)
    ro, rl = sdpa_reference(case)
    np.testing.assert_allclose(o, ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_dense_dv576_matches_sdpa():
    case = small_dense([70, 3], s_q=1, h_q=2, d_v=576)
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 576, case.softmax_scale)
    ro, rl = sdpa_reference(case)
    np.testing.assert_allclose(o, ro, rtol=1e-11, atol=1e-12)


def test_one_token_cache_returns_v_exactly():
    case = small_dense([1, 1], h_q=5)
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 512, case.softmax_scale)
    for b in range(2):
        v = contiguous_k(case, b)[0].numpy()
        np.testing.assert_array_equal(o[b, 0], np.broadcast_to(v[:512], (5, 512)))
        s = (case.q[b, 0].to(torch.float64).numpy() @ v) * case.softmax_scale
        np.testing.assert_allclose(lse[b, 0], s, rtol=1e-14, atol=1e-14)


def test_zero_query_gives_mean_of_v_and_log_length():
    case = small_dense([100, 7], h_q=2)
    case.q.zero_()
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 512, case.softmax_scale)
    for b, L in enumerate([100, 7]):
        mean = contiguous_k(case, b)[:, :512].mean(0).numpy()
        np.testing.assert_allclose(o[b, 0, 0], mean, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[b, 0], math.log(L), rtol=1e-14)


def test_paging_is_layout_invariant_bit_exact():
    """Same logical cache through a shuffled table and through the identity
    table: bit-identical results."""
    case = small_dense([150, 64, 1], h_q=3, seed=5)
    o1, l1 = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 512, case.softmax_scale)
    rows = [contiguous_k(case, b).to(torch.bfloat16) for b in range(case.batch)]
    pages = [(r.shape[0] + 63) // 64 for r in rows]
    kc = torch.zeros((sum(pages), 64, 1, 576), dtype=torch.bfloat16)
    bt = torch.full_like(case.block_table, -1)
    p0 = 0
    for b, r in enumerate(rows):
        kc.view(-1, 576)[p0 * 64:p0 * 64 + r.shape[0]] = r
        bt[b, :pages[b]] = torch.arange(p0, p0 + pages[b], dtype=torch.int32)
        p0 += pages[b]
    o2, l2 = oracle.dense_decode(case.q, kc, bt, case.cache_seqlens, 512, case.softmax_scale)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_split_partials_combine_to_unsplit():
    case = small_dense([300, 129], s_q=2, h_q=2, seed=9)
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 512, case.softmax_scale)
    cuts = [0, 64, 130, 200, 10 ** 6]
    parts = []
    for a, c in zip(cuts[:-1], cuts[1:]):
        lo = np.full(2, a, dtype=np.int32)
        hi = np.full(2, c, dtype=np.int32)
        parts.append(oracle.dense_decode(case.q, case.kcache, case.block_table,
                                         case.cache_seqlens, 512, case.softmax_scale,
                                         token_lo=lo, token_hi=hi))
    for b in range(2):
        for i in range(2):
            for h in range(2):
                lse_i = np.array([p[1][b, i, h] for p in parts])
                o_i = np.stack([p[0][b, i, h] for p in parts])
                oc, lc = oracle.combine(lse_i, o_i)
                np.testing.assert_allclose(oc, o[b, i, h], rtol=1e-12, atol=1e-13)
                np.testing.assert_allclose(lc, lse[b, i, h], rtol=1e-13)


def test_causal_row0_equals_shorter_single_query():
    case = small_dense([90], s_q=2, h_q=3, seed=11)
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 512, case.softmax_scale)
    sl = torch.tensor([89], dtype=torch.int32)
    o1, l1 = oracle.dense_decode(case.q[:, :1].contiguous(), case.kcache, case.block_table, sl,
                                 512, case.softmax_scale)
    np.testing.assert_array_equal(o[:, 0], o1[:, 0])
    np.testing.assert_array_equal(lse[:, 0], l1[:, 0])


def test_empty_sequence_gives_zero_and_neg_inf():
    case = small_dense([0, 10], h_q=2)
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 512, case.softmax_scale)
    assert (o[0] == 0).all() and np.isneginf(lse[0]).all()
    assert np.isfinite(lse[1]).all()


def test_sampled_rows_equal_full_rows():
    case = small_dense([40, 77], s_q=2, h_q=3, seed=4)
    o, lse = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                 512, case.softmax_scale)
    rows = np.array([0, 5, 7, 11])
    os_, ls_ = oracle.dense_decode(case.q, case.kcache, case.block_table, case.cache_seqlens,
                                   512, case.softmax_scale, rows=rows)
    np.testing.assert_array_equal(os_, o.reshape(-1, 512)[rows])
    np.testing.assert_array_equal(ls_, lse.reshape(-1)[rows])


# ------------------------------------------------------------- fused path

def fused_library_reference(case, positions=None):
    """The fused step chain built from library routines in fp64: torch rms_norm,
    numpy complex rotation, torch SDPA, complex conjugate rotation, and the
    float8_e4m3fn cast of o/scale (ratio rounded to fp32).  The query of
    sequence b sits at positions[b] (default L - 1)."""
    b, _, h, _ = case.q_raw.shape
    theta_k = 10000.0 ** (-np.arange(32) * 2.0 / 64.0)
    codes = np.zeros((b, h, 576), dtype=np.uint8)
    scales = np.zeros((b, h))
    lses = np.zeros((b, h))
    pres = np.zeros((b, h, 576))
    for bi in range(b):
        L = int(case.cache_seqlens[bi])
        pos = L - 1 if positions is None else positions[bi]
        x = case.q_raw[bi, 0].to(torch.float64)
        y = F.rms_norm(x, (576,), weight=case.gain.to(torch.float64), eps=case.eps).numpy()
        z = (y[:, 512::2] + 1j * y[:, 513::2]) * np.exp(1j * pos * theta_k)
        y[:, 512::2], y[:, 513::2] = z.real, z.imag
        K = contiguous_k(case, bi)
        q = torch.tensor(y).to(torch.bfloat16).to(torch.float64)  # attention input in bf16
        o = F.scaled_dot_product_attention(q[None], K[None], K[None],
                                           scale=case.softmax_scale)[0].numpy()
        lses[bi] = torch.logsumexp((q @ K.T) * case.softmax_scale, dim=-1).numpy()
        w = (o[:, 512::2] + 1j * o[:, 513::2]) * np.exp(-1j * pos * theta_k)
        o[:, 512::2], o[:, 513::2] = w.real, w.imag
        amax = np.abs(o).max(axis=1)
        sc = np.where(amax > 0, amax / 448.0, 1.0)
        ratio = torch.tensor((o / sc[:, None]).astype(np.float32))
        codes[bi] = ratio.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        scales[bi] = sc
        pres[bi] = o
    return codes, scales, lses, pres


def test_fused_matches_library_chain():
    case = W.fused(seed=3, seqlens=[1, 70, 257], h_q=4)
    codes, sc, lse, pre = oracle.fused_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                              case.kcache, case.block_table, case.cache_seqlens,
                                              case.softmax_scale, want_pre_cast=True)
    rc, rs, rl, rp = fused_library_reference(case)
    np.testing.assert_allclose(pre[:, 0], rp, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(sc[:, 0], rs, rtol=1e-10)
    np.testing.assert_allclose(lse[:, 0], rl, rtol=1e-12, atol=1e-12)
    # both encode the same fp32 ratio except where the fp64 values differ in
    # the last bits across a rounding boundary: demand near-total agreement
    agree = (codes[:, 0] == rc).mean()
    assert agree > 0.999, agree


def test_fused_reduces_to_dense_without_norm_and_rotation():
    """Unit gain, eps = 0, position 0: RoPE is the identity and RMSNorm only
    scales q, which the dense oracle sees after the same scaling."""
    case = W.fused(seed=4, seqlens=[50, 3], h_q=2)
    case.gain = torch.ones(576)
    pos = torch.zeros(2, dtype=torch.int32)
    codes, sc, lse, pre = oracle.fused_decode(case.q_raw, case.gain, 0.0, 10000.0, case.kcache,
                                              case.block_table, case.cache_seqlens,
                                              case.softmax_scale, positions=pos,
                                              want_pre_cast=True)
    x = case.q_raw.to(torch.float64)
    rms = torch.sqrt((x * x).mean(-1, keepdim=True))
    qn = (x / rms).to(torch.bfloat16)  # normalised query, in the attention's bf16
    for b in range(2):
        for h in range(2):
            dcase = W.DenseCase(q=qn[b:b + 1, :, h:h + 1].contiguous(),
                                kcache=case.kcache, block_table=case.block_table[b:b + 1],
                                cache_seqlens=case.cache_seqlens[b:b + 1], s_q=1, h_q=1, d_v=576,
                                causal=False, softmax_scale=case.softmax_scale)
            o, l = oracle.dense_decode(dcase.q, dcase.kcache, dcase.block_table,
                                       dcase.cache_seqlens, 576, dcase.softmax_scale,
                                       causal=False)
            np.testing.assert_allclose(pre[b, 0, h], o[0, 0, 0], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(lse[b, 0, h], l[0, 0, 0], rtol=1e-12)


def test_fused_relative_position_invariance():
    """Rotating q and every cached RoPE dim by the same extra angle leaves the
    scores, hence LSE, unchanged; the output's RoPE dims come back through the
    conjugate rotation at the shifted position."""
    case = W.fused(seed=5, seqlens=[40], h_q=2)
    _, _, lse0 = oracle.fused_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                     case.kcache, case.block_table, case.cache_seqlens,
                                     case.softmax_scale)
    # shift every cached token's rope dims by +delta and the query position too
    delta = 37
    kc = case.kcache.clone()
    flat = kc.view(-1, 576).to(torch.float64)
    rope = flat[:, 512:].numpy()
    z = (rope[:, 0::2] + 1j * rope[:, 1::2]) * np.exp(1j * delta * 10000.0 **
                                                       (-np.arange(32) * 2.0 / 64.0))
    rot = np.empty_like(rope)
    rot[:, 0::2], rot[:, 1::2] = z.real, z.imag
    # keep exact invariance: compare against the unrotated cache run in fp64
    # through the dense oracle is not possible with bf16 storage, so instead
    # compare LSE up to the bf16 rounding of the rotated cache.
    flat[:, 512:] = torch.tensor(rot)
    kc.view(-1, 576)[:] = flat.to(torch.bfloat16)
    pos = case.cache_seqlens - 1 + delta
    _, _, lse1 = oracle.fused_decode(case.q_raw, case.gain, case.eps, case.rope_base, kc,
                                     case.block_table, case.cache_seqlens, case.softmax_scale,
                                     positions=pos)
    np.testing.assert_allclose(lse1, lse0, atol=2e-3)
    # and with a zero shift the explicit-position path is bit-identical
    _, _, lse2 = oracle.fused_decode(case.q_raw, case.gain, case.eps, case.rope_base,
                                     case.kcache, case.block_table, case.cache_seqlens,
                                     case.softmax_scale, positions=case.cache_seqlens - 1)
    np.testing.assert_array_equal(lse2, lse0)


# ------------------------------------------------------------ sparse path

def dequant_cache_torch(cache):
    """Library decode of the 656-byte rows: torch float8 view * fp32 scale."""
    rows = cache.reshape(-1, 656)
    codes = rows[:, :512].contiguous().view(torch.float8_e4m3fn).to(torch.float64)
    scales = rows[:, 512:528].contiguous().view(torch.float32).to(torch.float64)
    nope = codes.view(-1, 4, 128) * scales.view(-1, 4, 1)
    rope = rows[:, 528:].contiguous().view(torch.bfloat16).to(torch.float64)
    return torch.cat([nope.view(-1, 512), rope], dim=1)


def attention_rows(rows):
    """What the attention sees: the dequantised rows rounded to bf16 by torch
    (round to nearest even)."""
    return dequant_cache_torch(rows).to(torch.bfloat16).to(torch.float64)


def test_row656_decode_matches_torch_and_encoder_error_bound():
    g = torch.Generator().manual_seed(0)
    x = torch.randn((64, 512), generator=g)
    rope = torch.randn((64, 64), generator=g).to(torch.bfloat16)
    rows = W.quantize_rows656(x, rope)
    ref = dequant_cache_torch(rows)
    for r in (0, 13, 63):
        np.testing.assert_array_equal(oracle.decode_row656(rows[r]), ref[r].numpy())
    # quantisation error within half a code step at each value's magnitude,
    # rope dims exact
    dec = torch.stack([torch.tensor(oracle.decode_row656(rows[r])) for r in range(64)])
    scale = rows[:, 512:528].contiguous().view(torch.float32).to(torch.float64)
    s = scale.repeat_interleave(128, dim=1)
    v = (x.to(torch.float64) / s).abs()
    step = torch.where(v < 2 ** -6, torch.full_like(v, 2 ** -9),
                       2.0 ** (torch.floor(torch.log2(v.clamp_min(2 ** -6))) - 3))
    assert ((dec[:, :512] - x.to(torch.float64)).abs() <= 0.5 * step * s + 1e-12).all()
    np.testing.assert_array_equal(dec[:, 512:].numpy(), rope.to(torch.float64).numpy())


def sparse_small(seed=0, seqlens=(300, 130), topk=96, h_q=3, invalid_frac=0.05):
    return W.sparse(seed=seed, batch=len(seqlens), h_q=h_q, seqlens=list(seqlens), topk=topk,
                    invalid_frac=invalid_frac)


def test_sparse_matches_sdpa_on_dequantised_rows():
    case = sparse_small()
    o, lse = oracle.sparse_decode(case.q, case.kcache, case.indices, 512, case.softmax_scale)
    K = attention_rows(case.kcache)
    for b in range(case.batch):
        idx = case.indices[b, 0]
        sel = K[idx[idx >= 0].long()]
        q = case.q[b, 0].to(torch.float64)
        ro = F.scaled_dot_product_attention(q[None], sel[None], sel[None, :, :512],
                                            scale=case.softmax_scale)[0]
        rl = torch.logsumexp((q @ sel.T) * case.softmax_scale, dim=-1)
        np.testing.assert_allclose(o[b, 0], ro.numpy(), rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[b, 0], rl.numpy(), rtol=1e-12)


def test_sparse_all_tokens_equals_dense_noncausal():
    """indices = every token in logical order (physical slots through the
    table) equals non-causal dense attention over the dequantised cache."""
    case = sparse_small(seqlens=(100,), topk=100, invalid_frac=0.0)
    L = 100
    t = torch.arange(L)
    phys = case.block_table[0].long()[t // 64] * 64 + t % 64
    idx = phys.to(torch.int32).view(1, 1, L)
    o, lse = oracle.sparse_decode(case.q, case.kcache, idx, 512, case.softmax_scale)
    K = attention_rows(case.kcache)[phys]
    q = case.q[0, 0].to(torch.float64)
    ro = F.scaled_dot_product_attention(q[None], K[None], K[None, :, :512],
                                        scale=case.softmax_scale)[0]
    np.testing.assert_allclose(o[0, 0], ro.numpy(), rtol=1e-11, atol=1e-12)


def test_sparse_permutation_and_invalid_slots():
    case = sparse_small(seed=2, invalid_frac=0.0)
    o, lse = oracle.sparse_decode(case.q, case.kcache, case.indices, 512, case.softmax_scale)
    perm = torch.randperm(case.topk, generator=torch.Generator().manual_seed(0))
    o2, l2 = oracle.sparse_decode(case.q, case.kcache, case.indices[..., perm].contiguous(), 512,
                                  case.softmax_scale)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    # inserting -1 entries equals removing those slots
    ix = case.indices.clone()
    ix[..., ::5] = -1
    o3, l3 = oracle.sparse_decode(case.q, case.kcache, ix, 512, case.softmax_scale)
    keep = torch.ones(case.topk, dtype=torch.bool)
    keep[::5] = False
    o4, l4 = oracle.sparse_decode(case.q, case.kcache, case.indices[..., keep].contiguous(), 512,
                                  case.softmax_scale)
    np.testing.assert_array_equal(o3, o4)
    np.testing.assert_array_equal(l3, l4)
    # all invalid -> zero output, -inf LSE
    o5, l5 = oracle.sparse_decode(case.q, case.kcache, torch.full_like(ix, -1), 512,
                                  case.softmax_scale)
    assert (o5 == 0).all() and np.isneginf(l5).all()


def test_sparse_index_handling_logical_vs_physical():
    """The generator's physical slots equal block_table[t // 64] * 64 + t % 64
    of logical tokens drawn inside [0, L): every valid slot lies in a block
    owned by its own sequence, slots are distinct, and exactly
    round(5% * topk) entries are -1."""
    seqlens = (300, 130)
    case = sparse_small(seed=3, seqlens=seqlens)
    for b, L in enumerate(seqlens):
        own = set(case.block_table[b, :(L + 63) // 64].tolist())
        row = case.indices[b, 0]
        idx = row[row >= 0]
        assert len(set(idx.tolist())) == idx.numel()  # without replacement
        for s in idx.tolist():
            assert s // 64 in own
        assert int((row < 0).sum()) == round(0.05 * case.topk)

"""Pins of the oracle's V4.1 cache paths against facts that do not come from
the oracle:
  - FP8, 528-byte rows (512 E4M3 codes over the whole 512-dim latent, then 16
    E8M0 scales, one per 32 codes): torch's float8_e4m3fn and float8_e8m0fnu
    casts, the quantisation error bound, the one-slot case and the
    invariances of sparse attention;
  - FP4, 288-byte rows (512 E2M1 codes two per byte, then 32 E4M3 scales, one
    per 16 codes): the E2M1 value table of the format, torch's float8_e4m3fn
    cast for the scales, exactly representable values coming back exactly;
  - both: torch SDPA on independently dequantised rows."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
from mla_paged_kv_03_b200 import workloads as W


def dequant528_torch(rows):
    """[n, 528] uint8 -> fp64 [n, 512] with torch's own float8 decoders."""
    rows = rows.reshape(-1, 528)
    codes = rows[:, :512].contiguous().view(torch.float8_e4m3fn).to(torch.float64)
    scale = rows[:, 512:].contiguous().view(torch.float8_e8m0fnu).to(torch.float64)
    return codes * scale.repeat_interleave(32, dim=1)


def test_e8m0_decode_matches_torch_exhaustive():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = oracle.e8m0_decode(codes.numpy())
    finite = np.isfinite(ref)
    np.testing.assert_array_equal(got[finite], ref[finite])
    assert np.isnan(got[255]) and np.isnan(ref[255]) and finite[:255].all()
    assert got[127] == 1.0 and got[128] == 2.0 and got[126] == 0.5


def test_row528_decode_matches_torch_and_error_bound():
    g = torch.Generator().manual_seed(0)
    x = torch.randn((64, 512), generator=g) * torch.exp2(torch.randint(-6, 7, (64, 1), generator=g))
    x[3, 64:96] = 0.0  # an all-zero group: scale byte 127, codes 0
    rows = W.quantize_rows528(x)
    ref = dequant528_torch(rows)
    dec = torch.stack([torch.tensor(oracle.decode_row528(rows[r])) for r in range(64)])
    np.testing.assert_array_equal(dec.numpy(), ref.numpy())
    assert (rows[3, 512 + 2] == 127) and (dec[3, 64:96] == 0).all()
    # every stored scale is the smallest power of two with absmax / scale <= 448
    s = rows[:, 512:].to(torch.float64) - 127
    amax = x.view(64, 16, 32).abs().amax(dim=2).to(torch.float64)
    nz = amax > 0
    assert ((amax / torch.exp2(s))[nz] <= 448).all() and ((amax / torch.exp2(s - 1))[nz] > 448).all()
    # quantisation error within half a code step at each value's magnitude
    sc = torch.exp2(s).repeat_interleave(32, dim=1)
    v = (x.to(torch.float64) / sc).abs()
    step = torch.where(v < 2 ** -6, torch.full_like(v, 2 ** -9),
                       2.0 ** (torch.floor(torch.log2(v.clamp_min(2 ** -6))) - 3))
    assert ((dec - x.to(torch.float64)).abs() <= 0.5 * step * sc + 1e-30).all()


def small(seed=0, seqlens=(300, 130), topk=96, h_q=3, invalid_frac=0.05, s_q=1):
    return W.sparse_v41(seed=seed, batch=len(seqlens), h_q=h_q, s_q=s_q, seqlens=list(seqlens),
                        topk=topk, invalid_frac=invalid_frac)


def test_sparse_v41_matches_sdpa_on_dequantised_rows():
    case = small(s_q=2)
    o, lse = oracle.sparse_decode_v41(case.q, case.kcache, case.indices, case.softmax_scale)
    K = dequant528_torch(case.kcache)
    for b in range(case.batch):
        for i in range(case.s_q):
            idx = case.indices[b, i]
            sel = K[idx[idx >= 0].long()]
            q = case.q[b, i].to(torch.float64)
            ro = F.scaled_dot_product_attention(q[None], sel[None], sel[None],
                                                scale=case.softmax_scale)[0]
            rl = torch.logsumexp((q @ sel.T) * case.softmax_scale, dim=-1)
            np.testing.assert_allclose(o[b, i], ro.numpy(), rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(lse[b, i], rl.numpy(), rtol=1e-12)


def test_sparse_v41_one_slot_returns_its_row_exactly():
    case = small(seqlens=(70,), topk=1, invalid_frac=0.0)
    o, lse = oracle.sparse_decode_v41(case.q, case.kcache, case.indices, case.softmax_scale)
    row = dequant528_torch(case.kcache)[int(case.indices[0, 0, 0])]
    for h in range(case.h_q):
        np.testing.assert_array_equal(o[0, 0, h], row.numpy())
        s = float(case.q[0, 0, h].to(torch.float64) @ row) * case.softmax_scale
        assert abs(lse[0, 0, h] - s) <= 1e-12 * max(1.0, abs(s))


def test_sparse_v41_permutation_and_invalid_slots():
    case = small(seed=2, invalid_frac=0.0)
    o, lse = oracle.sparse_decode_v41(case.q, case.kcache, case.indices, case.softmax_scale)
    perm = torch.randperm(case.topk, generator=torch.Generator().manual_seed(0))
    o2, _ = oracle.sparse_decode_v41(case.q, case.kcache, case.indices[..., perm].contiguous(),
                                     case.softmax_scale)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    ix = case.indices.clone()
    ix[..., ::7] = -1
    o3, l3 = oracle.sparse_decode_v41(case.q, case.kcache, ix, case.softmax_scale)
    keep = torch.ones(case.topk, dtype=torch.bool)
    keep[::7] = False
    o4, l4 = oracle.sparse_decode_v41(case.q, case.kcache, case.indices[..., keep].contiguous(),
                                      case.softmax_scale)
    np.testing.assert_array_equal(o3, o4)
    np.testing.assert_array_equal(l3, l4)
    o5, l5 = oracle.sparse_decode_v41(case.q, case.kcache, torch.full_like(ix, -1),
                                      case.softmax_scale)
    assert (o5 == 0).all() and np.isneginf(l5).all()


# ------------------------------------------------------- V4.1 FP4 (288 B)

# The E2M1 format's values for codes 0..7 (sign bit 3 negates them).
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def dequant288_torch(rows):
    """[n, 288] uint8 -> fp64 [n, 512]: nibbles unpacked low-then-high with
    the format's value table, scales by torch's float8_e4m3fn decoder."""
    rows = rows.reshape(-1, 288)
    b = rows[:, :256].to(torch.int64)
    codes = torch.stack([b & 0xF, b >> 4], dim=-1).reshape(-1, 512)
    table = torch.tensor(E2M1_TABLE + [-v for v in E2M1_TABLE], dtype=torch.float64)
    vals = table[codes]
    scale = rows[:, 256:].contiguous().view(torch.float8_e4m3fn).to(torch.float64)
    return vals * scale.repeat_interleave(16, dim=1)


def test_e2m1_decode_matches_format_table():
    got = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    want = np.array(E2M1_TABLE + [-v for v in E2M1_TABLE])
    np.testing.assert_array_equal(np.abs(got), np.abs(want))
    assert (np.signbit(got[8:])).all() and not np.signbit(got[:8]).any()


def test_row288_decode_matches_torch_and_exact_values_roundtrip():
    g = torch.Generator().manual_seed(1)
    x = torch.randn((48, 512), generator=g)
    rows = W.quantize_rows288(x)
    ref = dequant288_torch(rows)
    dec = torch.stack([torch.tensor(oracle.decode_row288(rows[r])) for r in range(48)])
    np.testing.assert_array_equal(dec.numpy(), ref.numpy())
    # values that are exactly code * scale (absmax = 6 * scale) come back exactly
    scales = torch.tensor([0.25, 1.0, 0.09375, 3.5], dtype=torch.float32)  # all e4m3 values
    idx = torch.randint(0, 16, (4, 32, 16), generator=g)
    table = torch.tensor(E2M1_TABLE + [-v for v in E2M1_TABLE])
    vals = table[idx]
    vals[..., 0] = 6.0  # pin each group's absmax so that absmax / 6 is the scale
    group_scale = scales[torch.randint(0, 4, (4, 32), generator=g)].view(4, 32, 1)
    exact = (vals * group_scale).reshape(4, 512)
    rows2 = W.quantize_rows288(exact)
    dec2 = torch.stack([torch.tensor(oracle.decode_row288(rows2[r])) for r in range(4)])
    np.testing.assert_array_equal(dec2.numpy(), exact.to(torch.float64).numpy())


def test_sparse_v41_fp4_matches_sdpa_on_dequantised_rows():
    case = W.sparse_v41_fp4(seed=4, batch=2, h_q=3, s_q=2, seqlens=[300, 130], topk=96,
                            invalid_frac=0.05)
    o, lse = oracle.sparse_decode_v41(case.q, case.kcache, case.indices, case.softmax_scale)
    K = dequant288_torch(case.kcache)
    for b in range(case.batch):
        for i in range(case.s_q):
            idx = case.indices[b, i]
            sel = K[idx[idx >= 0].long()]
            q = case.q[b, i].to(torch.float64)
            ro = F.scaled_dot_product_attention(q[None], sel[None], sel[None],
                                                scale=case.softmax_scale)[0]
            rl = torch.logsumexp((q @ sel.T) * case.softmax_scale, dim=-1)
            np.testing.assert_allclose(o[b, i], ro.numpy(), rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(lse[b, i], rl.numpy(), rtol=1e-12)


def test_v41_generators_index_recipe():
    """Both V4.1 generators draw each query's valid slots without replacement
    from blocks its own sequence owns, with round(5% * topk) entries -1, and
    reproduce the same draw from the same seed."""
    for fp4 in (False, True):
        seqlens = (300, 130)
        case = W.sparse_v41(seed=6, batch=2, h_q=2, seqlens=list(seqlens), topk=96, fp4=fp4)
        for b, L in enumerate(seqlens):
            own = set(case.block_table[b, :(L + 63) // 64].tolist())
            row = case.indices[b, 0]
            idx = row[row >= 0]
            assert len(set(idx.tolist())) == idx.numel()
            assert all(s // 64 in own for s in idx.tolist())
            assert int((row < 0).sum()) == round(0.05 * case.topk)
        again = W.sparse_v41(seed=6, batch=2, h_q=2, seqlens=list(seqlens), topk=96, fp4=fp4)
        assert torch.equal(case.kcache, again.kcache) and torch.equal(case.indices, again.indices)

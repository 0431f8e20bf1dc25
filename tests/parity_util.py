"""Shared helpers of the GPU parity tests: tolerances and comparisons
(the thresholds are the ones stated for this library's outputs)."""
import numpy as np
import torch

# bf16 outputs: |o - ref| <= ATOL + RTOL * |ref|; LSE within 1e-3 absolute.
ATOL = 1e-2
RTOL = 1e-2
LSE_ATOL = 1e-3


def assert_out_close(out, ref, what="O"):
    o = out.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    err = np.abs(o - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                             f"first {idx.tolist()} got {o[bad][:5]} want {ref[bad][:5]}; "
                             f"max err {err.max():.3e}")


def assert_lse_close(lse, ref):
    g = lse.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    both_inf = np.isneginf(g) & np.isneginf(ref)
    with np.errstate(invalid="ignore"):
        ok = both_inf | (np.abs(g - ref) <= LSE_ATOL)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        raise AssertionError(f"LSE: {(~ok).sum()} bad; first {idx.tolist()} got {g[~ok][:5]} "
                             f"want {ref[~ok][:5]}")


def e4m3_neighbours(a, b):
    """Codes equal or one step apart on the E4M3 number line (same sign, or
    both within one step of zero)."""
    a = a.astype(np.int32)
    b = b.astype(np.int32)
    same_sign = (a & 0x80) == (b & 0x80)
    mag_a, mag_b = a & 0x7F, b & 0x7F
    close = same_sign & (np.abs(mag_a - mag_b) <= 1)
    near_zero = (mag_a <= 1) & (mag_b <= 1)
    return (a == b) | close | near_zero


def assert_fp8_close(codes, scale, ref_codes, ref_scale, min_equal=0.999):
    c = codes.detach().cpu().numpy().reshape(ref_codes.shape)
    s = scale.detach().float().cpu().numpy().astype(np.float64).reshape(ref_scale.shape)
    eq = (c == ref_codes).mean()
    assert eq >= min_equal, f"only {eq:.5f} of E4M3 codes equal the oracle's"
    nb = e4m3_neighbours(c, ref_codes)
    if not nb.all():
        bad = np.argwhere(~nb)[:5]
        det = [(tuple(int(v) for v in i), hex(int(c[tuple(i)])), hex(int(ref_codes[tuple(i)])))
               for i in bad]
        raise AssertionError(f"{(~nb).sum()} codes more than one step from the oracle's: "
                             f"(index, gpu, oracle) {det}")
    rel = np.abs(s - ref_scale) / np.maximum(np.abs(ref_scale), 1e-30)
    assert (rel <= 1e-3).all(), f"scale rel err {rel.max():.3e}"


def full_size_rows(rows_per_unit, unit_sizes, n_random, seed):
    """Rows checked in a full-size parity test: n_random rows drawn at random,
    plus every row of the first unit (sequence, query pair or token), of the
    largest one and of the last one, so that every head, every split of a
    long sequence and every role a CTA takes is covered at least once."""
    unit_sizes = np.asarray(unit_sizes)
    n_units = unit_sizes.size
    total = n_units * rows_per_unit
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(total, size=min(n_random, total), replace=False).tolist())
    for u in {0, int(np.argmax(unit_sizes)), n_units - 1}:
        rows.update(range(u * rows_per_unit, (u + 1) * rows_per_unit))
    return np.array(sorted(rows), dtype=np.int64)

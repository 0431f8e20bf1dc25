"""Split-KV planner (host build of the same routine the device runs):
bit-exact coverage of every (sequence, tile) pair, split counts and balance."""
import random

import pytest
import torch

from mla_paged_kv_03_b200 import binding as B

TILE = 128
OVERHEAD = 2


def tiles_of(L):
    return (L + TILE - 1) // TILE if L > 0 else 1


def expand(meta, ns, seqlens):
    """Walk the metadata like the kernel does -> list per part of (b, lo, hi, split)."""
    parts = []
    for p in range(meta.shape[0]):
        b0, t0, b1, t1, s0 = [int(v) for v in meta[p, :5]]
        segs = []
        for b in range(b0, b1 + 1):
            lo = t0 if b == b0 else 0
            hi = t1 if b == b1 else tiles_of(seqlens[b])
            if lo < hi:
                segs.append((b, lo, hi, s0 if b == b0 else 0))
        parts.append(segs)
    return parts


def check_plan(seqlens, parts_n):
    meta, ns = B.mla_get_metadata_host(seqlens, 16, parts_n)
    parts = expand(meta, ns, seqlens)
    seen = {b: [] for b in range(len(seqlens))}
    for segs in parts:
        for (b, lo, hi, s) in segs:
            seen[b].append((s, lo, hi))
    assert int(ns[0]) == 0
    for b, L in enumerate(seqlens):
        segs = sorted(seen[b])
        # splits numbered 0..n-1, contiguous, covering [0, tiles) exactly once, in order
        assert [s for s, _, _ in segs] == list(range(len(segs)))
        cur = 0
        for _, lo, hi in segs:
            assert lo == cur and hi > lo
            cur = hi
        assert cur == tiles_of(L)
        assert int(ns[b + 1] - ns[b]) == len(segs)
    # parts are contiguous runs in (b, tile) order
    flat = [(b, lo) for segs in parts for (b, lo, hi, s) in segs]
    assert flat == sorted(flat)
    return meta, ns, parts


@pytest.mark.parametrize("seqlens", [
    [0], [1], [63, 64, 65], [127, 128, 129], [37, 200], [0, 0, 0, 5],
    [16384] + [1] * 50, [1] * 300, list(range(0, 5000, 97)),
])
@pytest.mark.parametrize("parts_n", [1, 2, 7, 74, 148, 500])
def test_plan_covers_every_tile_once(seqlens, parts_n):
    check_plan(seqlens, parts_n)


def test_plan_random_mixes_and_balance():
    rng = random.Random(0)
    for trial in range(40):
        b = rng.randint(1, 200)
        seqlens = [int(rng.choice([rng.randint(0, 300), rng.randint(1000, 20000)])) for _ in range(b)]
        parts_n = rng.choice([1, 3, 74, 148])
        meta, ns, parts = check_plan(seqlens, parts_n)
        total = sum(tiles_of(L) + OVERHEAD for L in seqlens)
        target = -(-total // parts_n)
        costs = [sum(hi - lo + OVERHEAD for (_, lo, hi, _) in segs) for segs in parts]
        # every part but the last stays within one segment overhead of the target
        for c in costs[:-1]:
            assert c <= target + OVERHEAD + 1
        assert sum(costs) >= total


def test_plan_uniform_lengths_split_evenly():
    meta, ns, parts = check_plan([65536 // 32] * 32, 74)
    costs = [sum(hi - lo + OVERHEAD for (_, lo, hi, _) in segs) for segs in parts]
    nonempty = [c for c in costs if c]
    assert max(nonempty) - min(nonempty) <= 2 * OVERHEAD + 2


def test_plan_rejects_bad_arguments():
    with pytest.raises(B.MLAError):
        B.mla_get_metadata_host([5, -1], 16, 4)
    with pytest.raises(B.MLAError):
        B.mla_get_metadata_host([5], 16, 0)
    with pytest.raises(B.MLAError):
        B.mla_get_metadata_host([5], 16, 4, h_kv=2)


try:
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=200, deadline=None)
    @given(seqlens=st.lists(st.one_of(st.integers(0, 300), st.integers(1000, 70000)),
                            min_size=1, max_size=120),
           parts_n=st.integers(1, 600))
    def test_plan_property_coverage_and_balance(seqlens, parts_n):
        """Any length mix and partition count: every (sequence, tile) pair is
        covered exactly once, in order, and no part exceeds the target width
        by more than one segment overhead."""
        meta, ns, parts = check_plan(seqlens, parts_n)
        total = sum(tiles_of(L) + OVERHEAD for L in seqlens)
        target = -(-total // parts_n)
        for segs in parts:
            assert sum(hi - lo + OVERHEAD for (_, lo, hi, _) in segs) <= target + OVERHEAD + 1
except ImportError:  # pragma: no cover
    pass

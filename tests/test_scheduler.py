"""Split-KV planner (host build of the same routine the device runs):
bit-exact coverage of every (sequence, tile) pair, split counts and balance."""
import random

import pytest
import torch

from mla_paged_kv_03_b200 import binding as B

TILE = 128


def _planner_constants():
    """The planner's cost of a tile and the segment overheads, read from the
    library's shared header (kPlanTileCost, MLA_PLAN_OVH_* defaults)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "mla_paged_kv_03_b200", "csrc", "mla_common.h")).read()
    tile = int(re.search(r"kPlanTileCost = (\d+);", src).group(1))
    ovh = {k: int(v) for k, v in re.findall(r"#define MLA_PLAN_OVH_(\w+) (\d+)", src)}
    min_cta = int(re.search(r"kPlanMinWidthCta = (\d+) \* kPlanTileCost;", src).group(1)) * tile
    return tile, ovh, min_cta


TILE_COST, OVH, MIN_WIDTH_CTA = _planner_constants()


def overhead_for(heads_per_kv):
    return OVH["PAGE"] if heads_per_kv <= 32 else (OVH["CTA"] if heads_per_kv <= 64 else OVH["PAIR"])


def granule_for(heads_per_kv):
    return 2 if heads_per_kv > 64 else 1


def min_width_for(heads_per_kv):
    """The 1-CTA kernel's parts are at least two tiles wide."""
    return MIN_WIDTH_CTA if 32 < heads_per_kv <= 64 else 0


def target_width(seqlens, parts_n, heads_per_kv):
    u = granule_for(heads_per_kv) * TILE_COST
    return max(-(-plan_total(seqlens, heads_per_kv) // parts_n), u, min_width_for(heads_per_kv))


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
            hi = min(t1, tiles_of(seqlens[b])) if b == b1 else tiles_of(seqlens[b])
            if lo < hi:
                segs.append((b, lo, hi, s0 if b == b0 else 0))
        parts.append(segs)
    return parts


def seg_cost(lo, hi, heads_per_kv):
    """Planner cost of a segment of tiles [lo, hi): its granules and one overhead."""
    g = granule_for(heads_per_kv)
    return g * TILE_COST * (-(-(hi - lo) // g)) + overhead_for(heads_per_kv)


def plan_total(seqlens, heads_per_kv):
    g = granule_for(heads_per_kv)
    return sum(g * TILE_COST * (-(-tiles_of(L) // g)) + overhead_for(heads_per_kv)
               for L in seqlens)


def check_plan(seqlens, parts_n, heads_per_kv=16):
    meta, ns = B.mla_get_metadata_host(seqlens, heads_per_kv, parts_n)
    parts = expand(meta, ns, seqlens)
    g = granule_for(heads_per_kv)
    for segs in parts:
        for (b, lo, hi, s) in segs:
            # splits start on a granule; only a sequence's last split may be ragged
            assert lo % g == 0
            assert (hi - lo) % g == 0 or hi == tiles_of(seqlens[b])
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
    for heads_per_kv in (16, 64, 128):
        check_plan(seqlens, parts_n, heads_per_kv)


@pytest.mark.parametrize("heads_per_kv", [16, 64, 128])
def test_plan_random_mixes_and_balance(heads_per_kv):
    rng = random.Random(heads_per_kv)
    o = overhead_for(heads_per_kv)
    for trial in range(40):
        b = rng.randint(1, 200)
        seqlens = [int(rng.choice([rng.randint(0, 300), rng.randint(1000, 20000)])) for _ in range(b)]
        parts_n = rng.choice([1, 3, 74, 148])
        meta, ns, parts = check_plan(seqlens, parts_n, heads_per_kv)
        u = granule_for(heads_per_kv) * TILE_COST
        total = plan_total(seqlens, heads_per_kv)
        target = target_width(seqlens, parts_n, heads_per_kv)
        costs = [sum(seg_cost(lo, hi, heads_per_kv) for (_, lo, hi, _) in segs) for segs in parts]
        # every part stays within one granule and one segment overhead of the target
        for c in costs:
            assert c <= target + u + o
        assert sum(costs) >= total


def test_plan_uniform_lengths_split_evenly():
    o, u = overhead_for(128), 2 * TILE_COST
    meta, ns, parts = check_plan([65536 // 32] * 32, 74, heads_per_kv=128)
    costs = [sum(seg_cost(lo, hi, 128) for (_, lo, hi, _) in segs) for segs in parts]
    nonempty = [c for c in costs if c]
    assert max(nonempty) - min(nonempty) <= 2 * o + 2 * u


def test_plan_parts_narrower_than_a_tile():
    """More parts than quarter-tile units: the width stays one tile, so no
    split count includes a part that holds none of the sequence's tiles."""
    for seqlens in ([1], [1, 1], [130, 0, 5], [64] * 10):
        check_plan(seqlens, 500)
        check_plan(seqlens, 500, heads_per_kv=128)


def test_plan_minimum_width_of_the_one_cta_kernel():
    """Batch 1 on the 1-CTA kernel (64 rows per KV head): parts are at least
    two tiles wide, so fewer parts than SMs hold work and the rest are empty;
    the page kernel's plan of the same sequence splits it more finely."""
    L = 17000  # 133 tiles
    meta, ns, parts = check_plan([L], 148, heads_per_kv=64)
    tiles = [sum(hi - lo for (_, lo, hi, _) in segs) for segs in parts]
    used = [t for t in tiles if t]
    assert all(t >= 2 for t in used[:-1])
    # (the first parts lie inside the sequence's overhead and stay empty too)
    assert len(used) <= -(-plan_total([L], 64) // target_width([L], 148, 64)) < 148
    assert int(ns[1]) == len(used)
    # the page kernel's plan of the same sequence (no minimum) uses ~all parts
    _, ns16, _ = check_plan([L], 148, heads_per_kv=16)
    assert int(ns16[1]) > len(used)


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
           parts_n=st.integers(1, 600), heads_per_kv=st.sampled_from([16, 64, 128]))
    def test_plan_property_coverage_and_balance(seqlens, parts_n, heads_per_kv):
        """Any length mix and partition count: every (sequence, tile) pair is
        covered exactly once, in order, and no part exceeds the target width
        by more than one tile and one segment overhead."""
        o = overhead_for(heads_per_kv)
        u = granule_for(heads_per_kv) * TILE_COST
        meta, ns, parts = check_plan(seqlens, parts_n, heads_per_kv)
        target = target_width(seqlens, parts_n, heads_per_kv)
        for segs in parts:
            cost = sum(seg_cost(lo, hi, heads_per_kv) for (_, lo, hi, _) in segs)
            assert cost <= target + u + o
except ImportError:  # pragma: no cover
    pass

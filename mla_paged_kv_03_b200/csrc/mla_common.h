// mla_common.h -- constants, device status codes and the split-KV planner
// shared by the host entry points and the device kernels of libmla_b200.
#pragma once
#include <cstdint>

#ifdef __CUDACC__
#define MLA_HD __host__ __device__
#else
#define MLA_HD
#endif

namespace mla {

// Latent geometry of MLA: one shared KV head of 576 dims, 512 "nope" dims
// followed by 64 decoupled-RoPE dims; V is a prefix of the latent row.
// [FlashMLA (AI Wiki), "How does MLA differ from MHA and GQA?"]
constexpr int kD = 576;
constexpr int kNope = 512;
constexpr int kRope = 64;
constexpr int kPage = 64;        // paged cache block size [FlashMLA (AI Wiki), "What is FlashMLA?"]
constexpr int kRow656 = 656;     // FP8 cache row [FlashMLA (AI Wiki), "The FP8 and FP4 KV cache"]

// Kernel tiling: 128-token tiles (two pages), at most 64 query rows per CTA,
// 64-dim (128-byte) column chunks in the SW128 layout.
constexpr int kTileT = 128;
constexpr int kRowsPerCta = 64;
constexpr int kChunkD = 64;
constexpr int kNumChunks = kD / kChunkD;  // 9

// Planner cost of one work segment beyond its tiles (Q load, pipeline fill,
// epilogue), in tile units.
constexpr int kSegmentOverheadTiles = 2;

// Metadata row per SM part: {begin_b, begin_tile, end_b, end_tile,
// first_split, 0, 0, 0}; end_tile is exclusive within batch end_b.
constexpr int kMetaInts = 8;

// Device status codes (upper 16 bits of the status word).
constexpr int MLA_DEVERR_TIMEOUT = 1;
constexpr int MLA_DEVERR_BAD_INDEX = 2;

constexpr unsigned long long kWaitBudgetNs = 2000000000ull;  // 2 s per wait

MLA_HD inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Tiles (of 128 tokens) a sequence of length L contributes.  An empty
// sequence still owns one (fully masked) tile so that some CTA writes its
// O = 0, LSE = -inf result.
MLA_HD inline int tiles_of(int L) { return L > 0 ? ceil_div(L, kTileT) : 1; }

// Greedy dealing of tiles to parts with a cost cap `target` per part; a
// segment costs its tiles plus kSegmentOverheadTiles.  `tiles[b]` is
// tiles_of(seqlens[b]).  Returns the number of parts used (stops counting at
// max_parts + 1); writes the plan when metadata != nullptr.
MLA_HD inline int deal_tiles(const int32_t* tiles, int batch, long long target, int max_parts,
                             int32_t* metadata, int32_t* num_splits) {
  int p = 0;
  long long used = 0;
  bool part_open = false;
  if (num_splits) num_splits[0] = 0;
  for (int b = 0; b < batch; ++b) {
    const int n = tiles[b];
    int t = 0;
    int splits = 0;
    while (t < n) {
      if (part_open && used + kSegmentOverheadTiles + 1 > target) {
        ++p;
        used = 0;
        part_open = false;
        if (!metadata && p >= max_parts) return max_parts + 1;  // does not fit
      }
      const long long avail = target - used - kSegmentOverheadTiles;
      int take = static_cast<int>(avail < 1 ? 1 : (avail < n - t ? avail : n - t));
      if (metadata && p >= max_parts - 1) take = n - t;  // the last part takes the rest
      if (metadata) {
        int32_t* m = metadata + p * kMetaInts;
        if (!part_open) {
          m[0] = b;
          m[1] = t;
          m[4] = splits;
        }
        m[2] = b;
        m[3] = t + take;
      }
      part_open = true;
      used += take + kSegmentOverheadTiles;
      t += take;
      ++splits;
    }
    if (num_splits) num_splits[b + 1] = num_splits[b] + splits;
  }
  return part_open ? p + 1 : p;
}

// Parts used by the greedy dealing of deal_tiles() with cost cap `target`,
// one arithmetic step per sequence: after the sequence's first segment fills
// the open part, every further segment takes a fresh part of target - overhead
// tiles.  Returns max_parts + 1 as soon as the count exceeds max_parts.
MLA_HD inline int count_parts(const int32_t* tiles, int batch, long long target, int max_parts) {
  const long long o = kSegmentOverheadTiles;
  const long long full = target - o;  // tiles of a segment that fills a part
  long long p = 0, used = 0;
  bool open = false;
  for (int b = 0; b < batch; ++b) {
    const long long n = tiles[b];
    if (open && used + o + 1 > target) {
      ++p;
      used = 0;
      if (p >= max_parts) return max_parts + 1;
    }
    const long long avail = target - used - o;
    open = true;
    if (n <= avail) {
      used += n + o;
      continue;
    }
    const long long r = n - avail;           // tiles left after filling the open part
    const long long k = (r + full - 1) / full;  // further segments, one part each
    p += k;
    if (p >= max_parts) return max_parts + 1;
    used = r - (k - 1) * full + o;
  }
  return static_cast<int>(open ? p + 1 : p);
}

// Caps checked one by one above the lower bound before the planner falls
// back to bisection (the device planner checks them in parallel).
constexpr int kPlanWindow = 256;

// Smallest cap >= lo in the window for which the dealing fits, else the
// bisection boundary beyond it (the whole load in one part always fits).
MLA_HD inline long long plan_cap_beyond_window(const int32_t* tiles, int batch, int num_parts,
                                               long long lo, long long total) {
  long long a = lo + kPlanWindow;
  long long b = total > a ? total : a;
  while (a < b) {
    const long long mid = a + (b - a) / 2;
    if (count_parts(tiles, batch, mid, num_parts) <= num_parts)
      b = mid;
    else
      a = mid + 1;
  }
  return a;
}

// Lower bound of the cap: the mean cost per part, at least one tile.
MLA_HD inline long long plan_lower_bound(long long total, int num_parts) {
  long long lo = (total + num_parts - 1) / num_parts;
  return lo < kSegmentOverheadTiles + 1 ? kSegmentOverheadTiles + 1 : lo;
}

MLA_HD inline void plan_mark_empty(int32_t* m, int batch) {
  m[0] = batch;  // empty part: begins after every sequence
  m[1] = 0;
  m[2] = batch - 1;
  m[3] = 0;
  m[4] = m[5] = m[6] = m[7] = 0;
}

// Split-KV planner.  Finds the smallest per-part cost cap for which the
// greedy dealing (sequences in order, tiles of 128 tokens, a segment costing
// its tiles plus kSegmentOverheadTiles) fits in `num_parts` parts, then
// writes metadata[num_parts][8] and the prefix sums num_splits[batch + 1]
// (num_splits[b+1] - num_splits[b] = number of parts holding tiles of
// sequence b).  Each part covers one contiguous run of (sequence, tile)
// pairs; unused parts are marked empty (begin_seq > end_seq).  The caps
// lo .. lo + kPlanWindow - 1 above the lower bound are tried in order
// (the optimum lies within a few tiles of the bound), then bisection.
// `tiles` holds tiles_of() of every sequence.  The device planner
// (mla_plan_kernel) reaches the same cap.
MLA_HD inline void plan_splits_tiles(const int32_t* tiles, int batch, int num_parts,
                                     int32_t* metadata, int32_t* num_splits) {
  for (int p = 0; p < num_parts; ++p) plan_mark_empty(metadata + p * kMetaInts, batch);
  long long total = 0;
  for (int b = 0; b < batch; ++b) total += tiles[b] + kSegmentOverheadTiles;
  const long long lo = plan_lower_bound(total, num_parts);
  long long cap = -1;
  for (int k = 0; k < kPlanWindow && cap < 0; ++k)
    if (count_parts(tiles, batch, lo + k, num_parts) <= num_parts) cap = lo + k;
  if (cap < 0) cap = plan_cap_beyond_window(tiles, batch, num_parts, lo, total);
  deal_tiles(tiles, batch, cap, num_parts, metadata, num_splits);
}

}  // namespace mla

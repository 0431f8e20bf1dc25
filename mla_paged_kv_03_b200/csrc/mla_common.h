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
constexpr int kRow528 = 528;     // V4.1 FP8 cache row (512 e4m3 + 16 e8m0), same section
constexpr int kRow288 = 288;     // V4.1 FP4 cache row (512 e2m1 + 32 e4m3), same section
constexpr int kRowBf16 = 1152;   // plain bf16 latent row of 576 dims (sparse prefill)

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

// The planner counts in int32: the total cost sum(tiles + overhead) of a
// call must stay below this (checked by the entry points).
constexpr long long kPlanMaxTotal = (1LL << 30);

// ------------------------------------------------------- split-KV planner
//
// The sequences' work is laid out on one cost line: sequence b occupies
// [C[b], C[b+1]) with C[b+1] = C[b] + kSegmentOverheadTiles + tiles_of(L_b);
// its overhead positions come first and tile t sits at C[b] + overhead + t.
// The line is cut into num_parts intervals of width W = ceil(total /
// num_parts); part p takes the tiles whose positions fall in [pW, (p+1)W).
// Each part therefore covers one contiguous run of (sequence, tile) pairs and
// costs at most W plus one segment overhead (that of a sequence continued
// from the previous part).  Every quantity below is a closed form of C, so
// the device planner computes all parts and sequences in parallel and the
// host planner reaches the identical result with plain loops.

MLA_HD inline int plan_width(int total, int num_parts) {
  const int w = (total + num_parts - 1) / num_parts;
  return w < 1 ? 1 : w;
}

// Sequence b with C[b] <= x < C[b+1] (C holds batch + 1 prefix sums).
MLA_HD inline int plan_seq_at(const int32_t* C, int batch, int x) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (C[mid] <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// Parts holding tiles of sequence b: [plan_first_part(b), plan_last_part(b)].
MLA_HD inline int plan_first_part(const int32_t* C, int b, int w) {
  return (C[b] + kSegmentOverheadTiles) / w;
}
MLA_HD inline int plan_last_part(const int32_t* C, int b, int w) { return (C[b + 1] - 1) / w; }

MLA_HD inline void plan_mark_empty(int32_t* m, int batch) {
  m[0] = batch;  // empty part: begins after every sequence
  m[1] = 0;
  m[2] = batch - 1;
  m[3] = 0;
  m[4] = m[5] = m[6] = m[7] = 0;
}

// Metadata row of part p: {begin_b, begin_tile, end_b, end_tile (exclusive),
// first_split, 0, 0, 0}, or an empty row.
MLA_HD inline void plan_part_row(const int32_t* C, int batch, int w, int p, int32_t* m) {
  const int o = kSegmentOverheadTiles;
  const int total = C[batch];
  const long long s64 = static_cast<long long>(p) * w;
  if (batch == 0 || s64 >= total) {
    plan_mark_empty(m, batch);
    return;
  }
  const int s = static_cast<int>(s64);
  const int e = (total - s > w) ? s + w : total;  // interval [s, e)
  const int b0 = plan_seq_at(C, batch, s);
  int t0 = s - C[b0] - o;
  if (t0 < 0) t0 = 0;  // s inside b0's overhead: its first tile
  int b1 = plan_seq_at(C, batch, e - 1);
  int t1 = e - 1 - C[b1] - o;  // last tile in the interval
  if (t1 < 0) {                // e - 1 inside b1's overhead: the previous sequence's last tile
    --b1;
    if (b1 >= 0) t1 = C[b1 + 1] - C[b1] - o - 1;
  }
  if (b1 < b0 || (b1 == b0 && t1 < t0)) {  // only overhead positions
    plan_mark_empty(m, batch);
    return;
  }
  m[0] = b0;
  m[1] = t0;
  m[2] = b1;
  m[3] = t1 + 1;
  m[4] = p - plan_first_part(C, b0, w);
  m[5] = m[6] = m[7] = 0;
}

// Host planner: metadata[num_parts][8] and num_splits[batch + 1] from the
// per-sequence tile counts (same result as the device planner).
inline void plan_splits_host(const int32_t* tiles, int batch, int num_parts, int32_t* metadata,
                             int32_t* num_splits, int32_t* C /* batch + 1 scratch */) {
  C[0] = 0;
  for (int b = 0; b < batch; ++b) C[b + 1] = C[b] + tiles[b] + kSegmentOverheadTiles;
  const int w = plan_width(C[batch], num_parts);
  for (int p = 0; p < num_parts; ++p) plan_part_row(C, batch, w, p, metadata + p * kMetaInts);
  num_splits[0] = 0;
  for (int b = 0; b < batch; ++b)
    num_splits[b + 1] = num_splits[b] + plan_last_part(C, b, w) - plan_first_part(C, b, w) + 1;
}

}  // namespace mla

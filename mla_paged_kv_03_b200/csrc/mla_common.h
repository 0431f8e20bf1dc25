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

// Kernel tiling: 128-token tiles (two pages), at most 64 query rows per CTA,
// 64-dim (128-byte) column chunks in the SW128 layout.
constexpr int kTileT = 128;
constexpr int kRowsPerCta = 64;
constexpr int kChunkD = 64;
constexpr int kNumChunks = kD / kChunkD;  // 9

// Planner costs, in units of a quarter tile (32 tokens): a tile costs
// kPlanTileCost; one work segment (a sequence, or the part of one, that a CTA
// takes) costs a further overhead for its Q load, pipeline fill and epilogue.
// Work is dealt in granules of whole tiles: two for the CTA-pair kernel, which
// steps over 256 tokens at a time (a split of an odd tile count would leave
// half a step idle), one tile for the others.  The overhead and the granule
// depend on the kernel that will run, which the planner knows from the rows
// per KV head; the overheads are the fastest values of sweeps over the
// benchmark workloads on B200.  A part of the 1-CTA kernel is also at least
// two tiles wide: at batch 1 (the fused decode) one-tile parts leave the
// attention kernel latency-bound and make the combine read 148 partials per
// row, and two-tile parts were the fastest step of a sweep over 1..8 tiles.
constexpr int kPlanTileCost = 4;
#ifndef MLA_PLAN_OVH_PAGE
#define MLA_PLAN_OVH_PAGE 4
#endif
#ifndef MLA_PLAN_OVH_CTA
#define MLA_PLAN_OVH_CTA 16
#endif
#ifndef MLA_PLAN_OVH_PAIR
#define MLA_PLAN_OVH_PAIR 8
#endif
constexpr int kPlanOverheadPage = MLA_PLAN_OVH_PAGE;  // <= 32 rows per KV head (page kernel)
constexpr int kPlanOverheadCta = MLA_PLAN_OVH_CTA;    // 33..64 rows (1-CTA kernel)
constexpr int kPlanOverheadPair = MLA_PLAN_OVH_PAIR;  // > 64 rows (CTA-pair kernel)

constexpr int kPlanMinWidthCta = 2 * kPlanTileCost;

// The planner's constants for the kernel that serves `heads_per_kv` rows:
// segment overhead o, granule g (tiles) and minimum part width (cost units).
struct PlanParams {
  int o, g, wmin;
};
MLA_HD inline PlanParams plan_params(int heads_per_kv) {
  if (heads_per_kv <= 32) return {kPlanOverheadPage, 1, 0};
  if (heads_per_kv <= 64) return {kPlanOverheadCta, 1, kPlanMinWidthCta};
  return {kPlanOverheadPair, 2, 0};
}

// Metadata row per SM part: {begin_b, begin_tile, end_b, end_tile,
// first_split, 0, 0, 0}; end_tile is exclusive within batch end_b (it may pass
// that sequence's last tile, see the planner below).
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

// Planner granules (of g tiles) a sequence of length L contributes.
MLA_HD inline int granules_of(int L, int g) { return (tiles_of(L) + g - 1) / g; }

// The planner counts in int32: the total cost sum(tiles + overhead) of a
// call must stay below this (checked by the entry points).
constexpr long long kPlanMaxTotal = (1LL << 30);

// ------------------------------------------------------- split-KV planner
//
// The sequences' work is laid out on one cost line: with granules of g tiles,
// each costing u = g * kPlanTileCost, sequence b occupies [C[b], C[b+1]) with
// C[b+1] = C[b] + o + u * granules_of(L_b, g) (o the segment overhead); its
// overhead comes first and granule t starts at C[b] + o + u t.  The line is
// cut into num_parts intervals of width W = ceil(total / num_parts) (or the
// kernel's minimum width, when larger; the parts past the end stay empty); part p
// takes the granules whose start falls in [pW, (p+1)W).  Each part therefore
// covers one contiguous run of (sequence, tile) pairs and costs at most W plus
// one granule and one segment overhead (that of a sequence continued from the
// previous part).  Tile indices in the metadata are granule indices times g;
// a part's end tile may pass its last sequence's tiles by less than g (the
// kernels clamp it).  Every quantity below is a closed form of C, so the
// device planner computes all parts and sequences in parallel and the host
// planner reaches the identical result with plain loops.

// At least one granule (u) wide, so that every interval lying within a
// sequence's granules holds a granule start (the split counts rely on that),
// and at least the kernel's minimum width.
MLA_HD inline int plan_width(int total, int num_parts, const PlanParams& pp) {
  const int w = (total + num_parts - 1) / num_parts;
  const int u = pp.g * kPlanTileCost;
  const int m = u > pp.wmin ? u : pp.wmin;
  return w < m ? m : w;
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

// Parts holding tiles of sequence b: [plan_first_part(b), plan_last_part(b)]
// (the parts of its first and last granule starts; u = granule cost).
MLA_HD inline int plan_first_part(const int32_t* C, int b, int w, int o) {
  return (C[b] + o) / w;
}
MLA_HD inline int plan_last_part(const int32_t* C, int b, int w, int u) {
  return (C[b + 1] - u) / w;
}

MLA_HD inline void plan_mark_empty(int32_t* m, int batch) {
  m[0] = batch;  // empty part: begins after every sequence
  m[1] = 0;
  m[2] = batch - 1;
  m[3] = 0;
  m[4] = m[5] = m[6] = m[7] = 0;
}

// Metadata row of part p: {begin_b, begin_tile, end_b, end_tile (exclusive),
// first_split, 0, 0, 0}, or an empty row.
MLA_HD inline void plan_part_row(const int32_t* C, int batch, int w, int o, int g, int p,
                                 int32_t* m) {
  const int u = g * kPlanTileCost;
  const int total = C[batch];
  const long long s64 = static_cast<long long>(p) * w;
  if (batch == 0 || s64 >= total) {
    plan_mark_empty(m, batch);
    return;
  }
  const int s = static_cast<int>(s64);
  const int e = (total - s > w) ? s + w : total;  // interval [s, e)
  // first granule starting at or after s
  int b0 = plan_seq_at(C, batch, s);
  const int r0 = s - C[b0] - o;
  int t0 = r0 <= 0 ? 0 : (r0 + u - 1) / u;
  if (C[b0] + o + u * t0 >= C[b0 + 1]) {  // past b0's last granule start
    ++b0;
    t0 = 0;
  }
  // last granule starting before e
  int b1 = plan_seq_at(C, batch, e - 1);
  const int r1 = e - 1 - C[b1] - o;
  int t1 = r1 < 0 ? -1 : r1 / u;
  if (t1 < 0) {  // e - 1 inside b1's overhead: the previous sequence's last granule
    --b1;
    if (b1 >= 0) t1 = (C[b1 + 1] - C[b1] - o) / u - 1;
  }
  if (b0 >= batch || b1 < b0 || (b1 == b0 && t1 < t0)) {  // no tile starts in [s, e)
    plan_mark_empty(m, batch);
    return;
  }
  m[0] = b0;
  m[1] = t0 * g;
  m[2] = b1;
  m[3] = (t1 + 1) * g;
  m[4] = p - plan_first_part(C, b0, w, o);
  m[5] = m[6] = m[7] = 0;
}

// Host planner: metadata[num_parts][8] and num_splits[batch + 1] from the
// per-sequence granule counts and the kernel's planner constants (same
// result as the device planner).
inline void plan_splits_host(const int32_t* granules, int batch, int num_parts,
                             const PlanParams& pp, int32_t* metadata, int32_t* num_splits,
                             int32_t* C /* batch + 1 scratch */) {
  const int o = pp.o, g = pp.g;
  const int u = g * kPlanTileCost;
  C[0] = 0;
  for (int b = 0; b < batch; ++b) C[b + 1] = C[b] + o + u * granules[b];
  const int w = plan_width(C[batch], num_parts, pp);
  for (int p = 0; p < num_parts; ++p)
    plan_part_row(C, batch, w, o, g, p, metadata + p * kMetaInts);
  num_splits[0] = 0;
  for (int b = 0; b < batch; ++b)
    num_splits[b + 1] =
        num_splits[b] + plan_last_part(C, b, w, u) - plan_first_part(C, b, w, o) + 1;
}

}  // namespace mla

// pair_kernel.cuh -- 2-CTA (cta_group::2) sm_100a MLA decode for 65..128 query
// rows per latent KV head (e.g. 128 heads, s_q = 1), d_v = 512.
//
// Same computation as decode_kernel.cuh (softmax(scale Q K^T) V with V = the
// first d_v latent dims, plus LSE; [FlashMLA (AI Wiki), "How does MLA differ
// from MHA and GQA?", "Interfaces"]), in the conventional orientation: query
// rows on the UMMA M axis.  A pair of CTAs on two SMs runs M = 128, N = 256
// UMMAs over steps of 256 tokens (two scheduler tiles):
//   S[128 rows, 256 tok]   = Q[128, 576] . K_step[256 tok, 576]^T          (36 UMMAs)
//   O[128 rows, 256 d_j]  += P[128, 256 tok] . V_j[256 tok, 256 d]^T, j < 2 (32 UMMAs)
// Each CTA holds 64 of the rows (its Q and P), 128 of the step's tokens (two
// pages) for QK, and 128 of each 256-dim V slice for PV; the tensor cores read
// the partner's halves directly.  Per step each CTA moves 272 KB into shared
// memory in 16 KB stages.  In each CTA's TMEM a 64-row accumulator of N
// columns lies in lanes 0..63 for columns [0, N/2) and lanes 64..127 for
// [N/2, N), so thread (lane L) of the softmax warpgroup owns row L % 64 for
// the tokens (or output dims) of half L / 64.
//
// The MMA and loader warps run their loops warp-wide and let one elected
// lane issue each group of eight UMMAs (or the TMA copies): the per-group
// address arithmetic then stays warp-uniform, and a group of eight N = 256
// UMMAs covers the cost of the barrier waits between groups.
//
// Roles (warps): 0, 10, 11 loaders (both CTAs), 1 MMA issuer (leader CTA)
// and TMEM owner (both), 2..9 two softmax / epilogue warpgroups (both).
//
// Gather mode (sparse prefill): a unit is one query token, and its "cache" is
// the rows of a bf16 [s_kv, 576] array that the token's index list names.
// The loaders fetch them with TMA gather4 copies (four named rows, one 64-dim
// chunk each), so neighbouring tokens that select the same rows share them
// through L2; the softmax masks the entries that name no row.
#pragma once
#include "decode_kernel.cuh"

namespace mla {

namespace pcfg {
constexpr int kRows = 64;                          // query rows per CTA
constexpr int kStepT = 2 * kTileT;                 // tokens per step
constexpr int kBox = 64 * 128;                     // one TMA box: 64 rows x 64 bf16
constexpr int kQBytes = kNumChunks * kBox;         // 73728: [9 chunks][64 rows][64 d]
constexpr int kStage = 2 * kBox;                   // 16 KB ring stage
// One ring of 16 KB stages, consumed in UMMA order (the 9 K stages of step
// i, then the 8 V stages of step i - 1).  A TMA-issuing warp only sustains
// about 25 B/clk, so kLoaders warps fill the ring round-robin (stage load j
// by loader j % kLoaders).
#ifndef MLA_PAIR_STAGES
#define MLA_PAIR_STAGES 7
#endif
#ifndef MLA_PAIR_LOADERS
#define MLA_PAIR_LOADERS 3
#endif
constexpr int kNStage = MLA_PAIR_STAGES;
constexpr int kLoaders = MLA_PAIR_LOADERS;
static_assert(kLoaders >= 1 && kLoaders <= 3, "1 to 3 loader warps");
constexpr int kPBytes = 4 * kBox;                  // [4 token chunks][64 rows][64 tok] bf16
constexpr int kQOff = 0;
constexpr int kRingOff = kQOff + kQBytes;
constexpr int kPOff = kRingOff + kNStage * kStage;
constexpr int kBarOff = kPOff + kPBytes;
constexpr int kMiscBytes = 4096;
constexpr int kSmemBytes = kBarOff + kMiscBytes + 1024;
constexpr int kTmemCols = 512;
constexpr int kSCol = 0;    // S buffers at columns [0,128) and [128,256)
constexpr int kOCol = 256;  // O slice j (256 output dims) at columns 256 + 128 j
constexpr int kSoftmaxWarps = 8;  // two warpgroups, each on half of a lane half's columns
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
// Loader warps: 0, then 10, 11 after the softmax warps.
constexpr int kThreads = 32 * (2 + kSoftmaxWarps + kLoaders - 1);
}  // namespace pcfg
static_assert(pcfg::kSmemBytes <= 232448, "pair kernel shared memory above the sm_100 limit");

struct __align__(8) PairCtrl {
  uint64_t full[pcfg::kNStage], empty[pcfg::kNStage];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, p_empty;
  uint64_t o_free, drain;
  uint32_t tmem_base, pad;
  float red[2][4][64];  // [step parity][column quarter][row] partial row max
  float lred[4][64];    // [column quarter][row] partial row sums
};
static_assert(sizeof(PairCtrl) <= pcfg::kMiscBytes, "pair control block too large");

// Bounded wait, uniform over the softmax warps (barrier id 3): every thread
// waits, then the warps agree, so that all take the same path even if one
// of them timed out.
__device__ __forceinline__ bool sm_wait_cluster(uint64_t* bar, uint32_t parity, int site) {
  const bool mine = ptx::mbar_wait_cluster(bar, parity, site);
  uint32_t all;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 3, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(all)
      : "r"(mine ? 1 : 0), "n"(pcfg::kSoftmaxThreads));
  return all != 0;
}

// Warp-uniform bounded wait (every lane waits, the warp agrees).
__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity, int site) {
  const bool mine = ptx::mbar_wait_cluster(bar, parity, site);
  return __all_sync(0xffffffffu, mine);
}

// kGather: the tokens of a unit are rows of a bf16 array named by per-unit
// index lists (sparse prefill): K and V come in by TMA gather4 loads of four
// rows at a time (tm_kv is then a map with a box one row high), and entries
// that name no row are masked.
template <bool kGather>
__global__ void __launch_bounds__(pcfg::kThreads, 1)
    mla_pair_decode_kernel(const __grid_constant__ CUtensorMap tm_q3,
                           const __grid_constant__ CUtensorMap tm_kv,
                           const __grid_constant__ CUtensorMap tm_v3, const DecodeParams P) {
  using namespace pcfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kQOff;
  uint8_t* sRing = smem + kRingOff;
  uint8_t* sP = smem + kPOff;
  PairCtrl& C = *reinterpret_cast<PairCtrl*>(smem + kBarOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();  // 0 = leader (issues the UMMAs)
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int part = pair / P.n_groups;
  const int grp = pair % P.n_groups;  // 128-row group

  const int nqk = P.qk_chunks ? P.qk_chunks : kNumChunks;  // 64-dim chunks of q . k
  ptx::grid_dep_wait();    // the planner's metadata is complete
  ptx::grid_dep_launch();  // the combine grid may be scheduled as CTAs retire
  const int32_t* meta = P.metadata + part * kMetaInts;
  if (meta[0] > meta[2]) return;  // empty part: both CTAs of the pair leave together

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNStage; ++i) {
      ptx::mbar_init(&C.full[i], 1);
      ptx::mbar_init(&C.empty[i], 1);
    }
    ptx::mbar_init(&C.q_full, 1);
    ptx::mbar_init(&C.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&C.s_full[i], 1);
      ptx::mbar_init(&C.s_empty[i], 2 * kSoftmaxWarps);  // each softmax warp of both CTAs
    }
    ptx::mbar_init(&C.p_full, 2 * kSoftmaxWarps);
    ptx::mbar_init(&C.p_empty, 1);
    ptx::mbar_init(&C.o_free, 2 * kSoftmaxWarps);
    ptx::mbar_init(&C.drain, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&C.tmem_base, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_q3);
    ptx::prefetch_tmap(&tm_kv);
    ptx::prefetch_tmap(&tm_v3);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // barriers of both CTAs initialised before any remote use
  ptx::tc_fence_after();
  const uint32_t tmem = C.tmem_base;

  // leader-side barrier addresses in the shared::cluster window
  auto leader_addr = [&](uint64_t* bar) { return ptx::mapa_shared(ptx::smem_u32(bar), 0); };

  UnitIter it;
  it.init(meta);

  // Physical block of logical page `page`; pages past the sequence or past
  // this split's last tile load `fallback` instead (their tokens are masked).
  auto page_block = [&](const Unit& un, int page, int fallback) -> int {
    const int npg = (un.L + kPage - 1) / kPage;  // <= max_pages
    const int end = min(npg, 2 * un.hi);
    const int pg = page < end ? page : fallback;
    const int blk = pg < npg ? P.block_table[(size_t)un.b * P.max_pages + pg] : 0;
    return clamp_block(blk, P.num_blocks);
  };
  // Gather mode: the row of index entry e of unit `un` (row 0, masked, for an
  // entry past the unit's length or naming no row).
  auto gather_row = [&](const Unit& un, int e) -> int {
    if (e >= un.L) return 0;
    const int r = P.gather_idx[(size_t)un.b * P.gather_stride + e];
    return (r >= 0 && r < P.gather_rows) ? r : 0;
  };
  // Debug slot trace of the pages a load reads (pages a load only pads with
  // are not recorded).
  auto trace_if_real = [&](const Unit& un, int page, int blk, int planes) {
    const int npg = (un.L + kPage - 1) / kPage;
    if (page < npg && page < 2 * un.hi) trace_page(P, un.b, page, blk, planes);
  };

  if (warp == 0 || warp >= 2 + kSoftmaxWarps) {
    // ======================= loaders (both CTAs); warp 0 also loads Q =======================
    const int role = warp == 0 ? 0 : warp - (1 + kSoftmaxWarps);  // 0 .. kLoaders - 1
    uint32_t st_it = 0;  // stage loads so far (every loader counts all of them)
    int u_idx = 0;
    Unit u;
    bool ok = true;
    // Next stage load: `mine` tells whether this warp issues it; if so, waits
    // (warp-wide) for the stage to be free.
    auto acquire = [&](int& s, bool& mine) -> bool {
      const uint32_t idx = st_it++;
      mine = static_cast<int>(idx % kLoaders) == role;
      s = static_cast<int>(idx % kNStage);
      if (!mine) return true;
      return warp_wait_cluster(&C.empty[s], ((idx / kNStage) & 1) ^ 1, 0x41);
    };
    // K of step i: chunk c = [this CTA's 128 tokens (two pages)][64 dims]
    auto load_k = [&](const Unit& un, int i) -> bool {
      if constexpr (kGather) {
        // this CTA's 128 entries of the step: lane l loads rows 4l .. 4l + 3
        const int e0 = un.lo * kTileT + kStepT * i + 128 * static_cast<int>(rank) + 4 * lane;
        int r[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) r[k] = gather_row(un, e0 + k);
        if (role == 0) {
          // an entry past the rows is an input fault (negative ones mark unused entries)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (e0 + k < un.L && P.gather_idx[(size_t)un.b * P.gather_stride + e0 + k] >= P.gather_rows)
              ptx::set_error(MLA_DEVERR_BAD_INDEX, 0x46);
        }
        if (P.trace && role == 0) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int e = e0 + k;
            if (e < un.L) {
              const int raw = P.gather_idx[(size_t)un.b * P.gather_stride + e];
              const bool ok_row = raw >= 0 && raw < P.gather_rows;
              P.trace[(size_t)un.b * P.gather_stride + e] = ok_row ? raw : -1;
              P.trace[P.trace_plane + (size_t)un.b * P.gather_stride + e] = ok_row ? e : -1;
            }
          }
        }
        for (int c = 0; c < nqk; ++c) {
          int s;
          bool mine;
          if (!acquire(s, mine)) return false;
          if (!mine) continue;
          const uint32_t bar = leader_addr(&C.full[s]);
          if (leader && ptx::elect_one_sync()) ptx::mbar_arrive_expect_tx(&C.full[s], 2u * kStage);
          __syncwarp();
          ptx::tma_gather4_pair(sRing + s * kStage + lane * 512, &tm_kv, bar, c * kChunkD, r[0],
                                r[1], r[2], r[3]);
          __syncwarp();
        }
        return true;
      }
      const int p0 = 2 * (un.lo + 2 * i);
      const int kb0 = page_block(un, p0 + 2 * static_cast<int>(rank), p0);
      const int kb1 = page_block(un, p0 + 2 * static_cast<int>(rank) + 1, p0);
      if (P.trace && role == 0) {
        trace_if_real(un, p0 + 2 * static_cast<int>(rank), kb0, 1);
        trace_if_real(un, p0 + 2 * static_cast<int>(rank) + 1, kb1, 1);
      }
      for (int c = 0; c < nqk; ++c) {
        int s;
        bool mine;
        if (!acquire(s, mine)) return false;
        if (!mine) continue;
        if (ptx::elect_one_sync()) {
          if (leader) ptx::mbar_arrive_expect_tx(&C.full[s], 2u * kStage);
          const uint32_t bar = leader_addr(&C.full[s]);
          uint8_t* dst = sRing + s * kStage;
          ptx::tma_load_2d_pair(dst, &tm_kv, bar, c * kChunkD, kb0 * kPage);
          ptx::tma_load_2d_pair(dst + kBox, &tm_kv, bar, c * kChunkD, kb1 * kPage);
        }
        __syncwarp();
      }
      return true;
    };
    // V of step i: stage (j, q) = [page q][this CTA's 128 dims of slice j], one 3-D box
    auto load_v = [&](const Unit& un, int i) -> bool {
      if constexpr (kGather) {
        // stage (j, q): entries [64 q, 64 q + 64) of the step, this CTA's 128
        // dims of slice j; lane l loads rows 4 (l % 16) .. + 3 of chunk l / 16
        const int h = lane >> 4;
        int r[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            r[q][k] = gather_row(un, un.lo * kTileT + kStepT * i + 64 * q + 4 * (lane & 15) + k);
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            int s;
            bool mine;
            if (!acquire(s, mine)) return false;
            if (!mine) continue;
            const uint32_t bar = leader_addr(&C.full[s]);
            if (leader && ptx::elect_one_sync())
              ptx::mbar_arrive_expect_tx(&C.full[s], 2u * kStage);
            __syncwarp();
            ptx::tma_gather4_pair(sRing + s * kStage + h * kBox + (lane & 15) * 512, &tm_kv, bar,
                                  kChunkD * (4 * j + 2 * static_cast<int>(rank) + h), r[q][0],
                                  r[q][1], r[q][2], r[q][3]);
            __syncwarp();
          }
        return true;
      }
      const int p0 = 2 * (un.lo + 2 * i);
      int vb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) vb[q] = page_block(un, p0 + q, p0);
      if (P.trace && role == 0)
        for (int q = 0; q < 4; ++q) trace_if_real(un, p0 + q, vb[q], 2);
      for (int j = 0; j < 2; ++j)
        for (int q = 0; q < 4; ++q) {
          int s;
          bool mine;
          if (!acquire(s, mine)) return false;
          if (!mine) continue;
          if (ptx::elect_one_sync()) {
            if (leader) ptx::mbar_arrive_expect_tx(&C.full[s], 2u * kStage);
            ptx::tma_load_3d_pair(sRing + s * kStage, &tm_v3, leader_addr(&C.full[s]), 0,
                                  vb[q] * kPage, 4 * j + 2 * static_cast<int>(rank));
          }
          __syncwarp();
        }
      return true;
    };
    while (ok && it.next<kDense>(P, u)) {
      const int n = (u.hi - u.lo + 1) >> 1;
      if (role == 0) {
        if (!warp_wait_cluster(&C.q_empty, (u_idx & 1) ^ 1, 0x42)) {
          ok = false;
          break;
        }
        const int row0 = u.b * P.R + grp * 128 + static_cast<int>(rank) * kRows;
        if (ptx::elect_one_sync()) {
          if (leader) ptx::mbar_arrive_expect_tx(&C.q_full, 2u * nqk * kBox);
          ptx::tma_load_3d_pair(sQ, &tm_q3, leader_addr(&C.q_full), 0, row0, 0);
        }
        __syncwarp();
      }
      for (int i = 0; i < n && ok; ++i) {
        ok = load_k(u, i);
        if (ok && i >= 1) ok = load_v(u, i - 1);
      }
      if (ok) ok = load_v(u, n - 1);
      ++u_idx;
    }
    // drain: wait (bounded) until this warp's last loads into each stage landed
    // (the MMA issuer consumed them and released the stage).
    for (int i = 0; i < kNStage && i < static_cast<int>(st_it); ++i) {
      const uint32_t last = st_it - 1 - i;
      if (static_cast<int>(last % kLoaders) != role) continue;
      warp_wait_cluster(&C.empty[last % kNStage], (last / kNStage) & 1, 0x43);
    }
  } else if (warp == 1) {
    // ============================== MMA issuer (leader) ==============================
    if (leader) {
      const uint32_t idesc_qk = ptx::idesc_bf16_f32(128, 256, 0, 0);
      const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, 256, 0, 1);
      const ptx::DescWords dq = ptx::desc_words(ptx::smem_u32(sQ), 16, 1024, ptx::kLayoutSW128);
      const ptx::DescWords dk = ptx::desc_words(ptx::smem_u32(sRing), 16, 1024, ptx::kLayoutSW128);
      // V^T is MN-major: two 64-dim column blocks kBox apart, 8-token groups 1 KB apart
      const ptx::DescWords dv = ptx::desc_words(ptx::smem_u32(sRing), kBox, 1024, ptx::kLayoutSW128);
      const ptx::DescWords dp = ptx::desc_words(ptx::smem_u32(sP), 16, 1024, ptx::kLayoutSW128);
      uint32_t st_it = 0, gt = 0;
      int u_idx = 0;
      Unit u;
      bool ok = true;
      auto next_stage = [&](int& s) -> bool {
        s = static_cast<int>(st_it % kNStage);
        const uint32_t round = st_it / kNStage;
        ++st_it;
        return warp_wait_cluster(&C.full[s], round & 1, 0x51);
      };
      // 4 UMMAs: S += Q chunk c . K stage s (K = 64 dims)
      auto qk_chunk = [&](uint32_t d_tmem, int s, int c) {
        const uint32_t a = dq.lo + ((c * kBox) >> 4);
        const uint32_t b = dk.lo + ((s * kStage) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_f16_ss_pair_w(d_tmem, a + ((kk * 32) >> 4), dq.hi, b + ((kk * 32) >> 4), dk.hi,
                                  idesc_qk, (c | kk) ? 1u : 0u);
      };
      // 4 UMMAs: O_j += P token chunk t . V stage s (K = 64 tokens)
      auto pv_page = [&](uint32_t d_tmem, int s, int t, bool zero) {
        const uint32_t a = dp.lo + ((t * kBox) >> 4);
        const uint32_t b = dv.lo + ((s * kStage) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_f16_ss_pair_w(d_tmem, a + ((kk * 32) >> 4), dp.hi, b + ((kk * 2048) >> 4), dv.hi,
                                  idesc_pv, (zero && kk == 0) ? 0u : 1u);
      };
      auto do_qk = [&](uint32_t g) -> bool {
        const int sb = g & 1;
        if (!warp_wait_cluster(&C.s_empty[sb], ((g >> 1) & 1) ^ 1, 0x52)) return false;
        const uint32_t d_tmem = tmem + kSCol + sb * 128;
        for (int c0 = 0; c0 < nqk; c0 += 2) {
          const bool two = c0 + 1 < nqk;
          int s0 = 0, s1 = 0;
          if (!next_stage(s0)) return false;
          if (two && !next_stage(s1)) return false;
          ptx::tc_fence_after();
          if (ptx::elect_one_sync()) {
            qk_chunk(d_tmem, s0, c0);
            ptx::umma_commit_pair_mc(&C.empty[s0], 0x3);
            if (two) {
              qk_chunk(d_tmem, s1, c0 + 1);
              ptx::umma_commit_pair_mc(&C.empty[s1], 0x3);
            }
            if (c0 + 2 >= nqk) ptx::umma_commit_pair_mc(&C.s_full[sb], 0x3);
          }
          __syncwarp();
        }
        return true;
      };
      auto do_pv = [&](uint32_t g, bool first_of_unit) -> bool {
        if (!warp_wait_cluster(&C.p_full, g & 1, 0x53)) return false;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t d_tmem = tmem + kOCol + j * 128;
#pragma unroll
          for (int t = 0; t < 4; t += 2) {
            int s0 = 0, s1 = 0;
            if (!next_stage(s0) || !next_stage(s1)) return false;
            ptx::tc_fence_after();
            if (ptx::elect_one_sync()) {
              pv_page(d_tmem, s0, t, first_of_unit && t == 0);
              ptx::umma_commit_pair_mc(&C.empty[s0], 0x3);
              pv_page(d_tmem, s1, t + 1, false);
              ptx::umma_commit_pair_mc(&C.empty[s1], 0x3);
              if (j == 1 && t == 2) ptx::umma_commit_pair_mc(&C.p_empty, 0x3);
            }
            __syncwarp();
          }
        }
        return true;
      };
      while (ok && it.next<kDense>(P, u)) {
        if (!warp_wait_cluster(&C.q_full, u_idx & 1, 0x54)) break;
        ptx::tc_fence_after();
        const int n = (u.hi - u.lo + 1) >> 1;
        const uint32_t g0 = gt;
        for (int i = 0; i < n && ok; ++i) {
          ok = do_qk(g0 + i);
          if (ok && i == n - 1) {
            if (ptx::elect_one_sync()) ptx::umma_commit_pair_mc(&C.q_empty, 0x3);
            __syncwarp();
          }
          if (ok && i >= 1) {
            if (i == 1) {
              if (!warp_wait_cluster(&C.o_free, (u_idx & 1) ^ 1, 0x55)) {
                ok = false;
                break;
              }
              ptx::tc_fence_after();
            }
            ok = do_pv(g0 + i - 1, i == 1);
          }
        }
        if (ok) {
          if (n == 1) {
            if (!warp_wait_cluster(&C.o_free, (u_idx & 1) ^ 1, 0x56)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
          }
          ok = do_pv(g0 + n - 1, n == 1);
        }
        gt += n;
        ++u_idx;
      }
      if (ptx::elect_one_sync()) ptx::umma_commit_pair_mc(&C.drain, 0x1);
      __syncwarp();
      warp_wait_cluster(&C.drain, 0, 0x57);
    }
  } else {
    // ============================== softmax / epilogue (both CTAs) ==============================
    // Warp w (2..9) reads TMEM lanes 32 (w % 4) .. + 31; warpgroup wg = (w - 2) / 4
    // takes columns [64 wg, 64 wg + 64) of its lane half: 64 of the step's
    // tokens for S and P, and O slice wg (256 output dims) in the epilogue.
    const int wq = warp & 3;
    const int wg = (warp - 2) >> 2;
    const int L = wq * 32 + lane;   // TMEM lane
    const int r = L & 63;           // row of this CTA
    const int h = L >> 6;           // lane half
    const int quarter = 2 * h + wg;  // the thread's quarter of a row's S columns
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int rg = grp * 128 + static_cast<int>(rank) * kRows + r;  // row in [0, R)
    const bool row_valid = rg < P.R;
    const uint32_t s_empty_l = leader_addr(&C.s_empty[0]);
    const uint32_t p_full_l = leader_addr(&C.p_full);
    const uint32_t o_free_l = leader_addr(&C.o_free);
    uint32_t gt = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    while (ok && it.next<kDense>(P, u)) {
      const int n = (u.hi - u.lo + 1) >> 1;
      int lim = 0;
      if (row_valid) {
        lim = P.causal ? u.L - P.s_q + 1 + rg / P.h_q : u.L;
        lim = lim < 0 ? 0 : lim;
        lim = min(lim, u.hi * kTileT);  // tokens of later splits belong to them
      }
      float m_used = -INFINITY, lsum = 0.f;
      for (int i = 0; i < n && ok; ++i) {
        const uint32_t g = gt + i;
        const int sb = g & 1;
        // gather mode: which of this quarter's 64 entries name a row
        uint32_t vmask[2] = {0xffffffffu, 0xffffffffu};
        if constexpr (kGather) {
          const int e = u.lo * kTileT + kStepT * i + 64 * quarter + lane;
          int r0 = 0, r1 = 0;
          if (e < u.L) r0 = P.gather_idx[(size_t)u.b * P.gather_stride + e];
          if (e + 32 < u.L) r1 = P.gather_idx[(size_t)u.b * P.gather_stride + e + 32];
          vmask[0] = __ballot_sync(0xffffffffu, r0 >= 0 && r0 < P.gather_rows);
          vmask[1] = __ballot_sync(0xffffffffu, r1 >= 0 && r1 < P.gather_rows);
        }
        ok = sm_wait_cluster(&C.s_full[sb], (g >> 1) & 1, 0x61);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t s_addr = lane_addr + kSCol + sb * 128 + 64 * wg;
        const int nvalid = lim - ((u.lo + 2 * i) * kTileT + 64 * quarter);
        // One pass with the running maximum m: P = 2^(scale*s - m).  When some
        // row's maximum exceeds m_used by more than the threshold (always on a
        // unit's first step), all softmax warps redo the pass with the new
        // maximum.
        uint32_t pk[32];
        float lstep = 0.f, alpha = 1.f, m = m_used;
        bool rescaled = false;
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
          float mx = -INFINITY;
          lstep = 0.f;
          float xa[32], xb[32];
          ptx::tmem_ld32(s_addr, xa);
          ptx::tmem_ld_wait_regs(xa);
          ptx::tmem_ld32(s_addr + 32, xb);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            float* x = cc ? xb : xa;
            if (cc) ptx::tmem_ld_wait_regs(xb);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const bool v0 = 32 * cc + j < nvalid && ((vmask[cc] >> j) & 1u);
              const bool v1 = 32 * cc + j + 1 < nvalid && ((vmask[cc] >> (j + 1)) & 1u);
              mx = v0 ? fmaxf(mx, x[j]) : mx;
              mx = v1 ? fmaxf(mx, x[j + 1]) : mx;
              const float p0 = v0 ? ex2(fmaf(x[j], P.scale_log2, -m)) : 0.f;
              const float p1 = v1 ? ex2(fmaf(x[j + 1], P.scale_log2, -m)) : 0.f;
              lstep += p0 + p1;
              pk[16 * cc + j / 2] = ptx::pack_bf16x2(p0, p1);
            }
          }
          if (pass == 1) break;
          const float mxs = (mx == -INFINITY) ? -INFINITY : mx * P.scale_log2;
          const bool need = mxs > m_used + cfg::kRescaleThreshold;
          uint32_t any_need;
          asm volatile(
              "{\n\t.reg .pred p, q;\n\t"
              "setp.ne.b32 p, %1, 0;\n\t"
              "bar.red.or.pred q, 2, %2, p;\n\t"
              "selp.u32 %0, 1, 0, q;\n\t}"
              : "=r"(any_need)
              : "r"(need ? 1 : 0), "n"(kSoftmaxThreads));
          if (!any_need) break;
          // uniform over the softmax warps: exchange row maxima, new m_used
          C.red[g & 1][quarter][r] = mxs;
          ptx::named_bar_sync(1, kSoftmaxThreads);
          const float row_mx = fmaxf(fmaxf(C.red[g & 1][0][r], C.red[g & 1][1][r]),
                                     fmaxf(C.red[g & 1][2][r], C.red[g & 1][3][r]));
          const float m_new = fmaxf(m_used, row_mx);
          alpha = (m_new == -INFINITY) ? 1.f : ex2(m_used - m_new);
          lsum *= alpha;
          m_used = m_new;
          m = m_new;
          rescaled = true;
        }
        lsum += lstep;
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_remote(s_empty_l + sb * 8);
        // P buffer free and O stable once PV(g - 1) completed
        ok = sm_wait_cluster(&C.p_empty, (g & 1) ^ 1, 0x63);
        if (!ok) break;
        ptx::tc_fence_after();
        if (rescaled && i > 0) {  // this warpgroup's O slice
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            const uint32_t a = lane_addr + kOCol + 128 * wg + 32 * c;
            ptx::tmem_ld32(a, o);
            ptx::tmem_ld_wait_regs(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            ptx::tmem_st32(a, o);
          }
          ptx::tmem_st_wait();
        }
        // row r of token chunk `quarter` (K-major, 128-byte swizzle)
        uint8_t* prow = sP + quarter * kBox + r * 128;
#pragma unroll
        for (int uu = 0; uu < 8; ++uu)
          *reinterpret_cast<uint4*>(prow + ((uu ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * uu], pk[4 * uu + 1], pk[4 * uu + 2], pk[4 * uu + 3]);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_remote(p_full_l);
      }
      if (!ok) break;

      // ---- epilogue: warpgroup wg writes O slice wg (dims 256 wg + 128 h + ...)
      C.lred[quarter][r] = lsum;
      ptx::named_bar_sync(1, kSoftmaxThreads);
      const float l = (C.lred[0][r] + C.lred[1][r]) + (C.lred[2][r] + C.lred[3][r]);
      ptx::named_bar_sync(1, kSoftmaxThreads);  // lred reusable
      const uint32_t glast = gt + n - 1;
      ok = sm_wait_cluster(&C.p_empty, glast & 1, 0x64);
      if (!ok) break;
      ptx::tc_fence_after();
      const bool partial = P.always_partial || u.nsplit > 1;
      const int ws_row = ((P.ws_base ? P.ws_base[u.b] : P.num_splits[u.b]) + u.split) * P.R + rg;
      float inv = l > 0.f ? 1.0f / l : 0.f;
      float lv = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      if (!partial && P.sink) {
        // attention sink of the row's head (a logit without a value row): it
        // joins the normaliser, l' = l + 2^(sink - m) (max-shifted); a row
        // split over several parts gets it in the combine instead
        const float sk = P.sink[rg % P.h_q];
        if (sk != -INFINITY) {
          if (l > 0.f) {
            const float s2 = sk * 1.4426950408889634f;
            const float mp = fmaxf(m_used, s2);
            const float f = ex2(m_used - mp);
            const float l2 = l * f + ex2(s2 - mp);
            inv = f / l2;
            lv = (mp + __log2f(l2)) * 0.69314718055994531f;
          } else {
            lv = sk;  // no row: O stays 0
          }
        }
      }
      const bool ws32 = (reinterpret_cast<uintptr_t>(P.ws_o) & 31) == 0;
      const bool out32 = (reinterpret_cast<uintptr_t>(P.out) & 31) == 0;
      float o[2][32];
      ptx::tmem_ld32(lane_addr + kOCol + 128 * wg, o[0]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        ptx::tmem_ld_wait_regs(o[c & 1]);
        if (c < 3) ptx::tmem_ld32(lane_addr + kOCol + 128 * wg + 32 * (c + 1), o[(c + 1) & 1]);
        const float* v = o[c & 1];
        if (row_valid) {
          const int d0 = 256 * wg + 128 * h + 32 * c;
          // A thread holds 32 consecutive dims of its row: whole 32-byte sectors
          // per store where the buffer's base is 32-byte aligned (rows are
          // multiples of 32 bytes), 16-byte stores otherwise.  (Staging O
          // through shared memory so that eight lanes write one 128-byte line
          // was measured slower: more store instructions.)
          if (partial && ws32) {
            float* dst = P.ws_o + (size_t)ws_row * P.d_v + d0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              ptx::st_global_v8(dst + 8 * q, v[8 * q] * inv, v[8 * q + 1] * inv,
                                v[8 * q + 2] * inv, v[8 * q + 3] * inv, v[8 * q + 4] * inv,
                                v[8 * q + 5] * inv, v[8 * q + 6] * inv, v[8 * q + 7] * inv);
          } else if (partial) {
            float4* dst = reinterpret_cast<float4*>(P.ws_o + (size_t)ws_row * P.d_v + d0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(v[4 * q] * inv, v[4 * q + 1] * inv, v[4 * q + 2] * inv,
                                   v[4 * q + 3] * inv);
          } else if (out32) {
            __nv_bfloat16* dst = P.out + ((size_t)u.b * P.R + rg) * P.d_v + d0;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const float* w = v + 16 * q;
              ptx::st_global_v8(dst + 16 * q, ptx::pack_bf16x2(w[0] * inv, w[1] * inv),
                                ptx::pack_bf16x2(w[2] * inv, w[3] * inv),
                                ptx::pack_bf16x2(w[4] * inv, w[5] * inv),
                                ptx::pack_bf16x2(w[6] * inv, w[7] * inv),
                                ptx::pack_bf16x2(w[8] * inv, w[9] * inv),
                                ptx::pack_bf16x2(w[10] * inv, w[11] * inv),
                                ptx::pack_bf16x2(w[12] * inv, w[13] * inv),
                                ptx::pack_bf16x2(w[14] * inv, w[15] * inv));
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(P.out + ((size_t)u.b * P.R + rg) * P.d_v + d0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(ptx::pack_bf16x2(v[8 * q] * inv, v[8 * q + 1] * inv),
                                  ptx::pack_bf16x2(v[8 * q + 2] * inv, v[8 * q + 3] * inv),
                                  ptx::pack_bf16x2(v[8 * q + 4] * inv, v[8 * q + 5] * inv),
                                  ptx::pack_bf16x2(v[8 * q + 6] * inv, v[8 * q + 7] * inv));
          }
        }
      }
      if (row_valid && quarter == 0) {
        if (partial)
          P.ws_lse[ws_row] = lv;
        else
          P.lse[(size_t)u.b * P.R + rg] = lv;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_remote(o_free_l);
      gt += n;
      ++u_idx;
    }
  }

  // ---- teardown: both CTAs finished with TMEM and all UMMAs drained
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace mla

// page_kernel.cuh -- page-resident sm_100a MLA decode for up to 32 query rows
// per latent KV head (e.g. 16 heads x 2 speculative queries), d_v = 512.
//
// Same computation as the other attention kernels (softmax(scale Q K^T) V with
// V = the first d_v latent dims, plus LSE; [FlashMLA (AI Wiki), "How does MLA
// differ from MHA and GQA?", "Interfaces"]).  With at most 32 query rows the
// kernel is bound by the cache read, so every 64-token page is fetched into
// shared memory once and serves both products:
//   S^T[64 tok, 32 rows]  = K_page[64 tok, 576] . Q[32 rows, 576]^T      (M = 64, 36 UMMAs)
//   O^T[128 d_j, 64 cols] += V_j^T[128 d, 64 tok] . P^T[64 cols, 64 tok]^T (M = 128, 16 UMMAs)
// The page is read K-major for QK and, through an MN-major descriptor, as V^T
// for PV.  P^T has 64 columns of which the last 32 stay zero.
//
// Memory pipeline.  A page is five load items: four 16 KB "pair slots" holding
// dims [128 j, 128 j + 128) (chunks 2j and 2j + 1, so that the M = 128 V^T
// operand of block j has a fixed 8 KB stride between its two 64-dim halves)
// and one 8 KB "rope slot" holding dims 512..575.  The two rings are as deep as
// shared memory allows (9 pair + 3 rope slots, 2.25 pages).  Pair slot j of a
// page is released as soon as PV block j has consumed it, the rope slot right
// after QK, so the loads of the next pages start while this one is still being
// multiplied.  QK of page k + 1 is issued ahead of PV of page k for the pair
// slots that have already landed.
//
// TMEM: an M = 64 accumulator puts token t in lane 32 (t / 16) + t % 16, so
// lanes 0..15 of the softmax warps receive the 64 tokens of a page (and share
// each token's R columns with lanes 16..31); the M = 128 O^T accumulators put
// output dim d in lane d % 128 of block d / 128.
//
// Roles (warps): 0 loader (and Q), 1 MMA issuer + TMEM owner, 2..9 two softmax
// / epilogue warpgroups, 10 second loader.
#pragma once
#include "decode_kernel.cuh"

namespace mla {

struct PageCfg {
  static constexpr int kRows = 32;  // query rows per CTA: N of QK, columns of P^T
  static constexpr int kSmWarps = 8;                      // two softmax warpgroups
  static constexpr int kSmThreads = 32 * kSmWarps;
  static constexpr int kWgCols = kRows / 2;               // S^T columns per warpgroup
  static constexpr int kCols = kRows / 4;                 // S^T columns per softmax thread
  static constexpr int kChunk = kPage * 128;              // [64 tok][64 d] bf16 = 8 KB
  static constexpr int kPairBytes = 2 * kChunk;           // chunks 2j, 2j + 1
  static constexpr int kQBytes = kNumChunks * kRows * 128;
  static constexpr int kPBuf = kPage * 128;               // P^T [64 tok][64 cols] bf16
  static constexpr int kNPBuf = 2;
  static constexpr int kCtrlBytes = 4096;
  static constexpr int kRopeSlots = 3;
  static constexpr int kFixed =
      kQBytes + kNPBuf * kPBuf + kRopeSlots * kChunk + kCtrlBytes + 1024;
  static constexpr int kPairSlots = (232448 - kFixed) / kPairBytes;
  static_assert(kPairSlots == 9, "pair ring depth");
  // pairs of page k + 1 that fit while page k holds its four
  static constexpr int kAheadPairs = kPairSlots - 4 < 4 ? kPairSlots - 4 : 4;
  static constexpr int kVBlocks = 4;                      // M = 128 blocks of O^T (512 dims)
  // shared memory layout (1 KB aligned operands)
  static constexpr int kQOff = 0;
  static constexpr int kPairOff = kQOff + kQBytes;
  static constexpr int kRopeOff = kPairOff + kPairSlots * kPairBytes;
  static constexpr int kPOff = kRopeOff + kRopeSlots * kChunk;
  static constexpr int kBarOff = kPOff + kNPBuf * kPBuf;
  static constexpr int kSmemBytes = kBarOff + kCtrlBytes + 1024;
  static_assert(kSmemBytes <= 232448, "page kernel shared memory above the sm_100 limit");
  // TMEM columns
  static constexpr int kSCol = 0;           // S^T buffers [0, R) and [R, 2R)
  static constexpr int kOCol = 2 * kRows;   // O^T block j at kOCol + 64 j (512 dims)
  static constexpr int kTmemCols = 512;
  static_assert(kOCol + 64 * kVBlocks <= kTmemCols, "TMEM columns");
  static constexpr int kThreads = 32 * (2 + kSmWarps + 1);  // loader, MMA, softmax, loader
};

struct __align__(8) PageCtrl {
  uint64_t pair_full[9], pair_empty[9];
  uint64_t rope_full[3], rope_empty[3];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_free, drain;
  uint32_t tmem_base, pad;
  float red[4][64];       // per-warp column reductions
  float m[64];            // per-column reference max (log2 domain)
  float alpha[64];        // per-column rescale factor, then 1/l in the epilogue
  int lim[64];            // per-column visible-token limit of the current unit
};
static_assert(sizeof(PageCtrl) <= 4096, "page control block too large");

// -------------------------------------------------------------------- kernel

__global__ void __launch_bounds__(PageCfg::kThreads, 1)
    mla_page_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_kv, const DecodeParams P) {
  using Cfg = PageCfg;
  constexpr int kRows = Cfg::kRows;
  constexpr int kCols = Cfg::kCols;
  constexpr int kChunk = Cfg::kChunk;
  constexpr int kPairBytes = Cfg::kPairBytes;
  constexpr int kNPair = Cfg::kPairSlots;
  constexpr int kNRope = Cfg::kRopeSlots;
  constexpr int kNPBuf = Cfg::kNPBuf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + Cfg::kQOff;
  uint8_t* sPair = smem + Cfg::kPairOff;
  uint8_t* sRope = smem + Cfg::kRopeOff;
  uint8_t* sP = smem + Cfg::kPOff;
  PageCtrl& C = *reinterpret_cast<PageCtrl*>(smem + Cfg::kBarOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int part = blockIdx.x / P.n_groups;
  const int grp = blockIdx.x % P.n_groups;

  ptx::grid_dep_wait();    // the planner's metadata is complete
  ptx::grid_dep_launch();  // the combine grid may be scheduled as CTAs retire
  const int32_t* meta = P.metadata + part * kMetaInts;
  if (meta[0] > meta[2]) return;  // empty part

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNPair; ++i) {
      ptx::mbar_init(&C.pair_full[i], 1);
      ptx::mbar_init(&C.pair_empty[i], 1);
    }
    for (int i = 0; i < kNRope; ++i) {
      ptx::mbar_init(&C.rope_full[i], 1);
      ptx::mbar_init(&C.rope_empty[i], 1);
    }
    ptx::mbar_init(&C.q_full, 1);
    ptx::mbar_init(&C.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&C.s_full[i], 1);
      ptx::mbar_init(&C.s_empty[i], Cfg::kSmWarps);  // one arrival per softmax warp
      ptx::mbar_init(&C.p_full[i], Cfg::kSmWarps);
      ptx::mbar_init(&C.p_empty[i], 1);
    }
    ptx::mbar_init(&C.o_free, Cfg::kSmWarps);
    ptx::mbar_init(&C.drain, 1);
    ptx::fence_mbar_init();
  }
  // P^T columns kRows..63 are never written: zero every buffer once
  for (int i = threadIdx.x; i < kNPBuf * Cfg::kPBuf / 16; i += Cfg::kThreads)
    reinterpret_cast<uint4*>(sP)[i] = make_uint4(0, 0, 0, 0);
  ptx::fence_proxy_async_smem();
  if (warp == 1) {
    ptx::tmem_alloc(&C.tmem_base, Cfg::kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_kv);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = C.tmem_base;

  UnitIter it;
  it.init(meta);
  // Pages [2 lo, min(2 hi, pages of the sequence)) of a unit; none for L = 0.
  auto page_range = [&](const Unit& u, int& p0, int& np) {
    const int npg = (u.L + kPage - 1) / kPage;  // <= max_pages
    p0 = 2 * u.lo;
    const int p1 = 2 * u.hi < npg ? 2 * u.hi : npg;
    np = p1 > p0 ? p1 - p0 : 0;
  };
  auto warp_wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, site));
  };

  if (warp == 0 || warp == 2 + Cfg::kSmWarps) {
    // ============================== loaders ==============================
    // Load items in order: per page its four pair slots, then its rope slot;
    // item i is issued by loader (i % 2), which waits for the slot first.
    const int role = warp == 0 ? 0 : 1;
    uint32_t pair_it = 0, rope_it = 0, item = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    while (ok && it.next<kDense>(P, u)) {
      if (role == 0) {
        if (!warp_wait(&C.q_empty, (u_idx & 1) ^ 1, 0x81)) break;
        if (ptx::elect_one_sync()) {
          ptx::mbar_arrive_expect_tx(&C.q_full, Cfg::kQBytes);
          ptx::tma_load_3d(sQ, &tm_q, &C.q_full, 0, u.b * P.R + grp * kRows, 0);
        }
        __syncwarp();
      }
      int p0, np;
      page_range(u, p0, np);
      for (int k = 0; k < np && ok; ++k) {
        const int blk =
            clamp_block(P.block_table[(size_t)u.b * P.max_pages + p0 + k], P.num_blocks);
        if (P.trace && role == 0) trace_page(P, u.b, p0 + k, blk, 3);  // a slot serves K and V
        for (int j = 0; j < 5 && ok; ++j) {
          const bool mine = static_cast<int>(item++ & 1) == role;
          if (j < 4) {
            const uint32_t idx = pair_it++;
            if (!mine) continue;
            const int s = idx % kNPair;
            if (!warp_wait(&C.pair_empty[s], ((idx / kNPair) & 1) ^ 1, 0x82)) {
              ok = false;
              break;
            }
            if (ptx::elect_one_sync()) {
              uint8_t* dst = sPair + s * kPairBytes;
              ptx::mbar_arrive_expect_tx(&C.pair_full[s], kPairBytes);
              ptx::tma_load_2d(dst, &tm_kv, &C.pair_full[s], 128 * j, blk * kPage);
              ptx::tma_load_2d(dst + kChunk, &tm_kv, &C.pair_full[s], 128 * j + 64, blk * kPage);
            }
            __syncwarp();
          } else {
            const uint32_t idx = rope_it++;
            if (!mine) continue;
            const int s = idx % kNRope;
            if (!warp_wait(&C.rope_empty[s], ((idx / kNRope) & 1) ^ 1, 0x83)) {
              ok = false;
              break;
            }
            if (ptx::elect_one_sync()) {
              ptx::mbar_arrive_expect_tx(&C.rope_full[s], kChunk);
              ptx::tma_load_2d(sRope + s * kChunk, &tm_kv, &C.rope_full[s], kNope, blk * kPage);
            }
            __syncwarp();
          }
        }
      }
      ++u_idx;
    }
    // No TMA write left in flight: the final load of each slot has landed (a
    // wait on a load the other loader issued returns as soon as it lands too).
    for (int i = 0; i < kNPair && i < static_cast<int>(pair_it); ++i) {
      const uint32_t last = pair_it - 1 - i;
      ptx::mbar_wait(&C.pair_full[last % kNPair], (last / kNPair) & 1, 0x84);
    }
    for (int i = 0; i < kNRope && i < static_cast<int>(rope_it); ++i) {
      const uint32_t last = rope_it - 1 - i;
      ptx::mbar_wait(&C.rope_full[last % kNRope], (last / kNRope) & 1, 0x85);
    }
    if (role == 0 && u_idx > 0) ptx::mbar_wait(&C.q_full, (u_idx - 1) & 1, 0x86);
    __syncwarp();
  } else if (warp == 1) {
    // ============================== MMA issuer ==============================
    const uint32_t idesc_qk = ptx::idesc_bf16_f32(64, kRows, 0, 0);
    const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, 64, 1, 1);
    const ptx::DescWords dpair = ptx::desc_words(ptx::smem_u32(sPair), 16, 1024, ptx::kLayoutSW128);
    const ptx::DescWords drope = ptx::desc_words(ptx::smem_u32(sRope), 16, 1024, ptx::kLayoutSW128);
    const ptx::DescWords dq = ptx::desc_words(ptx::smem_u32(sQ), 16, 1024, ptx::kLayoutSW128);
    // V^T: MN-major, 64-dim halves one chunk apart, 8-token groups 1 KB apart
    const ptx::DescWords dvp =
        ptx::desc_words(ptx::smem_u32(sPair), kChunk, 1024, ptx::kLayoutSW128);
    const ptx::DescWords dp = ptx::desc_words(ptx::smem_u32(sP), 16, 1024, ptx::kLayoutSW128);
    uint32_t pg_it = 0, gt = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    // 8 UMMAs: S^T += K chunks 2j, 2j + 1 of page gi . Q^T
    auto qk_pair = [&](uint32_t gi, int j, uint32_t d_tmem, bool first) {
      const uint32_t idx = gi * 4 + j;
      const uint32_t a0 = dpair.lo + (((idx % kNPair) * kPairBytes) >> 4);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_f16_ss_w(d_tmem, a0 + ((h * kChunk + kk * 32) >> 4), dpair.hi,
                             dq.lo + (((2 * j + h) * (kRows * 128) + kk * 32) >> 4), dq.hi,
                             idesc_qk, (first && h == 0 && kk == 0) ? 0u : 1u);
    };
    // 4 UMMAs: S^T += K chunk 8 (dims 512..575) of page gi . Q^T
    auto qk_rope = [&](uint32_t gi, uint32_t d_tmem) {
      const uint32_t a0 = drope.lo + (((gi % kNRope) * kChunk) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        ptx::umma_f16_ss_w(d_tmem, a0 + ((kk * 32) >> 4), drope.hi,
                           dq.lo + ((8 * (kRows * 128) + kk * 32) >> 4), dq.hi, idesc_qk, 1u);
    };
    auto pair_landed = [&](uint32_t gi, int j) -> bool {
      const uint32_t idx = gi * 4 + j;
      return __all_sync(0xffffffffu,
                        ptx::mbar_test(&C.pair_full[idx % kNPair], (idx / kNPair) & 1));
    };
    while (ok && it.next<kDense>(P, u)) {
      if (!warp_wait(&C.q_full, u_idx & 1, 0x94)) break;
      ptx::tc_fence_after();
      int p0, np;
      page_range(u, p0, np);
      const uint32_t g0 = gt, it0 = pg_it;
      int ahead = 0;  // pairs of the current page issued during the previous page
      for (int k = 0; k < np && ok; ++k) {
        const uint32_t g = g0 + k, gi = it0 + k;
        const int sb = g & 1;
        const uint32_t d_s = tmem + Cfg::kSCol + kRows * sb;
        // ---- QK(k): the pairs not issued ahead, then the rope chunk
        if (ahead == 0 && !warp_wait(&C.s_empty[sb], ((g >> 1) & 1) ^ 1, 0x92)) {
          ok = false;
          break;
        }
        for (int j = ahead; j < 4 && ok; ++j) {
          const uint32_t idx = gi * 4 + j;
          if (!warp_wait(&C.pair_full[idx % kNPair], (idx / kNPair) & 1, 0x91)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          if (ptx::elect_one_sync()) qk_pair(gi, j, d_s, j == 0);
          __syncwarp();
        }
        if (!ok) break;
        if (!warp_wait(&C.rope_full[gi % kNRope], (gi / kNRope) & 1, 0x93)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (ptx::elect_one_sync()) {
          qk_rope(gi, d_s);
          ptx::umma_commit(&C.s_full[sb]);
          ptx::umma_commit(&C.rope_empty[gi % kNRope]);  // V is dims 0..511
          if (k == np - 1) ptx::umma_commit(&C.q_empty);  // the unit's last QK reads Q
        }
        __syncwarp();
        // ---- QK(k + 1) ahead of PV(k), for the pairs that have already landed
        ahead = 0;
        if (k + 1 < np) {
          const uint32_t g1 = g + 1;
          const int sb1 = g1 & 1;
          if (!warp_wait(&C.s_empty[sb1], ((g1 >> 1) & 1) ^ 1, 0x95)) {
            ok = false;
            break;
          }
          while (ahead < Cfg::kAheadPairs && pair_landed(gi + 1, ahead)) {
            ptx::tc_fence_after();
            if (ptx::elect_one_sync())
              qk_pair(gi + 1, ahead, tmem + Cfg::kSCol + kRows * sb1, ahead == 0);
            __syncwarp();
            ++ahead;
          }
        }
        // ---- PV(k)
        if (k == 0) {
          // the previous unit's epilogue has read O
          if (!warp_wait(&C.o_free, (u_idx & 1) ^ 1, 0x96)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
        }
        const int pb = g % kNPBuf;
        if (!warp_wait(&C.p_full[pb], (g / kNPBuf) & 1, 0x97)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t b0 = dp.lo + ((pb * Cfg::kPBuf) >> 4);
#pragma unroll
        for (int j = 0; j < Cfg::kVBlocks; ++j) {
          if (ptx::elect_one_sync()) {
            const uint32_t idx = gi * 4 + j;
            const uint32_t a0 = dvp.lo + (((idx % kNPair) * kPairBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              ptx::umma_f16_ss_w(tmem + Cfg::kOCol + 64 * j, a0 + ((kk * 2048) >> 4), dvp.hi,
                                 b0 + ((kk * 2048) >> 4), dp.hi, idesc_pv,
                                 (k == 0 && kk == 0) ? 0u : 1u);
            ptx::umma_commit(&C.pair_empty[idx % kNPair]);  // block j's pair slot is done
            if (j == Cfg::kVBlocks - 1) ptx::umma_commit(&C.p_empty[pb]);
          }
          __syncwarp();
        }
      }
      if (ok && np == 0) {
        if (!warp_wait(&C.o_free, (u_idx & 1) ^ 1, 0x98)) break;
        if (ptx::elect_one_sync()) ptx::umma_commit(&C.q_empty);
        __syncwarp();
      }
      pg_it += np;
      gt += np;
      ++u_idx;
    }
    if (ptx::elect_one_sync()) ptx::umma_commit(&C.drain);
    __syncwarp();
    ptx::mbar_wait(&C.drain, 0, 0x99);
    __syncwarp();
  } else {
    // ======================= softmax / epilogue (warps 2..9) =======================
    // Two warpgroups; warpgroup wg takes the query columns [wg R/2, wg R/2 + R/2).
    // Lanes 0..15 of each warp receive the S^T rows of 16 tokens; lane l and
    // lane l + 16 then share token 16 wq + l, lane l taking the first R/4 of
    // the warpgroup's columns and lane l + 16 the other R/4 (by shuffles).
    constexpr int kWgCols = Cfg::kWgCols;
    const int wq = warp & 3;                   // TMEM lane quarter
    const int wg = (warp - 2) >> 2;            // warpgroup
    const int wt = threadIdx.x - 64;           // 0..255
    const int half = lane >> 4;                // column half of this lane
    const int cw = kWgCols * wg;               // the warpgroup's first column
    const int cb = cw + kCols * half;          // this thread's first column
    const int t = 16 * wq + (lane & 15);       // token within the page
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    constexpr int kSm = Cfg::kSmThreads;
    // kWgCols consecutive TMEM columns of this thread's lane
    auto tmem_ld_wg = [&](uint32_t a, float* v) {
      if constexpr (kWgCols == 16) {
        ptx::tmem_ld16(a, v);
        ptx::tmem_ld_wait_regs16(v);
      } else {
        ptx::tmem_ld32(a, v);
        ptx::tmem_ld_wait_regs(v);
      }
    };
    auto tmem_st_wg = [&](uint32_t a, const float* v) {
      if constexpr (kWgCols == 16)
        ptx::tmem_st16(a, v);
      else
        ptx::tmem_st32(a, v);
    };
    uint32_t gt = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    while (ok && it.next<kDense>(P, u)) {
      int p0, np;
      page_range(u, p0, np);
      if (wt < kRows) {
        const int rg = grp * kRows + wt;
        int lim = 0;
        if (rg < P.R) {
          lim = P.causal ? u.L - P.s_q + 1 + rg / P.h_q : u.L;
          lim = lim < 0 ? 0 : lim;
        }
        C.lim[wt] = lim;
        C.m[wt] = -INFINITY;
      }
      ptx::named_bar_sync(1, kSm);
      int min_lim = 1 << 30;
      for (int c = 0; c < kRows; ++c)
        if (grp * kRows + c < P.R && C.lim[c] < min_lim) min_lim = C.lim[c];
      float lsum[kCols];
#pragma unroll
      for (int i = 0; i < kCols; ++i) lsum[i] = 0.f;

      for (int k = 0; k < np && ok; ++k) {
        const uint32_t g = gt + k;
        const int sb = g & 1;
        if (!wg_wait(&C.s_full[sb], (g >> 1) & 1, 0xA1, 3, kSm)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float x[kCols];
        {
          float raw[kWgCols];
          tmem_ld_wg(lane_addr + Cfg::kSCol + kRows * sb + cw, raw);
#pragma unroll
          for (int i = 0; i < kCols; ++i) {
            const float hi = __shfl_sync(0xffffffffu, raw[kCols + i], lane & 15);
            x[i] = half ? hi : raw[i];
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&C.s_empty[sb]);

        const int T = (p0 + k) * kPage + t;
        const bool need_mask = (p0 + k + 1) * kPage > min_lim;
        int need = 0;
#pragma unroll
        for (int i = 0; i < kCols; ++i) {
          float v = x[i] * P.scale_log2;
          if (need_mask && T >= C.lim[cb + i]) v = -INFINITY;
          x[i] = v;
          need |= (v > C.m[cb + i] + cfg::kRescaleThreshold);
        }
        uint32_t any_need;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.ne.b32 p, %1, 0;\n\t"
            "bar.red.or.pred q, 2, %2, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(any_need)
            : "r"(need), "n"(kSm));
        if (any_need) {
          // raise the reference max to this page's exact column max
#pragma unroll
          for (int i = 0; i < kCols; ++i) {
            float v = x[i];
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if ((lane & 15) == 0) C.red[wq][cb + i] = v;
          }
          ptx::named_bar_sync(1, kSm);
          if (wt < kRows) {
            const float tm =
                fmaxf(fmaxf(C.red[0][wt], C.red[1][wt]), fmaxf(C.red[2][wt], C.red[3][wt]));
            const float mo = C.m[wt];
            const float mn = fmaxf(mo, tm);
            C.alpha[wt] = (mn == -INFINITY) ? 1.f : ex2(mo - mn);
            C.m[wt] = mn;
          }
          ptx::named_bar_sync(1, kSm);
#pragma unroll
          for (int i = 0; i < kCols; ++i) lsum[i] *= C.alpha[cb + i];
          if (k > 0) {
            // O holds the sum through PV(g - 1): wait for it, then rescale this
            // dim lane's columns of the warpgroup in every block
            const uint32_t gp = g - 1;
            if (!wg_wait(&C.p_empty[gp % kNPBuf], (gp / kNPBuf) & 1, 0xA2, 3, kSm)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
#pragma unroll 1
            for (int j = 0; j < Cfg::kVBlocks; ++j) {
              float o[kWgCols];
              const uint32_t a = lane_addr + Cfg::kOCol + 64 * j + cw;
              tmem_ld_wg(a, o);
#pragma unroll
              for (int c = 0; c < kWgCols; ++c) o[c] *= C.alpha[cw + c];
              tmem_st_wg(a, o);
            }
            ptx::tmem_st_wait();
          }
        }
        // P buffer free once PV(g - kNPBuf) completed
        const int pb = g % kNPBuf;
        if (!wg_wait(&C.p_empty[pb], ((g / kNPBuf) & 1) ^ 1, 0xA3, 3, kSm)) {
          ok = false;
          break;
        }
        {
          uint8_t* prow = sP + pb * Cfg::kPBuf + t * 128;
#pragma unroll
          for (int uu = 0; uu < kCols / 8; ++uu) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * uu + 2 * e;
              const volatile float* mv = &C.m[cb + i];
              const float m0 = mv[0], m1 = mv[1];
              const float q0 = (x[i] == -INFINITY) ? 0.f : ex2(x[i] - m0);
              const float q1 = (x[i + 1] == -INFINITY) ? 0.f : ex2(x[i + 1] - m1);
              pk[e] = ptx::pack_bf16x2(q0, q1);
              lsum[i] += q0;
              lsum[i + 1] += q1;
            }
            const int unit = cb / 8 + uu;  // 16-byte unit = columns 8 unit .. 8 unit + 7
            *reinterpret_cast<uint4*>(prow + ((unit ^ (t & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&C.p_full[pb]);
      }
      if (!ok) break;

      // ---- epilogue: l = column sums over the page tokens
#pragma unroll
      for (int i = 0; i < kCols; ++i) {
        float v = lsum[i];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((lane & 15) == 0) C.red[wq][cb + i] = v;
      }
      ptx::named_bar_sync(1, kSm);
      const bool partial = P.always_partial || u.nsplit > 1;
      const int ws_row0 =
          ((P.ws_base ? P.ws_base[u.b] : P.num_splits[u.b]) + u.split) * P.R + grp * kRows;
      const int rows_here = min(kRows, P.R - grp * kRows);
      if (wt < kRows) {
        const float l = (C.red[0][wt] + C.red[1][wt]) + (C.red[2][wt] + C.red[3][wt]);
        C.alpha[wt] = l > 0.f ? 1.0f / l : 0.f;  // reused as 1/l (0: empty row)
        if (wt < rows_here) {
          const float lv = l > 0.f ? (C.m[wt] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
          if (partial)
            P.ws_lse[ws_row0 + wt] = lv;
          else
            P.lse[(size_t)u.b * P.R + grp * kRows + wt] = lv;
        }
      }
      ptx::named_bar_sync(1, kSm);
      if (np > 0) {
        const uint32_t glast = gt + np - 1;
        if (!wg_wait(&C.p_empty[glast % kNPBuf], (glast / kNPBuf) & 1, 0xA4, 3, kSm)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
      }
      const size_t row_first = partial ? (size_t)ws_row0 : (size_t)u.b * P.R + grp * kRows;
#pragma unroll 1
      for (int j = 0; j < Cfg::kVBlocks; ++j) {
        const int d = 128 * j + 32 * wq + lane;  // this thread's TMEM lane = output dim
        float o[kWgCols];
        if (np > 0) tmem_ld_wg(lane_addr + Cfg::kOCol + 64 * j + cw, o);
        if (d < P.d_v) {
          // consecutive lanes write consecutive dims of one row at a time
          const size_t e0 = (row_first + cw) * P.d_v + d;
          float* wo = P.ws_o + e0;
          __nv_bfloat16* bo = P.out + e0;
#pragma unroll
          for (int c = 0; c < kWgCols; ++c) {
            if (cw + c < rows_here) {
              const float a = C.alpha[cw + c];
              const float v = (np > 0 && a != 0.f) ? o[c] * a : 0.f;
              if (partial)
                *wo = v;
              else
                *bo = __float2bfloat16_rn(v);
            }
            wo += P.d_v;
            bo += P.d_v;
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&C.o_free);
      ptx::named_bar_sync(1, kSm);  // C.alpha / C.red / C.lim reusable
      gt += np;
      ++u_idx;
    }
  }

  // ---- teardown: the MMA pipe has drained; release TMEM
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace mla

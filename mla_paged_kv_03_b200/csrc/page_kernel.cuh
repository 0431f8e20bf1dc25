// page_kernel.cuh -- page-resident sm_100a MLA decode for up to 32 query rows
// per latent KV head (e.g. 16 heads x 2 speculative queries), d_v = 512.
//
// Same computation as decode_kernel.cuh (softmax(scale Q K^T) V with V = the
// first d_v latent dims, plus LSE; [FlashMLA (AI Wiki), "How does MLA differ
// from MHA and GQA?", "Interfaces"]).  With so few query rows the kernel is
// bound by the cache read, so every 64-token page is fetched into shared
// memory once, by one 72 KB TMA box, and serves both products:
//   S^T[64 tok, 32 rows]   = K_page[64 tok, 576] . Q[32 rows, 576]^T      (M = 64, 36 UMMAs)
//   O^T[128 d_j, 64 cols] += V_j^T[128 d, 64 tok] . P^T[64 cols, 64 tok]^T (M = 128, 16 UMMAs)
// The page is read K-major for QK and, through an MN-major descriptor, as V^T
// for PV.  P^T has 64 columns of which the last 32 stay zero.  Two page slots
// alternate: while page k is multiplied, page k + 1 is loaded.
//
// TMEM: an M = 64 accumulator puts token t in lane 32 (t / 16) + t % 16, so
// lanes 0..15 of the softmax warps receive the 64 tokens of a page (and share
// each token's 32 columns with lanes 16..31); the M = 128 O^T accumulators
// put output dim d in lane d.
//
// Roles (warps): 0 loader (Q, pages), 1 MMA issuer + TMEM owner,
// 2..5 softmax / epilogue.
#pragma once
#include "decode_kernel.cuh"

namespace mla {

namespace gcfg {
constexpr int kRows = 32;                              // query rows per CTA (N of QK)
constexpr int kChunk = kPage * 128;                    // [64 tok][64 d] bf16 = 8 KB
constexpr int kPageBytes = kNumChunks * kChunk;        // 73728
constexpr int kQBytes = kNumChunks * kRows * 128;      // 36864: [9 chunks][32 rows][64 d]
constexpr int kPBytes = kPage * 128;                   // P^T [64 tok][64 cols] bf16
#ifndef MLA_PAGE_SLOTS
#define MLA_PAGE_SLOTS 2
#endif
constexpr int kSlots = MLA_PAGE_SLOTS;
constexpr int kQOff = 0;
constexpr int kSlotOff = kQOff + kQBytes;
constexpr int kPOff = kSlotOff + kSlots * kPageBytes;
constexpr int kBarOff = kPOff + 2 * kPBytes;
constexpr int kMiscBytes = 2048;
constexpr int kSmemBytes = kBarOff + kMiscBytes + 1024;
constexpr int kTmemCols = 512;
constexpr int kSCol = 0;   // S^T buffers: columns [0, 32) and [32, 64)
constexpr int kOCol = 64;  // O^T slice j (128 dims): columns 64 + 64 j
constexpr int kThreads = 192;
}  // namespace gcfg
static_assert(gcfg::kSmemBytes <= 232448, "page kernel shared memory above the sm_100 limit");
static_assert(gcfg::kSlotOff % 1024 == 0 && gcfg::kPOff % 1024 == 0, "1 KB aligned operands");

struct __align__(8) PageCtrl {
  uint64_t slot_full[gcfg::kSlots], slot_empty[gcfg::kSlots];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_free, drain;
  uint32_t tmem_base, pad;
  float red[4][32];  // per-warp column reductions
  float m[32];       // per-column reference max (log2 domain)
  float alpha[32];   // per-column rescale factor, then 1/l in the epilogue
  int lim[32];       // per-column visible-token limit of the current unit
};
static_assert(sizeof(PageCtrl) <= gcfg::kMiscBytes, "page control block too large");

__global__ void __launch_bounds__(gcfg::kThreads, 1)
    mla_page_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_page, const DecodeParams P) {
  using namespace gcfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kQOff;
  uint8_t* sSlot = smem + kSlotOff;
  uint8_t* sP = smem + kPOff;
  PageCtrl& C = *reinterpret_cast<PageCtrl*>(smem + kBarOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int part = blockIdx.x;

  ptx::grid_dep_wait();    // the planner's metadata is complete
  ptx::grid_dep_launch();  // the combine grid may be scheduled as CTAs retire
  const int32_t* meta = P.metadata + part * kMetaInts;
  if (meta[0] > meta[2]) return;  // empty part

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      ptx::mbar_init(&C.slot_full[i], 1);
      ptx::mbar_init(&C.slot_empty[i], 1);
    }
    ptx::mbar_init(&C.q_full, 1);
    ptx::mbar_init(&C.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&C.s_full[i], 1);
      ptx::mbar_init(&C.s_empty[i], 4);  // one arrival per softmax warp
      ptx::mbar_init(&C.p_full[i], 4);
      ptx::mbar_init(&C.p_empty[i], 1);
    }
    ptx::mbar_init(&C.o_free, 4);
    ptx::mbar_init(&C.drain, 1);
    ptx::fence_mbar_init();
  }
  // P^T columns 32..63 are never written: zero both buffers once
  for (int i = threadIdx.x; i < 2 * kPBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(sP)[i] = make_uint4(0, 0, 0, 0);
  ptx::fence_proxy_async_smem();
  if (warp == 1) {
    ptx::tmem_alloc(&C.tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_page);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = C.tmem_base;

  UnitIter it;
  it.init(meta);
  // Pages [2 lo, min(2 hi, pages of the sequence)) of a unit; none for L = 0.
  auto page_range = [&](const Unit& u, int& p0, int& np) {
    int npg = (u.L + kPage - 1) / kPage;
    npg = npg < P.max_pages ? npg : P.max_pages;
    p0 = 2 * u.lo;
    const int p1 = 2 * u.hi < npg ? 2 * u.hi : npg;
    np = p1 > p0 ? p1 - p0 : 0;
  };
  auto warp_wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, site));
  };

  if (warp == 0) {
    // ============================== loader ==============================
    uint32_t pg_it = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    while (ok && it.next<kDense>(P, u)) {
      if (!warp_wait(&C.q_empty, (u_idx & 1) ^ 1, 0x81)) break;
      if (ptx::elect_one_sync()) {
        ptx::mbar_arrive_expect_tx(&C.q_full, kQBytes);
        ptx::tma_load_3d(sQ, &tm_q, &C.q_full, 0, u.b * P.R, 0);
      }
      __syncwarp();
      int p0, np;
      page_range(u, p0, np);
      for (int k = 0; k < np && ok; ++k) {
        const int slot = pg_it % kSlots;
        const uint32_t round = pg_it / kSlots;
        ++pg_it;
        if (!warp_wait(&C.slot_empty[slot], (round & 1) ^ 1, 0x82)) {
          ok = false;
          break;
        }
        const int blk =
            clamp_block(P.block_table[(size_t)u.b * P.max_pages + p0 + k], P.num_blocks);
        if (P.trace) trace_page(P, u.b, p0 + k, blk, 3);  // the slot serves K and V
        if (ptx::elect_one_sync()) {
          ptx::mbar_arrive_expect_tx(&C.slot_full[slot], kPageBytes);
          ptx::tma_load_3d(sSlot + slot * kPageBytes, &tm_page, &C.slot_full[slot], 0,
                           blk * kPage, 0);
        }
        __syncwarp();
      }
      ++u_idx;
    }
    // no TMA write left in flight: the final load of each slot has landed
    for (int i = 0; i < kSlots && i < static_cast<int>(pg_it); ++i) {
      const uint32_t last = pg_it - 1 - i;
      ptx::mbar_wait(&C.slot_full[last % kSlots], (last / kSlots) & 1, 0x83);
    }
    if (u_idx > 0) ptx::mbar_wait(&C.q_full, (u_idx - 1) & 1, 0x84);
    __syncwarp();
  } else if (warp == 1) {
    // ============================== MMA issuer ==============================
    const uint32_t idesc_qk = ptx::idesc_bf16_f32(64, kRows, 0, 0);
    const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, 64, 1, 1);
    const ptx::DescWords dk = ptx::desc_words(ptx::smem_u32(sSlot), 16, 1024, ptx::kLayoutSW128);
    const ptx::DescWords dq = ptx::desc_words(ptx::smem_u32(sQ), 16, 1024, ptx::kLayoutSW128);
    // V^T: MN-major, 64-dim blocks one chunk apart, 8-token groups 1 KB apart
    const ptx::DescWords dv = ptx::desc_words(ptx::smem_u32(sSlot), kChunk, 1024, ptx::kLayoutSW128);
    const ptx::DescWords dp = ptx::desc_words(ptx::smem_u32(sP), 16, 1024, ptx::kLayoutSW128);
    uint32_t pg_it = 0, gt = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    auto do_qk = [&](uint32_t g, int slot, uint32_t round) -> bool {
      const int sb = g & 1;
      if (!warp_wait(&C.s_empty[sb], ((g >> 1) & 1) ^ 1, 0x91)) return false;
      if (!warp_wait(&C.slot_full[slot], round & 1, 0x92)) return false;
      ptx::tc_fence_after();
      if (ptx::elect_one_sync()) {
        const uint32_t d_tmem = tmem + kSCol + 32 * sb;
        const uint32_t a0 = dk.lo + ((slot * kPageBytes) >> 4);
#pragma unroll
        for (int c = 0; c < kNumChunks; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16_ss_w(d_tmem, a0 + ((c * kChunk + kk * 32) >> 4), dk.hi,
                               dq.lo + ((c * (kRows * 128) + kk * 32) >> 4), dq.hi, idesc_qk,
                               (c | kk) ? 1u : 0u);
        ptx::umma_commit(&C.s_full[sb]);
      }
      __syncwarp();
      return true;
    };
    auto do_pv = [&](uint32_t g, int slot, bool first_of_unit) -> bool {
      const int pb = g & 1;
      if (!warp_wait(&C.p_full[pb], (g >> 1) & 1, 0x93)) return false;
      ptx::tc_fence_after();
      if (ptx::elect_one_sync()) {
        const uint32_t a0 = dv.lo + ((slot * kPageBytes) >> 4);
        const uint32_t b0 = dp.lo + ((pb * kPBytes) >> 4);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16_ss_w(tmem + kOCol + 64 * j, a0 + ((2 * j * kChunk + kk * 2048) >> 4),
                               dv.hi, b0 + ((kk * 2048) >> 4), dp.hi, idesc_pv,
                               (first_of_unit && kk == 0) ? 0u : 1u);
        ptx::umma_commit(&C.slot_empty[slot]);
        ptx::umma_commit(&C.p_empty[pb]);
      }
      __syncwarp();
      return true;
    };
    while (ok && it.next<kDense>(P, u)) {
      if (!warp_wait(&C.q_full, u_idx & 1, 0x94)) break;
      ptx::tc_fence_after();
      int p0, np;
      page_range(u, p0, np);
      // the previous unit's epilogue has read O: waited once per unit, before
      // the unit's first PV (or at its end when it has no page)
      auto wait_o_free = [&]() -> bool {
        if (!warp_wait(&C.o_free, (u_idx & 1) ^ 1, 0x95)) return false;
        ptx::tc_fence_after();
        return true;
      };
      const uint32_t g0 = gt, it0 = pg_it;
      // PV(k) follows QK(k), so that a slot is released as soon as its
      // page's softmax is done and the load of page k + 2 starts early.  QK(k
      // + 1) goes in between only when page k + 1 has already landed: the
      // tensor pipe then runs it during the softmax of page k, while PV(k)
      // never waits for a load.  (Always issuing QK(k + 1) first ties PV(k),
      // and with it the slot, to page k + 1's load; measured slower.)
      bool qk_ahead = false;
      for (int k = 0; k < np && ok; ++k) {
        const uint32_t idx = it0 + k;
        if (!qk_ahead) ok = do_qk(g0 + k, idx % kSlots, idx / kSlots);
        qk_ahead = false;
        if (ok && k + 1 < np) {
          const uint32_t nx = idx + 1;
          const bool landed = ptx::mbar_test(&C.slot_full[nx % kSlots], (nx / kSlots) & 1);
          if (__all_sync(0xffffffffu, landed)) {
            ok = do_qk(g0 + k + 1, nx % kSlots, nx / kSlots);
            qk_ahead = true;
          }
        }
        if (ok && k == 0) ok = wait_o_free();
        if (ok) ok = do_pv(g0 + k, idx % kSlots, k == 0);
      }
      if (ok && np == 0) ok = wait_o_free();
      if (ok) {
        if (ptx::elect_one_sync()) ptx::umma_commit(&C.q_empty);
        __syncwarp();
      }
      pg_it += np;
      gt += np;
      ++u_idx;
    }
    if (ptx::elect_one_sync()) ptx::umma_commit(&C.drain);
    __syncwarp();
    ptx::mbar_wait(&C.drain, 0, 0x96);
    __syncwarp();
  } else {
    // ============================== softmax / epilogue ==============================
    // Lanes 0..15 of each warp receive the S^T rows of 16 tokens; lane l and
    // lane l + 16 then share token 16 wq + l, lane l taking the query columns
    // 0..15 and lane l + 16 the columns 16..31 (handed over by shuffles).
    const int wq = warp & 3;                   // TMEM lane quarter
    const int wt = threadIdx.x - 64;           // 0..127
    const int half = lane >> 4;                // column half of this lane
    const int cb = 16 * half;                  // its first column
    const int t = 16 * wq + (lane & 15);       // token within the page
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    uint32_t gt = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    while (ok && it.next<kDense>(P, u)) {
      int p0, np;
      page_range(u, p0, np);
      if (wt < 32) {
        const int rg = wt;
        int lim = 0;
        if (rg < P.R) {
          lim = P.causal ? u.L - P.s_q + 1 + rg / P.h_q : u.L;
          lim = lim < 0 ? 0 : lim;
        }
        C.lim[wt] = lim;
        C.m[wt] = -INFINITY;
      }
      ptx::named_bar_sync(1, 128);
      int min_lim = 1 << 30;
      for (int c = 0; c < 32; ++c)
        if (c < P.R && C.lim[c] < min_lim) min_lim = C.lim[c];
      float lsum[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) lsum[i] = 0.f;

      for (int k = 0; k < np && ok; ++k) {
        const uint32_t g = gt + k;
        const int sb = g & 1;
        if (!wg_wait(&C.s_full[sb], (g >> 1) & 1, 0xA1, 3)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float x[16];
        {
          float raw[32];
          ptx::tmem_ld32(lane_addr + kSCol + 32 * sb, raw);
          ptx::tmem_ld_wait_regs(raw);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float hi = __shfl_sync(0xffffffffu, raw[16 + i], lane & 15);
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
        for (int i = 0; i < 16; ++i) {
          float v = x[i] * P.scale_log2;
          if (need_mask && T >= C.lim[cb + i]) v = -INFINITY;
          x[i] = v;
          need |= (v > C.m[cb + i] + cfg::kRescaleThreshold);
        }
        uint32_t any_need;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.ne.b32 p, %1, 0;\n\t"
            "bar.red.or.pred q, 2, 128, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(any_need)
            : "r"(need));
        if (any_need) {
          // raise the reference max to this page's exact column max
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float v = x[i];
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if ((lane & 15) == 0) C.red[wq][cb + i] = v;
          }
          ptx::named_bar_sync(1, 128);
          if (wt < 32) {
            const float tm = fmaxf(fmaxf(C.red[0][wt], C.red[1][wt]), fmaxf(C.red[2][wt], C.red[3][wt]));
            const float mo = C.m[wt];
            const float mn = fmaxf(mo, tm);
            C.alpha[wt] = (mn == -INFINITY) ? 1.f : ex2(mo - mn);
            C.m[wt] = mn;
          }
          ptx::named_bar_sync(1, 128);
#pragma unroll
          for (int i = 0; i < 16; ++i) lsum[i] *= C.alpha[cb + i];
          if (k > 0) {
            // O holds the sum through PV(g - 1): wait for it, rescale this dim lane
            const uint32_t gp = g - 1;
            if (!wg_wait(&C.p_empty[gp & 1], (gp >> 1) & 1, 0xA2, 3)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            for (int j = 0; j < 4; ++j) {
              float o[32];
              const uint32_t a = lane_addr + kOCol + 64 * j;
              ptx::tmem_ld32(a, o);
              ptx::tmem_ld_wait_regs(o);
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] *= C.alpha[c];
              ptx::tmem_st32(a, o);
            }
            ptx::tmem_st_wait();
          }
        }
        // P buffer free once PV(g - 2) completed
        const int pb = g & 1;
        if (!wg_wait(&C.p_empty[pb], ((g >> 1) & 1) ^ 1, 0xA3, 3)) {
          ok = false;
          break;
        }
        {
          uint8_t* prow = sP + pb * kPBytes + t * 128;
#pragma unroll
          for (int uu = 0; uu < 2; ++uu) {
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
            const int unit = 2 * half + uu;  // 16-byte unit = columns 8 unit .. 8 unit + 7
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
      for (int i = 0; i < 16; ++i) {
        float v = lsum[i];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((lane & 15) == 0) C.red[wq][cb + i] = v;
      }
      ptx::named_bar_sync(1, 128);
      const bool partial = P.always_partial || u.nsplit > 1;
      const int ws_row0 = (P.num_splits[u.b] + u.split) * P.R;
      const int rows_here = P.R < kRows ? P.R : kRows;
      if (wt < 32) {
        const float l = (C.red[0][wt] + C.red[1][wt]) + (C.red[2][wt] + C.red[3][wt]);
        C.alpha[wt] = l > 0.f ? 1.0f / l : 0.f;  // reused as 1/l (0: empty row)
        if (wt < rows_here) {
          const float lv = l > 0.f ? (C.m[wt] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
          if (partial)
            P.ws_lse[ws_row0 + wt] = lv;
          else
            P.lse[(size_t)u.b * P.R + wt] = lv;
        }
      }
      ptx::named_bar_sync(1, 128);
      if (np > 0) {
        const uint32_t glast = gt + np - 1;
        if (!wg_wait(&C.p_empty[glast & 1], (glast >> 1) & 1, 0xA4, 3)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
      }
      const size_t row_first = partial ? (size_t)ws_row0 : (size_t)u.b * P.R;
      for (int j = 0; j < 4; ++j) {
        const int d = 128 * j + 32 * wq + lane;  // this thread's TMEM lane = output dim
        float o[32];
        if (np > 0) {
          ptx::tmem_ld32(lane_addr + kOCol + 64 * j, o);
          ptx::tmem_ld_wait_regs(o);
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < rows_here) {
            const float a = C.alpha[c];
            const float v = (np > 0 && a != 0.f) ? o[c] * a : 0.f;
            if (partial)
              P.ws_o[(row_first + c) * P.d_v + d] = v;
            else
              P.out[(row_first + c) * P.d_v + d] = __float2bfloat16_rn(v);
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&C.o_free);
      ptx::named_bar_sync(1, 128);  // C.alpha / C.red / C.lim reusable
      gt += np;
      ++u_idx;
    }
  }

  // ---- teardown: the MMA pipe has drained; release TMEM
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mla

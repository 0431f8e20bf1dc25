// pair_kernel.cuh -- 2-CTA (cta_group::2) sm_100a MLA decode for 65..128 query
// rows per latent KV head (e.g. 128 heads, s_q = 1).
//
// Same computation as decode_kernel.cuh (softmax(scale Q K^T) V with V = the
// first d_v latent dims, plus LSE; [FlashMLA (AI Wiki), "How does MLA differ
// from MHA and GQA?", "Interfaces"]), in the conventional orientation: query
// rows on the UMMA M axis.  A pair of CTAs on two SMs runs M = 128 UMMAs:
//   S[128 rows, 128 tok]  = Q[128, 576] . K_tile[128 tok, 576]^T      (N = 128)
//   O[128 rows, 128 d_j] += P[128, 128 tok] . V_j[128 tok, 128 d]^T    (N = 128, j < 4)
// Each CTA holds 64 of the rows (its Q and P), one of the tile's two 64-token
// pages for QK, and one 64-dim half of each 128-dim V slice for PV; the tensor
// cores read the partner's halves directly.  Per 128-token tile each CTA moves
// 136 KB into shared memory, and every UMMA reads 4 KB of operands per 32
// tensor clocks.  In each CTA's TMEM a 64-row accumulator of N columns lies in
// lanes 0..63 for columns [0, N/2) and lanes 64..127 for [N/2, N), so thread
// (lane L) of the softmax warpgroup owns row L % 64 for tokens (or output
// dims) of half L / 64.
//
// Roles (warps): 0 loader (both CTAs), 1 MMA issuer (leader CTA) and TMEM
// owner (both), 2..5 softmax / epilogue (both).
#pragma once
#include "decode_kernel.cuh"

namespace mla {

namespace pcfg {
constexpr int kRows = 64;                          // query rows per CTA
constexpr int kQBytes = kNumChunks * kRows * 128;  // 73728
constexpr int kKChunk = 64 * 128;                  // [64 tokens][64 d] bf16
constexpr int kStage = 16384;                      // ring stage
#ifndef MLA_PAIR_STAGES
#define MLA_PAIR_STAGES 7
#endif
constexpr int kNStage = MLA_PAIR_STAGES;
constexpr int kPBytes = 2 * kRows * 128;           // [64 rows][128 tokens] bf16
constexpr int kQOff = 0;
constexpr int kRingOff = kQOff + kQBytes;
constexpr int kPOff = kRingOff + kNStage * kStage;
constexpr int kBarOff = kPOff + 2 * kPBytes;
constexpr int kMiscBytes = 3072;
constexpr int kSmemBytes = kBarOff + kMiscBytes + 1024;
constexpr int kTmemCols = 512;
constexpr int kSCol = 0;    // S buffers at columns [0,64) and [64,128)
constexpr int kOCol = 128;  // O slice j (128 output dims) at columns 128 + 64 j
constexpr int kThreads = 192;
constexpr int kKStages = 5;  // K chunk pairs {0,1} {2,3} {4,5} {6,7} {8}
}  // namespace pcfg

struct __align__(8) PairCtrl {
  uint64_t full[pcfg::kNStage], empty[pcfg::kNStage];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_free, drain;
  uint32_t tmem_base, pad;
  float red[2][2][64];  // [tile parity][token half][row] partial row max
  float lred[2][64];    // [token half][row] partial row sums
};
static_assert(sizeof(PairCtrl) <= pcfg::kMiscBytes, "pair control block too large");

// Warpgroup-uniform bounded wait with cluster-scope acquire (barrier id 3).
__device__ __forceinline__ bool wg_wait_cluster(uint64_t* bar, uint32_t parity, int site) {
  const bool mine = ptx::mbar_wait_cluster(bar, parity, site);
  uint32_t all;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 3, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(all)
      : "r"(mine ? 1 : 0));
  return all != 0;
}

__global__ void __launch_bounds__(pcfg::kThreads, 1)
    mla_pair_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_kv, const DecodeParams P) {
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
  const int nv = P.d_v / 128;         // PV slices of 128 dims (4)

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
      ptx::mbar_init(&C.s_empty[i], 8);  // one arrival per softmax warp of both CTAs
      ptx::mbar_init(&C.p_full[i], 8);
      ptx::mbar_init(&C.p_empty[i], 1);
    }
    ptx::mbar_init(&C.o_free, 8);
    ptx::mbar_init(&C.drain, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&C.tmem_base, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_kv);
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

  if (warp == 0) {
    // ============================== loader (both CTAs) ==============================
    if (lane == 0) {
      uint32_t st_it = 0;
      int u_idx = 0;
      Unit u;
      bool ok = true;
      // Returns the stage buffer after waiting for it to be free; the leader
      // posts the pair's transaction bytes on its own full barrier.
      auto acquire_stage = [&](uint32_t bytes_pair, uint8_t*& dst, uint32_t& bar) -> bool {
        const int s = st_it % kNStage;
        const uint32_t round = st_it / kNStage;
        ++st_it;
        if (!ptx::mbar_wait_cluster(&C.empty[s], (round & 1) ^ 1, 0x41)) return false;
        if (leader) ptx::mbar_arrive_expect_tx(&C.full[s], bytes_pair);
        dst = sRing + s * kStage;
        bar = leader_addr(&C.full[s]);
        return true;
      };
      auto page_block = [&](const Unit& un, int page, int fallback_page) -> int {
        int npg = (un.L + kPage - 1) / kPage;
        if (npg > P.max_pages) {
          ptx::set_error(MLA_DEVERR_BAD_INDEX, 0x45);
          npg = P.max_pages;
        }
        const int pg = page < npg ? page : fallback_page;
        const int blk = pg < npg ? P.block_table[(size_t)un.b * P.max_pages + pg] : 0;
        return clamp_block(blk, P.num_blocks);
      };
      auto load_k = [&](const Unit& un, int tile, int st) -> bool {
        const int c0 = 2 * st;
        const int nch = (c0 + 1 < kNumChunks) ? 2 : 1;
        uint8_t* dst;
        uint32_t bar;
        if (!acquire_stage(2u * nch * kKChunk, dst, bar)) return false;
        const int blk = page_block(un, 2 * tile + static_cast<int>(rank), 2 * tile);
        for (int j = 0; j < nch; ++j)
          ptx::tma_load_2d_pair(dst + j * kKChunk, &tm_kv, bar, (c0 + j) * kChunkD, blk * kPage);
        return true;
      };
      auto load_v = [&](const Unit& un, int tile, int j) -> bool {
        uint8_t* dst;
        uint32_t bar;
        if (!acquire_stage(2u * kStage, dst, bar)) return false;
        const int b0 = page_block(un, 2 * tile, 2 * tile);
        const int b1 = page_block(un, 2 * tile + 1, 2 * tile);
        const int x = (2 * j + static_cast<int>(rank)) * kChunkD;  // this CTA's 64-dim half
        ptx::tma_load_2d_pair(dst, &tm_kv, bar, x, b0 * kPage);
        ptx::tma_load_2d_pair(dst + kKChunk, &tm_kv, bar, x, b1 * kPage);
        return true;
      };
      while (ok && it.next<kDense>(P, u)) {
        if (!ptx::mbar_wait_cluster(&C.q_empty, (u_idx & 1) ^ 1, 0x42)) { ok = false; break; }
        if (leader) ptx::mbar_arrive_expect_tx(&C.q_full, 2u * kQBytes);
        const uint32_t qbar = leader_addr(&C.q_full);
        const int row0 = u.b * P.R + grp * 128 + static_cast<int>(rank) * kRows;
        for (int c = 0; c < kNumChunks; ++c)
          ptx::tma_load_2d_pair(sQ + c * (kRows * 128), &tm_q, qbar, c * kChunkD, row0);
        const int n = u.hi - u.lo;
        for (int k = 0; k < n && ok; ++k) {
          for (int st = 0; st < kKStages && ok; ++st) ok = load_k(u, u.lo + k, st);
          if (k >= 1)
            for (int j = 0; j < nv && ok; ++j) ok = load_v(u, u.lo + k - 1, j);
        }
        for (int j = 0; j < nv && ok; ++j) ok = load_v(u, u.hi - 1, j);
        ++u_idx;
      }
      // drain: wait (bounded) until the pair's last loads into each stage landed
      // (signalled on the leader's barriers; the MMA issuer consumed them).
      for (int i = 0; i < kNStage && i < static_cast<int>(st_it); ++i) {
        const uint32_t last = st_it - 1 - i;
        ptx::mbar_wait_cluster(&C.empty[last % kNStage], (last / kNStage) & 1, 0x43);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================== MMA issuer (leader) ==============================
    if (leader && lane == 0) {
      const uint32_t idesc_qk = ptx::idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t q_addr = ptx::smem_u32(sQ);
      const uint32_t ring_addr = ptx::smem_u32(sRing);
      const uint32_t p_addr = ptx::smem_u32(sP);
      uint32_t st_it = 0, gt = 0;
      int u_idx = 0;
      Unit u;
      bool ok = true;
      auto wait_stage = [&](uint32_t& addr) -> int {
        const int s = st_it % kNStage;
        const uint32_t round = st_it / kNStage;
        ++st_it;
        if (!ptx::mbar_wait_cluster(&C.full[s], round & 1, 0x51)) return -1;
        ptx::tc_fence_after();
        addr = ring_addr + s * kStage;
        return s;
      };
      const ptx::DescWords dq = ptx::desc_words(q_addr, 16, 1024, ptx::kLayoutSW128);
      const ptx::DescWords dr = ptx::desc_words(ring_addr, 16, 1024, ptx::kLayoutSW128);
      const ptx::DescWords dp = ptx::desc_words(p_addr, 16, 1024, ptx::kLayoutSW128);
      auto do_qk = [&](uint32_t g) -> bool {
        const int sb = g & 1;
        if (!ptx::mbar_wait_cluster(&C.s_empty[sb], ((g >> 1) & 1) ^ 1, 0x52)) return false;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + kSCol + sb * 64;
#pragma unroll
        for (int st = 0; st < kKStages; ++st) {
          uint32_t a0;
          const int s = wait_stage(a0);
          if (s < 0) return false;
          const uint32_t k_lo = dr.lo + ((s * kStage) >> 4);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int c = 2 * st + j;
            if (c < kNumChunks) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                ptx::umma_f16_ss_pair_w(d_tmem, dq.lo + ((c * (kRows * 128) + kk * 32) >> 4), dq.hi,
                                        k_lo + ((j * kKChunk + kk * 32) >> 4), dr.hi, idesc_qk,
                                        (c | kk) ? 1u : 0u);
            }
          }
          ptx::umma_commit_pair_mc(&C.empty[s], 0x3);
        }
        ptx::umma_commit_pair_mc(&C.s_full[sb], 0x3);
        return true;
      };
      auto do_pv = [&](uint32_t g, bool first_of_unit) -> bool {
        const int pb = g & 1;
        if (!ptx::mbar_wait_cluster(&C.p_full[pb], (g >> 1) & 1, 0x53)) return false;
        ptx::tc_fence_after();
        const uint32_t p_lo = dp.lo + ((pb * kPBytes) >> 4);
        for (int j = 0; j < nv; ++j) {
          uint32_t a0;
          const int s = wait_stage(a0);
          if (s < 0) return false;
          const uint32_t d_tmem = tmem + kOCol + j * 64;
          const uint32_t v_lo = dr.lo + ((s * kStage) >> 4);
          ptx::umma_f16_ss_pair_w(d_tmem, p_lo, dp.hi, v_lo, dr.hi, idesc_pv, first_of_unit ? 0u : 1u);
#pragma unroll
          for (int kk = 1; kk < kTileT / 16; ++kk)
            ptx::umma_f16_ss_pair_w(d_tmem, p_lo + (((kk >> 2) * kKChunk + (kk & 3) * 32) >> 4), dp.hi,
                                    v_lo + ((kk * 2048) >> 4), dr.hi, idesc_pv, 1u);
          ptx::umma_commit_pair_mc(&C.empty[s], 0x3);
        }
        ptx::umma_commit_pair_mc(&C.p_empty[pb], 0x3);
        return true;
      };
      while (ok && it.next<kDense>(P, u)) {
        if (!ptx::mbar_wait_cluster(&C.q_full, u_idx & 1, 0x54)) break;
        ptx::tc_fence_after();
        const int n = u.hi - u.lo;
        const uint32_t g0 = gt;
        for (int k = 0; k < n && ok; ++k) {
          ok = do_qk(g0 + k);
          if (ok && k == n - 1) ptx::umma_commit_pair_mc(&C.q_empty, 0x3);
          if (ok && k >= 1) {
            if (k == 1 && !ptx::mbar_wait_cluster(&C.o_free, (u_idx & 1) ^ 1, 0x55)) {
              ok = false;
              break;
            }
            ok = do_pv(g0 + k - 1, k == 1);
          }
        }
        if (ok) {
          if (n == 1 && !ptx::mbar_wait_cluster(&C.o_free, (u_idx & 1) ^ 1, 0x56)) {
            ok = false;
            break;
          }
          ok = do_pv(g0 + n - 1, n == 1);
        }
        gt += n;
        ++u_idx;
      }
      ptx::umma_commit_pair_mc(&C.drain, 0x1);
      ptx::mbar_wait_cluster(&C.drain, 0, 0x57);
    }
    __syncwarp();
  } else {
    // ============================== softmax / epilogue (both CTAs) ==============================
    const int wq = warp & 3;
    const int L = wq * 32 + lane;   // TMEM lane
    const int r = L & 63;           // row of this CTA
    const int h = L >> 6;           // token half (QK) / output-dim half (PV)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int rg = grp * 128 + static_cast<int>(rank) * kRows + r;  // row in [0, R)
    const bool row_valid = rg < P.R;
    const uint32_t s_empty_l = leader_addr(&C.s_empty[0]);
    const uint32_t p_full_l = leader_addr(&C.p_full[0]);
    const uint32_t o_free_l = leader_addr(&C.o_free);
    uint32_t gt = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    while (ok && it.next<kDense>(P, u)) {
      const int n = u.hi - u.lo;
      int lim = 0;
      if (row_valid) {
        lim = P.causal ? u.L - P.s_q + 1 + rg / P.h_q : u.L;
        lim = lim < 0 ? 0 : lim;
      }
      float m_used = -INFINITY, lsum = 0.f;
      for (int k = 0; k < n && ok; ++k) {
        const uint32_t g = gt + k;
        const int sb = g & 1;
        ok = wg_wait_cluster(&C.s_full[sb], (g >> 1) & 1, 0x61);
        if (!ok) break;
        ptx::tc_fence_after();
        float x[64];
        ptx::tmem_ld32(lane_addr + kSCol + sb * 64, x);
        ptx::tmem_ld32(lane_addr + kSCol + sb * 64 + 32, x + 32);
        ptx::tmem_ld_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(s_empty_l + sb * 8);
        const int tok0 = (u.lo + k) * kTileT + 64 * h;
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float v = (tok0 + j < lim) ? x[j] * P.scale_log2 : -INFINITY;
          x[j] = v;
          mx = fmaxf(mx, v);
        }
        C.red[g & 1][h][r] = mx;
        ptx::named_bar_sync(1, 128);
        const float row_mx = fmaxf(C.red[g & 1][0][r], C.red[g & 1][1][r]);
        const bool need = row_mx > m_used + cfg::kRescaleThreshold;
        uint32_t any_need;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.ne.b32 p, %1, 0;\n\t"
            "bar.red.or.pred q, 2, 128, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(any_need)
            : "r"(need ? 1 : 0));
        if (any_need) {  // warpgroup-uniform
          const float m_new = fmaxf(m_used, row_mx);
          const float alpha = (m_new == -INFINITY) ? 1.f : ex2(m_used - m_new);
          lsum *= alpha;
          m_used = m_new;
          if (k > 0) {
            const uint32_t gp = g - 1;
            ok = wg_wait_cluster(&C.p_empty[gp & 1], (gp >> 1) & 1, 0x62);
            if (!ok) break;
            ptx::tc_fence_after();
            for (int j = 0; j < nv; ++j) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                float o[32];
                const uint32_t a = lane_addr + kOCol + j * 64 + 32 * hh;
                ptx::tmem_ld32(a, o);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] *= alpha;
                ptx::tmem_st32(a, o);
              }
            }
            ptx::tmem_st_wait();
          }
        }
        // P buffer free once PV(g - 2) completed
        const int pb = g & 1;
        ok = wg_wait_cluster(&C.p_empty[pb], ((g >> 1) & 1) ^ 1, 0x63);
        if (!ok) break;
        uint8_t* prow = sP + pb * kPBytes + h * kKChunk + r * 128;
#pragma unroll
        for (int uu = 0; uu < 8; ++uu) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 8 * uu + 2 * e;
            const float p0 = (x[c] == -INFINITY) ? 0.f : ex2(x[c] - m_used);
            const float p1 = (x[c + 1] == -INFINITY) ? 0.f : ex2(x[c + 1] - m_used);
            pk[e] = ptx::pack_bf16x2(p0, p1);
            lsum += p0 + p1;
          }
          *reinterpret_cast<uint4*>(prow + ((uu ^ (r & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(p_full_l + pb * 8);
      }
      if (!ok) break;

      // ---- epilogue
      C.lred[h][r] = lsum;
      ptx::named_bar_sync(1, 128);
      const float l = C.lred[0][r] + C.lred[1][r];
      ptx::named_bar_sync(1, 128);  // lred reusable
      const uint32_t glast = gt + n - 1;
      ok = wg_wait_cluster(&C.p_empty[glast & 1], (glast >> 1) & 1, 0x64);
      if (!ok) break;
      ptx::tc_fence_after();
      const bool partial = P.always_partial || u.nsplit > 1;
      const int ws_row = (P.num_splits[u.b] + u.split) * P.R + rg;
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      for (int j = 0; j < nv; ++j) {
        float o[64];
        ptx::tmem_ld32(lane_addr + kOCol + j * 64, o);
        ptx::tmem_ld32(lane_addr + kOCol + j * 64 + 32, o + 32);
        ptx::tmem_ld_wait();
        if (row_valid) {
          const int d0 = 128 * j + 64 * h;
          if (partial) {
            float4* dst = reinterpret_cast<float4*>(P.ws_o + (size_t)ws_row * P.d_v + d0);
#pragma unroll
            for (int q = 0; q < 16; ++q)
              dst[q] = make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv,
                                   o[4 * q + 3] * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(P.out + ((size_t)u.b * P.R + rg) * P.d_v + d0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_uint4(ptx::pack_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                                  ptx::pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                  ptx::pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                  ptx::pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
          }
        }
      }
      if (row_valid && h == 0) {
        const float lv = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (partial)
          P.ws_lse[ws_row] = lv;
        else
          P.lse[(size_t)u.b * P.R + rg] = lv;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(o_free_l);
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

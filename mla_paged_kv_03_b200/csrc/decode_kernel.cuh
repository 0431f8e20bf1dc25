// decode_kernel.cuh -- persistent, warp-specialised sm_100a MLA decode kernel.
//
// What it computes, per query row r of a sequence b (one shared latent KV head
// of 576 dims, V = first d_v dims of the same row):
//   O[r] = softmax(scale * Q[r] K^T) V ,  LSE[r] = log sum exp(scale * Q[r] K^T)
// [FlashMLA (AI Wiki), "How does MLA differ from MHA and GQA?", "How is
//  FlashMLA designed?", "Interfaces"]
//
// Orientation.  All query rows (s_q * h_q, up to 64 per CTA) share one KV
// head, so the tensor-core tile puts TOKENS on the M axis and query rows on N:
//   S^T[128 tok, 64 rows]  = K_tile[128 tok, 576] . Q[64 rows, 576]^T   (QK)
//   O^T[128 d,   64 rows] += V^T[128 d, 128 tok] . P^T[64 rows, 128 tok]^T (PV)
// so M = 128 is always full even for 16 or 32 query rows.  S^T and O^T live in
// TMEM (fp32); the K tile in shared memory serves as the K-major A operand of
// QK and, read through an MN-major descriptor, as V^T for PV.
//
// Memory pipeline.  The cache is read in 128-token tiles (two 64-token pages
// found through the block table) split into 64-dim, 128-byte-wide chunks that
// TMA writes in the 128B-swizzled layout.  A ring of 32 KB "pair slots" (two
// chunks each) is consumed in a fixed order QK(0), QK(1), PV(0), QK(2), PV(1),
// ..., so the softmax of tile k overlaps QK of tile k+1.  V chunks are fetched
// a second time for PV (an L2 hit) instead of holding a whole 144 KB tile.
//
// Roles (warps):  0, 10, 11 = TMA loaders (0 also loads Q),  1 = MMA issuer +
//   TMEM owner,  2..9 = two softmax warpgroups (one thread per token lane of
//   the tile and 32 query-row columns each; also the epilogue).
//
// The fused variant differs only in P: it keeps P to about 16 bits as a bf16
// hi/lo pair (two PV UMMAs per k-step), so that O is accurate enough for its
// E4M3 output codes.  Its query arrives already normalised and rotated (the
// prologue kernel), and its epilogue always goes through the combine kernel.
//
// Softmax uses a lazily updated per-row reference max m: scores are
// exponentiated against m until some score exceeds m by more than 8 (log2
// units); only then is m raised and O, l rescaled.  The result is exact
// either way because O and l are formed against the same m (the "skip scale"
// idea of [FlashMLA (AI Wiki), "The Ascend kernel deep-dive"]).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "mla_common.h"
#include "ptx.cuh"

namespace mla {

enum Mode : int { kDense = 0, kFused = 1 };

struct DecodeParams {
  int batch;       // sequences
  int s_q, h_q;    // query tokens per sequence and heads
  int R;           // rows sharing one KV head: s_q*h_q
  int d_v;         // 512 or 576
  int n_groups;    // ceil(R / 64)
  int num_parts;   // scheduler parts; grid = num_parts * n_groups
  int num_blocks;  // cache blocks (dense/fused)
  int max_pages;
  int causal;
  int always_partial;  // write split partials even for unsplit sequences (fused)
  float scale_log2;    // softmax_scale * log2(e)
  const int32_t* block_table;
  const uint8_t* kcache;      // cache base (L2 prefetch of whole pages)
  const int32_t* seqlens;     // per sequence (dense/fused)
  const int32_t* metadata;    // [num_parts][8]
  const int32_t* num_splits;  // [batch + 1] prefix sums
  __nv_bfloat16* out;         // [batch*R, d_v] bf16 (unsplit rows)
  float* lse;                 // [batch*R]
  float* ws_o;                // [total_splits, R, d_v] fp32 partial O (normalised)
  float* ws_lse;              // [total_splits, R]
  // debug slot trace (null = off): int32 [2][batch][max_pages * 64], the
  // physical slot of every token whose cache row a kernel loaded, plane 0 for
  // the rows read as K, plane 1 for the rows read as V
  int32_t* trace;
  long long trace_plane;  // entries per plane
  // gather mode (CTA-pair kernel): the cache is a bf16 row array
  // [gather_rows, 576] and token t of unit b is row gather_idx[b *
  // gather_stride + t] (an entry outside [0, gather_rows) is masked)
  const int32_t* gather_idx;
  int gather_stride;
  int gather_rows;
  // split partials of sequence b start at ws row ws_base[b] (only split
  // sequences own rows), or at num_splits[b] when ws_base is null
  const int32_t* ws_base;
  // sparse prefill: per-head attention sink logits (natural-log units) or
  // null; folded into the rows the kernel finishes (unsplit ones)
  const float* sink;
  // CTA-pair kernel: 64-dim chunks of q . k, 9 (the 576-dim latent; 0 reads
  // as 9) or 8 (a 512-dim latent: q is [rows, 512], and the cache's dims
  // 512..575 are not read)
  int qk_chunks;
};

namespace cfg {
constexpr int kQBytes = kNumChunks * kRowsPerCta * 128;  // 73728
constexpr int kSubChunk = kTileT * 128;                  // 16384: [128 tok][64 d] bf16
constexpr int kPairBytes = 2 * kSubChunk;                // 32768
#ifndef MLA_RING_PAIRS
#define MLA_RING_PAIRS 3
#endif
#ifndef MLA_P_BUFFERS
#define MLA_P_BUFFERS 2
#endif
constexpr int kNPair = MLA_RING_PAIRS;                   // ring depth (pair slots)
constexpr int kNP = MLA_P_BUFFERS;                       // P buffer regions
constexpr int kPBytes = kTileT * 128;                    // [128 tok][64 rows] bf16
constexpr int kQOff = 0;
constexpr int kRingOff = kQOff + kQBytes;
constexpr int kPOff = kRingOff + kNPair * kPairBytes;
constexpr int kBarOff = kPOff + kNP * kPBytes;
constexpr int kMiscBytes = 4096;
constexpr int kSmemBytes = kBarOff + kMiscBytes + 1024;  // + alignment slack
constexpr int kTmemCols = 512;
constexpr int kSCol = 0;     // S^T buffers at cols [0,64) and [64,128)
constexpr int kOCol = 128;   // O^T chunk c at cols 128 + 64c (c < 5)
constexpr float kRescaleThreshold = 8.0f;  // log2 units
#ifndef MLA_PREFETCH_TILES
#define MLA_PREFETCH_TILES 0
#endif
constexpr int kPrefetchTiles = MLA_PREFETCH_TILES;  // pages of tile k + this are pulled into L2
}  // namespace cfg

// Softmax warpgroups (32 query-row columns each) and the named barrier that
// spans all of them (ids 1..6 are per-group).
constexpr int kSoftmaxGroups = 2;
constexpr int kBarAllSoftmax = 7;

// TMA loader warps filling the ring round-robin (one issuing warp sustains
// only about 25 B/clk): warp 0, then warps 10, 11 after the softmax groups.
#ifndef MLA_DECODE_LOADERS
#define MLA_DECODE_LOADERS 3
#endif
template <int kMode>
struct Loaders {
  static constexpr int value = MLA_DECODE_LOADERS;
};

template <int kMode>
struct Threads {
  // loader + MMA warps, softmax groups, extra loaders
  static constexpr int value = 64 + 128 * kSoftmaxGroups + 32 * (Loaders<kMode>::value - 1);
};

// Shared-memory control block (at kBarOff).
struct __align__(8) Ctrl {
  uint64_t slot_full[cfg::kNPair];
  uint64_t slot_empty[cfg::kNPair];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[cfg::kNP], p_empty[cfg::kNP];
  uint64_t o_free;
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t pad;
  float red[8][32];     // cross-warp reduction scratch [group*4 + warp][column]
  float m[64];          // per-column reference max (log2 domain)
  float alpha[64];      // per-column rescale factor, then 1/l in the epilogue
  int lim[64];          // per-column visible-token limit of the current unit
};
static_assert(sizeof(Ctrl) <= cfg::kMiscBytes, "control block too large");

struct Unit {
  int b, lo, hi, split, nsplit;
  int L;      // tokens attended: cache_seqlens[b], at most max_pages * 64
  int L_raw;  // cache_seqlens[b] as given (the planner counted its tiles)
};

// Iterates the (sequence, tile-range) segments of one scheduler part.
struct UnitIter {
  int b, b_first, b_end, t_begin, t_end, s_begin;
  __device__ void init(const int32_t* m) {
    b = b_first = m[0];
    t_begin = m[1];
    b_end = m[2];
    t_end = m[3];
    s_begin = m[4];
  }
  template <int kMode>
  __device__ bool next(const DecodeParams& P, Unit& u) {
    while (b <= b_end) {
      const int bb = b++;
      const int L_raw = P.seqlens[bb];
      const int lo = (bb == b_first) ? t_begin : 0;
      const int tiles = tiles_of(L_raw);  // the planner's tiles
      const int hi = (bb == b_end) ? min(t_end, tiles) : tiles;
      if (lo >= hi) continue;
      u.b = bb;
      u.lo = lo;
      u.hi = hi;
      u.split = (bb == b_first) ? s_begin : 0;
      u.nsplit = P.num_splits[bb + 1] - P.num_splits[bb];
      u.L_raw = L_raw;
      // A length beyond the block table's max_pages * 64 tokens is read as
      // that many (the block table names no further page) and recorded as an
      // input fault; tiles past it are fully masked, so every split the
      // planner counted still writes its (empty) partial.
      u.L = L_raw;
      if (L_raw > P.max_pages * kPage) {
        ptx::set_error(MLA_DEVERR_BAD_INDEX, 0x30);
        u.L = P.max_pages * kPage;
      }
      return true;
    }
    return false;
  }
};

// Warpgroup-uniform bounded wait: every thread of the 128-thread group waits,
// then the group agrees (barrier AND-reduction) so that all threads take the
// same path even if one of them timed out.
__device__ __forceinline__ bool wg_wait(uint64_t* bar, uint32_t parity, int site, int bar_id,
                                        int nthreads = 128) {
  const bool mine = ptx::mbar_wait(bar, parity, site);
  uint32_t all;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(all)
      : "r"(mine ? 1 : 0), "r"(bar_id), "r"(nthreads));
  return all != 0;
}

// cos/sin of theta = pos * inv_freq in fp64 (the fused prologue rounds the
// rotated query to bf16; computing it in fp64 makes that rounding decision
// agree with an fp64 reference except at exact ties).
__device__ __forceinline__ void rope_sincos64(double pos, double inv_freq, double* sn, double* cs) {
  sincos(pos * inv_freq, sn, cs);
}

// fp32 cos/sin for the output rotation: the angle is formed and reduced
// modulo 2*pi in fp64, the reduced angle in [-pi, pi] is evaluated in fp32.
__device__ __forceinline__ void rope_sincos(double pos, double inv_freq, float* sn, float* cs) {
  const double kTwoPi = 6.283185307179586476925286766559;
  const double theta = pos * inv_freq;
  const double r = fma(-rint(theta * (1.0 / kTwoPi)), kTwoPi, theta);
  __sincosf(static_cast<float>(r), sn, cs);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Debug slot trace: the calling warp records the physical slot (block * 64 +
// offset) of the 64 tokens of page `page` of sequence b, in plane 0 (bit 0
// of `planes`) and / or plane 1 (bit 1).
__device__ __forceinline__ void trace_page(const DecodeParams& P, int b, int page, int blk,
                                           int planes) {
  int32_t* t = P.trace + (size_t)b * P.max_pages * kPage + (size_t)page * kPage;
  for (int i = threadIdx.x & 31; i < kPage; i += 32) {
    if (planes & 1) t[i] = blk * kPage + i;
    if (planes & 2) t[P.trace_plane + i] = blk * kPage + i;
  }
}

__device__ __forceinline__ int clamp_block(int blk, int num_blocks) {
  if (blk < 0 || blk >= num_blocks) {
    ptx::set_error(MLA_DEVERR_BAD_INDEX, 0x51);
    return 0;
  }
  return blk;
}

// --------------------------------------------------------------------------
template <int kMode>
__global__ void __launch_bounds__(Threads<kMode>::value, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kv, const DecodeParams P) {
  using namespace cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kQOff;
  uint8_t* sRing = smem + kRingOff;
  uint8_t* sP = smem + kPOff;
  Ctrl& C = *reinterpret_cast<Ctrl*>(smem + kBarOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int part = blockIdx.x / P.n_groups;
  const int grp = blockIdx.x % P.n_groups;
  const int nv_pairs = (P.d_v + 127) / 128;  // PV pair slots per tile

  // P^T buffers: two alternating bf16 buffers, or (fused variant) one buffer
  // holding P as a bf16 hi/lo pair so that PV sees P to ~16 bits.
  constexpr bool kPSplit = (kMode == kFused);
  constexpr int NPm = kPSplit ? 1 : kNP;
  static_assert(!kPSplit || kNP >= 2, "the hi/lo P pair needs two P buffer regions");

  ptx::grid_dep_wait();    // the planner's metadata is complete
  ptx::grid_dep_launch();  // the combine grid may be scheduled as CTAs retire
  const int32_t* meta = P.metadata + part * kMetaInts;
  if (meta[0] > meta[2]) return;  // empty part: nothing to do (uniform exit)

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNPair; ++i) {
      ptx::mbar_init(&C.slot_full[i], 1);
      ptx::mbar_init(&C.slot_empty[i], 1);
    }
    ptx::mbar_init(&C.q_full, 1);
    ptx::mbar_init(&C.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&C.s_full[i], 1);
      ptx::mbar_init(&C.s_empty[i], 128 * kSoftmaxGroups);
    }
    for (int i = 0; i < kNP; ++i) {
      ptx::mbar_init(&C.p_full[i], 128 * kSoftmaxGroups);
      ptx::mbar_init(&C.p_empty[i], 1);
    }
    ptx::mbar_init(&C.o_free, 128 * kSoftmaxGroups);
    ptx::mbar_init(&C.drain, 1);

    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&C.tmem_base, kTmemCols);
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

  constexpr int kL = Loaders<kMode>::value;
  constexpr int kFirstExtraLoader = 2 + 4 * kSoftmaxGroups;
  if (warp == 0 || warp >= kFirstExtraLoader) {
    // ============================== loaders ==============================
    // Pair slot j of the ring is filled by loader warp j % kL (whole warp,
    // one elected lane issues the copies).  Warp 0 also loads Q.
    const int role = warp == 0 ? 0 : warp - kFirstExtraLoader + 1;
    uint32_t ring_it = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    auto load_pair = [&](const Unit& un, int tile, int pair, int planes) -> bool {
      const uint32_t idx = ring_it++;
      if (static_cast<int>(idx % kL) != role) return true;
      const int slot = idx % kNPair;
      const uint32_t round = idx / kNPair;
      bool w = ptx::mbar_wait(&C.slot_empty[slot], (round & 1) ^ 1, 0x01);
      if (!__all_sync(0xffffffffu, w)) return false;
      const int c0 = 2 * pair;
      const int nch = (c0 + 1 < kNumChunks) ? 2 : 1;
      const int tok0 = tile * kTileT;
      const int npg = (un.L + kPage - 1) / kPage;  // <= max_pages
      const int p0 = tok0 / kPage;
      int blk0 = p0 < npg ? P.block_table[(size_t)un.b * P.max_pages + p0] : 0;
      int blk1 = (p0 + 1 < npg) ? P.block_table[(size_t)un.b * P.max_pages + p0 + 1] : blk0;
      blk0 = clamp_block(blk0, P.num_blocks);
      blk1 = clamp_block(blk1, P.num_blocks);
      if (P.trace && pair == 0) {
        if (p0 < npg) trace_page(P, un.b, p0, blk0, planes);
        if (p0 + 1 < npg) trace_page(P, un.b, p0 + 1, blk1, planes);
      }
      if (ptx::elect_one_sync()) {
        ptx::mbar_arrive_expect_tx(&C.slot_full[slot], nch * kSubChunk);
        uint8_t* dst = sRing + slot * kPairBytes;
        for (int j = 0; j < nch; ++j) {
          const int x = (c0 + j) * kChunkD;
          ptx::tma_load_2d(dst + j * kSubChunk, &tm_kv, &C.slot_full[slot], x, blk0 * kPage);
          ptx::tma_load_2d(dst + j * kSubChunk + kSubChunk / 2, &tm_kv, &C.slot_full[slot], x,
                           blk1 * kPage);
        }
      }
      __syncwarp();
      return true;
    };
    while (ok && it.template next<kMode>(P, u)) {
      if (role == 0) {
        // Q rows [64*grp, 64*grp+64) of this sequence (or query pair); for the
        // fused variant the normalised, rotated rows of the prologue kernel
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&C.q_empty, (u_idx & 1) ^ 1, 0x02));
        if (ok && ptx::elect_one_sync()) {
          ptx::mbar_arrive_expect_tx(&C.q_full, kQBytes);
          const int row0 = u.b * P.R + grp * kRowsPerCta;
          for (int c = 0; c < kNumChunks; ++c)
            ptx::tma_load_2d(sQ + c * (kRowsPerCta * 128), &tm_q, &C.q_full, c * kChunkD, row0);
        }
        __syncwarp();
      }
      if (ok) {
        const int n = u.hi - u.lo;
        for (int k = 0; k < n && ok; ++k) {
          for (int pr = 0; pr < 5 && ok; ++pr) ok = load_pair(u, u.lo + k, pr, 1);
          if (k >= 1)
            for (int pr = 0; pr < nv_pairs && ok; ++pr) ok = load_pair(u, u.lo + k - 1, pr, 2);
        }
        for (int pr = 0; pr < nv_pairs && ok; ++pr) ok = load_pair(u, u.hi - 1, pr, 2);
      }
      ++u_idx;
    }
    // Never leave a TMA write in flight: wait (bounded) for the final load of
    // each slot if this warp issued it (an earlier load into a slot completed
    // before the slot could be reused).  In the normal path these phases
    // completed long ago and the waits return at once.
    for (int i = 0; i < kNPair && i < static_cast<int>(ring_it); ++i) {
      const uint32_t last = ring_it - 1 - i;
      if (static_cast<int>(last % kL) != role) continue;
      ptx::mbar_wait(&C.slot_full[last % kNPair], (last / kNPair) & 1, 0x03);
    }
    if (role == 0 && u_idx > 0) ptx::mbar_wait(&C.q_full, (u_idx - 1) & 1, 0x04);
    __syncwarp();
  } else if (warp == 1) {
    // ============================== MMA issuer ==============================
    // The whole warp runs the loop (its address arithmetic stays warp-uniform)
    // and one elected lane issues each slot's UMMAs and commits.
    const uint32_t idesc_qk = ptx::idesc_bf16_f32(128, kRowsPerCta, 0, 0);
    const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, kRowsPerCta, 1, 1);
    const uint32_t q_addr = ptx::smem_u32(sQ);
    const uint32_t ring_addr = ptx::smem_u32(sRing);
    const uint32_t p_addr = ptx::smem_u32(sP);
    uint32_t ring_it = 0, gt = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    auto warp_wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
      return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, site));
    };
    auto wait_slot = [&]() -> int {
      const int slot = ring_it % kNPair;
      const uint32_t round = ring_it / kNPair;
      ++ring_it;
      if (!warp_wait(&C.slot_full[slot], round & 1, 0x11)) return -1;
      ptx::tc_fence_after();
      return slot;
    };
    // Descriptor words of each operand's base; inner loops only add offsets.
    const ptx::DescWords dq = ptx::desc_words(q_addr, 16, 1024, ptx::kLayoutSW128);
    const ptx::DescWords dring = ptx::desc_words(ring_addr, 16, 1024, ptx::kLayoutSW128);
    const ptx::DescWords dv = ptx::desc_words(ring_addr, kSubChunk, 1024, ptx::kLayoutSW128);
    const ptx::DescWords dp = ptx::desc_words(p_addr, 16, 1024, ptx::kLayoutSW128);
    auto do_qk = [&](uint32_t g) -> bool {
      const int sb = g & 1;
      if (!warp_wait(&C.s_empty[sb], ((g >> 1) & 1) ^ 1, 0x12)) return false;
      ptx::tc_fence_after();
      const uint32_t d_tmem = tmem + kSCol + sb * kRowsPerCta;
#pragma unroll
      for (int pr = 0; pr < 5; ++pr) {
        const int slot = wait_slot();
        if (slot < 0) return false;
        if (ptx::elect_one_sync()) {
          const uint32_t a_lo = dring.lo + ((slot * kPairBytes) >> 4);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int c = 2 * pr + j;
            if (c < kNumChunks) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                ptx::umma_f16_ss_w(d_tmem, a_lo + ((j * kSubChunk + kk * 32) >> 4), dring.hi,
                                   dq.lo + ((c * (kRowsPerCta * 128) + kk * 32) >> 4), dq.hi,
                                   idesc_qk, (c | kk) ? 1u : 0u);
            }
          }
          ptx::umma_commit(&C.slot_empty[slot]);
          if (pr == 4) ptx::umma_commit(&C.s_full[sb]);
        }
        __syncwarp();
      }
      return true;
    };
    auto do_pv = [&](uint32_t g, bool first_of_unit) -> bool {
      const int pb = g % NPm;
      if (!warp_wait(&C.p_full[pb], (g / NPm) & 1, 0x13)) return false;
      ptx::tc_fence_after();
      const uint32_t b_lo = dp.lo + ((pb * kPBytes) >> 4);
      for (int pr = 0; pr < nv_pairs; ++pr) {
        const int slot = wait_slot();
        if (slot < 0) return false;
        if (ptx::elect_one_sync()) {
          const uint32_t d_tmem = tmem + kOCol + pr * kRowsPerCta;
          const uint32_t a_lo = dv.lo + ((slot * kPairBytes) >> 4);
          // first k-step of the unit's first tile starts the accumulator
          ptx::umma_f16_ss_w(d_tmem, a_lo, dv.hi, b_lo, dp.hi, idesc_pv, first_of_unit ? 0u : 1u);
          if (kPSplit)
            ptx::umma_f16_ss_w(d_tmem, a_lo, dv.hi, b_lo + (kPBytes >> 4), dp.hi, idesc_pv, 1u);
#pragma unroll
          for (int kk = 1; kk < kTileT / 16; ++kk) {
            ptx::umma_f16_ss_w(d_tmem, a_lo + ((kk * 2048) >> 4), dv.hi, b_lo + ((kk * 2048) >> 4),
                               dp.hi, idesc_pv, 1u);
            if (kPSplit)  // + V^T . P_lo^T
              ptx::umma_f16_ss_w(d_tmem, a_lo + ((kk * 2048) >> 4), dv.hi,
                                 b_lo + ((kPBytes + kk * 2048) >> 4), dp.hi, idesc_pv, 1u);
          }
          ptx::umma_commit(&C.slot_empty[slot]);
          if (pr == nv_pairs - 1) ptx::umma_commit(&C.p_empty[pb]);
        }
        __syncwarp();
      }
      return true;
    };
    while (ok && it.template next<kMode>(P, u)) {
      if (!warp_wait(&C.q_full, u_idx & 1, 0x14)) break;
      ptx::tc_fence_after();
      const int n = u.hi - u.lo;
      const uint32_t g0 = gt;
      for (int k = 0; k < n && ok; ++k) {
        ok = do_qk(g0 + k);
        if (ok && k == n - 1) {
          if (ptx::elect_one_sync()) ptx::umma_commit(&C.q_empty);
          __syncwarp();
        }
        if (ok && k >= 1) {
          if (k == 1 && !warp_wait(&C.o_free, (u_idx & 1) ^ 1, 0x15)) {
            ok = false;
            break;
          }
          ok = do_pv(g0 + k - 1, k == 1);
        }
      }
      if (ok) {
        if (n == 1 && !warp_wait(&C.o_free, (u_idx & 1) ^ 1, 0x16)) {
          ok = false;
          break;
        }
        ok = do_pv(g0 + n - 1, n == 1);
      }
      gt += n;
      ++u_idx;
    }
    // Drain the tensor pipe before TMEM is released.
    if (ptx::elect_one_sync()) ptx::umma_commit(&C.drain);
    __syncwarp();
    ptx::mbar_wait(&C.drain, 0, 0x17);
    __syncwarp();
  } else if (warp >= 2 && warp < 2 + 4 * kSoftmaxGroups) {
    // ============================== softmax / epilogue ==============================
    // Two warpgroups; group sg owns query-row columns [32*sg, 32*sg + 32).
    const int sg = (warp - 2) >> 2;
    const int cb = 32 * sg;               // first column of this group
    const int wq = warp & 3;              // TMEM lane quarter of this warp
    const int t = wq * 32 + lane;         // token lane within the tile (0..127)
    const int wt = (threadIdx.x - 64) & 127;  // thread index within the warpgroup
    const int bar_sync = 1 + 3 * sg, bar_or = 2 + 3 * sg, bar_and = 3 + 3 * sg;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    uint32_t gt = 0;
    int u_idx = 0;
    Unit u;
    bool ok = true;
    while (ok && it.template next<kMode>(P, u)) {
      const int n = u.hi - u.lo;
      // ---- per-unit column limits (visible tokens of each query row)
      if (wt < 32) {
        const int rg = grp * kRowsPerCta + cb + wt;
        int lim = 0;
        if (rg < P.R) {
          if (!P.causal) {
            lim = u.L;
          } else {
            lim = u.L - P.s_q + 1 + rg / P.h_q;
            lim = lim < 0 ? 0 : lim;
          }
        }
        C.lim[cb + wt] = lim;
        C.m[cb + wt] = -INFINITY;
      }
      ptx::named_bar_sync(bar_sync, 128);  // C.lim, C.m of this group visible

      int min_lim = 1 << 30;
      for (int c = 0; c < 32; ++c) {
        const int rg = grp * kRowsPerCta + cb + c;
        if (rg < P.R && C.lim[cb + c] < min_lim) min_lim = C.lim[cb + c];
      }
      float lsum[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) lsum[c] = 0.f;

      for (int k = 0; k < n && ok; ++k) {
        const uint32_t g = gt + k;
        const int sb = g & 1;
        if (!wg_wait(&C.s_full[sb], (g >> 1) & 1, 0x22, bar_and)) { ok = false; break; }
        ptx::tc_fence_after();
        float x[32];
        ptx::tmem_ld32(lane_addr + kSCol + sb * kRowsPerCta + cb, x);
        ptx::tmem_ld_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&C.s_empty[sb]);

        const int tile_tok0 = (u.lo + k) * kTileT;
        const int T = tile_tok0 + t;
        const bool need_mask = tile_tok0 + kTileT > min_lim;
        int need = 0;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float v = x[c] * P.scale_log2;
          if (need_mask && T >= C.lim[cb + c]) v = -INFINITY;
          x[c] = v;
          need |= (v > C.m[cb + c] + kRescaleThreshold);
        }
        uint32_t any_need;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.ne.b32 p, %1, 0;\n\t"
            "bar.red.or.pred q, %2, 128, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(any_need)
            : "r"(need), "r"(bar_or));
        if (any_need) {
          // Raise the reference max to this tile's exact column max.
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float v = x[c];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) C.red[4 * sg + wq][c] = v;
          }
          ptx::named_bar_sync(bar_sync, 128);
          if (wt < 32) {
            const float tm = fmaxf(fmaxf(C.red[4 * sg][wt], C.red[4 * sg + 1][wt]),
                                   fmaxf(C.red[4 * sg + 2][wt], C.red[4 * sg + 3][wt]));
            const float mo = C.m[cb + wt];
            const float mn = fmaxf(mo, tm);
            C.alpha[cb + wt] = (mn == -INFINITY) ? 1.f : ex2(mo - mn);
            C.m[cb + wt] = mn;
          }
          ptx::named_bar_sync(bar_sync, 128);
#pragma unroll
          for (int c = 0; c < 32; ++c) lsum[c] *= C.alpha[cb + c];
          if (k > 0) {
            // O holds the sum through PV(g-1): wait for it, rescale this lane.
            const uint32_t gp = g - 1;
            if (!wg_wait(&C.p_empty[gp % NPm], (gp / NPm) & 1, 0x23, bar_and)) { ok = false; break; }
            ptx::tc_fence_after();
            for (int pr = 0; pr < nv_pairs; ++pr) {
              float o[32];
              const uint32_t a = lane_addr + kOCol + pr * kRowsPerCta + cb;
              ptx::tmem_ld32(a, o);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] *= C.alpha[cb + c];
              ptx::tmem_st32(a, o);
            }
            ptx::tmem_st_wait();
          }
        }
        // P buffer free once PV(g - NPm) completed
        const int pb = g % NPm;
        if (!wg_wait(&C.p_empty[pb], ((g / NPm) & 1) ^ 1, 0x24, bar_and)) { ok = false; break; }
        // probabilities: bf16 (or a bf16 hi/lo pair) for the PV operand, fp32
        // for the row sums l
        uint8_t* prow = sP + pb * kPBytes + t * 128;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          uint32_t pk[4], pl[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 8 * uu + 2 * e;
            // fresh shared-memory reads (not registers kept from the check above)
            const volatile float* mv = &C.m[cb + c];
            const float m0 = mv[0], m1 = mv[1];
            const float p0 = (x[c] == -INFINITY) ? 0.f : ex2(x[c] - m0);
            const float p1 = (x[c + 1] == -INFINITY) ? 0.f : ex2(x[c + 1] - m1);
            pk[e] = ptx::pack_bf16x2(p0, p1);
            if (kPSplit)
              pl[e] = ptx::pack_bf16x2(p0 - __uint_as_float(pk[e] << 16),
                                       p1 - __uint_as_float(pk[e] & 0xFFFF0000u));
            lsum[c] += p0;
            lsum[c + 1] += p1;
          }
          const int unit = 4 * sg + uu;  // 16-byte unit = rows 8*unit .. 8*unit+7
          *reinterpret_cast<uint4*>(prow + ((unit ^ (t & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          if (kPSplit)
            *reinterpret_cast<uint4*>(prow + kPBytes + ((unit ^ (t & 7)) << 4)) =
                make_uint4(pl[0], pl[1], pl[2], pl[3]);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&C.p_full[pb]);
      }
      if (!ok) break;

      // ---- epilogue: l = column sums over the 128 token lanes
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float v = lsum[c];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) C.red[4 * sg + wq][c] = v;
      }
      ptx::named_bar_sync(bar_sync, 128);
      const bool partial = P.always_partial || u.nsplit > 1;
      const int ws_row0 = ((P.ws_base ? P.ws_base[u.b] : P.num_splits[u.b]) + u.split) * P.R;
      const int rows_here = min(kRowsPerCta, P.R - grp * kRowsPerCta);
      if (wt < 32) {
        const float l = (C.red[4 * sg][wt] + C.red[4 * sg + 1][wt]) +
                        (C.red[4 * sg + 2][wt] + C.red[4 * sg + 3][wt]);
        C.alpha[cb + wt] = l > 0.f ? 1.0f / l : 0.f;  // reused as 1/l
        if (cb + wt < rows_here) {
          const int rg = grp * kRowsPerCta + cb + wt;
          const float lv =
              l > 0.f ? (C.m[cb + wt] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
          if (partial)
            P.ws_lse[ws_row0 + rg] = lv;
          else
            P.lse[(size_t)u.b * P.R + rg] = lv;
        }
      }
      ptx::named_bar_sync(bar_sync, 128);
      const uint32_t glast = gt + n - 1;
      if (!wg_wait(&C.p_empty[glast % NPm], (glast / NPm) & 1, 0x25, bar_and)) { ok = false; break; }
      ptx::tc_fence_after();
      const int ncols = min(32, rows_here - cb);  // valid columns of this group
      const size_t row_first = partial ? (size_t)ws_row0 + grp * kRowsPerCta + cb
                                       : (size_t)u.b * P.R + grp * kRowsPerCta + cb;
      for (int pr = 0; pr < nv_pairs; ++pr) {
        const int d = pr * 128 + t;
        float o[32];
        ptx::tmem_ld32(lane_addr + kOCol + pr * kRowsPerCta + cb, o);
        ptx::tmem_ld_wait();
        if (d < P.d_v && ncols > 0) {
          if (partial) {
            float* dst = P.ws_o + row_first * P.d_v + d;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < ncols) dst[(size_t)c * P.d_v] = o[c] * C.alpha[cb + c];
          } else {
            __nv_bfloat16* dst = P.out + row_first * P.d_v + d;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < ncols) dst[(size_t)c * P.d_v] = __float2bfloat16_rn(o[c] * C.alpha[cb + c]);
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&C.o_free);
      ptx::named_bar_sync(bar_sync, 128);  // C.alpha / C.red / C.lim reusable
      gt += n;
      ++u_idx;
    }
  }

  // ---- teardown: every role has finished issuing; wait for the MMA pipe to
  // drain before releasing TMEM.
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mla

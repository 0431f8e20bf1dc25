// sparse_gather.cuh -- first step of token-level sparse decode: gather the
// selected rows of an FP8 latent cache, dequantise them to bf16 and compact
// each query's valid tokens into a dense paged buffer that the dense decode
// kernels then attend over.
//
// Cache rows (per token), [FlashMLA (AI Wiki), "The FP8 and FP4 KV cache"]:
//  - 656 bytes: [512 x E4M3 codes][4 x fp32 scale, one per 128 codes]
//    [64 x bf16 RoPE dims]; a nope value is code * scale.
//  - 528 bytes (V4.1): [512 x E4M3 codes over the whole 512-dim latent]
//    [16 x E8M0 scale, one per 32 codes]; a value is code * 2^(e - 127).
//  - 288 bytes (V4.1 FP4): [512 x E2M1 codes, two per byte, code 2i in the
//    low nibble of byte i][32 x E4M3 scale, one per 16 codes].
//  For both V4.1 rows the buffer row stays 576 wide with dims 512..575 zero,
//  and the 512-wide query rows are copied into a 576-wide buffer with zero
//  dims 512..575, so that q . k and the first 512 dims of V are unchanged.
// Indices (per (sequence, query) pair): physical slots, -1 (or any value
// outside [0, num_slots)) marks an unused entry; the block table of the cache
// is not used.  [FlashMLA (AI Wiki), "Interfaces"]
//
// Attention is invariant to the order of the attended tokens, so the valid
// tokens of pair b are written in index order to rows [0, n_b) of b's region
// of the buffer (pages of 64 rows, b's pages numbered b * pages_per_pair + p),
// n_b goes to seqlens[b], and the dense kernels run with that identity block
// table, no causal mask and lengths n_b.  A pair without valid tokens gets
// n_b = 0, hence O = 0 and LSE = -inf.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "mla_common.h"
#include "ptx.cuh"

namespace mla {

constexpr int kGatherTokens = 64;  // tokens per CTA = one page of the buffer
constexpr int kGatherCtaThreads = 256;
constexpr int kRowUnits = kD / 8;  // 16-byte bf16 output units per row (72)

struct GatherParams {
  const uint8_t* cache;     // [num_slots, row bytes]: 656, 528 or 288
  long long num_slots;
  const int32_t* indices;   // [pairs, topk]
  int topk;
  int pages_per_pair;       // ceil(topk / 64)
  __nv_bfloat16* rows;      // [pairs * pages_per_pair * 64, 576]
  int32_t* block_table;     // [pairs, pages_per_pair]
  int32_t* seqlens;         // [pairs]
  // V4.1 rows (528 / 288 bytes) only: query rows [pairs * h_q, 512] are
  // widened into [pairs * h_q, 576]
  const __nv_bfloat16* q512;
  __nv_bfloat16* q576;
  int h_q;
  // debug slot trace (null = off): int32 [2][pairs][topk]; plane 0 holds the
  // slot each entry read (-1 for an unused entry), plane 1 the row of the
  // compacted buffer it went to (-1 likewise)
  int32_t* trace;
  long long trace_plane;  // entries per plane
};

// E8M0 byte -> fp32: 2^(e - 127) (e = 0 is the fp32 subnormal 2^-127),
// 0xFF -> NaN.
__device__ __forceinline__ float e8m0_to_float(uint32_t e) {
  if (e == 0xFFu) return __int_as_float(0x7FC00000);
  return e == 0u ? __int_as_float(0x00400000) : __int_as_float(static_cast<int>(e << 23));
}

__device__ __forceinline__ bool gather_valid(int idx, long long num_slots) {
  return idx >= 0 && static_cast<long long>(idx) < num_slots;
}

// a * b rounded to odd in fp32: the truncated product, with its last bit set
// when the product was inexact.  Rounding that to nearest bf16 (16 bits
// shorter) gives the correctly rounded bf16 of the exact product, with no
// double-rounding error (rounding to odd: Boldo and Melquiond, "Emulation of
// FMA and correctly rounded sums: proved algorithms using rounding to odd",
// IEEE Transactions on Computers 57(4), 2008).
__device__ __forceinline__ float mul_round_odd(float a, float b) {
  const float p = __fmul_rz(a, b);
  const float e = __fmaf_rz(a, b, -p);  // the exact remainder of the truncation
  return e != 0.f ? __uint_as_float(__float_as_uint(p) | 1u) : p;
}

// Eight E2M1 codes (4 bytes, low nibble first) -> four f16x2 pairs through the
// hardware pair conversion (byte j -> pair j, low nibble -> low half).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}

// grid (pages_per_pair, pairs): CTA (c, b) handles indices [64c, 64c + 64) of pair b.
// Register caps: the FP8 variants would take about 100 registers (2 CTAs per
// SM) and are held to 3 CTAs; the FP4 and bf16 variants fit 4.
template <int kRowBytes>
constexpr int gather_min_ctas() {
  return kRowBytes == kRow288 ? 4 : 3;
}

template <int kRowBytes>
__global__ void __launch_bounds__(kGatherCtaThreads, gather_min_ctas<kRowBytes>())
    mla_sparse_gather_kernel(const GatherParams G) {
  static_assert(kRowBytes == kRow656 || kRowBytes == kRow528 || kRowBytes == kRow288,
                "656-, 528- or 288-byte rows");
  constexpr bool kV41 = kRowBytes == kRow528 || kRowBytes == kRow288;  // 512-dim latent
  constexpr bool kFp4 = kRowBytes == kRow288;
  __shared__ int s_red[kGatherCtaThreads / 32];
  __shared__ int s_idx[kGatherTokens];
  __shared__ int s_dst[kGatherTokens];  // destination row within the pair, or -1
  __shared__ int s_base;
  ptx::grid_dep_wait();
  const int c = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* idx_b = G.indices + (size_t)b * G.topk;
  const int lim = G.topk;

  // valid tokens in the pair's earlier chunks: this chunk's first output row
  int cnt = 0;
  for (int j = tid; j < c * kGatherTokens && j < lim; j += kGatherCtaThreads)
    cnt += gather_valid(__ldg(idx_b + j), G.num_slots) ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) s_red[warp] = cnt;

  // this chunk: validity and rank among the chunk's valid tokens (warps 0, 1)
  if (tid < kGatherTokens) {
    const int j = c * kGatherTokens + tid;
    const int idx = j < lim ? __ldg(idx_b + j) : -1;
    bool v = gather_valid(idx, G.num_slots);
    if (j < lim && idx >= 0 && !v) ptx::set_error(MLA_DEVERR_BAD_INDEX, 0x80);
    const unsigned m = __ballot_sync(0xffffffffu, v);
    s_idx[tid] = idx;
    s_dst[tid] = v ? __popc(m & ((1u << lane) - 1)) : -1;  // rank within the warp
    if (tid == 0) s_base = __popc(m);  // valid tokens among the chunk's first 32
  }
  __syncthreads();
  if (tid == 0) {
    int before = 0;
    for (int w = 0; w < kGatherCtaThreads / 32; ++w) before += s_red[w];
    s_red[0] = before;
  }
  __syncthreads();
  const int before = s_red[0];
  if (tid < kGatherTokens && s_dst[tid] >= 0)
    s_dst[tid] += before + (tid >= 32 ? s_base : 0);
  __syncthreads();
  if (G.trace && tid < kGatherTokens && c * kGatherTokens + tid < G.topk) {
    int32_t* t = G.trace + (size_t)b * G.topk + c * kGatherTokens + tid;
    t[0] = s_dst[tid] >= 0 ? s_idx[tid] : -1;
    t[G.trace_plane] = s_dst[tid];
  }

  __nv_bfloat16* out_b = G.rows + (size_t)b * G.pages_per_pair * kGatherTokens * kD;
  if (tid == 0) G.block_table[(size_t)b * G.pages_per_pair + c] = b * G.pages_per_pair + c;
  if (c == G.pages_per_pair - 1) {
    // the pair's length, and zeros for the rest of its last page: the decode
    // kernel masks those tokens, but multiplies their rows by P = 0
    __shared__ int s_n;
    if (tid == 0) {
      int n = 0;
      for (int t = 0; t < kGatherTokens; ++t) n += s_dst[t] >= 0 ? 1 : 0;
      s_n = before + n;
      G.seqlens[b] = s_n;
    }
    __syncthreads();
    const int n = s_n;
    // a pair without valid tokens still has its first page read (fully masked)
    const int end = n > 0 ? (n + kGatherTokens - 1) / kGatherTokens * kGatherTokens : kGatherTokens;
    for (int item = tid; item < (end - n) * kRowUnits; item += kGatherCtaThreads)
      *reinterpret_cast<uint4*>(out_b + (size_t)(n + item / kRowUnits) * kD + 8 * (item % kRowUnits)) =
          make_uint4(0, 0, 0, 0);
  }

  {
    // dequantise: per token 32 units of 16 codes (two 16-byte bf16 outputs
    // each) and 8 units of the dims 512..575 (bf16 RoPE dims, or zeros for the
    // 528-byte rows); all loads of a thread are issued before any conversion so
    // that they overlap
    constexpr int kUnits = kNope / 16 + kRope / 8;  // 40
    constexpr int kPer = kGatherTokens * kUnits / kGatherCtaThreads;  // 10
    static_assert(kGatherTokens * kUnits % kGatherCtaThreads == 0, "even split");
    uint4 raw[kPer];
    float sc[kPer];      // 656-byte rows: the fp32 scale
    uint32_t eb[kPer];   // 528-byte rows: the E8M0 byte, converted after all loads
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int item = tid + k * kGatherCtaThreads;
      const int t = item / kUnits, u = item % kUnits;
      raw[k] = make_uint4(0, 0, 0, 0);
      sc[k] = 0.f;
      eb[k] = 127u;
      if (s_dst[t] >= 0) {
        const uint8_t* row = G.cache + (size_t)s_idx[t] * kRowBytes;
        if (u < kNope / 16 && kFp4) {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(row) + u);  // 16 codes
          raw[k] = make_uint4(v.x, v.y, 0u, 0u);
          eb[k] = __ldg(row + kNope / 2 + u);
        } else if (u < kNope / 16) {
          raw[k] = __ldg(reinterpret_cast<const uint4*>(row) + u);
          if (kV41)
            eb[k] = __ldg(row + kNope + (u >> 1));
          else
            sc[k] = __ldg(reinterpret_cast<const float*>(row + kNope) + (u >> 3));
        } else if (!kV41) {
          raw[k] = __ldg(reinterpret_cast<const uint4*>(row + kNope + 16) + (u - kNope / 16));
        }
      }
    }
    if (kV41 && G.q576) {
      // the pair's query rows widened to 576 dims (72 16-byte units a row),
      // spread over all pages_per_pair CTAs of the pair, while the row loads
      // above are in flight
      const int n_items = G.h_q * kRowUnits;
      for (int item = c * kGatherCtaThreads + tid; item < n_items;
           item += G.pages_per_pair * kGatherCtaThreads) {
        const size_t r = (size_t)b * G.h_q + item / kRowUnits;
        const int uu = item % kRowUnits;
        const uint4 v = uu < kNope / 8
                            ? __ldg(reinterpret_cast<const uint4*>(G.q512 + r * kNope) + uu)
                            : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(G.q576 + r * kD + 8 * uu) = v;
      }
    }

#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int item = tid + k * kGatherCtaThreads;
      const int t = item / kUnits, u = item % kUnits;
      const int dst = s_dst[t];
      if (dst < 0) continue;
      __nv_bfloat16* orow = out_b + (size_t)dst * kD;
      if (u < kNope / 16 && kFp4) {
        // code * scale in f16 is exact (at most 6 significant bits, |x| <= 2688),
        // and so is its bf16 rounding
        uint32_t s2;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;"
            : "=r"(s2)
            : "h"(static_cast<uint16_t>((eb[k] & 0xFFu) * 0x0101u)));
        const __half2 scl2 = *reinterpret_cast<const __half2*>(&s2);
        uint32_t h[8];
        e2m1x8_to_f16x2(raw[k].x, *reinterpret_cast<uint32_t(*)[4]>(&h[0]));
        e2m1x8_to_f16x2(raw[k].y, *reinterpret_cast<uint32_t(*)[4]>(&h[4]));
        uint32_t r[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float2 f = __half22float2(__hmul2(*reinterpret_cast<const __half2*>(&h[q]), scl2));
          r[q] = ptx::pack_bf16x2(f.x, f.y);
        }
        *reinterpret_cast<uint4*>(orow + 16 * u) = make_uint4(r[0], r[1], r[2], r[3]);
        *reinterpret_cast<uint4*>(orow + 16 * u + 8) = make_uint4(r[4], r[5], r[6], r[7]);
      } else if (u < kNope / 16) {
        const uint32_t words[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
        const float scl = kV41 ? e8m0_to_float(eb[k]) : sc[k];
        uint32_t r[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t h0, h1;
          const uint16_t lo16 = static_cast<uint16_t>(words[q] & 0xFFFF);
          const uint16_t hi16 = static_cast<uint16_t>(words[q] >> 16);
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h0) : "h"(lo16));
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h1) : "h"(hi16));
          const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
          const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
          // code * scale rounded once to bf16; with the power-of-two E8M0 scales
          // the product is exact already
          if (kV41) {
            r[2 * q] = ptx::pack_bf16x2(f0.x * scl, f0.y * scl);
            r[2 * q + 1] = ptx::pack_bf16x2(f1.x * scl, f1.y * scl);
          } else {
            r[2 * q] = ptx::pack_bf16x2(mul_round_odd(f0.x, scl), mul_round_odd(f0.y, scl));
            r[2 * q + 1] = ptx::pack_bf16x2(mul_round_odd(f1.x, scl), mul_round_odd(f1.y, scl));
          }
        }
        *reinterpret_cast<uint4*>(orow + 16 * u) = make_uint4(r[0], r[1], r[2], r[3]);
        *reinterpret_cast<uint4*>(orow + 16 * u + 8) = make_uint4(r[4], r[5], r[6], r[7]);
      } else {
        *reinterpret_cast<uint4*>(orow + kNope + 8 * (u - kNope / 16)) = raw[k];
      }
    }
  }
}

}  // namespace mla

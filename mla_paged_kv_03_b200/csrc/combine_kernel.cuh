// combine_kernel.cuh -- split-KV merge and the fused output epilogue.
//
// For a row split into n partial results (O_i normalised, LSE_i):
//   LSE = log sum_i exp(LSE_i)  (max-subtracted),  O = sum_i exp(LSE_i - LSE) O_i
// The pages imply this step through the per-batch split counts returned by
// the metadata call and the LSE returned with every output
// [FlashMLA Ampere port README, "Usage"; FlashMLA (AI Wiki), "Interfaces"].
//
// Fused variant (d_v = 576): after the merge, the conjugate RoPE rotates
// O[512:576] by -theta at the query position, the row's absmax sets the fp32
// scale = absmax / 448, and O / scale is cast to E4M3 (round to nearest even,
// saturating).  [FlashMLA fused norm-RoPE-attention-RoPE-cast kernel card]
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "mla_common.h"
#include "decode_kernel.cuh"

namespace mla {

struct CombineParams {
  int batch, R, d_v, h_q;
  const int32_t* num_splits;  // [batch + 1]
  const int32_t* ws_base;     // [batch] first partial row of each split sequence, or null
                              // (then num_splits[b])
  const float* ws_o;          // [total_splits, R, d_v]
  const float* ws_lse;        // [total_splits, R]
  __nv_bfloat16* out;         // dense: [batch*R, d_v]
  float* lse;                 // [batch*R]
  // fused
  uint8_t* out_fp8;           // [batch*R, 576]
  float* out_scale;           // [batch*R]
  const int32_t* seqlens;
  const int32_t* positions;   // nullable: L - 1
  double inv_freq[kRope / 2]; // base^(-2k/64), computed on the host in fp64
  int row_per_cta;            // 1: a CTA's warps share one row's splits (few rows)
  // optional: the rows are those of the sequences seq_list[0 .. list_len)
  // (-1 entries are skipped) instead of all batch sequences
  const int32_t* seq_list;
  int list_len;
  const float* sink;          // nullable: per-head sink logits joining the normaliser
};

__device__ __forceinline__ uint32_t cvt_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(a), "f"(b));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(c), "f"(d));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// One warp per row: lane l owns the float4 groups l, l + 32, ... of the row
// (d_v / 4 = 128 or 144 groups); split weights are formed 32 at a time, one
// per lane, and broadcast with shuffles.  With few rows and many splits
// (row_per_cta) the CTA's warps take every kCombineWarps-th split of one row
// and add their sums in shared memory.
__device__ __forceinline__ void fma_acc(float4& a, float w, const float4 v) {
  a.x += w * v.x;
  a.y += w * v.y;
  a.z += w * v.z;
  a.w += w * v.w;
}

constexpr int kCombineMaxSplits = 1024;  // splits of one sequence (<= SM parts)
constexpr int kCombineWarps = 8;
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kCombineGroups = (kD / 4 + 31) / 32;  // float4 groups per lane (5)

// kPairs: splits are taken two at a time (both loads in flight before the
// FMAs).  It needs more registers (two CTAs per SM instead of four), so the
// host selects it only when the grid fits in one wave at that occupancy.
template <bool kFusedOut, bool kPairs>
__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(const CombineParams P) {
  __shared__ float4 s_acc[kCombineWarps - 1][kD / 4];
  ptx::grid_dep_wait();  // the decode kernel's partials are complete
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool shared_row = P.row_per_cta != 0;
  const long long row_id =
      shared_row ? blockIdx.x : static_cast<long long>(blockIdx.x) * kCombineWarps + warp;
  const int nseq = P.seq_list ? P.list_len : P.batch;
  if (row_id >= static_cast<long long>(nseq) * P.R) return;
  const int b = P.seq_list ? P.seq_list[row_id / P.R] : static_cast<int>(row_id / P.R);
  if (b < 0) return;
  const int r = static_cast<int>(row_id % P.R);
  const int n = P.num_splits[b + 1] - P.num_splits[b];
  const int base = P.ws_base ? P.ws_base[b] : P.num_splits[b];
  if (!kFusedOut && n <= 1) return;  // written directly by the decode kernel

  // LSE of the merged row: max-subtracted log-sum-exp of the split LSEs
  const float* lse_i = P.ws_lse + (size_t)base * P.R + r;
  float m = -INFINITY;
  for (int i = lane; i < n; i += 32) m = fmaxf(m, lse_i[(size_t)i * P.R]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.f;
  if (m != -INFINITY)
    for (int i = lane; i < n; i += 32) sum += expf(lse_i[(size_t)i * P.R] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  float lse = (m == -INFINITY) ? -INFINITY : m + logf(sum);
  if (P.sink) {
    // the head's sink logit joins the normaliser (no value row)
    const float sk = P.sink[r % P.h_q];
    if (sk != -INFINITY) {
      if (lse == -INFINITY) {
        lse = sk;
      } else {
        const float mp = fmaxf(lse, sk);
        lse = mp + logf(expf(lse - mp) + expf(sk - mp));
      }
    }
  }

  // O = sum_i exp(LSE_i - LSE) O_i
  const int ngroups = P.d_v / 4;
  const float4* src0 = reinterpret_cast<const float4*>(P.ws_o + ((size_t)base * P.R + r) * P.d_v);
  const size_t stride = (size_t)P.R * P.d_v / 4;  // float4s between consecutive splits
  float4 acc[kCombineGroups];
#pragma unroll
  for (int j = 0; j < kCombineGroups; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int k_first = shared_row ? warp : 0;
  const int k_step = shared_row ? kCombineWarps : 1;
  for (int c0 = 0; c0 < n; c0 += 32) {
    float wl = 0.f;
    if (c0 + lane < n) {
      const float li = lse_i[(size_t)(c0 + lane) * P.R];
      wl = (lse == -INFINITY || li == -INFINITY) ? 0.f : expf(li - lse);
    }
    const int cn = min(32, n - c0);
    int k = k_first;
    for (; kPairs && k + k_step < cn; k += 2 * k_step) {
      const float w0 = __shfl_sync(0xffffffffu, wl, k);
      const float w1 = __shfl_sync(0xffffffffu, wl, k + k_step);
      const float4* s0 = src0 + (size_t)(c0 + k) * stride;
      const float4* s1 = s0 + (size_t)k_step * stride;
      float4 v0[kCombineGroups], v1[kCombineGroups];
#pragma unroll
      for (int j = 0; j < kCombineGroups; ++j) {
        const int g = lane + 32 * j;
        if (g < ngroups) {
          v0[j] = s0[g];
          v1[j] = s1[g];
        }
      }
#pragma unroll
      for (int j = 0; j < kCombineGroups; ++j) {
        if (lane + 32 * j < ngroups) {
          fma_acc(acc[j], w0, v0[j]);
          fma_acc(acc[j], w1, v1[j]);
        }
      }
    }
    for (; k < cn; k += k_step) {
      const float w = __shfl_sync(0xffffffffu, wl, k);
      const float4* src = src0 + (size_t)(c0 + k) * stride;
#pragma unroll
      for (int j = 0; j < kCombineGroups; ++j) {
        const int g = lane + 32 * j;
        if (g < ngroups) fma_acc(acc[j], w, src[g]);
      }
    }
  }

  if (shared_row) {  // add the warps' partial sums; warp 0 finishes the row
    if (warp > 0) {
#pragma unroll
      for (int j = 0; j < kCombineGroups; ++j)
        if (lane + 32 * j < ngroups) s_acc[warp - 1][lane + 32 * j] = acc[j];
    }
    __syncthreads();
    if (warp > 0) return;
#pragma unroll
    for (int j = 0; j < kCombineGroups; ++j) {
      const int g = lane + 32 * j;
      if (g < ngroups)
        for (int w = 0; w < kCombineWarps - 1; ++w) {
          const float4 v = s_acc[w][g];
          acc[j].x += v.x;
          acc[j].y += v.y;
          acc[j].z += v.z;
          acc[j].w += v.w;
        }
    }
  }

  const size_t row = (size_t)b * P.R + r;
  if (!kFusedOut) {
#pragma unroll
    for (int j = 0; j < kCombineGroups; ++j) {
      const int g = lane + 32 * j;
      if (g < ngroups) {
        uint2 pk;
        pk.x = ptx::pack_bf16x2(acc[j].x, acc[j].y);
        pk.y = ptx::pack_bf16x2(acc[j].z, acc[j].w);
        *reinterpret_cast<uint2*>(P.out + row * P.d_v + 4 * g) = pk;
      }
    }
    if (lane == 0) P.lse[row] = lse;
    return;
  }

  // ---- fused epilogue: conjugate RoPE on dims 512..575, absmax, E4M3 cast
  const int L = P.seqlens[b];
  const double pos = P.positions ? static_cast<double>(P.positions[b]) : static_cast<double>(L - 1);
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kCombineGroups; ++j) {
    const int g = lane + 32 * j;
    if (g < ngroups && 4 * g >= kNope) {
      const int k0 = (4 * g - kNope) / 2;  // pair index of (x, y); (z, w) is k0 + 1
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float sn, c;
        rope_sincos(pos, P.inv_freq[k0 + e], &sn, &c);
        float& a = e ? acc[j].z : acc[j].x;
        float& bb = e ? acc[j].w : acc[j].y;
        const float na = a * c + bb * sn;  // rotate by -theta
        const float nb = -a * sn + bb * c;
        a = na;
        bb = nb;
      }
    }
    if (g < ngroups)
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(acc[j].x), fabsf(acc[j].y)),
                               fmaxf(fabsf(acc[j].z), fabsf(acc[j].w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? amax / 448.0f : 1.0f;
#pragma unroll
  for (int j = 0; j < kCombineGroups; ++j) {
    const int g = lane + 32 * j;
    if (g < ngroups)
      *reinterpret_cast<uint32_t*>(P.out_fp8 + row * kD + 4 * g) =
          cvt_e4m3x4(acc[j].x / scale, acc[j].y / scale, acc[j].z / scale, acc[j].w / scale);
  }
  if (lane == 0) {
    P.out_scale[row] = scale;
    P.lse[row] = lse;
  }
}

// Device-side planner: one CTA stages the cost prefix sums of at most
// kPlanMaxBatch sequences in shared memory (larger batches are rejected by
// the entry points) and evaluates the host planner's closed forms, every
// sequence and part in parallel.
constexpr int kPlanThreads = 256;
constexpr int kPlanMaxBatch = 8192;  // prefix sums live in shared memory

// Block-wide exclusive prefix sum of one value per thread; returns the
// thread's exclusive sum, and the block total through *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total) {
  __shared__ int s_warp[kPlanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kPlanThreads / 32; ++w) {
    const int t = s_warp[w];
    before += w < warp ? t : 0;
    all += t;
  }
  __syncthreads();  // s_warp reusable
  *total = all;
  return before + x - v;
}

// Split-KV planner of one CTA: the closed forms of mla_common.h evaluated in
// parallel (prefix sums by block scans, one metadata row per thread).
__device__ void plan_block(const int32_t* seqlens, int batch, int num_parts, const PlanParams pp,
                           int32_t* metadata, int32_t* num_splits, int32_t* ws_base,
                           int32_t* split_list, int list_cap) {
  const int o = pp.o, g = pp.g;
  const int u = g * kPlanTileCost;
  __shared__ int32_t C[kPlanMaxBatch + 1];
  const int tid = threadIdx.x;
  int carry = 0;
  for (int base = 0; base < batch; base += kPlanThreads) {
    const int b = base + tid;
    const int L = b < batch ? seqlens[b] : 0;
    const int v = b < batch ? o + u * granules_of(L, g) : 0;
    int chunk_total;
    const int ex = block_exclusive_scan(v, &chunk_total);
    if (b < batch) C[b] = carry + ex;
    carry += chunk_total;
  }
  if (tid == 0) C[batch] = carry;
  __syncthreads();
  const int w = plan_width(carry, num_parts, pp);
  for (int p = tid; p < num_parts; p += kPlanThreads)
    plan_part_row(C, batch, w, o, g, p, metadata + p * kMetaInts);
  int nsum = 0;
  if (tid == 0) num_splits[0] = 0;
  for (int base = 0; base < batch; base += kPlanThreads) {
    const int b = base + tid;
    const int v = b < batch ? plan_last_part(C, b, w, u) - plan_first_part(C, b, w, o) + 1 : 0;
    int chunk_total;
    const int ex = block_exclusive_scan(v, &chunk_total);
    if (b < batch) num_splits[b + 1] = nsum + ex + v;
    nsum += chunk_total;
  }
  if (ws_base) {
    // compact partial rows: only sequences split over several parts own rows
    // (at most 2 num_parts in all: a part holds at most two split segments)
    int wsum = 0;
    for (int base = 0; base < batch; base += kPlanThreads) {
      const int b = base + tid;
      const int v = b < batch ? plan_last_part(C, b, w, u) - plan_first_part(C, b, w, o) + 1 : 0;
      int chunk_total;
      const int ex = block_exclusive_scan(v > 1 ? v : 0, &chunk_total);
      if (b < batch) ws_base[b] = wsum + ex;
      wsum += chunk_total;
    }
  }
  if (split_list) {
    // the split sequences in order (at most num_parts - 1: each lies across
    // a part boundary), then -1 up to list_cap
    for (int i = tid; i < list_cap; i += kPlanThreads) split_list[i] = -1;
    __syncthreads();
    int ksum = 0;
    for (int base = 0; base < batch; base += kPlanThreads) {
      const int b = base + tid;
      const int v = b < batch ? plan_last_part(C, b, w, u) - plan_first_part(C, b, w, o) + 1 : 0;
      int chunk_total;
      const int ex = block_exclusive_scan(v > 1 ? 1 : 0, &chunk_total);
      if (b < batch && v > 1 && ksum + ex < list_cap) split_list[ksum + ex] = b;
      ksum += chunk_total;
    }
  }
}

__global__ void __launch_bounds__(kPlanThreads) mla_plan_kernel(const int32_t* seqlens, int batch,
                                                               int num_parts, const PlanParams pp,
                                                               int32_t* metadata,
                                                               int32_t* num_splits,
                                                               int32_t* ws_base,
                                                               int32_t* split_list, int list_cap) {
  ptx::grid_dep_wait();
  ptx::grid_dep_launch();  // the decode grid waits for this one at its start
  plan_block(seqlens, batch, num_parts, pp, metadata, num_splits, ws_base, split_list, list_cap);
}

}  // namespace mla

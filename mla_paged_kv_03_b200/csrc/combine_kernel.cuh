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
};

__device__ __forceinline__ uint32_t cvt_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(a), "f"(b));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(c), "f"(d));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// One CTA per row; thread i owns the float4 group i of the row (d_v / 4 = 128
// or 144 threads).  The split weights are formed once in shared memory.
constexpr int kCombineMaxSplits = 1024;  // splits of one sequence (<= SM parts)
constexpr int kCombineThreads = 160;

template <bool kFusedOut>
__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(const CombineParams P) {
  __shared__ float s_w[kCombineMaxSplits];
  __shared__ float s_red[kCombineThreads / 32];
  __shared__ float s_lse;
  ptx::grid_dep_wait();  // the decode kernel's partials are complete
  const int row_id = blockIdx.x;
  const int b = row_id / P.R;
  const int r = row_id % P.R;
  const int base = P.num_splits[b];
  const int n = P.num_splits[b + 1] - base;
  if (!kFusedOut && n <= 1) return;  // written directly by the decode kernel
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kCombineThreads / 32;

  // max over the split LSEs
  float m = -INFINITY;
  for (int i = tid; i < n; i += kCombineThreads) {
    const float li = P.ws_lse[(size_t)(base + i) * P.R + r];
    s_w[i] = li;
    m = fmaxf(m, li);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  m = s_red[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) m = fmaxf(m, s_red[w]);
  __syncthreads();
  float sum = 0.f;
  if (m != -INFINITY)
    for (int i = tid; i < n; i += kCombineThreads) sum += expf(s_w[i] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_red[warp] = sum;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += s_red[w];
    s_lse = (m == -INFINITY) ? -INFINITY : m + logf(t);
  }
  __syncthreads();
  const float lse = s_lse;
  for (int i = tid; i < n; i += kCombineThreads)
    s_w[i] = (lse == -INFINITY || s_w[i] == -INFINITY) ? 0.f : expf(s_w[i] - lse);
  __syncthreads();

  const int ngroups = P.d_v / 4;
  const int g = tid;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (g < ngroups) {
    const float4* src = reinterpret_cast<const float4*>(P.ws_o + ((size_t)base * P.R + r) * P.d_v) + g;
    const size_t stride = (size_t)P.R * P.d_v / 4;  // float4s between consecutive splits
    int i = 0;
    for (; i + 4 <= n; i += 4) {
      const float4 v0 = src[(i + 0) * stride], v1 = src[(i + 1) * stride];
      const float4 v2 = src[(i + 2) * stride], v3 = src[(i + 3) * stride];
      const float w0 = s_w[i], w1 = s_w[i + 1], w2 = s_w[i + 2], w3 = s_w[i + 3];
      acc.x += w0 * v0.x + w1 * v1.x + w2 * v2.x + w3 * v3.x;
      acc.y += w0 * v0.y + w1 * v1.y + w2 * v2.y + w3 * v3.y;
      acc.z += w0 * v0.z + w1 * v1.z + w2 * v2.z + w3 * v3.z;
      acc.w += w0 * v0.w + w1 * v1.w + w2 * v2.w + w3 * v3.w;
    }
    for (; i < n; ++i) {
      const float4 v = src[i * stride];
      const float w = s_w[i];
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
  }

  const size_t row = (size_t)b * P.R + r;
  if (!kFusedOut) {
    if (g < ngroups) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(P.out + row * P.d_v + 4 * g) = pk;
    }
    if (tid == 0) P.lse[row] = lse;
    return;
  }

  // ---- fused epilogue: conjugate RoPE on dims 512..575, absmax, E4M3 cast
  if (g < ngroups && 4 * g >= kNope) {
    const int L = P.seqlens[b];
    const double pos =
        P.positions ? static_cast<double>(P.positions[b]) : static_cast<double>(L - 1);
    const int k0 = (4 * g - kNope) / 2;  // pair index of (x, y); (z, w) is k0 + 1
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float sn, c;
      rope_sincos(pos, P.inv_freq[k0 + e], &sn, &c);
      float& a = e ? acc.z : acc.x;
      float& bb = e ? acc.w : acc.y;
      const float na = a * c + bb * sn;  // rotate by -theta
      const float nb = -a * sn + bb * c;
      a = na;
      bb = nb;
    }
  }
  float amax = 0.f;
  if (g < ngroups)
    amax = fmaxf(fmaxf(fabsf(acc.x), fabsf(acc.y)), fmaxf(fabsf(acc.z), fabsf(acc.w)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __syncthreads();
  if (lane == 0) s_red[warp] = amax;
  __syncthreads();
  amax = s_red[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) amax = fmaxf(amax, s_red[w]);
  const float scale = amax > 0.f ? amax / 448.0f : 1.0f;
  if (g < ngroups) {
    const uint32_t codes =
        cvt_e4m3x4(acc.x / scale, acc.y / scale, acc.z / scale, acc.w / scale);
    *reinterpret_cast<uint32_t*>(P.out_fp8 + row * kD + 4 * g) = codes;
  }
  if (tid == 0) {
    P.out_scale[row] = scale;
    P.lse[row] = lse;
  }
}

// Device-side planner: the block stages tiles_of(seqlens) in shared memory
// (or, for very large batches, in the caller's scratch), then one thread runs
// the same planner the host uses.
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
__device__ void plan_block(const int32_t* seqlens, int batch, int num_parts,
                           int32_t* metadata, int32_t* num_splits) {
  __shared__ int32_t C[kPlanMaxBatch + 1];
  const int tid = threadIdx.x;
  int carry = 0;
  for (int base = 0; base < batch; base += kPlanThreads) {
    const int b = base + tid;
    const int L = b < batch ? seqlens[b] : 0;
    const int v = b < batch ? tiles_of(L) + kSegmentOverheadTiles : 0;
    int chunk_total;
    const int ex = block_exclusive_scan(v, &chunk_total);
    if (b < batch) C[b] = carry + ex;
    carry += chunk_total;
  }
  if (tid == 0) C[batch] = carry;
  __syncthreads();
  const int w = plan_width(carry, num_parts);
  for (int p = tid; p < num_parts; p += kPlanThreads)
    plan_part_row(C, batch, w, p, metadata + p * kMetaInts);
  int nsum = 0;
  if (tid == 0) num_splits[0] = 0;
  for (int base = 0; base < batch; base += kPlanThreads) {
    const int b = base + tid;
    const int v = b < batch ? plan_last_part(C, b, w) - plan_first_part(C, b, w) + 1 : 0;
    int chunk_total;
    const int ex = block_exclusive_scan(v, &chunk_total);
    if (b < batch) num_splits[b + 1] = nsum + ex + v;
    nsum += chunk_total;
  }
}

__global__ void __launch_bounds__(kPlanThreads) mla_plan_kernel(const int32_t* seqlens, int batch,
                                                               int num_parts, int32_t* metadata,
                                                               int32_t* num_splits) {
  ptx::grid_dep_wait();
  ptx::grid_dep_launch();  // the decode grid waits for this one at its start
  plan_block(seqlens, batch, num_parts, metadata, num_splits);
}

}  // namespace mla

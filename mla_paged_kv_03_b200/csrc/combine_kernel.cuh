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

// One warp per row; lane l owns float4 groups l, l+32, ... of the row.
template <bool kFusedOut>
__global__ void __launch_bounds__(256) mla_combine_kernel(const CombineParams P) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= P.batch * P.R) return;
  const int b = warp / P.R;
  const int r = warp % P.R;
  const int base = P.num_splits[b];
  const int n = P.num_splits[b + 1] - base;
  if (!kFusedOut && n <= 1) return;  // written directly by the decode kernel

  float m = -INFINITY;
  for (int i = 0; i < n; ++i) m = fmaxf(m, P.ws_lse[(size_t)(base + i) * P.R + r]);
  float sum = 0.f;
  if (m != -INFINITY)
    for (int i = 0; i < n; ++i) sum += expf(P.ws_lse[(size_t)(base + i) * P.R + r] - m);
  const float lse = (m == -INFINITY) ? -INFINITY : m + logf(sum);

  constexpr int kMaxG = 5;  // float4 groups per lane (576 / 4 / 32 -> 5)
  const int ngroups = P.d_v / 4;
  float4 acc[kMaxG];
#pragma unroll
  for (int j = 0; j < kMaxG; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (m != -INFINITY) {
    for (int i = 0; i < n; ++i) {
      const float li = P.ws_lse[(size_t)(base + i) * P.R + r];
      if (li == -INFINITY) continue;
      const float w = expf(li - lse);
      const float4* src =
          reinterpret_cast<const float4*>(P.ws_o + ((size_t)(base + i) * P.R + r) * P.d_v);
#pragma unroll
      for (int j = 0; j < kMaxG; ++j) {
        const int g = lane + 32 * j;
        if (g < ngroups) {
          const float4 v = src[g];
          acc[j].x += w * v.x;
          acc[j].y += w * v.y;
          acc[j].z += w * v.z;
          acc[j].w += w * v.w;
        }
      }
    }
  }

  const size_t row = (size_t)b * P.R + r;
  if (!kFusedOut) {
#pragma unroll
    for (int j = 0; j < kMaxG; ++j) {
      const int g = lane + 32 * j;
      if (g < ngroups) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j].x, acc[j].y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j].z, acc[j].w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
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
  for (int j = 0; j < kMaxG; ++j) {
    const int g = lane + 32 * j;
    if (g < ngroups && 4 * g >= kNope) {
      const int k0 = (4 * g - kNope) / 2;  // pair index of (x, y); (z, w) is k0 + 1
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float s, c;
        rope_sincos(pos, P.inv_freq[k0 + e], &s, &c);
        float& a = e ? acc[j].z : acc[j].x;
        float& bb = e ? acc[j].w : acc[j].y;
        const float na = a * c + bb * s;   // rotate by -theta
        const float nb = -a * s + bb * c;
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
  for (int j = 0; j < kMaxG; ++j) {
    const int g = lane + 32 * j;
    if (g < ngroups) {
      const uint32_t codes = cvt_e4m3x4(acc[j].x / scale, acc[j].y / scale, acc[j].z / scale,
                                        acc[j].w / scale);
      *reinterpret_cast<uint32_t*>(P.out_fp8 + row * kD + 4 * g) = codes;
    }
  }
  if (lane == 0) {
    P.out_scale[row] = scale;
    P.lse[row] = lse;
  }
}

// Device-side planner launch: one thread runs the same planner the host uses.
__global__ void mla_plan_kernel(const int32_t* seqlens, int batch, int num_parts,
                                int32_t* metadata, int32_t* num_splits) {
  if (blockIdx.x == 0 && threadIdx.x == 0) plan_splits(seqlens, batch, num_parts, metadata, num_splits);
}

// Planner over `batch` items of equal length `len` (sparse decode).
__global__ void mla_plan_uniform_kernel(int len, int batch, int num_parts, int32_t* lens_scratch,
                                        int32_t* metadata, int32_t* num_splits) {
  for (int i = threadIdx.x; i < batch; i += blockDim.x) lens_scratch[i] = len;
  __syncthreads();
  if (threadIdx.x == 0) plan_splits(lens_scratch, batch, num_parts, metadata, num_splits);
}

}  // namespace mla

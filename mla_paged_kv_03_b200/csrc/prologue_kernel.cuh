// prologue_kernel.cuh -- the fused decode's query prologue: Q RMSNorm, then
// RoPE of dims 512..575 at the query position, rounded once to bf16.
// [FlashMLA fused norm-RoPE-attention-RoPE-cast kernel card, "Arithmetic
// intensity": the normalisation and the rotation of Q precede the attention]
//
//   y_d = q_d * g_d / sqrt(mean_d(q_d^2) + eps)            (d < 576)
//   (y_{512+2k}, y_{513+2k}) rotated by theta_k = pos * base^(-2k/64)
//
// The transform runs once per query row, here, rather than in every CTA of
// the attention grid that reads the row: a batch-1 decode otherwise repeats it
// for the same rows on every SM.  The rows are written as a plain [rows, 576]
// bf16 matrix, which the attention kernel then loads by TMA like a dense
// query.  The arithmetic is fp64 with one bf16 rounding at the end, so the
// rounding decision agrees with an fp64 reference except at exact ties.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "decode_kernel.cuh"

namespace mla {

struct FusedQParams {
  const __nv_bfloat16* q_raw;  // [rows, 576]; row r belongs to sequence r / R
  const float* gain;           // [576]
  float eps;
  const int32_t* positions;  // nullable: position = seqlens[b] - 1
  const int32_t* seqlens;    // [batch] (used only when positions is null)
  int rows;                  // batch * R
  int R;                     // query rows per sequence (h_q)
  double inv_freq[kRope / 2];  // base^(-2k/64), computed on the host in fp64
  __nv_bfloat16* q_out;        // [rows, 576]
};

constexpr int kPrologueWarps = 8;

// One warp per row; lane l holds the row's 16-byte units l, l + 32 and l + 64
// (dims 8u .. 8u + 7), and computes cos/sin of rotation pair l.
__global__ void __launch_bounds__(32 * kPrologueWarps)
    mla_fused_q_kernel(const FusedQParams P) {
  __shared__ double cs[kPrologueWarps][kRope / 2][2];
  // Launched in stream order (after all earlier work of the stream), so the
  // inputs are complete; the attention grid may start its setup now and
  // waits for this grid's completion before it reads the rows.
  ptx::grid_dep_launch();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kPrologueWarps + warp;
  if (r < P.rows) {
    const int b = r / P.R;
    const double pos = P.positions ? static_cast<double>(P.positions[b])
                                   : static_cast<double>(P.seqlens[b] - 1);
    double sn, c;
    rope_sincos64(pos, P.inv_freq[lane], &sn, &c);
    cs[warp][lane][0] = c;
    cs[warp][lane][1] = sn;
    __syncwarp();
    const __nv_bfloat16* src = P.q_raw + static_cast<size_t>(r) * kD;
    __nv_bfloat16* dst = P.q_out + static_cast<size_t>(r) * kD;
    uint4 w[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int uu = lane + 32 * j;
      w[j] = uu < kD / 8 ? *reinterpret_cast<const uint4*>(src + uu * 8) : make_uint4(0, 0, 0, 0);
    }
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w[j]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        ss = fma(static_cast<double>(f.x), static_cast<double>(f.x), ss);
        ss = fma(static_cast<double>(f.y), static_cast<double>(f.y), ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const double inv = 1.0 / sqrt(ss / static_cast<double>(kD) + P.eps);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int uu = lane + 32 * j;
      if (uu < kD / 8) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w[j]);
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(P.gain + uu * 8));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(P.gain + uu * 8 + 4));
        const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        double y[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h[e]);
          y[2 * e] = static_cast<double>(f.x) * inv * static_cast<double>(gv[2 * e]);
          y[2 * e + 1] = static_cast<double>(f.y) * inv * static_cast<double>(gv[2 * e + 1]);
        }
        if (uu >= kNope / 8) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k = (uu * 8 - kNope) / 2 + e;
            const double cc = cs[warp][k][0], s = cs[warp][k][1];
            const double a = y[2 * e], bq = y[2 * e + 1];
            y[2 * e] = a * cc - bq * s;
            y[2 * e + 1] = a * s + bq * cc;
          }
        }
        uint4 o;
        o.x = ptx::pack_bf16x2_f64(y[0], y[1]);
        o.y = ptx::pack_bf16x2_f64(y[2], y[3]);
        o.z = ptx::pack_bf16x2_f64(y[4], y[5]);
        o.w = ptx::pack_bf16x2_f64(y[6], y[7]);
        *reinterpret_cast<uint4*>(dst + uu * 8) = o;
      }
    }
  }
}

}  // namespace mla

// sink_kernel.cuh -- attention sinks of the sparse prefill: one logit per
// head that joins the softmax normaliser without a value row.  For a row with
// output O and log-sum-exp LSE over its tokens, and the head's sink logit s:
//   LSE' = log(e^LSE + e^s),   O' = O * e^(LSE - LSE')
// (a row without tokens keeps O = 0 and gets LSE' = s).  Applied in place
// after the split combine.  [FlashMLA (AI Wiki), "Interfaces": sparse prefill
// takes an optional attention-sink argument]
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace mla {

constexpr int kSinkWarps = 8;

// The sparse prefill's per-token lengths: topk_length[t] clamped to [0, topk],
// or topk for every token when no lengths are given.
__global__ void __launch_bounds__(256)
    mla_prefill_lengths_kernel(const int32_t* topk_len, int topk, int s_q, int32_t* out) {
  ptx::grid_dep_wait();
  const int t = blockIdx.x * 256 + threadIdx.x;
  if (t >= s_q) return;
  const int l = topk_len ? topk_len[t] : topk;
  out[t] = l < 0 ? 0 : (l < topk ? l : topk);
}

// One warp per (token, head) row of `d_v` bf16 values (d_v a multiple of 8).
__global__ void __launch_bounds__(32 * kSinkWarps)
    mla_sink_kernel(__nv_bfloat16* out, float* lse, const float* sink, long long rows, int h_q,
                    int d_v) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kSinkWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float s = sink[row % h_q];
  if (s == -INFINITY) return;
  const float l = lse[row];
  float lp, f;
  if (l == -INFINITY) {
    lp = s;
    f = 0.f;
  } else {
    const float m = fmaxf(l, s);
    lp = m + logf(expf(l - m) + expf(s - m));
    f = expf(l - lp);
  }
  uint4* o = reinterpret_cast<uint4*>(out + row * d_v);
  for (int u = lane; u < d_v / 8; u += 32) {
    uint4 v = o[u];
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      w[e] = ptx::pack_bf16x2(x.x * f, x.y * f);
    }
    o[u] = v;
  }
  if (lane == 0) lse[row] = lp;
}

}  // namespace mla

// prefill_kernel.cuh -- the sparse prefill's per-token top-k lengths.
// [FlashMLA (AI Wiki), "Interfaces": sparse prefill takes an optional
// per-token top-k length and an optional attention sink]
//
// The attention sinks themselves (one logit per head that joins the softmax
// normaliser without a value row: LSE' = log(e^LSE + e^s), O' = O e^(LSE -
// LSE'), and a row without tokens gets O = 0, LSE' = s) are folded into the
// rows' normalisation where each row is finished: the CTA-pair kernel's
// epilogue for tokens held by one part, the split combine for the others.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace mla {

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

}  // namespace mla

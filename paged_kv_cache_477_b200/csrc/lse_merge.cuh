// lse_merge.cuh -- combine split-KV decode partials by log-sum-exp.
//
// Flash-decoding's second step: each split of a long context wrote its
// normalised partial output and log2-sum-exp; this kernel weighs them into the
// final row ("从零构建CUDA推理引擎：Tiny-Infer项目的技术深度解析", section
// "Flash Attention：内存与计算的重平衡": the online softmax merges partial
// maxima and sums; the split form applies the same rule across CTAs).
#pragma once
#include "decode_attn.cuh"

namespace pkv {

// ----------------------------------------------------------------------------
// Log-sum-exp merge of split partials (log2 domain):
//   out = sum_c 2^{lse_c - M} o_c / sum_c 2^{lse_c - M},  M = max_c lse_c,
// over the splits that hold at least one key of the sequence.
// ----------------------------------------------------------------------------
struct MergeParams {
  __nv_bfloat16* out;         // [B][Hq][D]
  const float* o_part;        // [B][Hq][C][D]
  const float* lse_part;      // [B][Hq][C]
  const int32_t* context_lens;
  int32_t Hq, num_splits, pages_per_split, cap_tokens, window;
};

template <int D>
__global__ void __launch_bounds__(D) lse_merge_kernel(const __grid_constant__ MergeParams p) {
  grid_dependency_wait();  // the split kernel's partials (no-op when launched plainly)
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  int L = __ldg(p.context_lens + b);
  L = L < 0 ? 0 : (L > p.cap_tokens ? p.cap_tokens : L);
  const int npages = (L + kPageRows - 1) / kPageRows - window_first_key(L, p.window) / kPageRows;
  const int nval = (npages + p.pages_per_split - 1) / p.pages_per_split;
  const size_t row = (size_t)b * p.Hq + h;
  const float* lse = p.lse_part + row * p.num_splits;
  const float* o = p.o_part + row * p.num_splits * D;
  // Loads are issued MU splits at a time, predicated past nval, so a
  // sequence's splits cost two load round trips per MU of them instead of one
  // dependent load per split.  Every split below nval holds at least one page
  // and wrote its partial (o = 0 and lse = -inf when a window masked all its
  // rows).
  constexpr int MU = 8;
  float M = -INFINITY;
  for (int c0 = 0; c0 < nval; c0 += MU) {
    float l8[MU];
#pragma unroll
    for (int i = 0; i < MU; ++i) l8[i] = c0 + i < nval ? lse[c0 + i] : -INFINITY;
#pragma unroll
    for (int i = 0; i < MU; ++i) M = fmaxf(M, l8[i]);
  }
  float ws = 0.f, a = 0.f;
  for (int c0 = 0; c0 < nval; c0 += MU) {
    float l8[MU], o8[MU];
#pragma unroll
    for (int i = 0; i < MU; ++i) {
      const bool in = c0 + i < nval;
      l8[i] = in ? lse[c0 + i] : -INFINITY;
      o8[i] = in ? o[(size_t)(c0 + i) * D + d] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < MU; ++i) {
      const float w = l8[i] == -INFINITY ? 0.f : ex2(l8[i] - M);
      ws += w;
      a = fmaf(w, o8[i], a);
    }
  }
  p.out[row * D + d] = __float2bfloat16_rn(ws > 0.f ? a / ws : 0.f);
}

}  // namespace pkv

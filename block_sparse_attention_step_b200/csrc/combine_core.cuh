// Log-sum-exp merge of S split partials of one (b, query head) row:
//   lse = log sum_s e^{lse_s},  out[d] = sum_s e^{lse_s - lse} o_s[d]
// (empty splits carry lse_s = -inf and weigh nothing).
#pragma once

#include "seer_common.cuh"

namespace seer {

__device__ __forceinline__ uint16_t to_bf16_bits(float x) {
  const __nv_bfloat16 v = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t*>(&v);
}

struct LoadReadOnly {  // data written by an earlier kernel
  __device__ __forceinline__ float operator()(const float* p) const { return __ldg(p); }
};
struct LoadL2 {  // data written by other CTAs of this kernel
  __device__ __forceinline__ float operator()(const float* p) const { return __ldcg(p); }
};

// One output element of one (b, query head) row, every split's data loaded
// in a single batch (no dependent round trip per split):
//   m = max_s lse_s, w_s = e^{lse_s - m}, tot = sum_s w_s (in split order),
//   out = (sum_s w_s o_s) * (1 / tot), lse = m + log(tot).
// lse_row: [S]; o: split 0 of this dim (split stride kHeadDim).  Every thread
// computes the weights itself, so the result does not depend on how many
// threads share a row.
template <typename LOAD>
__device__ __forceinline__ float combine_element(const float* lse_row, const float* o, int S,
                                                 float* lse_merged, LOAD load) {
  constexpr int kChunk = 16;
  float m = -INFINITY;
  for (int s0 = 0; s0 < S; s0 += kChunk) {
    float v[kChunk];
#pragma unroll
    for (int i = 0; i < kChunk; ++i) v[i] = (s0 + i < S) ? load(lse_row + s0 + i) : -INFINITY;
#pragma unroll
    for (int i = 0; i < kChunk; ++i) m = fmaxf(m, v[i]);
  }
  float tot = 0.f, acc = 0.f;
  if (m != -INFINITY) {
    for (int s0 = 0; s0 < S; s0 += kChunk) {
      float l[kChunk], x[kChunk];
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        const bool in = s0 + i < S;
        l[i] = in ? load(lse_row + s0 + i) : -INFINITY;
        x[i] = in ? load(o + (int64_t)(s0 + i) * kHeadDim) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        if (s0 + i < S) {
          const float w = expf(l[i] - m);
          tot += w;
          if (w != 0.f) acc += w * x[i];
        }
      }
    }
  }
  *lse_merged = tot > 0.f ? m + logf(tot) : -INFINITY;
  return tot > 0.f ? acc * (1.f / tot) : 0.f;
}

}  // namespace seer

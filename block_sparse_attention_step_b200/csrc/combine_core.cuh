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
          tot = __fadd_rn(tot, w);
          if (w != 0.f) acc = __fmaf_rn(w, x[i], acc);
        }
      }
    }
  }
  *lse_merged = tot > 0.f ? m + logf(tot) : -INFINITY;
  return tot > 0.f ? __fmul_rn(acc, 1.f / tot) : 0.f;
}

// The same merge for one whole (b, query head) row by one warp: lane l takes
// dims 4l .. 4l+3 and every split's 4 values in one 16-byte load; the split
// weights come from the lse values through shuffles.  Same arithmetic in the
// same order as combine_element, so the same bits.  S <= 64; o_row 16-byte
// aligned.  out_row2 (optional) receives the same bf16 row.  PACKED: each
// lane stores its four values as one 8-byte word (both rows 8-byte aligned),
// so a warp writes a row in one contiguous 256-byte store.
template <typename LOAD4, bool PACKED = false>
__device__ __forceinline__ void combine_row_warp(const float* lse_row, const float* o_row, int S,
                                                 uint16_t* out_row, float* lse_out, LOAD4 load4,
                                                 uint16_t* out_row2 = nullptr) {
  const int lane = threadIdx.x & 31;
  const float la = lane < S ? __ldcg(lse_row + lane) : -INFINITY;
  const float lb = lane + 32 < S ? __ldcg(lse_row + lane + 32) : -INFINITY;
  float m = fmaxf(la, lb);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float tot = 0.f, acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const float l = __shfl_sync(0xffffffffu, s < 32 ? la : lb, s & 31);
      const float4 x = load4(o_row + (int64_t)s * kHeadDim + 4 * lane);
      const float w = expf(l - m);
      tot = __fadd_rn(tot, w);
      if (w != 0.f) {
        acc0 = __fmaf_rn(w, x.x, acc0);
        acc1 = __fmaf_rn(w, x.y, acc1);
        acc2 = __fmaf_rn(w, x.z, acc2);
        acc3 = __fmaf_rn(w, x.w, acc3);
      }
    }
  }
  const float r = tot > 0.f ? 1.f / tot : 0.f;
  const uint16_t v0 = to_bf16_bits(tot > 0.f ? __fmul_rn(acc0, r) : 0.f);
  const uint16_t v1 = to_bf16_bits(tot > 0.f ? __fmul_rn(acc1, r) : 0.f);
  const uint16_t v2 = to_bf16_bits(tot > 0.f ? __fmul_rn(acc2, r) : 0.f);
  const uint16_t v3 = to_bf16_bits(tot > 0.f ? __fmul_rn(acc3, r) : 0.f);
  if constexpr (PACKED) {
    const uint2 w = make_uint2((uint32_t)v0 | ((uint32_t)v1 << 16), (uint32_t)v2 | ((uint32_t)v3 << 16));
    *reinterpret_cast<uint2*>(out_row + 4 * lane) = w;
    if (out_row2 != nullptr) *reinterpret_cast<uint2*>(out_row2 + 4 * lane) = w;
  } else {
    out_row[4 * lane + 0] = v0;
    out_row[4 * lane + 1] = v1;
    out_row[4 * lane + 2] = v2;
    out_row[4 * lane + 3] = v3;
    if (out_row2 != nullptr) {
      out_row2[4 * lane + 0] = v0;
      out_row2[4 * lane + 1] = v1;
      out_row2[4 * lane + 2] = v2;
      out_row2[4 * lane + 3] = v3;
    }
  }
  if (lse_out != nullptr && lane == 0) *lse_out = tot > 0.f ? m + logf(tot) : -INFINITY;
}

struct Load4L2 {  // 16-byte loads of data written by other CTAs of this kernel
  __device__ __forceinline__ float4 operator()(const float* p) const {
    return __ldcg(reinterpret_cast<const float4*>(p));
  }
};

}  // namespace seer

// The one summation order every kernel uses for a pooled key (mean of the
// valid K rows of one block), so pooled keys agree bit for bit whichever
// kernel computes them: warp w of 8 adds rows w, w+8, w+16, ... in order into
// four running sums (lane l holds dims 4l .. 4l+3), then the 8 warp partials
// are added in warp order and divided by the number of valid rows.
#pragma once

#include "seer_common.cuh"

namespace seer {

constexpr int kPoolWarps = 8;

// base_lane: the block's row 0 for this KV head, already offset by 4 * lane.
__device__ __forceinline__ float4 pool_warp_partial(const uint16_t* base_lane,
                                                    int64_t stride_token, int valid, int warp) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  // at most bs / 8 = 16 rows per warp: fully unrolled so every load is in flight
#pragma unroll 16
  for (int t = warp; t < valid; t += kPoolWarps) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(base_lane + (int64_t)t * stride_token));
    a0 += __uint_as_float(v.x << 16);
    a1 += __uint_as_float(v.x & 0xffff0000u);
    a2 += __uint_as_float(v.y << 16);
    a3 += __uint_as_float(v.y & 0xffff0000u);
  }
  return make_float4(a0, a1, a2, a3);
}

// part: [kPoolWarps][kHeadDim] partials in shared memory.
__device__ __forceinline__ float pool_finish(const float* part, int d, int valid) {
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kPoolWarps; ++w) s += part[w * kHeadDim + d];
  return s / (float)valid;
}

// 128-dim dot product of a lane's 4 values with its 4 weights, summed over the
// warp with a fixed butterfly: the gate score order shared by every kernel.
__device__ __forceinline__ float warp_dot4(float4 a, float4 b) {
  float v = a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace seer

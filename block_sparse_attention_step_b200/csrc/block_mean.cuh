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
// The lane's four products are chained with explicit round-to-nearest
// intrinsics, which the compiler never re-contracts, so every kernel that
// inlines this gets the same bits.
__device__ __forceinline__ float warp_dot4(float4 a, float4 b) {
  float v = __fmaf_rn(a.w, b.w, __fmaf_rn(a.z, b.z, __fmaf_rn(a.y, b.y, __fmul_rn(a.x, b.x))));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Eight warp_dot4 at once, bit for bit: a[i] . b for i = 0..7 with 9 shuffles
// instead of 40.  Each exchange step pairs the same lanes as warp_dot4's
// butterfly (offsets 16, 8, 4, 2, 1) and adds the same two partial sums, but
// hands half of the rows still in play to the partner instead of all of
// them; lane l returns the product for row (l >> 2) & 7.
__device__ __forceinline__ float warp_dot4_x8(const float4 (&a)[8], float4 b) {
  const int lane = threadIdx.x & 31;
  float p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    p[i] = __fmaf_rn(a[i].w, b.w, __fmaf_rn(a[i].z, b.z, __fmaf_rn(a[i].y, b.y,
                                                                 __fmul_rn(a[i].x, b.x))));
  const bool hi4 = (lane & 16) != 0, hi3 = (lane & 8) != 0, hi2 = (lane & 4) != 0;
  float q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // keep rows 4*hi4 + i
    const float give = hi4 ? p[i] : p[4 + i];
    q[i] = (hi4 ? p[4 + i] : p[i]) + __shfl_xor_sync(0xffffffffu, give, 16);
  }
  float r[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {  // keep rows 4*hi4 + 2*hi3 + i
    const float give = hi3 ? q[i] : q[2 + i];
    r[i] = (hi3 ? q[2 + i] : q[i]) + __shfl_xor_sync(0xffffffffu, give, 8);
  }
  const float give = hi2 ? r[0] : r[1];  // keep row 4*hi4 + 2*hi3 + hi2
  float v = (hi2 ? r[1] : r[0]) + __shfl_xor_sync(0xffffffffu, give, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v;
}

}  // namespace seer

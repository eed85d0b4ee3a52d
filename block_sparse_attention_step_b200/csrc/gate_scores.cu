// a1: gate scores.  score[b,h,j] = gate_scale * g . kbar[b,h,j] with
// g = W[h] qbar and qbar the mean of the G query heads of KV head h.  The
// gate is query-aware without query pooling over time (SeerAttention-R
// Abstract); the mean over the GQA group of the per-head scores equals the
// score of the mean query because the score is linear in q.
//
// Grid (chunk of blocks, h, b); 256 threads.  Each CTA first forms g (the
// D x D mat-vec reads W[h] from L2: 64 KB shared by every CTA of head h),
// then streams its chunk of kbar rows, one warp per row, 4 rows in flight per
// warp, a 32-lane float4 dot product and a shuffle reduction per row.  The
// kbar stream is the HBM cost: NB * D * 4 bytes per (b, h).
#include "block_mean.cuh"
#include "seer_kernels.cuh"

namespace seer {

__global__ void __launch_bounds__(256) gate_scores_kernel(const GateParams p) {
  __shared__ __align__(16) float qbar[kHeadDim];
  __shared__ __align__(16) float gvec[kHeadDim];
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  const int j0 = blockIdx.x * p.blocks_per_cta;
  const int j1 = min(j0 + p.blocks_per_cta, p.max_blocks);
  float* out = p.scores + ((int64_t)b * p.Hkv + h) * p.max_blocks;

  if (j0 >= nb) {  // nothing valid in this chunk
    for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) out[j] = -INFINITY;
    return;
  }
  if (threadIdx.x < kHeadDim) {
    const uint16_t* qg = p.q + ((int64_t)b * p.Hq + (int64_t)h * p.G) * kHeadDim + threadIdx.x;
    float s = 0.f;
    for (int g = 0; g < p.G; ++g) s += __uint_as_float((uint32_t)__ldg(qg + g * kHeadDim) << 16);
    qbar[threadIdx.x] = s / (float)p.G;
  }
  __syncthreads();
  {
    const float4 qv = *reinterpret_cast<const float4*>(&qbar[4 * lane]);
    const float* W = p.w_gate + (int64_t)h * kHeadDim * kHeadDim;
#pragma unroll 4
    for (int row = warp; row < kHeadDim; row += 8) {
      const float4 w = __ldg(reinterpret_cast<const float4*>(W + row * kHeadDim + 4 * lane));
      const float v = warp_dot4(w, qv);
      if (lane == 0) gvec[row] = __fmul_rn(v, p.gate_scale);
    }
  }
  __syncthreads();
  const float4 gv = *reinterpret_cast<const float4*>(&gvec[4 * lane]);
  const float* kb = p.kbar + ((int64_t)b * p.Hkv + h) * p.max_blocks * kHeadDim + 4 * lane;
  bool bad = false;
  for (int jb = j0 + warp * 4; jb < j1; jb += 32) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u;
      v[u] = (j < nb && j < j1) ? __ldg(reinterpret_cast<const float4*>(kb + (int64_t)j * kHeadDim))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u;
      const float sc = warp_dot4(v[u], gv);
      if (lane == 0 && j < j1) {
        if (j < nb) {
          out[j] = sc;
          bad |= !isfinite(sc);
        } else {
          out[j] = -INFINITY;
        }
      }
    }
  }
  if (bad) flag_status(p.status, SEER_DEV_NONFINITE_SCORE);
}

cudaError_t run_gate_scores(const GateParams& p, int B, cudaStream_t stream) {
  dim3 grid((p.max_blocks + p.blocks_per_cta - 1) / p.blocks_per_cta, p.Hkv, B);
  gate_scores_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace seer

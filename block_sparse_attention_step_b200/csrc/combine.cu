// a4: log-sum-exp combine of the split-KV partials.
//   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) * o_s  (bf16, RNE)
// Empty splits carry lse_s = -inf and weigh nothing; if every split is empty
// the output is 0 and lse is -inf.
//
// One CTA of 128 threads (one per dim) per (b, query head).  The S weights are
// computed once into shared memory; each thread then reads its dim of every
// partial (coalesced 512-byte rows).
#include "seer_kernels.cuh"

namespace seer {

__global__ void __launch_bounds__(kHeadDim) combine_kernel(const CombineParams p) {
  __shared__ float w[kMaxSplits];
  __shared__ float inv_total, lse_total;
  const int64_t row = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;  // b * Hq + qh
  const float* lse = p.lse_part + row * p.S;
  if (threadIdx.x < 32) {
    float m = -INFINITY;
    for (int s = threadIdx.x; s < p.S; s += 32) m = fmaxf(m, __ldg(lse + s));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float tot = 0.f;
    for (int s = threadIdx.x; s < p.S; s += 32) {
      const float e = (m == -INFINITY) ? 0.f : expf(__ldg(lse + s) - m);
      w[s] = e;
      tot += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    if (threadIdx.x == 0) {
      inv_total = tot > 0.f ? 1.f / tot : 0.f;
      lse_total = tot > 0.f ? m + logf(tot) : -INFINITY;
    }
  }
  __syncthreads();
  const float* o = p.o_part + row * p.S * kHeadDim + threadIdx.x;
  float acc = 0.f;
  for (int s = 0; s < p.S; ++s) {
    const float ws = w[s];
    if (ws != 0.f) acc += ws * __ldg(o + (int64_t)s * kHeadDim);
  }
  const __nv_bfloat16 v = __float2bfloat16_rn(acc * inv_total);
  p.out[row * kHeadDim + threadIdx.x] = *reinterpret_cast<const uint16_t*>(&v);
  if (p.lse_out != nullptr && threadIdx.x == 0) p.lse_out[row] = lse_total;
}

cudaError_t run_combine(const CombineParams& p, int B, int Hq, cudaStream_t stream) {
  dim3 grid(Hq, B);
  combine_kernel<<<grid, kHeadDim, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace seer

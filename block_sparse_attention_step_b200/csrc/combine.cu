// a4: log-sum-exp combine of the split-KV partials.
//   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) * o_s  (bf16, RNE)
// Empty splits carry lse_s = -inf and weigh nothing; if every split is empty
// the output is 0 and lse is -inf.
//
// One CTA of 128 threads (one per dim) per (b, query head); each thread loads
// the row's S lse values and its dim of every partial in one batch.  In the
// whole step it is chained to the decode kernel by programmatic dependent
// launch and waits for it in griddepcontrol.wait.
#include "combine_core.cuh"
#include "seer_kernels.cuh"

namespace seer {

__global__ void __launch_bounds__(kHeadDim) combine_kernel(const CombineParams p) {
  pdl_wait();  // the partials come from the preceding decode grid
  const int64_t row = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;  // b * Hq + qh
  const int d = threadIdx.x;
  float lse;
  const float v = combine_element(p.lse_part + row * p.S, p.o_part + row * p.S * kHeadDim + d,
                                  p.S, &lse, LoadReadOnly{});
  const uint16_t bits = to_bf16_bits(v);
  p.out[row * kHeadDim + d] = bits;
  if (p.out_host != nullptr) p.out_host[row * kHeadDim + d] = bits;
  if (p.lse_out != nullptr && d == 0) p.lse_out[row] = lse;
}

// The step's chained combine: one warp per (b, query head) row
// (combine_row_warp: the same bits as combine_kernel), four rows per CTA,
// for partials on 16-byte boundaries; PACKED for 8-byte aligned outputs.
constexpr int kCombineRowsPerCta = 4;

template <bool PACKED>
__global__ void __launch_bounds__(kCombineRowsPerCta * 32)
    combine_rows_kernel(const CombineParams p, int rows) {
  pdl_wait();  // the partials come from the preceding decode grid
  const int row = blockIdx.x * kCombineRowsPerCta + (threadIdx.x >> 5);
  if (row >= rows) return;  // the whole warp
  combine_row_warp<Load4L2, PACKED>(
      p.lse_part + (int64_t)row * p.S, p.o_part + (int64_t)row * p.S * kHeadDim, p.S,
      p.out + (int64_t)row * kHeadDim, p.lse_out != nullptr ? p.lse_out + row : nullptr, Load4L2{},
      p.out_host != nullptr ? p.out_host + (int64_t)row * kHeadDim : nullptr);
}

cudaError_t run_combine_rows(const CombineParams& p, int B, int Hq, cudaStream_t stream,
                             bool pdl, bool packed) {
  const int rows = B * Hq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((rows + kCombineRowsPerCta - 1) / kCombineRowsPerCta);
  cfg.blockDim = dim3(kCombineRowsPerCta * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = packed ? cudaLaunchKernelEx(&cfg, combine_rows_kernel<true>, p, rows)
                         : cudaLaunchKernelEx(&cfg, combine_rows_kernel<false>, p, rows);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t run_combine(const CombineParams& p, int B, int Hq, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(Hq, B);
  cfg.blockDim = dim3(kHeadDim);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, combine_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace seer

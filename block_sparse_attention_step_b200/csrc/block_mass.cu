// Per-block attention mass of a decode step (the dense-mode target of the
// self-distilled gate, SeerAttention-R Abstract): for every (b, query head)
// and every selected block j,
//     mass_j = sum_{t in j, t < seqlen} p_t = sum_pieces e^{piece_lse - lse}
// where the decode kernel wrote each piece's ln sum_t e^{x_t} (16 tokens of
// one 64-token tile, natural log of the scaled scores) and lse is the row's
// merged log-sum-exp (the combine's lse output).  Blocks that were not
// selected carry no mass (0).
//
// One CTA of 256 threads per (b, query head): the (b, h) index row marks the
// selected blocks in shared memory, then one thread per block adds its pieces.
#include "seer_kernels.cuh"

namespace seer {

__global__ void __launch_bounds__(256) block_mass_kernel(const MassParams p) {
  __shared__ unsigned char selected[kMaxBlocks];
  const int b = blockIdx.y, qh = blockIdx.x;
  const int h = qh / p.G;
  const int64_t bh = (int64_t)b * p.Hkv + h;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  for (int j = threadIdx.x; j < p.max_blocks; j += blockDim.x) selected[j] = 0;
  __syncthreads();
  const int n = max(0, min(__ldg(p.n_sel + bh), p.k_max));
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int j = __ldg(p.idx + bh * p.k_max + i);
    if (j >= 0 && j < nb) selected[j] = 1;
  }
  __syncthreads();
  const int64_t row = (int64_t)b * p.Hq + qh;
  const float lse = __ldg(p.lse + row);
  const int pieces = (p.bs / kTileTokens) * 4;
  float* out = p.mass + row * p.max_blocks;
  for (int j = threadIdx.x; j < p.max_blocks; j += blockDim.x) {
    float m = 0.f;
    if (selected[j] && lse != -INFINITY) {
      const int subs = ceil_div_i(min(p.bs, L - j * p.bs), kTileTokens);
      const float* pl = p.block_lse + (row * p.max_blocks + j) * pieces;
      for (int q = 0; q < subs * 4; ++q) m += expf(__ldg(pl + q) - lse);
    }
    out[j] = m;
  }
}

cudaError_t run_block_mass(const MassParams& p, int B, cudaStream_t stream) {
  dim3 grid(p.Hq, B);
  block_mass_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace seer

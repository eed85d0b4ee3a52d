// a0: mean-pooled block keys kbar[b,h,j,:] = mean of K[b, t, h, :] over the
// valid tokens t < seqlen of block j.  Only keys are pooled: the SeerAttention-R
// Abstract removes query pooling for decoding, so the gate compares the raw
// decode query (projected) with one pooled key per block.
//
// One CTA of 8 warps per (block j, KV head h, sequence b).  Each lane reads 4
// dims (8 bytes) of a 256-byte K row, so a warp reads whole rows coalesced;
// warp w sums tokens w, w+8, ...; the 8 partial sums are added in a fixed
// order through shared memory (deterministic).  The incremental form runs one
// CTA per (b, h) on the newest block NB_b - 1 only: the block the appended
// token changed.
#include "block_mean.cuh"
#include "seer_kernels.cuh"

namespace seer {

__global__ void __launch_bounds__(256) pool_keys_kernel(const PoolParams p) {
  __shared__ __align__(16) float part[kPoolWarps][kHeadDim];
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  int j = blockIdx.x;
  if (p.incremental) {
    if (nb == 0) return;
    j = nb - 1;
  }
  float* dst = p.kbar + (((int64_t)b * p.Hkv + h) * p.max_blocks + j) * kHeadDim;
  const int valid = max(0, min(p.bs, L - j * p.bs));
  int64_t page = valid > 0 ? page_of(p.page_table, b, j, p.max_blocks) : 0;
  const bool bad_page = valid > 0 && (page < 0 || page >= p.num_pages);
  if (valid == 0 || bad_page) {
    if (bad_page && threadIdx.x == 0) flag_status(p.status, SEER_DEV_BAD_PAGE);
    if (threadIdx.x < kHeadDim) dst[threadIdx.x] = 0.f;
    return;
  }
  const uint16_t* base = p.k_pool + page * p.stride_page + (int64_t)h * p.stride_head + 4 * lane;
  const float4 a = pool_warp_partial(base, p.stride_token, valid, warp);
  *reinterpret_cast<float4*>(&part[warp][4 * lane]) = a;
  __syncthreads();
  if (threadIdx.x < kHeadDim) dst[threadIdx.x] = pool_finish(&part[0][0], threadIdx.x, valid);
}

cudaError_t run_pool_keys(const PoolParams& p, int B, cudaStream_t stream) {
  dim3 grid(p.incremental ? 1 : p.max_blocks, p.Hkv, B);
  pool_keys_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace seer

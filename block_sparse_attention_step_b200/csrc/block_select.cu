// a2: per-(b, h) top-k block selection (Agent Skill page, Step 1: top-k over
// the gate scores), exact and deterministic.
//
// Order: score descending, then block index ascending; -0.0 equals +0.0; NaN
// ranks below -inf.  The newest block NB-1, when forced, is taken first and
// counts toward k.  Output: the chosen indices ascending, -1 padded.
//
// One CTA of 1024 threads per (b, h); thread t owns one block (rows of at
// most 1024 blocks) or blocks 4t .. 4t+3, so a block-wide scan visits blocks
// in index order.  The value-binned select (one histogram pass over equal-
// width score bins, the threshold bin's few blocks ranked pairwise by order
// key and index) picks the blocks; rows whose threshold bin is crowded fall
// back to the 4-pass radix select.  No sort.
#include "seer_kernels.cuh"
#include "select_core.cuh"

namespace seer {

constexpr int kSelThreads = 1024;
constexpr int kSelItems = kMaxBlocks / kSelThreads;  // 4

__global__ void __launch_bounds__(kSelThreads) block_select_kernel(const SelectParams p) {
  __shared__ SelectSmem sm;
  const int b = blockIdx.y, h = blockIdx.x;
  const int64_t bh = (int64_t)b * p.Hkv + h;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  const float* row = p.scores + bh * p.max_blocks;
  const int k = __ldg(p.k_per_seq + b);
  if (nb <= kSelThreads)
    select_topk_binned<kSelThreads, 1>(row, nb, k, p.force_newest, p.k_max, p.idx + bh * p.k_max,
                                       p.n_sel + bh, p.status, sm);
  else
    select_topk_binned<kSelThreads, kSelItems>(row, nb, k, p.force_newest, p.k_max,
                                               p.idx + bh * p.k_max, p.n_sel + bh, p.status, sm);
}

cudaError_t run_block_select(const SelectParams& p, int B, cudaStream_t stream) {
  dim3 grid(p.Hkv, B);
  block_select_kernel<<<grid, kSelThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

// Unified cross-head selection (the LessIsMore abstract on the author page:
// one block ranking shared by every KV head instead of per-head subsets).
// One CTA per sequence adds the KV heads' score rows block by block, in head
// order, in fp32 (the aggregate; ranking by the sum is ranking by the mean),
// runs the same exact value-binned top-k on it, and writes the one index row
// to every head, so the decode kernel is unchanged.  Waits for the preceding
// grid (the gate scores) when chained by programmatic dependent launch.
__global__ void __launch_bounds__(kSelThreads) unified_select_kernel(const SelectParams p) {
  __shared__ SelectSmem sm;
  __shared__ float agg[kMaxBlocks];
  __shared__ int32_t chosen[kMaxBlocks];
  __shared__ int32_t n_chosen;
  const int b = blockIdx.x, tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  const float* rows = p.scores + (int64_t)b * p.Hkv * p.max_blocks;
  for (int j = tid; j < nb; j += kSelThreads) {
    float a = 0.f;
    for (int h = 0; h < p.Hkv; ++h) a += rows[(int64_t)h * p.max_blocks + j];
    agg[j] = a;
  }
  __syncthreads();
  const int k = __ldg(p.k_per_seq + b);
  if (nb <= kSelThreads)
    select_topk_binned<kSelThreads, 1>(agg, nb, k, p.force_newest, p.k_max, chosen, &n_chosen,
                                       p.status, sm);
  else
    select_topk_binned<kSelThreads, kSelItems>(agg, nb, k, p.force_newest, p.k_max, chosen,
                                               &n_chosen, p.status, sm);
  __syncthreads();
  for (int h = 0; h < p.Hkv; ++h) {
    const int64_t bh = (int64_t)b * p.Hkv + h;
    for (int q = tid; q < p.k_max; q += kSelThreads) p.idx[bh * p.k_max + q] = chosen[q];
    if (tid == 0) p.n_sel[bh] = n_chosen;
  }
}

cudaError_t run_unified_select(const SelectParams& p, int B, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, unified_select_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// k per sequence from seqlens (budget mode when budget > 0).
__global__ void fill_k_kernel(const int32_t* seqlens, int B, int bs, int permille, int budget,
                              int32_t* k_out) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
    const int L = max(0, __ldg(seqlens + b));
    const long long nb = (L + bs - 1) / bs;
    long long k;
    if (budget > 0) {
      k = budget / bs;
      if (k > nb) k = nb;
    } else {
      k = ((1000 - permille) * nb + 999) / 1000;
    }
    k_out[b] = (int32_t)(k < 1 ? 1 : k);
  }
}

cudaError_t run_fill_k(const int32_t* seqlens, int B, int bs, int permille, int budget,
                       int32_t* k_out, cudaStream_t stream) {
  const int threads = 256;
  const int blocks = (B + threads - 1) / threads;
  fill_k_kernel<<<blocks, threads, 0, stream>>>(seqlens, B, bs, permille, budget, k_out);
  return cudaGetLastError();
}

}  // namespace seer

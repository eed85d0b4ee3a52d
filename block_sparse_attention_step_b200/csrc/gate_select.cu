// a0 (incremental) + a1 + a2 fused for the decode step: one CTA per (b, h)
// refreshes the pooled key of the newest block, scores every block against
// the gate-projected query and selects the top-k, without a round trip of
// the scores through HBM and without two of the step's launches.
//
// Each CTA streams its kbar row (NB x 512 bytes) through three 64 KB shared-
// memory buffers with bulk copies, issued before the gate projection
// g = W qbar is formed so the projection hides under the first copies; the
// newest block's mean is recomputed from K with the same summation order as
// seer_pool_keys and written back; the scores (also written to the caller's
// scores buffer) stay in shared memory for the exact value-binned top-k.
// Results are identical to running seer_pool_keys (incremental),
// seer_gate_scores and seer_block_select one after another.
#include "block_mean.cuh"
#include "seer_kernels.cuh"
#include "select_core.cuh"

namespace seer {

constexpr int kGSThreads = 512;
constexpr int kGSWarps = kGSThreads / 32;
constexpr int kGSItems = kMaxBlocks / kGSThreads;  // 8
constexpr int kGSChunkRows = 128;                  // kbar rows per buffer
constexpr int kGSBuffers = 3;                      // 64 KB buffers in flight

struct GateSelectSmem {
  float buf[kGSBuffers][kGSChunkRows * kHeadDim];  // kbar rows in flight
  float scores[kMaxBlocks];
  float part[kPoolWarps * kHeadDim];
  float newest[kHeadDim];
  float qbar[kHeadDim];
  float gvec[kHeadDim];
  uint64_t bar[kGSBuffers];
  SelectSmem sel;
};

size_t gate_select_smem_bytes() { return sizeof(GateSelectSmem) + 128; }

__global__ void __launch_bounds__(kGSThreads, 1) gate_select_kernel(const GateSelectParams p) {
  extern __shared__ uint8_t gs_raw[];
  GateSelectSmem& sm = *reinterpret_cast<GateSelectSmem*>(
      (reinterpret_cast<uintptr_t>(gs_raw) + 127) & ~uintptr_t(127));
  const int b = blockIdx.y, h = blockIdx.x;
  const int64_t bh = (int64_t)b * p.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  const int nchunks = ceil_div_i(nb, kGSChunkRows);
  float* kb_row = p.kbar + bh * p.max_blocks * kHeadDim;

  if (tid == 0) {
    for (int i = 0; i < kGSBuffers; ++i) mbar_init(&sm.bar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Global memory is touched only from here on: wait for the preceding grid
  // (it may have produced q), then let the decode grid start launching.
  pdl_wait();
  pdl_launch_dependents();
  if (p.work_counter != nullptr && b == 0 && h == 0 && tid < 2) p.work_counter[tid] = 0u;
  const int k_row = __ldg(p.k_per_seq + b);  // used at the end; loaded early
  if (tid == 0) {
    for (int c = 0; c < kGSBuffers && c < nchunks; ++c) {
      const uint32_t bytes = (uint32_t)min(kGSChunkRows, nb - c * kGSChunkRows) * kHeadDim * 4;
      mbar_arrive_expect_tx(&sm.bar[c], bytes);
      bulk_copy_g2s(sm.buf[c], kb_row + (int64_t)c * kGSChunkRows * kHeadDim, bytes, &sm.bar[c]);
    }
  }

  // newest block's pooled key (incremental update), warps 0..7
  const bool refresh = p.incremental && nb > 0;
  int valid_new = 0;
  bool bad_page = false;
  if (refresh) {
    valid_new = L - (nb - 1) * p.bs;
    const int64_t page = page_of(p.page_table, b, nb - 1, p.max_blocks);
    bad_page = page < 0 || page >= p.num_pages;
    if (warp < kPoolWarps && !bad_page) {
      const uint16_t* base =
          p.k_pool + page * p.stride_page + (int64_t)h * p.stride_head + 4 * lane;
      const float4 a = pool_warp_partial(base, p.stride_token, valid_new, warp);
      *reinterpret_cast<float4*>(&sm.part[warp * kHeadDim + 4 * lane]) = a;
    }
  }
  // this warp's rows of W[h], in flight while the mean query is formed
  float4 wrow[kHeadDim / kGSWarps];
  {
    const float* W = p.w_gate + (int64_t)h * kHeadDim * kHeadDim;
#pragma unroll
    for (int r = 0; r < kHeadDim / kGSWarps; ++r)
      wrow[r] = __ldg(reinterpret_cast<const float4*>(W + (warp + r * kGSWarps) * kHeadDim + 4 * lane));
  }
  // mean query of the group, warps 8..11
  if (tid >= 256 && tid < 256 + kHeadDim) {
    const int d = tid - 256;
    const uint16_t* qg = p.q + ((int64_t)b * p.Hq + (int64_t)h * p.G) * kHeadDim + d;
    float s = 0.f;
    for (int g = 0; g < p.G; ++g) s += __uint_as_float((uint32_t)__ldg(qg + g * kHeadDim) << 16);
    sm.qbar[d] = s / (float)p.G;
  }
  __syncthreads();
  if (refresh && tid < kHeadDim) {
    float v = 0.f;
    if (!bad_page) v = pool_finish(sm.part, tid, valid_new);
    sm.newest[tid] = v;
    kb_row[(int64_t)(nb - 1) * kHeadDim + tid] = v;
    if (bad_page && tid == 0) flag_status(p.status, SEER_DEV_BAD_PAGE);
  }
  // g = gate_scale * W[h] qbar
  {
    const float4 qv = *reinterpret_cast<const float4*>(&sm.qbar[4 * lane]);
#pragma unroll
    for (int r = 0; r < kHeadDim / kGSWarps; ++r) {
      const float v = warp_dot4(wrow[r], qv);
      if (lane == 0) sm.gvec[warp + r * kGSWarps] = v * p.gate_scale;
    }
  }
  __syncthreads();

  // scores, chunk by chunk
  const float4 gv = *reinterpret_cast<const float4*>(&sm.gvec[4 * lane]);
  float* scores_out = p.scores + bh * p.max_blocks;
  bool bad = false;
  bool ok = true;
  for (int c = 0; c < nchunks; ++c) {
    const int slot = c % kGSBuffers;
    if (ok && !mbar_wait(&sm.bar[slot], (c / kGSBuffers) & 1)) {
      flag_status(p.status, SEER_DEV_TIMEOUT);
      ok = false;
    }
    const int rows = min(kGSChunkRows, nb - c * kGSChunkRows);
    const float* buf = sm.buf[slot];
    for (int r = warp; r < rows; r += kGSWarps) {
      const int j = c * kGSChunkRows + r;
      const float4 v = (refresh && j == nb - 1)
                           ? *reinterpret_cast<const float4*>(&sm.newest[4 * lane])
                           : *reinterpret_cast<const float4*>(&buf[r * kHeadDim + 4 * lane]);
      const float sc = warp_dot4(v, gv);
      if (lane == 0) {
        sm.scores[j] = sc;
        scores_out[j] = sc;
        bad |= !isfinite(sc);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();  // every warp is done with this buffer
    if (tid == 0 && ok && c + kGSBuffers < nchunks) {
      const int cn = c + kGSBuffers;
      const uint32_t bytes = (uint32_t)min(kGSChunkRows, nb - cn * kGSChunkRows) * kHeadDim * 4;
      mbar_arrive_expect_tx(&sm.bar[slot], bytes);
      bulk_copy_g2s(sm.buf[slot], kb_row + (int64_t)cn * kGSChunkRows * kHeadDim, bytes,
                    &sm.bar[slot]);
    }
  }
  if (bad) flag_status(p.status, SEER_DEV_NONFINITE_SCORE);
  for (int j = nb + tid; j < p.max_blocks; j += kGSThreads) scores_out[j] = -INFINITY;
  __syncthreads();

  if (nb <= kGSThreads)
    select_topk_binned<kGSThreads, 1>(sm.scores, nb, k_row, p.force_newest, p.k_max,
                                      p.idx + bh * p.k_max, p.n_sel + bh, p.status, sm.sel);
  else
    select_topk_binned<kGSThreads, kGSItems>(sm.scores, nb, k_row, p.force_newest, p.k_max,
                                             p.idx + bh * p.k_max, p.n_sel + bh, p.status,
                                             sm.sel);
}

cudaError_t run_gate_select(const GateSelectParams& p, int B, cudaStream_t stream, bool pdl) {
  const size_t smem = gate_select_smem_bytes();
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem_limit(gate_select_kernel, smem_set);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.Hkv, B);
  cfg.blockDim = dim3(kGSThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gate_select_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace seer

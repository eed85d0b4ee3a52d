// a0 (incremental) + a1 + a2 fused for the decode step: one CTA per (b, h)
// refreshes the pooled key of the newest block, scores every block against
// the gate-projected query and selects the top-k, without a round trip of
// the scores through HBM and without two of the step's launches.
//
// Each CTA (512 threads, one per SM) streams its kbar row (NB x 512 bytes)
// through three 64 KB shared-memory buffers with bulk copies, issued before
// the gate projection g = W qbar is formed so the projection hides under the
// first copies.  (Measured and dropped: 256-thread CTAs with 24 KB buffers,
// two per SM, for batches with more rows than SMs -- 5 % slower on the
// ragged batch, 60 % slower on the headline one; and each 64 KB chunk cut
// into 4-16 KB bulk copies -- slower at every size.)  The
// newest block's mean is recomputed from K with the same summation order as
// seer_pool_keys and written back; the scores (also written to the caller's
// scores buffer) stay in shared memory for the exact value-binned top-k.
// Results are identical to running seer_pool_keys (incremental),
// seer_gate_scores and seer_block_select one after another.
#include "block_mean.cuh"
#include "seer_kernels.cuh"
#include "select_core.cuh"

namespace seer {

template <int THREADS, int CHUNK_ROWS>
struct GateSelectShape {
  static constexpr int kWarps = THREADS / 32;
  static constexpr int kBuffers = 3;
  static constexpr int kItems = kMaxBlocks / THREADS;  // blocks per thread, long rows
  static_assert(kWarps >= kPoolWarps, "the pooled-key refresh uses 8 warps");
  static_assert(THREADS >= kHeadDim, "one thread per dimension for the mean query");
  static_assert(kHeadDim == 8 * kWarps && CHUNK_ROWS == 8 * kWarps,
                "every warp reduces 8 W rows and 8 kbar rows per chunk at once");
  struct Smem {
    float buf[kBuffers][CHUNK_ROWS * kHeadDim];  // kbar rows in flight
    float scores[kMaxBlocks];
    float part[kPoolWarps * kHeadDim];
    float newest[kHeadDim];
    float qbar[kHeadDim];
    float gvec[kHeadDim];
    uint64_t bar[kBuffers];
    SelectSmem sel;
  };
  static size_t smem_bytes() { return sizeof(Smem) + 128; }
};

using GSWide = GateSelectShape<512, 128>;   // one CTA per SM, 192 KB in flight

template <int THREADS, int CHUNK_ROWS, int MIN_BLOCKS>
__global__ void __launch_bounds__(THREADS, MIN_BLOCKS) gate_select_kernel(const GateSelectParams p) {
  using Shape = GateSelectShape<THREADS, CHUNK_ROWS>;
  using Smem = typename Shape::Smem;
  constexpr int kWarps = Shape::kWarps;
  constexpr int kBuffers = Shape::kBuffers;
  extern __shared__ uint8_t gs_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(gs_raw) + 127) &
                                      ~uintptr_t(127));
  const int b = blockIdx.y, h = blockIdx.x;
  const int64_t bh = (int64_t)b * p.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  const int nchunks = ceil_div_i(nb, CHUNK_ROWS);
  float* kb_row = p.kbar + bh * p.max_blocks * kHeadDim;

  if (tid == 0) {
    for (int i = 0; i < kBuffers; ++i) mbar_init(&sm.bar[i], 1);
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
    for (int c = 0; c < kBuffers && c < nchunks; ++c) {
      const uint32_t bytes = (uint32_t)min(CHUNK_ROWS, nb - c * CHUNK_ROWS) * kHeadDim * 4;
      mbar_arrive_expect_tx(&sm.bar[c], bytes);
      bulk_copy_g2s(sm.buf[c], kb_row + (int64_t)c * CHUNK_ROWS * kHeadDim, bytes, &sm.bar[c]);
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
  float4 wrow[kHeadDim / kWarps];
  {
    const float* W = p.w_gate + (int64_t)h * kHeadDim * kHeadDim;
#pragma unroll
    for (int r = 0; r < kHeadDim / kWarps; ++r)
      wrow[r] = __ldg(reinterpret_cast<const float4*>(W + (warp + r * kWarps) * kHeadDim + 4 * lane));
  }
  // mean query of the group (warps 8..11 of 16, or warps 0..3 of 8)
  constexpr int kQFirst = THREADS >= 512 ? 256 : 0;
  if (tid >= kQFirst && tid < kQFirst + kHeadDim) {
    const int d = tid - kQFirst;
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
  // g = gate_scale * W[h] qbar: this warp's 8 rows warp + 16 i in one reduction
  {
    const float4 qv = *reinterpret_cast<const float4*>(&sm.qbar[4 * lane]);
    const float v = warp_dot4_x8(wrow, qv);
    if ((lane & 3) == 0) sm.gvec[warp + ((lane >> 2) & 7) * kWarps] = __fmul_rn(v, p.gate_scale);
  }
  __syncthreads();

  // scores, chunk by chunk
  const float4 gv = *reinterpret_cast<const float4*>(&sm.gvec[4 * lane]);
  float* scores_out = p.scores + bh * p.max_blocks;
  bool bad = false;
  bool ok = true;
  for (int c = 0; c < nchunks; ++c) {
    const int slot = c % kBuffers;
    if (ok && !mbar_wait(&sm.bar[slot], (c / kBuffers) & 1)) {
      flag_status(p.status, SEER_DEV_TIMEOUT);
      ok = false;
    }
    const int rows = min(CHUNK_ROWS, nb - c * CHUNK_ROWS);
    const float* buf = sm.buf[slot];
    {  // this warp's 8 rows warp + 16 i of the chunk, one reduction
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = warp + i * kWarps;
        const int j = c * CHUNK_ROWS + r;
        v[i] = (r >= rows) ? make_float4(0.f, 0.f, 0.f, 0.f)
               : (refresh && j == nb - 1)
                   ? *reinterpret_cast<const float4*>(&sm.newest[4 * lane])
                   : *reinterpret_cast<const float4*>(&buf[r * kHeadDim + 4 * lane]);
      }
      const float sc = warp_dot4_x8(v, gv);
      const int r = warp + ((lane >> 2) & 7) * kWarps;
      if ((lane & 3) == 0 && r < rows) {
        const int j = c * CHUNK_ROWS + r;
        sm.scores[j] = sc;
        scores_out[j] = sc;
        bad |= !isfinite(sc);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();  // every warp is done with this buffer
    if (tid == 0 && ok && c + kBuffers < nchunks) {
      const int cn = c + kBuffers;
      const uint32_t bytes = (uint32_t)min(CHUNK_ROWS, nb - cn * CHUNK_ROWS) * kHeadDim * 4;
      mbar_arrive_expect_tx(&sm.bar[slot], bytes);
      bulk_copy_g2s(sm.buf[slot], kb_row + (int64_t)cn * CHUNK_ROWS * kHeadDim, bytes,
                    &sm.bar[slot]);
    }
  }
  if (bad) flag_status(p.status, SEER_DEV_NONFINITE_SCORE);
  for (int j = nb + tid; j < p.max_blocks; j += THREADS) scores_out[j] = -INFINITY;
  if (p.scores_only) return;  // uniform: the cross-head select runs next
  __syncthreads();

  if (nb <= THREADS)
    select_topk_binned<THREADS, 1>(sm.scores, nb, k_row, p.force_newest, p.k_max,
                                   p.idx + bh * p.k_max, p.n_sel + bh, p.status, sm.sel);
  else
    select_topk_binned<THREADS, Shape::kItems>(sm.scores, nb, k_row, p.force_newest, p.k_max,
                                               p.idx + bh * p.k_max, p.n_sel + bh, p.status,
                                               sm.sel);
}

template <typename Shape, int THREADS, int CHUNK_ROWS, int MIN_BLOCKS>
static cudaError_t launch_gate_select(const GateSelectParams& p, int B, cudaStream_t stream,
                                      bool pdl) {
  auto kern = gate_select_kernel<THREADS, CHUNK_ROWS, MIN_BLOCKS>;
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem_limit(kern, smem_set);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.Hkv, B);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = Shape::smem_bytes();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t run_gate_select(const GateSelectParams& p, int B, cudaStream_t stream, bool pdl) {
  return launch_gate_select<GSWide, 512, 128, 1>(p, B, stream, pdl);
}

}  // namespace seer

// a0 (incremental) + a1 + a2 fused for the decode step: one CTA per (b, h)
// refreshes the pooled key of the newest block, scores every block against
// the gate-projected query and selects the top-k, without a round trip of
// the scores through HBM and without two of the step's launches.
//
// Each CTA (512 threads, one per SM) streams its kbar row (NB x 512 bytes)
// through three 64 KB shared-memory buffers with bulk copies: the first at
// once (128 rows, before the row length is known), the others right after
// the newest block's K loads (so those queue behind one chunk, not three),
// all before the gate projection g = W qbar is formed, which hides under the
// copies.  (Measured and dropped: 256-thread CTAs with 24 KB buffers, two per
// SM, for batches with more rows than SMs -- 5 % slower on the ragged batch,
// 60 % slower on the headline one; and each 64 KB chunk cut into 4-16 KB bulk
// copies -- slower at every size.)  The
// newest block's mean is recomputed from K with the same summation order as
// seer_pool_keys and written back; the scores (also written to the caller's
// scores buffer) stay in shared memory for the exact value-binned top-k.
// Results are identical to running seer_pool_keys (incremental),
// seer_gate_scores and seer_block_select one after another.
#include "gate_row.cuh"

namespace seer {

constexpr int kGSThreads = 512;
constexpr int kGSWorkers = 16;                   // every warp scores
constexpr int kGSChunkRows = 8 * kGSWorkers;     // 128 kbar rows = 64 KB per buffer
constexpr int kGSBuffers = 3;

struct GateSelectSmem {
  float buf[kGSBuffers][kGSChunkRows * kHeadDim];  // kbar rows in flight
  GateRowScratch row;                              // 16-byte aligned (float4 members)
  float part[kPoolWarps * kHeadDim];               // newest-block pooling partials
  uint64_t bar[kGSBuffers];
};
static_assert(offsetof(GateSelectSmem, row) % 16 == 0 && offsetof(GateSelectSmem, part) % 16 == 0 &&
                  offsetof(GateSelectSmem, bar) % 8 == 0,
              "gate kernel shared-memory carve alignment");

// Publishes row bh (after a barrier that follows its gate row): its indices,
// kbar row, appended K/V row and query copy are visible to the decode grid,
// whose TMA and bulk copies read the last two, once the flag is.  The epoch
// does not move before every row is out (the decode grid's last CTA
// advances it).
__device__ __forceinline__ void publish_row(const GateSelectParams& p, int bh) {
  if (p.row_flag == nullptr || bh < 0) return;
  const uint32_t value = *reinterpret_cast<const volatile uint32_t*>(p.epoch) + 1u;
  __threadfence();
  fence_proxy_async_global();
  st_release_gpu(p.row_flag + bh, value);
}

__global__ void __launch_bounds__(kGSThreads, 1) gate_select_kernel(const GateSelectParams p) {
  extern __shared__ uint8_t gs_raw[];
  GateSelectSmem& sm = *reinterpret_cast<GateSelectSmem*>(
      (reinterpret_cast<uintptr_t>(gs_raw) + 127) & ~uintptr_t(127));
  const int b = blockIdx.y, h = blockIdx.x;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGSBuffers; ++i) mbar_init(&sm.bar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Global memory is touched only from here on: wait for the preceding grid
  // (it may have produced q or the appended K/V), then let the decode grid
  // start launching.
  pdl_wait();
  pdl_launch_dependents();
  if (p.work_counter != nullptr && b == 0 && h == 0 && threadIdx.x < 2)
    p.work_counter[threadIdx.x] = 0u;
  uint32_t seq = 0;
  const ChunkRing<kGSBuffers> ring = {{sm.buf[0], sm.buf[1], sm.buf[2]}};
  gate_row<kGSThreads, kGSWorkers, kGSBuffers, 256, kHeadDim, 1, true>(p, b, h, ring, sm.bar, seq,
                                                                       sm.row, sm.part);
  if (p.row_flag != nullptr) {
    __syncthreads();  // every thread's writes of the row come before the flag
    if (threadIdx.x == 0) publish_row(p, b * p.Hkv + h);
  }
}

// The same rows for batches with more (b, h) rows than SMs: one persistent
// CTA per SM gates row after row, claiming rows two ahead (a counter at zero
// when the launch starts), and keeps one kbar chunk stream across its rows --
// the next row's first chunks are in flight while this one finishes and
// selects, and no CTA start-up or drain sits between rows.
__global__ void __launch_bounds__(kGSThreads, 1)
    gate_select_rows_kernel(const GateSelectParams p) {
  extern __shared__ uint8_t gs_raw[];
  GateSelectSmem& sm = *reinterpret_cast<GateSelectSmem*>(
      (reinterpret_cast<uintptr_t>(gs_raw) + 127) & ~uintptr_t(127));
  __shared__ int next_rows[2];
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGSBuffers; ++i) mbar_init(&sm.bar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  if (p.work_counter != nullptr && blockIdx.x == 0 && threadIdx.x < 2)
    p.work_counter[threadIdx.x] = 0u;
  const int rows = p.B * p.Hkv;
  const ChunkRing<kGSBuffers> ring = {{sm.buf[0], sm.buf[1], sm.buf[2]}};
  uint32_t seq = 0, ahead = 0;
  // Rows are claimed two ahead: the claim of the row after next goes out as a
  // row starts and is read when the next one starts, so its round trip hides
  // under a whole row (thread 0 holds it in `pending`).
  unsigned pending = 0xffffffffu;
  if (threadIdx.x == 0) {
    const unsigned v = atomicAdd(p.row_counter, 1u) + gridDim.x;
    next_rows[0] = v < (unsigned)rows ? (int)v : -1;
    if (v < (unsigned)rows) pending = atomicAdd(p.row_counter, 1u) + gridDim.x;
  }
  __syncthreads();
  int row = blockIdx.x, prev = -1;
  for (int it = 0; row < rows; ++it) {
    const int nxt = next_rows[it & 1];
    if (threadIdx.x == 0) {  // the row after nxt, and the claim after that one
      const bool more = nxt >= 0 && pending < (unsigned)rows;
      next_rows[(it + 1) & 1] = more ? (int)pending : -1;
      pending = more ? atomicAdd(p.row_counter, 1u) + gridDim.x : 0xffffffffu;
    }
    // the previous row, out since the barrier that ended it; its fences run
    // on warp 1 while the other warps start this row
    if (threadIdx.x == 32) publish_row(p, prev);
    gate_row<kGSThreads, kGSWorkers, kGSBuffers, 256, kHeadDim>(
        p, row / p.Hkv, row % p.Hkv, ring, sm.bar, seq, sm.row, sm.part, nxt >= 0 ? nxt / p.Hkv : -1,
        nxt >= 0 ? nxt % p.Hkv : 0, &ahead);
    __syncthreads();  // the row is out; next_rows[(it + 1) & 1] is written
    prev = row;
    row = nxt >= 0 ? nxt : rows;
  }
  if (threadIdx.x == 32) publish_row(p, prev);
  // the last CTA past its final claim puts the claiming words back to zero
  // for the next launch that shares them
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.row_done, 1u) == gridDim.x - 1) {
      atomicExch(p.row_counter, 0u);
      atomicExch(p.row_done, 0u);
    }
  }
}

cudaError_t run_gate_select_rows(const GateSelectParams& p, int num_sms, cudaStream_t stream,
                                 bool pdl) {
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem_limit(gate_select_rows_kernel, smem_set);
  if (e != cudaSuccess) return e;
  const int rows = p.B * p.Hkv;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows < num_sms ? rows : num_sms);
  cfg.blockDim = dim3(kGSThreads);
  cfg.dynamicSmemBytes = sizeof(GateSelectSmem) + 128;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gate_select_rows_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t run_gate_select(const GateSelectParams& p, int B, cudaStream_t stream, bool pdl) {
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem_limit(gate_select_kernel, smem_set);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.Hkv, B);
  cfg.blockDim = dim3(kGSThreads);
  cfg.dynamicSmemBytes = sizeof(GateSelectSmem) + 128;
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

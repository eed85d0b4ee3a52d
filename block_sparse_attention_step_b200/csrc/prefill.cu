// Prefill with query pooling (the SeerAttention form that SeerAttention-R
// drops for decoding, paper summary page, Abstract), for a whole sequence at
// once:
//   * prefill_gate_select_kernel, one CTA per (b, h, query block i): the
//     pooled query qbar_i (mean over the block's query tokens and the group's
//     G heads), g = gate_scale * W[h] qbar_i, scores g . kbar_j for the
//     causal prefix j <= i, then the exact top-k_i with block i forced (the
//     value-binned select of the decode step);
//   * prefill_attention_kernel, one CTA per (b, query head, 64-token query
//     tile): the selected key blocks of the tile's query block stream in by
//     TMA (the decode's tensor maps, 64 tokens x 64 dims per box), and four
//     math warps (16 query tokens each) run S = Q K^T, the causal and tail
//     masks, the online softmax and O += P V on the tensor cores
//     (mma.sync m16n8k16 bf16, P rounded to bf16 as in FlashAttention),
//     writing bf16 out and the natural-log lse.
// Every wait is bounded (SEER_DEV_TIMEOUT); nothing traps.
#include "block_mean.cuh"
#include "seer_kernels.cuh"
#include "select_core.cuh"
#include "tcgen05.cuh"

namespace seer {

// ------------------------------------------------------------ gate + select
constexpr int kPGThreads = 256;
constexpr int kPGWarps = kPGThreads / 32;  // 8: 16 W rows and 8 kbar rows per warp at a time

struct PrefillGateSmem {
  float scores[kMaxBlocks];
  float qpart[kPGWarps][kHeadDim];
  float qbar[kHeadDim];
  float gvec[kHeadDim];
  SelectSmem sel;
};

__device__ __forceinline__ int prefill_k(const PrefillParams& p, int n_cand) {
  long long k;
  if (p.budget_tokens > 0) {
    k = p.budget_tokens / p.bs;
    if (k > n_cand) k = n_cand;
  } else {
    k = ((long long)(1000 - p.sparsity_permille) * n_cand + 999) / 1000;
  }
  return (int)(k < 1 ? 1 : k);
}

__global__ void __launch_bounds__(kPGThreads, 3) prefill_gate_select_kernel(const PrefillParams p) {
  __shared__ __align__(16) PrefillGateSmem sm;
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row = ((int64_t)b * p.Hkv + h) * p.max_blocks + i;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  int32_t* idx_row = p.idx + row * p.k_max;
  float* scores_row = p.scores ? p.scores + row * p.max_blocks : nullptr;
  if (i >= nb) {  // a query block past the sequence: nothing selected
    for (int q = tid; q < p.k_max; q += kPGThreads) idx_row[q] = -1;
    if (scores_row)
      for (int j = tid; j < p.max_blocks; j += kPGThreads) scores_row[j] = -INFINITY;
    if (tid == 0) p.n_sel[row] = 0;
    return;
  }
  // pooled query: the block's (token, head) rows of the group, row r to warp
  // r % 8 (a row is 256 contiguous bytes; lane l takes dims 4l .. 4l+3), eight
  // rows in flight per warp; the eight warp partials are added in warp order
  const int lo = i * p.bs, hi = min(lo + p.bs, L);
  {
    const int nrows = (hi - lo) * p.G;
    const uint16_t* q0 = p.q + (((int64_t)b * p.max_blocks * p.bs + lo) * p.Hq + (int64_t)h * p.G) *
                                   kHeadDim + 4 * lane;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
    for (int rr = warp; rr < nrows; rr += kPGWarps) {
      const int t = rr / p.G, g = rr - t * p.G;
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(q0 + ((int64_t)t * p.Hq + g) * kHeadDim));
      a0 += __uint_as_float(v.x << 16);
      a1 += __uint_as_float(v.x & 0xffff0000u);
      a2 += __uint_as_float(v.y << 16);
      a3 += __uint_as_float(v.y & 0xffff0000u);
    }
    *reinterpret_cast<float4*>(&sm.qpart[warp][4 * lane]) = make_float4(a0, a1, a2, a3);
  }
  // this warp's W rows warp + 8 r (16 of them), in flight meanwhile
  float4 wrow[kHeadDim / kPGWarps];
  {
    const float* W = p.w_gate + (int64_t)h * kHeadDim * kHeadDim;
#pragma unroll
    for (int r = 0; r < kHeadDim / kPGWarps; ++r)
      wrow[r] = __ldg(reinterpret_cast<const float4*>(W + (warp + r * kPGWarps) * kHeadDim + 4 * lane));
  }
  __syncthreads();
  if (tid < kHeadDim) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kPGWarps; ++w) s += sm.qpart[w][tid];
    sm.qbar[tid] = s / (float)((hi - lo) * p.G);
  }
  __syncthreads();
  {
    const float4 qv = *reinterpret_cast<const float4*>(&sm.qbar[4 * lane]);
#pragma unroll
    for (int g8 = 0; g8 < 2; ++g8) {
      float4 w8[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) w8[r] = wrow[g8 * 8 + r];
      const float v = warp_dot4_x8(w8, qv);
      if ((lane & 3) == 0)
        sm.gvec[warp + (g8 * 8 + ((lane >> 2) & 7)) * kPGWarps] = __fmul_rn(v, p.gate_scale);
    }
  }
  __syncthreads();
  // scores of the causal prefix j <= i, 8 rows per warp per pass
  const int n_cand = i + 1;
  const float4 gv = *reinterpret_cast<const float4*>(&sm.gvec[4 * lane]);
  const float* kb = p.kbar + ((int64_t)b * p.Hkv + h) * p.max_blocks * kHeadDim;
  bool bad = false;
  for (int base = 0; base < n_cand; base += 8 * kPGWarps) {
    float4 v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int j = base + warp + r * kPGWarps;
      v[r] = j < n_cand ? __ldg(reinterpret_cast<const float4*>(kb + (int64_t)j * kHeadDim + 4 * lane))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float sc = warp_dot4_x8(v, gv);
    const int j = base + warp + ((lane >> 2) & 7) * kPGWarps;
    if ((lane & 3) == 0 && j < n_cand) {
      sm.scores[j] = sc;
      if (scores_row) scores_row[j] = sc;
      bad |= !isfinite(sc);
    }
  }
  if (bad) flag_status(p.status, SEER_DEV_NONFINITE_SCORE);
  if (scores_row)
    for (int j = n_cand + tid; j < p.max_blocks; j += kPGThreads) scores_row[j] = -INFINITY;
  __syncthreads();
  const int k = prefill_k(p, n_cand);
  if (n_cand <= kPGThreads)
    select_topk_binned<kPGThreads, 1>(sm.scores, n_cand, k, 1, p.k_max, idx_row, p.n_sel + row,
                                      p.status, sm.sel);
  else if (n_cand <= 2 * kPGThreads)
    select_topk_binned<kPGThreads, 2>(sm.scores, n_cand, k, 1, p.k_max, idx_row, p.n_sel + row,
                                      p.status, sm.sel);
  else
    select_topk_binned<kPGThreads, kMaxBlocks / kPGThreads>(sm.scores, n_cand, k, 1, p.k_max,
                                                             idx_row, p.n_sel + row, p.status,
                                                             sm.sel);
}

cudaError_t run_prefill_gate_select(const PrefillParams& p, cudaStream_t stream) {
  dim3 grid(p.max_blocks, p.Hkv, p.B);
  prefill_gate_select_kernel<<<grid, kPGThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- attention
//
// One CTA per (b, KV head h, 64-token query tile, pair of the group's query
// heads), longest causal prefixes first.  Its 128 query rows (64 tokens x 2
// heads; a group of odd size repeats its last head in the last pair, whose
// copy is computed and dropped) form the M = 128 side of the fifth-generation
// tensor-core MMAs, with both accumulators in tensor memory:
//   S = Q K^T  (N = 64 keys, K = 128 dims: 8 MMAs of K = 16)
//   O += P V   (N = 128 dims, K = 64 keys: 4 MMAs of K = 16)
// Warp roles (192 threads): warp 0 issues the TMA loads (Q once; K and V of
// every key tile of the selected blocks, 64 keys each, in 3 K and 2 V
// stages); warp 1 allocates 256 TMEM columns (S double-buffered in 2 x 64,
// O in 128) and one of its threads issues the MMAs; warps 2-5 (one query row
// per thread, TMEM lane = row) read S, apply the causal and sequence masks,
// run the online softmax in the exp2 domain and write P as bf16 into the
// shared-memory slot the tile's K occupied (S = Q K^T is done with it), in
// the 128-byte swizzled K-major layout the MMA reads.  The running maximum
// is a reference that moves only when a row's maximum grows by more than
// 2^8; O (in TMEM) and l are then rescaled by the same factor, so the
// result is exact for any reference.  Key rows past the sequence are zeroed
// in V before P V runs.  Stage hand-offs go through mbarriers; tcgen05.commit
// arrives on them when the MMAs finish.  Every wait is bounded
// (SEER_DEV_TIMEOUT); TMEM is freed on every path.
constexpr int kTCThreads = 192;
constexpr int kTCRows = 128;                      // MMA M: 64 tokens x 2 heads
constexpr int kTCKStages = 3, kTCVStages = 2;
constexpr int kTCBox = 64 * 128;                  // one TMA box: 64 rows x 64 bf16 dims
constexpr int kTCTile = 2 * kTCBox;               // 64 keys x 128 dims (K or V)
constexpr int kTCQBytes = kTCRows * kHeadDim * 2; // 2 boxes of 128 rows
constexpr int kTCData = kTCQBytes + (kTCKStages + kTCVStages) * kTCTile;  // 112 KB
constexpr size_t kTCSmem = (size_t)kTCData + 1024;  // + barriers and alignment slack
constexpr uint32_t kTCCols = 256;                 // S0 [0,64), S1 [64,128), O [128,256)
constexpr float kTCRescale = 8.f;                 // log2 growth that moves the reference
constexpr uint32_t kIdescS = tc_idesc_bf16(128, 64, 0, 0);    // Q (K-major) x K (K-major)
constexpr uint32_t kIdescPV = tc_idesc_bf16(128, 128, 0, 1);  // P (K-major) x V (MN-major)

struct TcBars {
  uint64_t q_full;
  uint64_t k_full[kTCKStages], k_empty[kTCKStages];
  uint64_t v_full[kTCVStages], v_empty[kTCVStages];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, pv_done[2], mma_done;  // P V of tile j completes on pv_done[j & 1]
  int2 meta[kTCKStages];  // per K stage: (first key token, valid keys) or (0, -1): no more
  uint32_t tmem_base;
};
static_assert(sizeof(TcBars) <= 256, "barrier block");

__device__ __forceinline__ uint64_t tc_kdesc(uint32_t addr) { return tc_desc_sw128(addr, 16, 1024); }

__global__ void __launch_bounds__(kTCThreads, 2)
    prefill_attention_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  extern __shared__ uint8_t tc_raw[];
  // 1024-byte aligned data (the 128-byte swizzle atom); the barriers go into
  // the slack in front when there are 256 bytes of it, else behind the data
  const uintptr_t raw = reinterpret_cast<uintptr_t>(tc_raw);
  uint8_t* data = reinterpret_cast<uint8_t*>((raw + 1023) & ~uintptr_t(1023));
  TcBars* bars = reinterpret_cast<TcBars*>(
      (uintptr_t)data - raw >= 256 ? tc_raw : data + kTCData);
  uint8_t* q_s = data;
  uint8_t* k_ring = data + kTCQBytes;
  uint8_t* v_ring = k_ring + kTCKStages * kTCTile;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Lq = p.max_blocks * p.bs;
  const int ntiles = Lq / kTileTokens;
  const int tile = ntiles - 1 - (int)blockIdx.x;  // longest causal prefixes first
  const int npairs = (p.G + 1) >> 1;
  const int h = (int)blockIdx.y / npairs, pair = (int)blockIdx.y - h * npairs;
  const int b = blockIdx.z;
  const int g0 = 2 * pair;
  const bool two = g0 + 1 < p.G;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, Lq));
  const int t0 = tile * kTileTokens;
  if (t0 >= L) return;  // the whole CTA: no query token here
  const int t_last = min(t0 + kTileTokens - 1, L - 1);
  const int qb = t0 / p.bs;  // query block of this tile
  const int64_t row = ((int64_t)b * p.Hkv + h) * p.max_blocks + qb;
  // after a wait has run out somewhere in the grid, later CTAs do no work
  // (each run-out wait costs about a second)
  if (p.status != nullptr &&
      (*reinterpret_cast<const volatile int32_t*>(p.status) & SEER_DEV_TIMEOUT))
    return;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kTCKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kTCVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], 4);
    }
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->pv_done[0], 1);
    mbar_init(&bars->pv_done[1], 1);
    mbar_init(&bars->mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTCCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ================================================================ copies
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      // Q is read by this CTA alone; K and V tiles by every query tile that
      // selected their block and by the group's other head pairs
      const uint64_t q_policy = policy_evict_first();
      const uint64_t policy = policy_evict_normal();
      // Q: rows 0-63 = tokens t0.. of head g0, rows 64-127 = head g0 + 1;
      // dims 0-63 in the first 16 KB, 64-127 in the second
      mbar_arrive_expect_tx(&bars->q_full, kTCQBytes);
      for (int half = 0; half < 2; ++half)
        for (int gs = 0; gs < 2; ++gs) {
          const int qh = h * p.G + (two ? g0 + gs : g0);
          tma_load_4d(q_s + half * (kTCQBytes / 2) + gs * kTCBox, &tm_q, 64 * half, qh, t0, b,
                      &bars->q_full, q_policy);
        }
      const int n = max(0, min(__ldg(p.n_sel + row), p.k_max));
      const int nb = ceil_div_i(L, p.bs);
      uint32_t kn = 0, vn = 0;  // K / V tiles issued
      bool ok = true;
      for (int q = 0; q < n && ok; ++q) {
        const int j = __ldg(p.idx + row * p.k_max + q);
        if (j < 0 || j >= nb || j > qb) {
          flag_status(p.status, SEER_DEV_BAD_INDEX);
          continue;
        }
        const int64_t page = page_of(p.page_table, b, j, p.max_blocks);
        if (page < 0 || page >= p.num_pages) {
          flag_status(p.status, SEER_DEV_BAD_PAGE);
          continue;
        }
        for (int e = 0; e * kTileTokens < p.bs; ++e) {
          const int s0 = j * p.bs + e * kTileTokens;
          if (s0 >= L || s0 > t_last) break;  // nothing a query of this tile may see
          const int t = e * kTileTokens;
          const int c1 = p.token_inner ? t : h, c2 = p.token_inner ? h : t;
          const int ks = kn % kTCKStages;
          if (!mbar_wait(&bars->k_empty[ks], ((kn / kTCKStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          bars->meta[ks] = make_int2(s0, min(kTileTokens, L - s0));
          mbar_arrive_expect_tx(&bars->k_full[ks], kTCTile);
          uint8_t* kd = k_ring + ks * kTCTile;
          tma_load_4d(kd, &tm_k, 0, c1, c2, (int)page, &bars->k_full[ks], policy);
          tma_load_4d(kd + kTCBox, &tm_k, 64, c1, c2, (int)page, &bars->k_full[ks], policy);
          ++kn;
          const int vs = vn % kTCVStages;
          if (!mbar_wait(&bars->v_empty[vs], ((vn / kTCVStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->v_full[vs], kTCTile);
          uint8_t* vd = v_ring + vs * kTCTile;
          tma_load_4d(vd, &tm_v, 0, c1, c2, (int)page, &bars->v_full[vs], policy);
          tma_load_4d(vd + kTCBox, &tm_v, 64, c1, c2, (int)page, &bars->v_full[vs], policy);
          ++vn;
        }
      }
      bool marked = false;
      if (ok) {  // end marker: a K stage with no data
        const int ks = kn % kTCKStages;
        if (mbar_wait(&bars->k_empty[ks], ((kn / kTCKStages) & 1) ^ 1)) {
          bars->meta[ks] = make_int2(0, -1);
          mbar_arrive(&bars->k_full[ks]);
          marked = true;
        }
      }
      if (!marked) flag_status(p.status, SEER_DEV_TIMEOUT);
      // Let this CTA's copies land before it retires: the newest copy of
      // each stage (older ones were consumed before their stage was reused;
      // with the end marker posted, the marker's stage holds no copy).
      for (uint32_t k = 1; k <= (uint32_t)kTCKStages && k <= kn; ++k) {
        const uint32_t c = kn - k;
        if (marked && c % kTCKStages == kn % kTCKStages) continue;
        if (!mbar_wait(&bars->k_full[c % kTCKStages], (c / kTCKStages) & 1))
          flag_status(p.status, SEER_DEV_TIMEOUT);
      }
      for (uint32_t k = 1; k <= (uint32_t)kTCVStages && k <= vn; ++k) {
        const uint32_t c = vn - k;
        if (!mbar_wait(&bars->v_full[c % kTCVStages], (c / kTCVStages) & 1))
          flag_status(p.status, SEER_DEV_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0) {
      bool ok = mbar_wait(&bars->q_full, 0);
      const uint32_t q_addr = smem_u32(q_s);
      auto issue_pv = [&](uint32_t jj) -> bool {
        if (!mbar_wait(&bars->p_full, jj & 1)) return false;
        const int vs = jj % kTCVStages;
        if (!mbar_wait(&bars->v_full[vs], (jj / kTCVStages) & 1)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(k_ring + (jj % kTCKStages) * kTCTile);
        const uint32_t va = smem_u32(v_ring + vs * kTCTile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_f16_ss(tmem + 128, tc_kdesc(pa + 32 * kk), tc_desc_sw128(va + 2048 * kk, kTCBox, 1024),
                        kIdescPV, (jj > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&bars->pv_done[jj & 1]);
        tc_commit(&bars->k_empty[jj % kTCKStages]);
        tc_commit(&bars->v_empty[vs]);
        return true;
      };
      uint32_t it = 0;
      while (ok) {
        const int ks = it % kTCKStages;
        if (!mbar_wait(&bars->k_full[ks], (it / kTCKStages) & 1)) {
          ok = false;
          break;
        }
        if (bars->meta[ks].y < 0) break;  // no more key tiles
        const int sb = it & 1;
        if (it >= 2 && !mbar_wait(&bars->s_free[sb], ((it >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ka = smem_u32(k_ring + ks * kTCTile);
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {
          const uint32_t off = (k8 >> 2) * (kTCQBytes / 2) + 32 * (k8 & 3);
          const uint32_t koff = (k8 >> 2) * kTCBox + 32 * (k8 & 3);
          tc_mma_f16_ss(tmem + 64 * sb, tc_kdesc(q_addr + off), tc_kdesc(ka + koff), kIdescS,
                        k8 > 0 ? 1u : 0u);
        }
        tc_commit(&bars->s_full[sb]);
        if (it >= 1 && !issue_pv(it - 1)) {
          ok = false;
          break;
        }
        ++it;
      }
      if (ok && it >= 1) ok = issue_pv(it - 1);
      if (ok) {  // tell the softmax warps there is no tile `it`
        const int sb = it & 1;
        if (it >= 2) ok = mbar_wait(&bars->s_free[sb], ((it >> 1) & 1) ^ 1);
        if (ok) mbar_arrive(&bars->s_full[sb]);
      }
      if (!ok) flag_status(p.status, SEER_DEV_TIMEOUT);
      // every MMA this thread issued has finished before TMEM is freed
      tc_commit(&bars->mma_done);
      if (!mbar_wait(&bars->mma_done, 0)) flag_status(p.status, SEER_DEV_TIMEOUT);
    }
  } else {
    // ============================================================ softmax
    const int quarter = warp & 3;               // TMEM lanes 32 * quarter ..
    const int r = 32 * quarter + lane;          // this thread's row
    const int tq = t0 + (r & 63);               // its query token
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * quarter) << 16);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    // P V of tile k completes on pv_done[k & 1], as that barrier's (k >> 1)-th
    // phase.  Tile j waits for tile j - 2's (long finished) so that neither
    // barrier ever runs two phases ahead of what this warp has seen; only an
    // O rescale waits for tile j - 1's.
    uint32_t pv_seen0 = 0u, pv_seen1 = 0u;  // phases observed on pv_done[0] / [1]
    auto wait_pv = [&](uint32_t k) -> bool {
      const uint32_t b = k & 1u, ph = k >> 1;
      if ((b ? pv_seen1 : pv_seen0) > ph) return true;
      const bool r = mbar_wait(&bars->pv_done[b], ph & 1u);
      if (b) pv_seen1 = ph + 1u;
      else pv_seen0 = ph + 1u;
      return r;
    };
    uint32_t it = 0;
    for (;; ++it) {
      const int sb = it & 1, ks = it % kTCKStages;
      ok = mbar_wait(&bars->s_full[sb], (it >> 1) & 1);
      ok = ok && mbar_wait(&bars->k_full[ks], (it / kTCKStages) & 1);  // meta of this tile
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int2 mt = bars->meta[ks];
      if (mt.y < 0) break;  // no more key tiles
      uint32_t sv[64];
      __syncwarp();
      tmem_ld64(lane_addr + 64 * sb, sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free[sb]);
      // visible keys of this row: c < lim (inside the sequence, not after tq);
      // eight independent partial maxima and sums keep the dependent chains
      // short (two softmax warps per scheduler hide little latency)
      const int lim = min(mt.y, tq - mt.x + 1);
      float x[64];
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        x[c] = c < lim ? __uint_as_float(sv[c]) * p.scale_log2 : -INFINITY;
        m8[c & 7] = fmaxf(m8[c & 7], x[c]);
      }
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_ref + kTCRescale) {
        if (m_ref != -INFINITY) {
          alpha = fast_exp2(m_ref - mx);
          rescale = true;
        }
        m_ref = mx;
      }
      const float ref = m_ref == -INFINITY ? 0.f : m_ref;
      float s8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) s8[i] = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        x[c] = fast_exp2(x[c] - ref);  // exp2(-inf) = 0 for masked keys
        s8[c & 7] += x[c];
      }
      const float sum = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
      l = l * alpha + sum;
      if (it >= 2) ok = wait_pv(it - 2);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (__any_sync(0xffffffffu, rescale)) {
        // O is stable once the previous tile's P V has finished
        if (it >= 1) ok = wait_pv(it - 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t o[32];
          __syncwarp();
          tmem_ld32(lane_addr + 128 + 32 * c4, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          __syncwarp();
          tmem_st32(lane_addr + 128 + 32 * c4, o);
        }
      }
      // key rows past the sequence may hold anything: zero them in V
      if (mt.y < kTileTokens) {
        const int vs = it % kTCVStages;
        if (!mbar_wait(&bars->v_full[vs], (it / kTCVStages) & 1)) ok = false;
        uint8_t* vd = v_ring + vs * kTCTile;
        const int nz = (kTileTokens - mt.y) * 16;  // 16-byte pieces (2 boxes x 8 per row)
        for (int i = r; i < nz && ok; i += kTCRows) {
          const int key = mt.y + (i >> 4), piece = i & 15;
          *reinterpret_cast<uint4*>(vd + (piece >> 3) * kTCBox + key * 128 + (piece & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      // P (bf16) into the K slot of this tile: row r, 128-byte swizzled
      uint8_t* prow = k_ring + ks * kTCTile + r * 128;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint4 v;
        v.x = pack_bf16x2(x[8 * c8 + 0], x[8 * c8 + 1]);
        v.y = pack_bf16x2(x[8 * c8 + 2], x[8 * c8 + 3]);
        v.z = pack_bf16x2(x[8 * c8 + 4], x[8 * c8 + 5]);
        v.w = pack_bf16x2(x[8 * c8 + 6], x[8 * c8 + 7]);
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (!ok) flag_status(p.status, SEER_DEV_TIMEOUT);
    // ---- epilogue: the last P V, then normalise, bf16 out, natural-log lse
    bool have_o = ok && it >= 1;
    if (have_o) {
      if (it >= 2) have_o = wait_pv(it - 2);
      have_o = wait_pv(it - 1) && have_o;
      have_o = __all_sync(0xffffffffu, have_o);
      if (!have_o) flag_status(p.status, SEER_DEV_TIMEOUT);
    }
    tc_fence_after();
    const int gs = r >> 6;
    const int qh = h * p.G + g0 + gs;
    const bool store = (gs == 0 || two) && tq < L;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    uint16_t* orow = p.out + (((int64_t)b * Lq + tq) * p.Hq + qh) * kHeadDim;
#pragma unroll 1
    for (int c2 = 0; c2 < 2; ++c2) {
      uint32_t o[64];
      if (have_o) {
        __syncwarp();
        tmem_ld64(lane_addr + 128 + 64 * c2, o);
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) o[e] = 0u;
      }
      if (store) {
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * e8 + 0]) * inv, __uint_as_float(o[8 * e8 + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(o[8 * e8 + 2]) * inv, __uint_as_float(o[8 * e8 + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(o[8 * e8 + 4]) * inv, __uint_as_float(o[8 * e8 + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(o[8 * e8 + 6]) * inv, __uint_as_float(o[8 * e8 + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + 64 * c2 + 8 * e8) = v;
        }
      }
    }
    if (store && p.lse != nullptr)
      p.lse[((int64_t)b * p.Hq + qh) * Lq + tq] =
          l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTCCols);
  }
}

cudaError_t run_prefill_attention(const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const PrefillParams& p,
                                  cudaStream_t stream) {
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem_limit(prefill_attention_kernel, smem_set);
  if (e != cudaSuccess) return e;
  dim3 grid(p.max_blocks * p.bs / kTileTokens, p.Hkv * ((p.G + 1) / 2), p.B);
  prefill_attention_kernel<<<grid, kTCThreads, kTCSmem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace seer

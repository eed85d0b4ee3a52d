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
constexpr int kPAMathWarps = 4;                          // 16 query tokens each
constexpr int kPAThreads = (kPAMathWarps + 1) * 32;      // + the copy warp
constexpr int kPAStages = 3;
constexpr int kPAHalf = kTileTokens * 64 * 2;            // 64 tokens x 64 dims bf16
constexpr int kPAStageBytes = 4 * kPAHalf;               // K lo, K hi, V lo, V hi
constexpr size_t kPABars = (size_t)kPAStages * kPAStageBytes;
constexpr size_t kPASmem = 1024 + kPABars + 16 * kPAStages + 8 * kPAStages;

__device__ __forceinline__ uint32_t ld_bf16x2(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint32_t*>(p));
}

__global__ void __launch_bounds__(kPAThreads, 2)
    prefill_attention_kernel(const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  extern __shared__ uint8_t pa_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pa_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPABars);
  uint64_t* empty = full + kPAStages;
  int2* meta = reinterpret_cast<int2*>(empty + kPAStages);  // (first key token, valid keys)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Lq = p.max_blocks * p.bs;
  const int ntiles = Lq / kTileTokens;
  const int tile = ntiles - 1 - (int)blockIdx.x;  // longest causal prefixes first
  const int qh = blockIdx.y, b = blockIdx.z, h = qh / p.G;
  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, Lq));
  const int t0 = tile * kTileTokens;
  if (t0 >= L) return;  // the whole CTA: no query token here
  const int t_last = min(t0 + kTileTokens - 1, L - 1);
  const int qb = t0 / p.bs;  // query block of this tile
  const int64_t row = ((int64_t)b * p.Hkv + h) * p.max_blocks + qb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPAStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kPAMathWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kPAMathWarps) {
    // ================================================================ copies
    if (lane != 0) return;
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    const uint64_t policy = policy_evict_first();
    const int n = max(0, min(__ldg(p.n_sel + row), p.k_max));
    const int nb = ceil_div_i(L, p.bs);
    uint32_t issued = 0;
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
        const int slot = issued % kPAStages;
        if (!mbar_wait(&empty[slot], ((issued / kPAStages) & 1) ^ 1)) {
          flag_status(p.status, SEER_DEV_TIMEOUT);
          ok = false;
          break;
        }
        meta[slot] = make_int2(s0, min(kTileTokens, L - s0));
        mbar_arrive_expect_tx(&full[slot], kPAStageBytes);
        const int t = e * kTileTokens;
        const int c1 = p.token_inner ? t : h, c2 = p.token_inner ? h : t;
        uint8_t* st = ring + slot * kPAStageBytes;
        tma_load_4d(st + 0 * kPAHalf, &tm_k, 0, c1, c2, (int)page, &full[slot], policy);
        tma_load_4d(st + 1 * kPAHalf, &tm_k, 64, c1, c2, (int)page, &full[slot], policy);
        tma_load_4d(st + 2 * kPAHalf, &tm_v, 0, c1, c2, (int)page, &full[slot], policy);
        tma_load_4d(st + 3 * kPAHalf, &tm_v, 64, c1, c2, (int)page, &full[slot], policy);
        ++issued;
      }
    }
    bool marked = false;
    if (ok) {  // end marker: a stage with no data
      const int slot = issued % kPAStages;
      if (mbar_wait(&empty[slot], ((issued / kPAStages) & 1) ^ 1)) {
        meta[slot] = make_int2(0, -1);
        mbar_arrive(&full[slot]);
        marked = true;
      } else {
        flag_status(p.status, SEER_DEV_TIMEOUT);
      }
    }
    // Let every copy this CTA started land before it retires.  With the end
    // marker posted, the stage that last used the marker's slot was released
    // by every math warp (so its copy landed), and its full barrier has moved
    // on by the marker's phase: a parity wait on it could not tell the two
    // apart, so it is left out.
    const uint32_t in_flight = marked ? kPAStages - 1 : kPAStages;
    for (uint32_t k = 0; k < in_flight && k < issued; ++k) {
      const uint32_t s = issued - 1 - k;
      if (!mbar_wait(&full[s % kPAStages], (s / kPAStages) & 1))
        flag_status(p.status, SEER_DEV_TIMEOUT);
    }
    return;
  }

  // ================================================================== math
  const int r = lane >> 2, c = lane & 3;
  const int ta = t0 + warp * 16 + r, tb = ta + 8;  // this thread's two query rows
  // Q as the A operand (16 tokens x 128 dims), straight from global memory
  uint32_t qa[8][4];
  {
    const uint16_t* qra = p.q + (((int64_t)b * Lq + ta) * p.Hq + qh) * kHeadDim + 2 * c;
    const uint16_t* qrb = p.q + (((int64_t)b * Lq + tb) * p.Hq + qh) * kHeadDim + 2 * c;
    const bool ina = ta < L, inb = tb < L;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = ina ? ld_bf16x2(qra + 16 * ks) : 0u;
      qa[ks][1] = inb ? ld_bf16x2(qrb + 16 * ks) : 0u;
      qa[ks][2] = ina ? ld_bf16x2(qra + 16 * ks + 8) : 0u;
      qa[ks][3] = inb ? ld_bf16x2(qrb + 16 * ks + 8) : 0u;
    }
  }
  float o[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;

  for (int k = 0;; ++k) {
    const int slot = k % kPAStages;
    if (!mbar_wait(&full[slot], (k / kPAStages) & 1)) {
      flag_status(p.status, SEER_DEV_TIMEOUT);
      break;
    }
    const int2 mt = meta[slot];
    if (mt.y < 0) break;  // end marker
    const int s0 = mt.x, valid = mt.y;
    const uint32_t kbase = smem_u32(ring + slot * kPAStageBytes);
    const uint32_t vbase = kbase + 2 * kPAHalf;

    // ---- S = Q K^T (16 tokens x 64 keys), K rows as the B operand
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
      for (int kp = 0; kp < 4; ++kp) {
        const int key = nt * 8 + (lane & 7);
        const int chunk = 4 * kp + (lane >> 3);
        const uint32_t addr = kbase + (chunk >> 3) * kPAHalf + key * 128 +
                              (((chunk & 7) ^ (key & 7)) << 4);
        uint32_t x0, x1, x2, x3;
        ldmatrix_x4(addr, x0, x1, x2, x3);
        mma_bf16_16816(s[nt], qa[2 * kp], x0, x1);
        mma_bf16_16816(s[nt], qa[2 * kp + 1], x2, x3);
      }
    }
    // ---- causal and tail masks, online softmax in the exp2 domain
    float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nt * 8 + 2 * c + (e & 1);
        const int tq = e < 2 ? ta : tb;
        const bool masked = col >= valid || s0 + col > tq;
        s[nt][e] = masked ? -INFINITY : s[nt][e] * p.scale_log2;
      }
      mxa = fmaxf(mxa, fmaxf(s[nt][0], s[nt][1]));
      mxb = fmaxf(mxb, fmaxf(s[nt][2], s[nt][3]));
    }
    mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
    mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
    mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
    mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
    const float na = fmaxf(ma, mxa), nbm = fmaxf(mb, mxb);
    const float ua = na == -INFINITY ? 0.f : na, ub = nbm == -INFINITY ? 0.f : nbm;
    const float alpha_a = fast_exp2(ma - ua), alpha_b = fast_exp2(mb - ub);
    ma = na;
    mb = nbm;
    float suma = 0.f, sumb = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = fast_exp2(s[nt][0] - ua);
      s[nt][1] = fast_exp2(s[nt][1] - ua);
      s[nt][2] = fast_exp2(s[nt][2] - ub);
      s[nt][3] = fast_exp2(s[nt][3] - ub);
      suma += s[nt][0] + s[nt][1];
      sumb += s[nt][2] + s[nt][3];
    }
    la = la * alpha_a + suma;
    lb = lb * alpha_b + sumb;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      o[dt][0] *= alpha_a;
      o[dt][1] *= alpha_a;
      o[dt][2] *= alpha_b;
      o[dt][3] *= alpha_b;
    }
    // ---- O += P V: P (from the S accumulators) rounded to bf16, V by ldmatrix.trans
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t ph[4];
      ph[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      ph[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      ph[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      ph[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      // tail keys (past the sequence) may hold anything: zero their V
      const int k0 = 16 * kk + 2 * c;
      const uint32_t m0 = (k0 < valid ? 0x0000ffffu : 0u) | (k0 + 1 < valid ? 0xffff0000u : 0u);
      const uint32_t m1 =
          (k0 + 8 < valid ? 0x0000ffffu : 0u) | (k0 + 9 < valid ? 0xffff0000u : 0u);
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        const int key = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int chunk = 2 * dp + (lane >> 4);
        const uint32_t addr = vbase + (chunk >> 3) * kPAHalf + key * 128 +
                              (((chunk & 7) ^ (key & 7)) << 4);
        uint32_t v0, v1, v2, v3;
        ldmatrix_x4_trans(addr, v0, v1, v2, v3);
        v0 &= m0;
        v1 &= m1;
        v2 &= m0;
        v3 &= m1;
        mma_bf16_16816(o[2 * dp], ph, v0, v1);
        mma_bf16_16816(o[2 * dp + 1], ph, v2, v3);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }

  // ---- epilogue: normalise, bf16 out, natural-log lse
  la += __shfl_xor_sync(0xffffffffu, la, 1);
  la += __shfl_xor_sync(0xffffffffu, la, 2);
  lb += __shfl_xor_sync(0xffffffffu, lb, 1);
  lb += __shfl_xor_sync(0xffffffffu, lb, 2);
  const float ia = la > 0.f ? 1.f / la : 0.f, ib = lb > 0.f ? 1.f / lb : 0.f;
  if (ta < L) {
    uint32_t* oa = reinterpret_cast<uint32_t*>(p.out + (((int64_t)b * Lq + ta) * p.Hq + qh) * kHeadDim);
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) oa[(dt * 8 + 2 * c) / 2] = pack_bf16x2(o[dt][0] * ia, o[dt][1] * ia);
    if (p.lse != nullptr && c == 0)
      p.lse[((int64_t)b * p.Hq + qh) * Lq + ta] = la > 0.f ? (ma + log2f(la)) * kLn2 : -INFINITY;
  }
  if (tb < L) {
    uint32_t* ob = reinterpret_cast<uint32_t*>(p.out + (((int64_t)b * Lq + tb) * p.Hq + qh) * kHeadDim);
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) ob[(dt * 8 + 2 * c) / 2] = pack_bf16x2(o[dt][2] * ib, o[dt][3] * ib);
    if (p.lse != nullptr && c == 0)
      p.lse[((int64_t)b * p.Hq + qh) * Lq + tb] = lb > 0.f ? (mb + log2f(lb)) * kLn2 : -INFINITY;
  }
}

cudaError_t run_prefill_attention(const CUtensorMap& tk, const CUtensorMap& tv,
                                  const PrefillParams& p, cudaStream_t stream) {
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem_limit(prefill_attention_kernel, smem_set);
  if (e != cudaSuccess) return e;
  dim3 grid(p.max_blocks * p.bs / kTileTokens, p.Hq, p.B);
  prefill_attention_kernel<<<grid, kPAThreads, kPASmem, stream>>>(tk, tv, p);
  return cudaGetLastError();
}

}  // namespace seer

// a3: split-KV sparse flash-decoding over the selected KV blocks.
//
// What it computes (Agent Skill page "Sparse Attention Reasoning", Step 4):
// for every (sequence b, KV head h, split s) the G query heads of the group
// attend, with softmax scale 1/sqrt(D), only the tokens t < seqlen_b of the
// blocks idx[b,h, floor(s*n/S) .. floor((s+1)*n/S)); the result is one
// normalised partial output and its log-sum-exp per query head.
//
// How it runs on sm_100a:
//   * persistent CTAs (one per SM) walk a static list of (b, h, s) items;
//   * one producer thread streams 64-token tiles of the selected K and V
//     blocks (4 boxes of 64 tokens x 64 dims, 128-byte swizzled) with 4-D
//     TMA loads into an NSTAGES-deep shared-memory ring guarded by mbarriers;
//     page lookup, block index and stride handling all live in the tensor
//     map coordinates, so the gather costs no address arithmetic in the math
//     warps;
//   * NGROUPS groups of 4 math warps take alternate tiles; inside a group each
//     warp owns 16 tokens of the tile and computes S = Q K^T and O += P V with
//     mma.sync m16n8k16 (the group's G <= 16 query heads are the 16 rows, so
//     each K/V byte is read from HBM once for all G heads), online softmax in
//     the exp2 domain with warp-quad shuffles, P fed to the tensor cores as a
//     bf16 hi + lo pair so the weights keep ~16 bits;
//   * at the end of an item the 4*NGROUPS warps merge their (m, l, O) through
//     shared memory and write o_part / lse_part.
// Every mbarrier wait is bounded (SEER_DEV_TIMEOUT); nothing traps.
#include "seer_kernels.cuh"

namespace seer {

constexpr int kHalfTileBytes = kTileTokens * 64 * 2;  // 64 tokens x 64 dims bf16
constexpr int kStageBytes = 4 * kHalfTileBytes;       // K lo, K hi, V lo, V hi

template <int NGROUPS, int NSTAGES>
struct DecodeShape {
  static constexpr int kMathWarps = 4 * NGROUPS;
  static constexpr int kThreads = (kMathWarps + 1) * 32;
  static size_t smem_bytes(int G) {
    return 1024 /* alignment slack */ + (size_t)NSTAGES * kStageBytes +
           2 * NSTAGES * sizeof(uint64_t) + (size_t)kMathWarps * 2 * kMaxGroup * sizeof(float) +
           (size_t)kMathWarps * G * kHeadDim * sizeof(float);
  }
};

// One work item: (b, h, split s) and the slice [lo, hi) of its index row.
struct Item {
  int b, h, s, L, nb, lo, hi;
};

__device__ __forceinline__ Item decode_item(const DecodeParams& p, int item) {
  Item it;
  const int bh = item / p.S;
  it.s = item - bh * p.S;
  it.b = bh / p.Hkv;
  it.h = bh - it.b * p.Hkv;
  int L = __ldg(p.seqlens + it.b);
  L = max(0, min(L, p.max_blocks * p.bs));
  it.L = L;
  it.nb = ceil_div_i(L, p.bs);
  int n = __ldg(p.n_sel + bh);
  n = max(0, min(n, p.k_max));
  it.lo = (int)(((long long)it.s * n) / p.S);
  it.hi = (int)(((long long)(it.s + 1) * n) / p.S);
  return it;
}

// Block index i of the item's row, or -1 if it is not a valid block.
__device__ __forceinline__ int block_at(const DecodeParams& p, const Item& it, int i) {
  const int j = __ldg(p.idx + (int64_t)(it.b * p.Hkv + it.h) * p.k_max + i);
  return (j >= 0 && j < it.nb) ? j : -1;
}

template <int NGROUPS, int NSTAGES>
__global__ void __launch_bounds__(DecodeShape<NGROUPS, NSTAGES>::kThreads, 1)
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using Shape = DecodeShape<NGROUPS, NSTAGES>;
  constexpr int kMathWarps = Shape::kMathWarps;
  constexpr int kMathThreads = kMathWarps * 32;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(ring + NSTAGES * kStageBytes);
  uint64_t* empty_bar = full_bar + NSTAGES;
  float* m_sh = reinterpret_cast<float*>(empty_bar + NSTAGES);  // [warps][16]
  float* l_sh = m_sh + kMathWarps * kMaxGroup;                   // [warps][16]
  float* o_sh = l_sh + kMathWarps * kMaxGroup;                   // [warps][G][128]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 4);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kMathWarps) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    const uint64_t policy = policy_evict_first();
    uint32_t issued = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
      const Item it = decode_item(p, item);
      for (int i = it.lo; i < it.hi && ok; ++i) {
        const int j = block_at(p, it, i);
        if (j < 0) {
          flag_status(p.status, SEER_DEV_BAD_INDEX);
          continue;
        }
        int64_t page = page_of(p.page_table, it.b, j, p.max_blocks);
        if (page < 0 || page >= p.num_pages) {
          flag_status(p.status, SEER_DEV_BAD_PAGE);
          page = 0;  // keep the copy inside the pool; the result is flagged
        }
        for (int sub = 0; sub < p.bs / kTileTokens; ++sub) {
          const int tok0 = j * p.bs + sub * kTileTokens;
          if (tok0 >= it.L) break;
          const int slot = issued % NSTAGES;
          const uint32_t phase = (issued / NSTAGES) & 1;
          if (!mbar_wait(&empty_bar[slot], phase ^ 1)) {
            flag_status(p.status, SEER_DEV_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* st = ring + slot * kStageBytes;
          mbar_arrive_expect_tx(&full_bar[slot], kStageBytes);
          const int t = sub * kTileTokens;
          const int c1 = p.token_inner ? t : it.h;
          const int c2 = p.token_inner ? it.h : t;
          const int pg = (int)page;
          tma_load_4d(st + 0 * kHalfTileBytes, &tm_k, 0, c1, c2, pg, &full_bar[slot], policy);
          tma_load_4d(st + 1 * kHalfTileBytes, &tm_k, 64, c1, c2, pg, &full_bar[slot], policy);
          tma_load_4d(st + 2 * kHalfTileBytes, &tm_v, 0, c1, c2, pg, &full_bar[slot], policy);
          tma_load_4d(st + 3 * kHalfTileBytes, &tm_v, 64, c1, c2, pg, &full_bar[slot], policy);
          ++issued;
        }
      }
    }
    // Let every copy this CTA started land before the CTA can retire.
    for (uint32_t k = 0; k < NSTAGES && k < issued; ++k) {
      const uint32_t s_it = issued - 1 - k;
      mbar_wait(&full_bar[s_it % NSTAGES], (s_it / NSTAGES) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- math warps
  const int group = warp / 4;
  const int wq = warp % 4;         // which 16 tokens of a tile
  const int r = lane >> 2;         // fragment row (query head) r and r + 8
  const int c = lane & 3;          // fragment column pair
  const int G = p.G;
  uint32_t stage_iter = 0;
  bool ok = true;

  for (int item = blockIdx.x; item < p.num_items; item += gridDim.x) {
    const Item it = decode_item(p, item);

    // Q fragments: rows = the group's query heads (zero past G), 8 k-steps.
    uint32_t qa[8][4];
    {
      const uint16_t* qrow0 = p.q + ((int64_t)it.b * p.Hq + (int64_t)it.h * G + r) * kHeadDim;
      const uint16_t* qrow1 = qrow0 + 8 * kHeadDim;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int d0 = kk * 16 + 2 * c;
        qa[kk][0] = (r < G) ? __ldg(reinterpret_cast<const uint32_t*>(qrow0 + d0)) : 0u;
        qa[kk][1] = (r + 8 < G) ? __ldg(reinterpret_cast<const uint32_t*>(qrow1 + d0)) : 0u;
        qa[kk][2] = (r < G) ? __ldg(reinterpret_cast<const uint32_t*>(qrow0 + d0 + 8)) : 0u;
        qa[kk][3] = (r + 8 < G) ? __ldg(reinterpret_cast<const uint32_t*>(qrow1 + d0 + 8)) : 0u;
      }
    }

    float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 domain) of rows r, r+8
    float l0 = 0.f, l1 = 0.f;              // this thread's share of the row sums
    float o[16][4];
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;

    for (int i = it.lo; i < it.hi; ++i) {
      const int j = block_at(p, it, i);
      if (j < 0) continue;
      for (int sub = 0; sub < p.bs / kTileTokens; ++sub) {
        const int tok0 = j * p.bs + sub * kTileTokens;
        if (tok0 >= it.L) break;
        const uint32_t my_iter = stage_iter++;
        if ((int)(my_iter % NGROUPS) != group) continue;
        const int slot = my_iter % NSTAGES;
        const uint32_t phase = (my_iter / NSTAGES) & 1;
        if (ok && !mbar_wait(&full_bar[slot], phase)) {
          flag_status(p.status, SEER_DEV_TIMEOUT);
          ok = false;
        }
        if (ok) {
          const uint32_t k_base = smem_u32(ring + slot * kStageBytes);
          const uint32_t v_base = k_base + 2 * kHalfTileBytes;
          const int valid = it.L - tok0;  // >= 1; < 64 only on the newest tile

          // ---- S = Q K^T for this warp's 16 tokens (2 n-tiles of 8)
          float s[2][4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
            const int tok = wq * 16 + nt * 8 + (lane & 7);
            const int mi = lane >> 3;
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
              const int half = kp >> 1;
              const int chunk = (kp & 1) * 4 + mi;
              const uint32_t addr = k_base + half * kHalfTileBytes + tok * 128 +
                                    ((chunk ^ (tok & 7)) << 4);
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4(addr, b0, b1, b2, b3);
              mma_bf16_16816(s[nt], qa[2 * kp], b0, b1);
              mma_bf16_16816(s[nt], qa[2 * kp + 1], b2, b3);
            }
          }
          // ---- scale, mask tokens past the sequence end, online softmax
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int t_rel = wq * 16 + nt * 8 + 2 * c;
            const bool v0 = t_rel < valid, v1 = t_rel + 1 < valid;
            s[nt][0] = v0 ? s[nt][0] * p.scale_log2 : -INFINITY;
            s[nt][1] = v1 ? s[nt][1] * p.scale_log2 : -INFINITY;
            s[nt][2] = v0 ? s[nt][2] * p.scale_log2 : -INFINITY;
            s[nt][3] = v1 ? s[nt][3] * p.scale_log2 : -INFINITY;
          }
          float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
          float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
          const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
          const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
          const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
          const float a0 = fast_exp2(m0 - mu0), a1 = fast_exp2(m1 - mu1);
          m0 = mn0;
          m1 = mn1;
          float pr[2][4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            pr[nt][0] = fast_exp2(s[nt][0] - mu0);
            pr[nt][1] = fast_exp2(s[nt][1] - mu0);
            pr[nt][2] = fast_exp2(s[nt][2] - mu1);
            pr[nt][3] = fast_exp2(s[nt][3] - mu1);
          }
          l0 = l0 * a0 + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
          l1 = l1 * a1 + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
#pragma unroll
          for (int nd = 0; nd < 16; ++nd) {
            o[nd][0] *= a0;
            o[nd][1] *= a0;
            o[nd][2] *= a1;
            o[nd][3] *= a1;
          }
          // P as a bf16 pair hi + lo (hi = RNE(p), lo = RNE(p - hi)): the
          // product P V then carries p to ~2^-16 instead of bf16's 2^-9, so
          // heavy-tailed V rows do not amplify the rounding of the weights.
          uint32_t pa[4], pl[4];
          split_bf16x2(pr[0][0], pr[0][1], pa[0], pl[0]);
          split_bf16x2(pr[0][2], pr[0][3], pa[1], pl[1]);
          split_bf16x2(pr[1][0], pr[1][1], pa[2], pl[2]);
          split_bf16x2(pr[1][2], pr[1][3], pa[3], pl[3]);

          // ---- O += P V (V tile rows past the end are zeroed in registers:
          // their P is 0 but the slot may hold anything, NaN included)
          uint32_t vmask_lo = 0xffffffffu, vmask_hi = 0xffffffffu;
          if (valid < kTileTokens) {
            const int t0 = wq * 16 + 2 * c, t1 = t0 + 8;
            vmask_lo = (t0 < valid ? 0x0000ffffu : 0u) | (t0 + 1 < valid ? 0xffff0000u : 0u);
            vmask_hi = (t1 < valid ? 0x0000ffffu : 0u) | (t1 + 1 < valid ? 0xffff0000u : 0u);
          }
          const int mi = lane >> 3;
          const int vtok = wq * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
          for (int dp = 0; dp < 8; ++dp) {
            const int half = dp >> 2;
            const int chunk = (dp & 3) * 2 + (mi >> 1);
            const uint32_t addr = v_base + half * kHalfTileBytes + vtok * 128 +
                                  ((chunk ^ (vtok & 7)) << 4);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(addr, b0, b1, b2, b3);
            b0 &= vmask_lo;
            b1 &= vmask_hi;
            b2 &= vmask_lo;
            b3 &= vmask_hi;
            mma_bf16_16816(o[2 * dp], pa, b0, b1);
            mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
            mma_bf16_16816(o[2 * dp], pl, b0, b1);
            mma_bf16_16816(o[2 * dp + 1], pl, b2, b3);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);
      }
    }

    // ---- merge the math warps' partial softmax states for this item
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (c == 0) {
      m_sh[warp * kMaxGroup + r] = m0;
      l_sh[warp * kMaxGroup + r] = l0;
      m_sh[warp * kMaxGroup + r + 8] = m1;
      l_sh[warp * kMaxGroup + r + 8] = l1;
    }
    float* ow = o_sh + (size_t)warp * G * kHeadDim;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      const int d = nd * 8 + 2 * c;
      if (r < G) *reinterpret_cast<float2*>(ow + r * kHeadDim + d) = make_float2(o[nd][0], o[nd][1]);
      if (r + 8 < G)
        *reinterpret_cast<float2*>(ow + (r + 8) * kHeadDim + d) = make_float2(o[nd][2], o[nd][3]);
    }
    named_barrier_sync(1, kMathThreads);
    for (int e = threadIdx.x; e < G * kHeadDim; e += kMathThreads) {
      const int g = e / kHeadDim, d = e - g * kHeadDim;
      float mt = -INFINITY;
#pragma unroll
      for (int w = 0; w < kMathWarps; ++w) mt = fmaxf(mt, m_sh[w * kMaxGroup + g]);
      const int64_t row = ((int64_t)it.b * p.Hq + (int64_t)it.h * G + g) * p.S + it.s;
      if (mt == -INFINITY) {
        p.o_part[row * kHeadDim + d] = 0.f;
        if (d == 0) p.lse_part[row] = -INFINITY;
        continue;
      }
      float lt = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < kMathWarps; ++w) {
        const float f = fast_exp2(m_sh[w * kMaxGroup + g] - mt);
        lt += l_sh[w * kMaxGroup + g] * f;
        acc += o_sh[((size_t)w * G + g) * kHeadDim + d] * f;
      }
      p.o_part[row * kHeadDim + d] = acc / lt;
      if (d == 0) p.lse_part[row] = (mt + log2f(lt)) * kLn2;
    }
    named_barrier_sync(1, kMathThreads);
  }
}

// ------------------------------------------------------------------ launcher
template <int NGROUPS, int NSTAGES>
static cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv,
                                 const DecodeParams& p, int num_sms, cudaStream_t stream) {
  using Shape = DecodeShape<NGROUPS, NSTAGES>;
  const size_t smem = Shape::smem_bytes(p.G);
  auto kern = sparse_decode_kernel<NGROUPS, NSTAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = p.num_items < num_sms ? p.num_items : num_sms;
  kern<<<grid, Shape::kThreads, smem, stream>>>(tk, tv, p);
  return cudaGetLastError();
}

cudaError_t run_sparse_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                              int num_sms, cudaStream_t stream) {
  return launch_decode<2, 4>(tk, tv, p, num_sms, stream);
}

}  // namespace seer

// a2: per-(b, h) top-k block selection (Agent Skill page, Step 1: top-k over
// the gate scores), exact and deterministic.
//
// Order: score descending, then block index ascending; -0.0 equals +0.0; NaN
// ranks below -inf.  The newest block NB-1, when forced, is taken first and
// counts toward k.  Output: the chosen indices ascending, -1 padded.
//
// One CTA of 1024 threads per (b, h); thread t owns blocks 4t .. 4t+3 so a
// block-wide scan visits blocks in index order.  Scores become order-
// preserving 32-bit keys; a 4-pass MSB radix select (8-bit digits, shared-
// memory histograms, one warp picking the digit) finds the k'-th largest key
// T and how many keys equal to T are still needed; a scan over "key == T"
// ranks the ties by index, and a second scan compacts the chosen blocks in
// ascending order.  No sort, no data-dependent loop bounds beyond NB.
#include "seer_kernels.cuh"

namespace seer {

constexpr int kSelThreads = 1024;
constexpr int kSelItems = kMaxBlocks / kSelThreads;  // 4

// Order-preserving key: larger score -> larger key; NaN -> 0 (lowest).
__device__ __forceinline__ uint32_t order_key(float f, bool& nan_seen) {
  if (f != f) {
    nan_seen = true;
    return 0u;
  }
  uint32_t u = __float_as_uint(f);
  if (f == 0.0f) u = 0u;  // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the CTA in thread order; returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int& total, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  total = warp_sums[31];
  const int before = (warp > 0) ? warp_sums[warp - 1] : 0;
  __syncthreads();  // warp_sums may be reused right after
  return before + x - v;
}

__global__ void __launch_bounds__(kSelThreads) block_select_kernel(const SelectParams p) {
  __shared__ int hist[256];
  __shared__ int warp_sums[32];
  __shared__ int pick_digit, pick_above;

  const int b = blockIdx.y, h = blockIdx.x;
  const int64_t bh = (int64_t)b * p.Hkv + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  int L = __ldg(p.seqlens + b);
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  int k = __ldg(p.k_per_seq + b);
  if (k < 1) k = 1;
  if (k > p.k_max) {
    k = p.k_max;
    if (tid == 0) flag_status(p.status, SEER_DEV_K_CLAMPED);
  }
  const int n = min(k, nb);
  const int forced = (p.force_newest && n > 0) ? 1 : 0;
  const int cand = nb - forced;  // candidates: blocks 0 .. cand-1
  const int want = n - forced;   // picked on merit
  const float* row = p.scores + bh * p.max_blocks;

  uint32_t key[kSelItems];
  bool nan_seen = false;
#pragma unroll
  for (int i = 0; i < kSelItems; ++i) {
    const int j = tid * kSelItems + i;
    key[i] = (j < cand) ? order_key(__ldg(row + j), nan_seen) : 0u;
  }
  if (nan_seen) flag_status(p.status, SEER_DEV_NONFINITE_SCORE);

  bool sel[kSelItems];
  if (want >= cand) {
#pragma unroll
    for (int i = 0; i < kSelItems; ++i) sel[i] = (tid * kSelItems + i) < cand;
  } else if (want <= 0) {
#pragma unroll
    for (int i = 0; i < kSelItems; ++i) sel[i] = false;
  } else {
    uint32_t prefix = 0u, mask = 0u;
    int remaining = want;  // rank (from the top) of the threshold key
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      if (tid < 256) hist[tid] = 0;
      __syncthreads();
#pragma unroll
      for (int i = 0; i < kSelItems; ++i) {
        const int j = tid * kSelItems + i;
        if (j < cand && (key[i] & mask) == prefix) atomicAdd(&hist[(key[i] >> shift) & 255], 1);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l covers digits 255-8l down to 248-8l (descending)
        int cnt[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cnt[e] = hist[255 - 8 * lane - e];
          tot += cnt[e];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int excl = incl - tot;
        if (excl < remaining && remaining <= incl) {
          int acc = excl;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (acc + cnt[e] >= remaining) {
              pick_digit = 255 - 8 * lane - e;
              pick_above = acc;
              break;
            }
            acc += cnt[e];
          }
        }
      }
      __syncthreads();
      remaining -= pick_above;
      prefix |= (uint32_t)pick_digit << shift;
      mask |= 0xffu << shift;
      __syncthreads();
    }
    // keys > prefix are in; `remaining` keys equal to prefix, lowest index first
    int eq_local = 0;
#pragma unroll
    for (int i = 0; i < kSelItems; ++i) eq_local += ((tid * kSelItems + i) < cand && key[i] == prefix);
    int eq_total;
    int eq_rank = block_exclusive_scan(eq_local, eq_total, warp_sums);
#pragma unroll
    for (int i = 0; i < kSelItems; ++i) {
      const int j = tid * kSelItems + i;
      const bool valid = j < cand;
      if (valid && key[i] == prefix) {
        sel[i] = eq_rank < remaining;
        ++eq_rank;
      } else {
        sel[i] = valid && key[i] > prefix;
      }
    }
  }
  if (forced) {
#pragma unroll
    for (int i = 0; i < kSelItems; ++i)
      if (tid * kSelItems + i == nb - 1) sel[i] = true;
  }
  int local = 0;
#pragma unroll
  for (int i = 0; i < kSelItems; ++i) local += sel[i];
  int total;
  int pos = block_exclusive_scan(local, total, warp_sums);
  int32_t* out = p.idx + bh * p.k_max;
#pragma unroll
  for (int i = 0; i < kSelItems; ++i) {
    if (sel[i]) {
      if (pos < p.k_max) out[pos] = tid * kSelItems + i;
      ++pos;
    }
  }
  for (int q = total + tid; q < p.k_max; q += kSelThreads) out[q] = -1;
  if (tid == 0) p.n_sel[bh] = total;
}

cudaError_t run_block_select(const SelectParams& p, int B, cudaStream_t stream) {
  dim3 grid(p.Hkv, B);
  block_select_kernel<<<grid, kSelThreads, 0, stream>>>(p);
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

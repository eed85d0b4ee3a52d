// Exact top-k of one score row (Agent Skill page, Step 1: top-k over the gate
// scores; ties to the lower block index, optional forced newest block,
// ascending output, from the step specification), two ways: select_topk (a
// radix select: the standalone selection kernel, and the fused gate +
// selection kernel on rows longer than its CTA) and select_topk_sorted (a
// bitonic sort in registers: the fused kernel on rows of at most 512 blocks).
// Both are exact, so they return the same rows.
//
// select_topk: THREADS threads own ITEMS consecutive blocks each, so block-wide scans run
// in index order.  Scores map to order-preserving 32-bit keys (-0.0 as +0.0,
// NaN lowest); a 4-pass MSB radix select (8-bit digits) finds the k'-th
// largest key and how many keys equal to it are still needed; a scan over
// "key == threshold" ranks the ties by index, and a second scan writes the
// chosen indices in ascending order, padded with -1 to k_max.
#pragma once

#include "seer_common.cuh"

namespace seer {

struct SelectSmem {
  int hist[256];
  int warp_sums[32];
  int pick_digit;
  int pick_above;
};

__device__ __forceinline__ uint32_t order_key(float f, bool& nan_seen) {
  if (f != f) {
    nan_seen = true;
    return 0u;
  }
  uint32_t u = __float_as_uint(f);
  if (f == 0.0f) u = 0u;  // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the CTA in thread order; returns it, total in `total`.
template <int THREADS>
__device__ __forceinline__ int block_exclusive_scan(int v, int& total, int* warp_sums) {
  constexpr int kWarps = THREADS / 32;
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
    int w = lane < kWarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  total = warp_sums[kWarps - 1];
  const int before = (warp > 0) ? warp_sums[warp - 1] : 0;
  __syncthreads();  // warp_sums may be reused right after
  return before + x - v;
}

// Selects from row[0 .. nb) (global or shared), writes out[0 .. k_max) and
// *n_out.  k < 1 counts as 1; k > k_max is clamped (SEER_DEV_K_CLAMPED).
// Every thread of the CTA must call it (it synchronises).
template <int THREADS, int ITEMS>
__device__ void select_topk(const float* row, int nb, int k, int force_newest, int k_max,
                            int32_t* out, int32_t* n_out, int32_t* status, SelectSmem& sm) {
  static_assert(THREADS * ITEMS >= kMaxBlocks, "one item per block");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (k < 1) k = 1;
  if (k > k_max) {
    k = k_max;
    if (tid == 0) flag_status(status, SEER_DEV_K_CLAMPED);
  }
  const int n = min(k, nb);
  const int forced = (force_newest && n > 0) ? 1 : 0;
  const int cand = nb - forced;  // candidates: blocks 0 .. cand-1
  const int want = n - forced;   // picked on merit

  uint32_t key[ITEMS];
  bool nan_seen = false;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const int j = tid * ITEMS + i;
    key[i] = (j < cand) ? order_key(row[j], nan_seen) : 0u;
  }
  if (nan_seen) flag_status(status, SEER_DEV_NONFINITE_SCORE);

  bool sel[ITEMS];
  if (want >= cand) {
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) sel[i] = (tid * ITEMS + i) < cand;
  } else if (want <= 0) {
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) sel[i] = false;
  } else {
    uint32_t prefix = 0u, mask = 0u;
    int remaining = want;  // rank (from the top) of the threshold key
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int e = tid; e < 256; e += THREADS) sm.hist[e] = 0;
      __syncthreads();
      // warp-aggregated: lanes holding the same digit add once (gate scores
      // crowd into few digits, which would serialise per-lane atomics)
#pragma unroll
      for (int i = 0; i < ITEMS; ++i) {
        const int j = tid * ITEMS + i;
        const bool in = j < cand && (key[i] & mask) == prefix;
        const int digit = in ? (int)((key[i] >> shift) & 255u) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, digit);
        if (in && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[digit], __popc(peers));
      }
      __syncthreads();
      if (warp == 0) {
        // lane l covers digits 255-8l down to 248-8l (descending)
        int cnt[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cnt[e] = sm.hist[255 - 8 * lane - e];
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
              sm.pick_digit = 255 - 8 * lane - e;
              sm.pick_above = acc;
              break;
            }
            acc += cnt[e];
          }
        }
      }
      __syncthreads();
      remaining -= sm.pick_above;
      prefix |= (uint32_t)sm.pick_digit << shift;
      mask |= 0xffu << shift;
      __syncthreads();
    }
    // keys > prefix are in; `remaining` keys equal to prefix, lowest index first
    int eq_local = 0;
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) eq_local += ((tid * ITEMS + i) < cand && key[i] == prefix);
    int eq_total;
    int eq_rank = block_exclusive_scan<THREADS>(eq_local, eq_total, sm.warp_sums);
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
      const int j = tid * ITEMS + i;
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
    for (int i = 0; i < ITEMS; ++i)
      if (tid * ITEMS + i == nb - 1) sel[i] = true;
  }
  int local = 0;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) local += sel[i];
  int total;
  int pos = block_exclusive_scan<THREADS>(local, total, sm.warp_sums);
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    if (sel[i]) {
      if (pos < k_max) out[pos] = tid * ITEMS + i;
      ++pos;
    }
  }
  for (int q = total + tid; q < k_max; q += THREADS) out[q] = -1;
  if (tid == 0) *n_out = total;
}

// The same selection by sorting, for rows of at most THREADS blocks: thread t
// holds key t (order_key(score) << 32 | ~index: score descending, then lower
// index first; the forced newest block gets the top key; padding 0) and a
// bitonic network sorts them descending -- stages with stride < 32 through
// warp shuffles, the others through a double-buffered shared array, one
// barrier each -- so thread t ends up holding the t-th largest key.  The first
// n_sel keys mark their blocks and a scan writes them in ascending order.
// Exact, like select_topk.  xchg: 2 * THREADS keys; flags: >= nb ints.
template <int THREADS>
__device__ void select_topk_sorted(const float* row, int nb, int k, int force_newest, int k_max,
                                   int32_t* out, int32_t* n_out, int32_t* status, uint64_t* xchg,
                                   int* flags, int* warp_sums) {
  static_assert(THREADS >= 32 && (THREADS & (THREADS - 1)) == 0, "power-of-two CTA");
  const int tid = threadIdx.x;
  if (k < 1) k = 1;
  if (k > k_max) {
    k = k_max;
    if (tid == 0) flag_status(status, SEER_DEV_K_CLAMPED);
  }
  const int n = min(k, nb);
  const bool forced = force_newest && n > 0;
  int np = 32;
  while (np < nb) np <<= 1;  // nb <= THREADS by contract
  bool nan_seen = false;
  uint64_t key = 0;  // padding sorts last
  if (tid < nb) {
    const uint32_t hi = (forced && tid == nb - 1) ? 0xffffffffu : order_key(row[tid], nan_seen);
    key = ((uint64_t)hi << 32) | (uint32_t)(~(uint32_t)tid);
  }
  if (nan_seen) flag_status(status, SEER_DEV_NONFINITE_SCORE);
  int buf = 0;
  for (int size = 2; size <= np; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      uint64_t other;
      if (stride < 32) {
        other = __shfl_xor_sync(0xffffffffu, key, stride);
      } else {
        if (tid < np) xchg[buf * THREADS + tid] = key;
        __syncthreads();
        other = (tid < np) ? xchg[buf * THREADS + (tid ^ stride)] : 0;
        buf ^= 1;  // the next exchange writes the other half: no second barrier
      }
      const bool desc = (tid & size) == 0;
      const bool lower = (tid & stride) == 0;
      const bool keep_max = (lower == desc);
      key = keep_max ? (key > other ? key : other) : (key < other ? key : other);
    }
  }
  for (int i = tid; i < nb; i += THREADS) flags[i] = 0;
  __syncthreads();
  if (tid < n) flags[~(uint32_t)(key & 0xffffffffu)] = 1;
  __syncthreads();
  const int mine = (tid < nb) ? flags[tid] : 0;
  int total;
  const int pos = block_exclusive_scan<THREADS>(mine, total, warp_sums);
  if (mine && pos < k_max) out[pos] = tid;
  for (int q = total + tid; q < k_max; q += THREADS) out[q] = -1;
  if (tid == 0) *n_out = total;
}

}  // namespace seer

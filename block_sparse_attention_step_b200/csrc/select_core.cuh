// Exact top-k of one score row (Agent Skill page, Step 1: top-k over the gate
// scores; ties to the lower block index, optional forced newest block,
// ascending output, from the step specification), two ways that return the
// same rows:
//
// select_topk (a radix select): THREADS threads own ITEMS consecutive blocks
// each, so block-wide scans run in index order.  Scores map to order-
// preserving 32-bit keys (-0.0 as +0.0, NaN lowest); a 4-pass MSB radix
// select (8-bit digits) finds the k'-th largest key and how many keys equal to
// it are still needed; a scan over "key == threshold" ranks the ties by index,
// and a second scan writes the chosen indices in ascending order, padded with
// -1 to k_max.
//
// select_topk_binned (the fast path): one pass of value bins instead of four
// digit passes.  Scores are spread over 254 equal-width bins between the
// row's finite minimum and maximum (NaN and -inf below, +inf and the forced
// block above); a bin index computed that way never decreases as the order
// key grows, so every block in a bin above the threshold bin outranks every
// block in or below it.  The few blocks of the threshold bin are ranked
// exactly by (order key, lower index) against one another.  A row whose
// threshold bin holds more than kBinCand blocks (all-equal scores, one
// extreme outlier) falls back to select_topk.
#pragma once

#include "seer_common.cuh"

namespace seer {

constexpr int kBinCand = 128;  // threshold-bin blocks ranked pairwise, else radix

struct SelectSmem {
  int hist[256];
  int warp_sums[32];
  int pick_digit;
  int pick_above;
  float wmin[32];
  float wmax[32];
  int cand_n;
  unsigned long long cand[kBinCand];
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

// Selects from row[0 .. nb) (global or shared; nb <= THREADS * ITEMS), writes
// out[0 .. k_max) and *n_out.  k < 1 counts as 1; k > k_max is clamped (SEER_DEV_K_CLAMPED).
// Every thread of the CTA must call it (it synchronises).
template <int THREADS, int ITEMS>
__device__ void select_topk(const float* row, int nb, int k, int force_newest, int k_max,
                            int32_t* out, int32_t* n_out, int32_t* status, SelectSmem& sm) {
  // precondition: nb <= THREADS * ITEMS (one item per block)
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

// Value-binned exact top-k (see the file comment).  Same contract and results
// as select_topk; every thread of the CTA must call it.
template <int THREADS, int ITEMS>
__device__ void select_topk_binned(const float* row, int nb, int k, int force_newest, int k_max,
                                   int32_t* out, int32_t* n_out, int32_t* status,
                                   SelectSmem& sm) {
  static_assert(THREADS % 32 == 0 && THREADS <= 1024, "whole warps");
  constexpr int kWarps = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int kk = k < 1 ? 1 : k;
  if (kk > k_max) kk = k_max;  // flagged by whichever path finishes
  const int n = min(kk, nb);
  const bool forced = force_newest && n > 0;

  // keys (order key << 32 | ~index; the forced block on top) and the finite
  // range of the scores competing on merit
  float sc[ITEMS];
  unsigned long long key[ITEMS];
  bool nan_seen = false;
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const int j = tid * ITEMS + i;
    sc[i] = 0.f;
    key[i] = 0ull;
    if (j < nb) {
      const float f = row[j];
      const bool top = forced && j == nb - 1;
      const uint32_t ok = top ? 0xffffffffu : order_key(f, nan_seen);
      key[i] = ((unsigned long long)ok << 32) | (uint32_t)(~(uint32_t)j);
      sc[i] = f;
      if (!top && isfinite(f)) {
        lo = fminf(lo, f);
        hi = fmaxf(hi, f);
      }
    }
  }
  for (int e = tid; e < 256; e += THREADS) sm.hist[e] = 0;
  if (tid == 0) sm.cand_n = 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    sm.wmin[warp] = lo;
    sm.wmax[warp] = hi;
  }
  __syncthreads();
  lo = lane < kWarps ? sm.wmin[lane] : INFINITY;
  hi = lane < kWarps ? sm.wmax[lane] : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  // bins: 0 = NaN and -inf, 1..254 = finite scores, 255 = +inf and the forced
  // block; inv = 0 (a single bin 1) when the range is empty, zero or overflows
  float inv = 0.f;
  if (hi > lo) {
    const float range = hi - lo;
    const float v = 253.5f / range;
    if (isfinite(range) && isfinite(v)) inv = v;
  }
  int bin[ITEMS];
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const int j = tid * ITEMS + i;
    int bi = -1;
    if (j < nb) {
      const float f = sc[i];
      if ((uint32_t)(key[i] >> 32) == 0xffffffffu || f == INFINITY) {
        bi = 255;
      } else if (!(f > -INFINITY)) {
        bi = 0;  // NaN or -inf
      } else {
        // inv > 0 only for a finite range, so f - lo cannot overflow
        bi = inv > 0.f ? 1 + min(253, __float2int_rz((f - lo) * inv)) : 1;
      }
      atomicAdd(&sm.hist[bi], 1);
    }
    bin[i] = bi;
  }
  if (nan_seen) flag_status(status, SEER_DEV_NONFINITE_SCORE);
  __syncthreads();
  // threshold bin: the highest bin d with (blocks in bins above d) < n
  if (warp == 0) {
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
    if (excl < n && n <= incl) {
      int acc = excl;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (acc + cnt[e] >= n) {
          sm.pick_digit = 255 - 8 * lane - e;
          sm.pick_above = acc;
          break;
        }
        acc += cnt[e];
      }
    }
    if (n <= 0 && lane == 0) {  // nothing to choose
      sm.pick_digit = 256;
      sm.pick_above = 0;
    }
  }
  __syncthreads();
  const int dstar = sm.pick_digit, above = sm.pick_above;
  const int c = dstar < 256 ? sm.hist[dstar] : 0;
  if (c > kBinCand) {  // uniform across the CTA
    __syncthreads();   // hist / pick_* are reused by the radix path
    select_topk<THREADS, ITEMS>(row, nb, k, force_newest, k_max, out, n_out, status, sm);
    return;
  }
  if (k > k_max && tid == 0) flag_status(status, SEER_DEV_K_CLAMPED);
  const int need = n - above;  // taken from the threshold bin
  bool sel[ITEMS];
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    sel[i] = bin[i] > dstar;
    if (bin[i] == dstar && need < c) sm.cand[atomicAdd(&sm.cand_n, 1)] = key[i];
    if (bin[i] == dstar && need >= c) sel[i] = true;
  }
  if (need < c) {  // uniform
    __syncthreads();
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
      if (bin[i] == dstar) {
        int rank = 0;
        for (int q = 0; q < c; ++q) rank += sm.cand[q] > key[i];
        sel[i] = rank < need;
      }
    }
  }
  // ascending compaction: warp scan, one barrier, warp-level scan of warp totals
  int local = 0;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) local += sel[i];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sm.warp_sums[warp] = incl;
  __syncthreads();
  int wv = lane < kWarps ? sm.warp_sums[lane] : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, wv, o);
    if (lane >= o) wv += y;
  }
  const int total = __shfl_sync(0xffffffffu, wv, kWarps - 1);
  const int wbase = __shfl_sync(0xffffffffu, wv, (warp + 31) & 31);
  int pos = (warp > 0 ? wbase : 0) + incl - local;
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

}  // namespace seer

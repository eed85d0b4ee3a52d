// One gate row -- a0 (incremental) + a1 + a2 for one (sequence b, KV head h) --
// as a device function that a whole CTA runs, shared by the gate + select
// kernel of the step (one row per CTA, 512 threads) and the single-launch
// fused step (rows of a persistent CTA, 320 threads):
//   * optionally append the new token's K and V rows at position L - 1 of the
//     paged cache (the step's KV append);
//   * g = gate_scale * W[h] qbar, qbar the mean of the group's queries;
//   * refresh the newest block's pooled key from K (the summation order of
//     seer_pool_keys; the appended token read from the new row itself) and
//     write it back to kbar;
//   * stream the kbar row through a ring of NBUF chunk buffers (bulk copies
//     on mbarriers; the first goes out as soon as the row length is known)
//     and score every block, 8 rows per worker warp per chunk in one
//     reduction that gives the same bits as warp_dot4 row by row;
//   * select the top-k with the exact value-binned select (or stop after the
//     scores when the unified cross-head select follows).
// Results are identical to seer_pool_keys (incremental), seer_gate_scores and
// seer_block_select run one after another.
#pragma once

#include "block_mean.cuh"
#include "seer_kernels.cuh"
#include "select_core.cuh"

namespace seer {

// Shared-memory scratch of a gate row besides the chunk buffers and the
// pooling partials.  newest, qbar and gvec are read and written as float4:
// the struct and those members sit on 16-byte boundaries.
struct alignas(16) GateRowScratch {
  float scores[kMaxBlocks];
  float newest[kHeadDim];
  float qbar[kHeadDim];
  float gvec[kHeadDim];
  SelectSmem sel;
};
static_assert(offsetof(GateRowScratch, newest) % 16 == 0 &&
                  offsetof(GateRowScratch, qbar) % 16 == 0 &&
                  offsetof(GateRowScratch, gvec) % 16 == 0 &&
                  offsetof(GateRowScratch, sel) % 8 == 0,
              "float4 members of the gate scratch on 16-byte boundaries");

// The kbar chunk buffers of a gate row: NBUF slots of CHUNK_ROWS rows each,
// anywhere in shared memory (16-byte aligned).
template <int NBUF>
struct ChunkRing {
  float* slot[NBUF];
};

// THREADS: the CTA (every thread calls this; it synchronises the CTA).
// WORKERS: warps 0 .. WORKERS-1 form g and the scores (8 W rows and 8 kbar
// rows per warp at a time, R8 such groups of kbar rows per chunk).
// CHUNK_ROWS = 8 * R8 * WORKERS kbar rows per buffer.
// Threads QFIRST .. QFIRST + QTHREADS - 1 form the mean query.  Thread 0
// issues the copies.  `seq` counts the chunks this CTA consumed before (slot
// and parity of the ring), so a persistent CTA's rows share one ring.
// A CTA that gates several rows streams them as one chunk sequence: `ahead`
// enters as the number of this row's chunks already issued by the previous
// row, and leaves as the number of the next row's chunks issued here (next_b
// < 0: no next row), so the next row's data is on its way while this row
// finishes and selects.
// Returns false when a wait ran out (SEER_DEV_TIMEOUT is flagged).
// SPEC_FIRST (a CTA that gates one row, nothing issued ahead): the first
// chunk goes out before the row length is known -- min(CHUNK_ROWS, NBmax)
// rows of the kbar row, all inside the kbar buffer, of which the row scores
// its first nb -- and an empty row waits for it before returning.
template <int THREADS, int WORKERS, int NBUF, int QFIRST, int QTHREADS, int R8 = 1,
          bool SPEC_FIRST = false>
__device__ bool gate_row(const GateSelectParams& p, int b, int h, const ChunkRing<NBUF>& ring,
                         uint64_t* bars, uint32_t& seq, GateRowScratch& gs, float* part,
                         int next_b = -1, int next_h = 0, uint32_t* ahead = nullptr) {
  constexpr int CHUNK_ROWS = 8 * R8 * WORKERS;
  constexpr int kWRows = kHeadDim / WORKERS;  // W rows per worker warp
  constexpr int kPoolRows = 128 / kPoolWarps;  // newest-block tokens per pooling warp (bs <= 128)
  // With 16 or more warps each newest-block token row is split between two
  // warps (dims 0..63 and 64..127), so each lane holds half as many words.
  constexpr int kPoolSplit = THREADS / 32 >= 2 * kPoolWarps ? 2 : 1;
  constexpr int kPoolWords = 2 / kPoolSplit;  // 32-bit words (bf16 pairs) per lane per token
  static_assert(THREADS % 32 == 0 && THREADS / 32 >= kPoolWarps, "pooling uses 8 warps");
  static_assert(WORKERS * 32 <= THREADS && kWRows % 8 == 0, "8 W rows per reduction");
  static_assert(kHeadDim % QTHREADS == 0 && QFIRST + QTHREADS <= THREADS, "mean query threads");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = (int64_t)b * p.Hkv + h;
  if (SPEC_FIRST && tid == 0) {
    const uint32_t bytes = (uint32_t)min(CHUNK_ROWS, p.max_blocks) * kHeadDim * 4;
    mbar_arrive_expect_tx(&bars[seq % NBUF], bytes);
    bulk_copy_g2s(ring.slot[seq % NBUF], p.kbar + bh * p.max_blocks * kHeadDim, bytes,
                  &bars[seq % NBUF]);
  }
  // Loads that need nothing else go out first: the row lengths, this warp's
  // rows of W[h] (rows warp + WORKERS * i) and, below, the group's queries.
  int L = __ldg(p.seqlens + b);
  const int Ln = next_b >= 0 ? __ldg(p.seqlens + next_b) : 0;
  const int k_row = __ldg(p.k_per_seq + b);
  float4 wrow[kWRows];
  if (warp < WORKERS) {
    const float* W = p.w_gate + (int64_t)h * kHeadDim * kHeadDim;
#pragma unroll
    for (int r = 0; r < kWRows; ++r)
      wrow[r] = __ldg(reinterpret_cast<const float4*>(W + (warp + r * WORKERS) * kHeadDim +
                                                      4 * lane));
  }
  L = max(0, min(L, p.max_blocks * p.bs));
  const int nb = ceil_div_i(L, p.bs);
  const int nchunks = ceil_div_i(nb, CHUNK_ROWS);
  float* kb_row = p.kbar + bh * p.max_blocks * kHeadDim;
  bool ok = true;
  // the chunk stream: this row's chunks, then the next row's
  const int next_nb = next_b >= 0 ? ceil_div_i(max(0, min(Ln, p.max_blocks * p.bs)), p.bs) : 0;
  const float* next_kb =
      next_b >= 0 ? p.kbar + ((int64_t)next_b * p.Hkv + next_h) * p.max_blocks * kHeadDim : nullptr;
  const int stream_len = nchunks + ceil_div_i(next_nb, CHUNK_ROWS);
  const uint32_t first = ahead != nullptr ? *ahead : 0u;  // already issued
  auto issue = [&](int u) {  // position u of the stream into slot (seq + u) % NBUF
    const uint32_t slot = (seq + u) % NBUF;
    const bool own = u < nchunks;
    const int c = own ? u : u - nchunks;
    const int rows_c = min(CHUNK_ROWS, (own ? nb : next_nb) - c * CHUNK_ROWS);
    const uint32_t bytes = (uint32_t)rows_c * kHeadDim * 4;
    mbar_arrive_expect_tx(&bars[slot], bytes);
    bulk_copy_g2s(ring.slot[slot], (own ? kb_row : next_kb) + (int64_t)c * CHUNK_ROWS * kHeadDim,
                  bytes, &bars[slot]);
  };
  // One chunk goes out as soon as the lengths are in; the other free slots
  // are filled once the newest block's K loads below are on their way, so
  // that those loads queue behind one chunk per row, not behind the whole
  // burst (g's own loads left before any of it).
  constexpr int kBurst = 1;
  if (tid == 0 && !SPEC_FIRST)
    for (int u = (int)first; u < kBurst && u < stream_len; ++u) issue(u);
  uint32_t issued = (uint32_t)max((int)first, min(NBUF, stream_len));

  // The newest block's page: the KV append writes the new token's K and V
  // rows of head h into it (position L - 1), and its pooled key is
  // refreshed from K below.
  const bool append = p.k_new != nullptr && L > 0;
  const bool refresh = p.incremental && nb > 0;
  const int valid_new = refresh ? L - (nb - 1) * p.bs : 0;
  int64_t new_page = 0;
  bool bad_page = false;
  if (append || refresh) {
    new_page = page_of(p.page_table, b, nb - 1, p.max_blocks);
    bad_page = new_page < 0 || new_page >= p.num_pages;
  }
  if (append && warp == 0 && !bad_page) {
    const int64_t off = new_page * p.stride_page + (int64_t)((L - 1) % p.bs) * p.stride_token +
                        (int64_t)h * p.stride_head + 4 * lane;
    const int64_t src = bh * kHeadDim + 4 * lane;
    *reinterpret_cast<uint2*>(p.k_pool_w + off) = __ldg(reinterpret_cast<const uint2*>(p.k_new + src));
    *reinterpret_cast<uint2*>(p.v_pool_w + off) = __ldg(reinterpret_cast<const uint2*>(p.v_new + src));
  }

  // mean query of the group
  if (tid >= QFIRST && tid < QFIRST + QTHREADS) {
    const int64_t row0 = ((int64_t)b * p.Hq + (int64_t)h * p.G) * kHeadDim;
    if (p.q_copy != nullptr) {
      // q in mapped host memory (16-byte aligned): the group's G rows, one
      // contiguous G x 256 bytes, cross PCIe as 16-byte words in one round
      // trip, are copied to q_copy for the decode and staged in the score
      // buffer (free until the chunk loop) for the mean below
      const uint4* src = reinterpret_cast<const uint4*>(p.q + row0);
      uint4* dst = reinterpret_cast<uint4*>(p.q_copy + row0);
      uint4* stage = reinterpret_cast<uint4*>(gs.scores);
      const int words = p.G * kHeadDim * 2 / 16;
      for (int w = tid - QFIRST; w < words; w += QTHREADS) {
        const uint4 v = __ldcg(src + w);
        stage[w] = v;
        dst[w] = v;
      }
      named_barrier_sync(2, QTHREADS);  // the mean-query threads only
    }
    const uint16_t* staged = reinterpret_cast<const uint16_t*>(gs.scores);
#pragma unroll
    for (int m = 0; m < kHeadDim / QTHREADS; ++m) {
      const int d = tid - QFIRST + m * QTHREADS;
      float s = 0.f;
      if (p.q_copy != nullptr) {
        for (int g = 0; g < p.G; ++g)
          s += __uint_as_float((uint32_t)staged[g * kHeadDim + d] << 16);
      } else {
        for (int g = 0; g < p.G; ++g)
          s += __uint_as_float((uint32_t)__ldg(p.q + row0 + d + g * kHeadDim) << 16);
      }
      gs.qbar[d] = s / (float)p.G;
    }
  }
  // The newest block's K rows go out now, behind one chunk per row: token t
  // to warp t % 8 (+ 8 for the upper half of the dims when split), lane l to
  // dims 4l .. 4l+3 (2l, 2l+1 of its half when split).  The appended token is
  // read from k_new itself, so no barrier has to order the append before
  // these loads.
  const int pool_warp = warp % kPoolWarps;
  const int pool_dim = (warp / kPoolWarps) * (kHeadDim / kPoolSplit) + 2 * kPoolWords * lane;
  const bool pooler = refresh && warp < kPoolWarps * kPoolSplit && !bad_page;
  uint32_t knew[kPoolRows][kPoolWords];
  if (pooler) {
    const uint16_t* base = p.k_pool + new_page * p.stride_page + (int64_t)h * p.stride_head + pool_dim;
    const uint16_t* appended = append ? p.k_new + bh * kHeadDim + pool_dim : nullptr;
#pragma unroll
    for (int i = 0; i < kPoolRows; ++i) {
      const int t = pool_warp + i * kPoolWarps;
      const uint16_t* src =
          (append && t == valid_new - 1) ? appended : base + (int64_t)t * p.stride_token;
      if constexpr (kPoolWords == 2) {
        const uint2 v = t < valid_new ? __ldg(reinterpret_cast<const uint2*>(src)) : make_uint2(0u, 0u);
        knew[i][0] = v.x;
        knew[i][1] = v.y;
      } else {
        knew[i][0] = t < valid_new ? __ldg(reinterpret_cast<const uint32_t*>(src)) : 0u;
      }
    }
  }
  // the newest block's mean over its valid tokens, summed in the order of
  // seer_pool_keys (per dim: the tokens of each residue mod 8 in order, then
  // the 8 partials in order), and written back to kbar
  auto pool_sum = [&]() {
    if (!pooler) return;
    float a[2 * kPoolWords] = {};
#pragma unroll
    for (int i = 0; i < kPoolRows; ++i) {
      if (pool_warp + i * kPoolWarps < valid_new) {
#pragma unroll
        for (int w = 0; w < kPoolWords; ++w) {
          a[2 * w] += __uint_as_float(knew[i][w] << 16);
          a[2 * w + 1] += __uint_as_float(knew[i][w] & 0xffff0000u);
        }
      }
    }
    float* dst = &part[pool_warp * kHeadDim + pool_dim];
    if constexpr (kPoolWords == 2)
      *reinterpret_cast<float4*>(dst) = make_float4(a[0], a[1], a[2], a[3]);
    else
      *reinterpret_cast<float2*>(dst) = make_float2(a[0], a[1]);
  };
  // Without the split the words would stay live across the projection: the
  // warps sum them as soon as they arrive instead.
  if constexpr (kPoolSplit == 1) pool_sum();
  __syncthreads();  // qbar
  if (tid == 0)
    for (int u = max((int)first, kBurst); u < NBUF && u < stream_len; ++u) issue(u);
  if (bad_page && tid == 0) flag_status(p.status, SEER_DEV_BAD_PAGE);
  // g = gate_scale * W[h] qbar, 8 rows per reduction
  if (warp < WORKERS) {
    const float4 qv = *reinterpret_cast<const float4*>(&gs.qbar[4 * lane]);
#pragma unroll
    for (int g8 = 0; g8 < kWRows / 8; ++g8) {
      float4 w8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w8[i] = wrow[g8 * 8 + i];
      const float v = warp_dot4_x8(w8, qv);
      if ((lane & 3) == 0)
        gs.gvec[warp + (g8 * 8 + ((lane >> 2) & 7)) * WORKERS] = __fmul_rn(v, p.gate_scale);
    }
  }
  if constexpr (kPoolSplit == 2) pool_sum();
  __syncthreads();
  if (refresh) {
    if (tid < kHeadDim) {
      const float v = bad_page ? 0.f : pool_finish(part, tid, valid_new);
      gs.newest[tid] = v;
      kb_row[(int64_t)(nb - 1) * kHeadDim + tid] = v;
    }
    __syncthreads();
  }

  // scores, chunk by chunk; thread 0 refills each buffer once it is read
  const float4 gv = *reinterpret_cast<const float4*>(&gs.gvec[4 * lane]);
  float* scores_out = p.scores + bh * p.max_blocks;
  bool bad = false;
  for (int c = 0; c < nchunks; ++c) {
    const uint32_t slot = (seq + c) % NBUF;
    if (ok && !mbar_wait(&bars[slot], ((seq + c) / NBUF) & 1)) {
      flag_status(p.status, SEER_DEV_TIMEOUT);
      ok = false;
    }
    const int rows = min(CHUNK_ROWS, nb - c * CHUNK_ROWS);
    const float* buf = ring.slot[slot];
    if (warp < WORKERS) {  // this warp's rows warp + WORKERS * i, 8 per reduction
#pragma unroll
      for (int g8 = 0; g8 < R8; ++g8) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = warp + (g8 * 8 + i) * WORKERS;
          const int j = c * CHUNK_ROWS + r;
          v[i] = (r >= rows) ? make_float4(0.f, 0.f, 0.f, 0.f)
                 : (refresh && j == nb - 1)
                     ? *reinterpret_cast<const float4*>(&gs.newest[4 * lane])
                     : *reinterpret_cast<const float4*>(&buf[r * kHeadDim + 4 * lane]);
        }
        const float sc = warp_dot4_x8(v, gv);
        const int r = warp + (g8 * 8 + ((lane >> 2) & 7)) * WORKERS;
        if ((lane & 3) == 0 && r < rows) {
          const int j = c * CHUNK_ROWS + r;
          gs.scores[j] = sc;
          scores_out[j] = sc;
          bad |= !isfinite(sc);
        }
      }
    }
    fence_proxy_async_smem();
    __syncthreads();  // every warp is done with this buffer
    if (c + NBUF < stream_len) {
      if (tid == 0 && ok) issue(c + NBUF);
      issued = max(issued, (uint32_t)(c + NBUF + 1));
    }
  }
  if (SPEC_FIRST && nchunks == 0) {  // the early chunk of an empty row
    if (ok && !mbar_wait(&bars[seq % NBUF], (seq / NBUF) & 1)) {
      flag_status(p.status, SEER_DEV_TIMEOUT);
      ok = false;
    }
    seq += 1;
  }
  seq += (uint32_t)nchunks;
  if (ahead != nullptr) *ahead = issued > (uint32_t)nchunks ? issued - (uint32_t)nchunks : 0u;
  if (bad) flag_status(p.status, SEER_DEV_NONFINITE_SCORE);
  for (int j = nb + tid; j < p.max_blocks; j += THREADS) scores_out[j] = -INFINITY;
  if (p.scores_only) return ok;  // uniform: the cross-head select runs next
  __syncthreads();

  constexpr int kLongItems = (kMaxBlocks + THREADS - 1) / THREADS;
  int32_t* idx_row = p.idx + bh * p.k_max;
  if (nb <= THREADS)
    select_topk_binned<THREADS, 1>(gs.scores, nb, k_row, p.force_newest, p.k_max, idx_row,
                                   p.n_sel + bh, p.status, gs.sel);
  else if (nb <= 2 * THREADS)
    select_topk_binned<THREADS, 2>(gs.scores, nb, k_row, p.force_newest, p.k_max, idx_row,
                                   p.n_sel + bh, p.status, gs.sel);
  else
    select_topk_binned<THREADS, kLongItems>(gs.scores, nb, k_row, p.force_newest, p.k_max,
                                            idx_row, p.n_sel + bh, p.status, gs.sel);
  return ok;
}

}  // namespace seer

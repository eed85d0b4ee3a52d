// a3: split-KV sparse flash-decoding over the selected KV blocks.
//
// What it computes (Agent Skill page "Sparse Attention Reasoning", Step 4):
// for every (sequence b, KV head h, split s) the G query heads of the group
// attend, with softmax scale 1/sqrt(D), only the tokens t < seqlen_b of the
// blocks idx[b,h, floor(s*n/S) .. floor((s+1)*n/S)); the result is one
// normalised partial output and its log-sum-exp per query head.
//
// How it runs on sm_100a (one persistent CTA per SM; the (b, h, s) items are
// handed out through a global counter when the caller gives one, so CTAs that
// stream faster take more items, else round-robin):
//   * scheduler warp: for each item it reads the item's index slice
//     and page numbers lane-parallel (the dependent global loads stay off the
//     copy path), publishes an item record (the G query rows, copied into
//     shared memory by a bulk copy, and the number of 64-token stages) in a
//     small ring, and appends one (page, head, sub-tile, valid tokens) entry
//     per stage to an entry ring;
//   * copy thread: pops entries and streams the selected K and V tiles with
//     4-D TMA loads (64 tokens x 64 dims per box, 128-byte swizzle, L2
//     evict-first, no multicast) into an NSTAGES-deep ring of 32 KB stages
//     whose per-stage metadata (valid tokens) rides along (4 stages);
//   * two groups of four math warps take alternate stages; each warp owns 16
//     tokens of a stage and never touches global memory in the loop.  The
//     tensor-core tile is "swap-AB": S^T = K q^T with the 16 tokens as M and
//     the query heads as N (8 per n-tile), O^T += V^T P^T with head_dim as M,
//     so a GQA group of G <= 8 heads costs one n-tile.  K and V fragments are
//     read with ldmatrix (conflict-free thanks to the swizzle) and the stage is
//     handed back to the copy thread before the softmax and P.V math;
//   * online softmax per head column in the exp2 domain; P^T enters the
//     tensor cores through movmatrix as a bf16 hi + lo pair (weights kept to
//     ~16 bits); tail tokens past seqlen are masked in registers;
//   * at the end of an item each math warp drops its (m, l, O) into a
//     shared-memory slot (mbarrier-counted) and goes on; two merge warps merge
//     the item's head rows into o_part / lse_part and free the slot, so the
//     math warps never stop at item boundaries (the one-slot shapes merge in
//     the math warps instead, one item later).
// After the persistent row-claiming gate grid, which publishes each row's
// flag as it finishes, the scheduler reads a row's indices once its flag is
// out instead of waiting for the whole gate grid (the ROWFLAGS instantiation).
// Every mbarrier wait is bounded (SEER_DEV_TIMEOUT); nothing traps.
#include "gate_row.cuh"
#include "combine_core.cuh"

#include <type_traits>

namespace seer {

constexpr int kHalfTileBytes = kTileTokens * 64 * 2;  // 64 tokens x 64 dims bf16
constexpr int kStageBytes = 4 * kHalfTileBytes;       // K lo, K hi, V lo, V hi
constexpr int kItemSlots = 3;
constexpr int kOStride = kHeadDim + 4;                 // padded merge row (floats)
constexpr int kEntries = 256;                          // stage entries in flight (power of 2)
// Queued stages left when the scheduler claims a CTA's next item from the
// shared counter (a build-time tuning constant).
#ifndef SEER_DECODE_CLAIM_AHEAD
#define SEER_DECODE_CLAIM_AHEAD 6
#endif

// The two-slot shapes hand each finished item's merge to warps of their own
// (in the single-launch step they also take part in the gate phase and the
// final combine); the one-slot shapes keep the merge in the math warps.
constexpr int kMergeWarpsPerCta = 2;
constexpr int merge_warps(int mslots, bool fused) {
  (void)fused;
  return mslots == 2 ? kMergeWarpsPerCta : 0;
}

template <int NT, int STAGES, int MSLOTS, int MW = 0>
struct DecodeShape {
  static constexpr int kMathWarps = 8;
  static constexpr int kMergeWarps = MW;
  // + copy warp + scheduler warp (+ merge warp)
  static constexpr int kThreads = (kMathWarps + 2 + MW) * 32;
  static constexpr int kGroups = 2;
  // Stage k goes to group k % kGroups and slot k % kStages.  The ring depth
  // must be a multiple of the group count so that every slot is always
  // consumed by the same group: a group then never waits on a slot two
  // phases ahead of it (a parity wait cannot tell phase k from k + 2).
  static constexpr int kStages = STAGES;
  static_assert(kStages % kGroups == 0, "each ring slot must belong to one group");
  static constexpr int kQSlotBytes = NT * 8 * kHeadDim * 2;  // the group's query rows
  // shared memory carve (offsets from the 1024-aligned base)
  static constexpr size_t kRing = 0;
  static constexpr size_t kQBuf = kRing + (size_t)kStages * kStageBytes;
  static constexpr size_t kBars = kQBuf + (size_t)kItemSlots * kQSlotBytes;
  static constexpr size_t kMeta = kBars + 8 * (2 * kStages + 2 * kItemSlots);
  static constexpr size_t kRec = (kMeta + 8 * kStages + 15) & ~size_t(15);
  static constexpr size_t kEnt = (kRec + 8 * kItemSlots + 15) & ~size_t(15);
  static constexpr size_t kEntCtl = kEnt + 16 * kEntries;  // tail, head
  // merge slots: per slot the 8 warps' (m, l) [warps][2][16], the item id and
  // a full / empty mbarrier pair, then the warps' O [warps][G][kOStride]
  static constexpr int kMSlots = MSLOTS;
  static constexpr size_t kMBars = kEntCtl + 16;
  static constexpr size_t kML = kMBars + 16 * kMSlots + 16;
  static constexpr size_t kMLBytes = (size_t)kMathWarps * 2 * kMaxGroup * 4;
  static constexpr size_t kO = kML + kMSlots * kMLBytes;
  __host__ __device__ static size_t o_slot_floats(int G) { return (size_t)kMathWarps * G * kOStride; }
  static size_t smem_bytes(int G) { return 1024 + kO + kMSlots * o_slot_floats(G) * 4; }
  // The single-launch step's gate rows stream kbar in 64 KB chunks (two
  // stage slots each) through the stage ring plus one more 64 KB slot when it
  // fits (192 KB in flight), else 32 KB chunks through the ring and one more
  // 32 KB slot; their scratch and chunk mbarriers sit in the merge area -- all
  // idle until the decode starts.
  static constexpr size_t kGateBars = (kML + sizeof(GateRowScratch) + 7) & ~size_t(7);
  static constexpr size_t kGateExtra = (kGateBars + 8 * (kStages + 2) + 127) & ~size_t(127);
  static constexpr bool kGateWide = 1024 + kGateExtra + 2 * kStageBytes + 512 <= 227 * 1024;
  static constexpr int kGateR8 = kGateWide ? 2 : 1;                  // 8-row groups per warp
  static constexpr int kGateSlots = kGateWide ? kStages / 2 + 1 : kStages + 1;
  static size_t smem_bytes_fused(int G) {
    const size_t gate = 1024 + kGateExtra + (size_t)(kGateWide ? 2 : 1) * kStageBytes;
    return smem_bytes(G) > gate ? smem_bytes(G) : gate;
  }
  static_assert(kRing % 1024 == 0 && kStageBytes % 1024 == 0, "swizzled TMA tiles need 1 KB");
  static_assert(kQBuf % 16 == 0 && kQSlotBytes % 16 == 0, "bulk copy destinations need 16 B");
  static_assert(kBars % 8 == 0 && kRec % 8 == 0 && kEnt % 16 == 0 && kMBars % 8 == 0 &&
                    kML % 16 == 0 && kO % 16 == 0,
                "shared-memory carve alignment");
};

__device__ __forceinline__ uint32_t ld_volatile(const uint32_t* p) {
  return *reinterpret_cast<const volatile uint32_t*>(p);
}

__device__ __forceinline__ void st_volatile(uint32_t* p, uint32_t v) {
  *reinterpret_cast<volatile uint32_t*>(p) = v;
}

struct ItemCoord {
  int b, h, s, L, nb, lo, hi;
  int64_t row;  // offset of the (b, h) index row
};

// Items run split-major (item = s * B * Hkv + bh): under the static
// round-robin over CTAs each CTA then sees consecutive split indices, whose
// sizes differ by at most one block, instead of one split index repeated.
__device__ __forceinline__ int item_bh(const DecodeParams& p, int item) {
  return item % (p.B * p.Hkv);
}

__device__ __forceinline__ ItemCoord item_coord(const DecodeParams& p, int item, int L, int n) {
  ItemCoord c;
  const int bh = item_bh(p, item);
  c.s = item / (p.B * p.Hkv);
  c.b = bh / p.Hkv;
  c.h = bh - c.b * p.Hkv;
  c.L = max(0, min(L, p.max_blocks * p.bs));
  c.nb = ceil_div_i(c.L, p.bs);
  n = max(0, min(n, p.k_max));
  c.lo = (int)(((long long)c.s * n) / p.S);
  c.hi = (int)(((long long)(c.s + 1) * n) / p.S);
  c.row = (int64_t)bh * p.k_max;
  return c;
}

// Index rows written while this grid runs (by its own gate rows, or by a
// gate grid that publishes each row) must come through L2.
template <bool CONCURRENT>
__device__ __forceinline__ int ld_row_data(const int32_t* ptr) {
  if constexpr (CONCURRENT) return __ldcg(ptr);
  else return __ldg(ptr);
}

// ROWFLAGS: the per-stage decode after a gate grid that publishes each row
// (f.ctl and f.row_flag set); the single-launch step (FUSED) always works
// with row flags.
template <int NT, int STAGES, int MSLOTS, bool MASS, bool FUSED, bool ROWFLAGS>
__global__ void __launch_bounds__(
    DecodeShape<NT, STAGES, MSLOTS, merge_warps(MSLOTS, FUSED)>::kThreads, 1)
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const DecodeParams p,
                         const FusedParams f) {
  using Shape = DecodeShape<NT, STAGES, MSLOTS, merge_warps(MSLOTS, FUSED)>;
  constexpr bool kMergeWarp = Shape::kMergeWarps > 0;
  static_assert(Shape::kMathWarps == 8 && Shape::kGroups == 2, "merge order assumes 2 x 4 warps");
  constexpr int kStages = Shape::kStages;
  constexpr int kQSlotBytes = Shape::kQSlotBytes;
  constexpr int kMathWarps = Shape::kMathWarps;
  constexpr int kMathThreads = kMathWarps * 32;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem + Shape::kRing;
  uint8_t* qbuf = smem + Shape::kQBuf;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Shape::kBars);
  uint64_t* empty_bar = full_bar + kStages;
  uint64_t* item_full = empty_bar + kStages;
  uint64_t* item_empty = item_full + kItemSlots;
  int2* stage_meta = reinterpret_cast<int2*>(smem + Shape::kMeta);  // (valid, block * 2 + sub)
  int2* item_rec = reinterpret_cast<int2*>(smem + Shape::kRec);  // (item, stages)
  int4* ent = reinterpret_cast<int4*>(smem + Shape::kEnt);  // (page, h | sub | valid, block, -)
  uint32_t* ent_tail = reinterpret_cast<uint32_t*>(smem + Shape::kEntCtl);
  uint32_t* ent_head = ent_tail + 1;
  uint64_t* state_full = reinterpret_cast<uint64_t*>(smem + Shape::kMBars);  // [MSLOTS]
  uint64_t* state_empty = state_full + MSLOTS;                                 // [MSLOTS]
  int* slot_item = reinterpret_cast<int*>(state_empty + MSLOTS);               // [MSLOTS]
  float* ml_base = reinterpret_cast<float*>(smem + Shape::kML);  // [slot][warps][m 16 | l 16]
  float* o_base = reinterpret_cast<float*>(smem + Shape::kO);    // [slot][warps][G][kOStride]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.G;
  const size_t o_slot = Shape::o_slot_floats(G);

  // Item number u's merge: every math warp's (m, l, O) of that item is in
  // merge slot u % MSLOTS once state_full completes (the caller has waited
  // for that when `waited`); threads tid = 0 .. nthr - 1 of the merging
  // warps take outputs e = tid, tid + nthr, ... of the G x D block, write
  // o_part / lse_part and free the slot.  Group (item's first stage's parity)
  // first, then the other group: the sums then run in the same order
  // whichever group took the item's first stage, so an item's partials do
  // not depend on which CTA ran it, what that CTA ran before, or which warps
  // merge it.  Merge warps take one head's row per pass (the head's weights
  // worked out once), math warps one output per pass: the same values in the
  // same order either way.
  // Single-launch step, phase C: the LSE combine of this CTA's rows by the
  // math warps and merge warps, once every CTA of the grid has written its
  // last partials.  (Split-major items put every row's last split among the
  // last items, so waiting for the whole grid costs little over waiting per
  // row, and it takes one fence per warp instead of one per item.)
  auto phase_c = [&]() {
    constexpr int kCombineWarps = kMathWarps + Shape::kMergeWarps;
    __syncwarp();
    if (lane == 0) __threadfence();  // this warp's partials are out
    named_barrier_sync(1, kCombineWarps * 32);
    if (threadIdx.x == 0) {  // one arrival per CTA
      __threadfence();
      atomicAdd(f.ctl + 3, 1u);
      const uint32_t want = gridDim.x;
      const long long t0 = clock64();
      while (ld_acquire_gpu(f.ctl + 3) < want) {
        __nanosleep(64);
        if (clock64() - t0 > (1ll << 31)) {
          flag_status(p.status, SEER_DEV_TIMEOUT);
          break;
        }
      }
    }
    named_barrier_sync(1, kCombineWarps * 32);
    // one warp per (b, query head) row, spread over the combining warps of
    // the grid (merge warps follow the math warps)
    const int cw = warp < kMathWarps ? warp : warp - 2;
    const int qrows = p.B * p.Hq;
    for (int q = blockIdx.x * kCombineWarps + cw; q < qrows; q += gridDim.x * kCombineWarps)
      combine_row_warp(p.lse_part + (int64_t)q * p.S, p.o_part + (int64_t)q * p.S * kHeadDim,
                       p.S, f.out + (int64_t)q * kHeadDim,
                       f.lse_out != nullptr ? f.lse_out + q : nullptr, Load4L2{});
    // the last CTA through its combine puts the two counters back to zero
    // (every CTA has passed the wait above by then)
    if (threadIdx.x == 0 && atomicAdd(f.ctl + 4, 1u) == gridDim.x - 1) {
      atomicExch(f.ctl + 3, 0u);
      atomicExch(f.ctl + 4, 0u);
    }
  };

  auto merge_item = [&](int u, int tid, int nthr, bool waited, bool& okr) {
    const int ms = u % MSLOTS;
    const uint32_t use = (uint32_t)(u / MSLOTS);
    if (!waited && okr && !mbar_wait(&state_full[ms], use & 1)) {
      flag_status(p.status, SEER_DEV_TIMEOUT);
      okr = false;
    }
    const int mitem = slot_item[ms] >> 1;
    if (okr && mitem >= 0 && mitem < p.num_items) {
      const int first = slot_item[ms] & 1;
      const int bh = item_bh(p, mitem);
      const int s = mitem / (p.B * p.Hkv);
      const int b = bh / p.Hkv;
      const int h = bh - b * p.Hkv;
      const float* mls = ml_base + (size_t)ms * (Shape::kMLBytes / 4);
      const float* os = o_base + (size_t)ms * o_slot;
      if (waited) {
        // merge warps: one head's row per warp and pass, 4 outputs per lane
        // (d = 4 lane .. 4 lane + 3, float4 loads), the head's weights once
        const int d0 = 4 * lane;
        for (int g = tid; g < G; g += nthr) {
          float mt = -INFINITY;
#pragma unroll
          for (int w = 0; w < kMathWarps; ++w) mt = fmaxf(mt, mls[w * 2 * kMaxGroup + g]);
          const int64_t orow = ((int64_t)b * p.Hq + (int64_t)h * G + g) * p.S + s;
          float4* dst = reinterpret_cast<float4*>(p.o_part + orow * kHeadDim + d0);
          if (mt == -INFINITY) {
            *dst = make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane == 0) p.lse_part[orow] = -INFINITY;
            continue;
          }
          float fw[kMathWarps], lt = 0.f;
#pragma unroll
          for (int wr = 0; wr < kMathWarps; ++wr) {
            const int w = wr ^ (first << 2);  // kMathWarps == 8, groups of 4
            fw[wr] = fast_exp2(mls[w * 2 * kMaxGroup + g] - mt);
            lt = __fmaf_rn(mls[w * 2 * kMaxGroup + kMaxGroup + g], fw[wr], lt);
          }
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int wr = 0; wr < kMathWarps; ++wr) {
            const int w = wr ^ (first << 2);
            const float4 v =
                *reinterpret_cast<const float4*>(os + ((size_t)w * G + g) * kOStride + d0);
            acc.x = __fmaf_rn(v.x, fw[wr], acc.x);
            acc.y = __fmaf_rn(v.y, fw[wr], acc.y);
            acc.z = __fmaf_rn(v.z, fw[wr], acc.z);
            acc.w = __fmaf_rn(v.w, fw[wr], acc.w);
          }
          *dst = make_float4(acc.x / lt, acc.y / lt, acc.z / lt, acc.w / lt);
          if (lane == 0) p.lse_part[orow] = (mt + log2f(lt)) * kLn2;
        }
      } else {
        // the math warps: one output per thread and pass, weights on the fly
        for (int e = tid; e < G * kHeadDim; e += nthr) {
          const int g = e / kHeadDim, d = e - g * kHeadDim;
          float mt = -INFINITY;
#pragma unroll
          for (int w = 0; w < kMathWarps; ++w) mt = fmaxf(mt, mls[w * 2 * kMaxGroup + g]);
          const int64_t orow = ((int64_t)b * p.Hq + (int64_t)h * G + g) * p.S + s;
          if (mt == -INFINITY) {
            p.o_part[orow * kHeadDim + d] = 0.f;
            if (d == 0) p.lse_part[orow] = -INFINITY;
            continue;
          }
          float lt = 0.f, acc = 0.f;
#pragma unroll
          for (int wr = 0; wr < kMathWarps; ++wr) {
            const int w = wr ^ (first << 2);
            const float f = fast_exp2(mls[w * 2 * kMaxGroup + g] - mt);
            lt = __fmaf_rn(mls[w * 2 * kMaxGroup + kMaxGroup + g], f, lt);
            acc = __fmaf_rn(os[((size_t)w * G + g) * kOStride + d], f, acc);
          }
          p.o_part[orow * kHeadDim + d] = acc / lt;
          if (d == 0) p.lse_part[orow] = (mt + log2f(lt)) * kLn2;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&state_empty[ms]);
  };

  if (threadIdx.x == 0) {
    *ent_tail = 0;
    *ent_head = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 4);
    }
    for (int i = 0; i < kItemSlots; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], kMathWarps);
    }
    for (int i = 0; i < MSLOTS; ++i) {
      // every merge warp waits on state_full; whoever merges frees the slot
      mbar_init(&state_full[i], kMathWarps);
      mbar_init(&state_empty[i], kMergeWarp ? Shape::kMergeWarps : kMathWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  // Everything above touches only shared memory; from here on the kernel reads
  // what the preceding kernel wrote (the index rows) and writes what it may
  // still read (the partials).  Without row flags it waits for the whole
  // preceding grid.  With them (a gate grid that publishes each row) each
  // row's indices are read after its flag, and the partials are safe as they
  // are: the gate grid let this grid launch only after its own wait for the
  // kernel before it, the previous step's combine.  Then let the next one
  // launch.
  constexpr bool kRowFlags = FUSED || ROWFLAGS;
  if constexpr (!kRowFlags || FUSED) pdl_wait();
  pdl_launch_dependents();

  __shared__ uint32_t epoch_next;  // this launch's row-flag value
  if constexpr (!FUSED && kRowFlags) {
    if (threadIdx.x == 0) epoch_next = ld_volatile(f.ctl + 2) + 1u;
    __syncthreads();
  }
  // ---- single-launch step, phase A: the gate rows of this CTA (all threads)
  if constexpr (FUSED) {
    constexpr int kSlots = Shape::kGateSlots;
    static_assert(kStageBytes == 8 * kMathWarps * kHeadDim * 4, "a stage holds one kbar chunk");
    GateRowScratch& gs = *reinterpret_cast<GateRowScratch*>(smem + Shape::kML);
    uint64_t* gbar = reinterpret_cast<uint64_t*>(smem + Shape::kGateBars);
    constexpr int kR8 = Shape::kGateR8;
    constexpr size_t kChunkBytes = (size_t)kR8 * kStageBytes;  // 8 * R8 * 8 warps rows
    // the pooling partials of the newest block go to the query-row slots,
    // which the scheduler fills only once the decode starts
    static_assert((size_t)kItemSlots * Shape::kQSlotBytes >= (size_t)kPoolWarps * kHeadDim * 4,
                  "pooling partials fit in the query-row slots");
    float* gpart = reinterpret_cast<float*>(smem + Shape::kQBuf);
    ChunkRing<kSlots> gring;
#pragma unroll
    for (int i = 0; i < kSlots - 1; ++i)
      gring.slot[i] = reinterpret_cast<float*>(ring + i * kChunkBytes);
    gring.slot[kSlots - 1] = reinterpret_cast<float*>(smem + Shape::kGateExtra);
    if (threadIdx.x == 0) {
      epoch_next = *reinterpret_cast<volatile uint32_t*>(f.ctl + 2) + 1u;
      for (int i = 0; i < kSlots; ++i) mbar_init(&gbar[i], 1);
      fence_mbar_init();
    }
    __syncthreads();
    uint32_t gseq = 0, gahead = 0;
    const int rows = p.B * p.Hkv;
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
      const int nxt = row + (int)gridDim.x;  // this CTA's next row: its kbar streams in early
      gate_row<Shape::kThreads, kMathWarps, kSlots, kMathThreads, 64, kR8>(
          f.gate, row / p.Hkv, row % p.Hkv, gring, gbar, gseq, gs, gpart,
          nxt < rows ? nxt / p.Hkv : -1,
          nxt < rows ? nxt % p.Hkv : 0, &gahead);
      __syncthreads();  // the row's indices, kbar row and appended K/V are written
      if (threadIdx.x == 0) {
        __threadfence();
        fence_proxy_async_global();  // the appended rows are read by TMA elsewhere
        st_release_gpu(f.row_flag + row, epoch_next);
      }
    }
    __syncthreads();  // ring and merge area belong to the decode from here on
  }

  if (kMergeWarp && warp >= kMathWarps + 2) {
    // =========================================================== merge warps
    // Merge each item the math warps drop into a merge slot, one item behind
    // them, each warp its share of the item's head rows; an item id of -1 in
    // a slot ends the run.
    bool mok = true;
    for (int u = 0; mok; ++u) {
      const int ms = u % MSLOTS;
      if (!mbar_wait(&state_full[ms], (u / MSLOTS) & 1)) {
        flag_status(p.status, SEER_DEV_TIMEOUT);
        break;
      }
      if (slot_item[ms] < 0) break;
      merge_item(u, warp - (kMathWarps + 2), Shape::kMergeWarps, true, mok);
    }
    if constexpr (FUSED) phase_c();
    return;
  }

  if (warp == kMathWarps + 1) {
    // =============================================================== scheduler
    // Runs ahead of the copies: resolves each item's block indices and pages
    // (lane-parallel, dependent global loads off the copy path), publishes
    // the item record + query rows, and appends one entry per 64-token stage
    // to the entry ring read by the copy thread.
    int ok = 1;
    uint32_t tail = 0;
    // CTA c starts on item c.  Round-robin (no counter): the next item's
    // length and count are fetched one item ahead.  Shared counter: the next
    // item is claimed only once the copy thread is down to kClaimAhead queued
    // stages (plus the ring in flight, several microseconds of streaming that
    // hide the claim's round trips), so a CTA never sits on claimed items
    // while another runs dry and the CTAs finish together.
    const bool dyn = p.work_counter != nullptr;
    constexpr uint32_t kClaimAhead = SEER_DECODE_CLAIM_AHEAD;
    // with row flags a row's indices are read only once its gate row has
    // published them (bounded wait on the row flag, acquire)
    auto row_ready = [&](int bh) {
      if constexpr (kRowFlags) {
        if (lane == 0 && ok) {
          const long long t0 = clock64();
          while (ld_acquire_gpu(f.row_flag + bh) != epoch_next) {
            if (clock64() - t0 > (1ll << 31)) {
              flag_status(p.status, SEER_DEV_TIMEOUT);
              ok = 0;
              break;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    };
    int item = (int)blockIdx.x;
    int L_cur = 0, n_cur = 0;
    if (item < p.num_items) {
      const int bh = item_bh(p, item);
      row_ready(bh);
      L_cur = __ldg(p.seqlens + bh / p.Hkv);
      n_cur = ld_row_data<kRowFlags>(p.n_sel + bh);
    }
    int it_no = 0;
    for (; item < p.num_items && ok; ++it_no) {
      int nxt = p.num_items, L_nxt = 0, n_nxt = 0;
      if (!dyn && item + (int)gridDim.x < p.num_items) {
        nxt = item + (int)gridDim.x;
        const int bh = item_bh(p, nxt);
        row_ready(bh);
        L_nxt = __ldg(p.seqlens + bh / p.Hkv);
        n_nxt = ld_row_data<kRowFlags>(p.n_sel + bh);
      }
      const ItemCoord ic = item_coord(p, item, L_cur, n_cur);

      // stages of this item (the first 32 indices stay in registers)
      int j0 = -1, nst = 0;
      for (int base = ic.lo; base < ic.hi; base += 32) {
        const int i = base + lane;
        int cnt = 0;
        if (i < ic.hi) {
          const int j = ld_row_data<kRowFlags>(p.idx + ic.row + i);
          if (j >= 0 && j < ic.nb) cnt = ceil_div_i(min(p.bs, ic.L - j * p.bs), kTileTokens);
          if (base == ic.lo) j0 = j;
        }
        nst += __reduce_add_sync(0xffffffffu, cnt);
      }

      // item record + query rows
      const int islot = it_no % kItemSlots;
      const uint32_t iphase = (it_no / kItemSlots) & 1;
      if (lane == 0) {
        if (!mbar_wait(&item_empty[islot], iphase ^ 1)) {
          flag_status(p.status, SEER_DEV_TIMEOUT);
          ok = 0;
        } else {
          item_rec[islot] = make_int2(item, nst);
          const uint32_t qbytes = (uint32_t)(G * kHeadDim * 2);
          mbar_arrive_expect_tx(&item_full[islot], qbytes);
          bulk_copy_g2s(qbuf + islot * kQSlotBytes,
                        p.q + ((int64_t)ic.b * p.Hq + (int64_t)ic.h * G) * kHeadDim, qbytes,
                        &item_full[islot]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);

      // one entry per stage: (page, h | sub-tile | valid tokens)
      for (int base = ic.lo; base < ic.hi && ok; base += 32) {
        const int i = base + lane;
        int j = -1, pg = 0, ne = 0;
        if (i < ic.hi) {
          j = (base == ic.lo) ? j0 : ld_row_data<kRowFlags>(p.idx + ic.row + i);
          if (j < 0 || j >= ic.nb) {
            flag_status(p.status, SEER_DEV_BAD_INDEX);
            j = -1;
          } else {
            const int64_t page = page_of(p.page_table, ic.b, j, p.max_blocks);
            if (page < 0 || page >= p.num_pages) {
              flag_status(p.status, SEER_DEV_BAD_PAGE);
              pg = 0;  // keep the copy inside the pool; the result is flagged
            } else {
              pg = (int)page;
            }
            ne = ceil_div_i(min(p.bs, ic.L - j * p.bs), kTileTokens);
          }
        }
        int incl = ne;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (lane == 0) {  // wait for room in the entry ring
          const long long t0 = clock64();
          while (tail + (uint32_t)total - ld_volatile(ent_head) > (uint32_t)kEntries) {
            if (clock64() - t0 > (1ll << 31)) {
              flag_status(p.status, SEER_DEV_TIMEOUT);
              ok = 0;
              break;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        for (int e = 0; e < ne; ++e) {
          const int t = e * kTileTokens;
          const int valid = min(kTileTokens, ic.L - (j * p.bs + t));
          ent[(tail + incl - ne + e) & (kEntries - 1)] =
              make_int4(pg, (ic.h << 16) | (e << 8) | valid, j, 0);
        }
        tail += (uint32_t)total;
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          st_volatile(ent_tail, tail);
        }
        __syncwarp();
      }
      if (dyn && ok) {
        if (lane == 0) {  // wait until the copy thread is nearly through the queue
          const long long t0 = clock64();
          while (tail - ld_volatile(ent_head) > kClaimAhead) {
            if (clock64() - t0 > (1ll << 31)) {
              flag_status(p.status, SEER_DEV_TIMEOUT);
              ok = 0;
              break;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        unsigned v = 0u;
        if (lane == 0) v = atomicAdd(p.work_counter, 1u) + gridDim.x;
        v = __shfl_sync(0xffffffffu, v, 0);
        if (v < (unsigned)p.num_items) {
          nxt = (int)v;
          const int bh = item_bh(p, nxt);
          row_ready(bh);
          L_nxt = __ldg(p.seqlens + bh / p.Hkv);
          n_nxt = ld_row_data<kRowFlags>(p.n_sel + bh);
        }
      }
      item = nxt;
      L_cur = L_nxt;
      n_cur = n_nxt;
    }
    // end-of-items record for the math warps
    if (lane == 0) {
      const int islot = it_no % kItemSlots;
      if (mbar_wait(&item_empty[islot], ((it_no / kItemSlots) & 1) ^ 1)) {
        item_rec[islot] = make_int2(-1, 0);
        mbar_arrive(&item_full[islot]);
      } else {
        flag_status(p.status, SEER_DEV_TIMEOUT);
      }
    }
    // the last CTA to stop fetching puts the counter back to zero for the
    // next launch that shares it
    if (p.work_counter != nullptr && lane == 0) {
      __threadfence();
      if (atomicAdd(p.work_counter + 1, 1u) == gridDim.x - 1) {
        atomicExch(p.work_counter, 0u);
        atomicExch(p.work_counter + 1, 0u);
        // every CTA read the epoch before its first row: the next launch's
        // flags use the next value
        if constexpr (kRowFlags) atomicAdd(f.ctl + 2, 1u);
      }
    }
    // terminator (the copy thread stops on a negative page)
    if (lane == 0) {
      const long long t0 = clock64();
      bool room = true;
      while (tail + 1u - ld_volatile(ent_head) > (uint32_t)kEntries) {
        if (clock64() - t0 > (1ll << 31)) {
          flag_status(p.status, SEER_DEV_TIMEOUT);
          room = false;
          break;
        }
      }
      if (room) {
        ent[tail & (kEntries - 1)] = make_int4(-1, 0, 0, 0);
        __threadfence_block();
        st_volatile(ent_tail, tail + 1u);
      }
    }
    return;
  }

  if (warp == kMathWarps) {
    // ============================================================ copy thread
    if (lane != 0) return;
    const uint64_t policy = policy_evict_first();
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    uint32_t head = 0, issued = 0;
    for (;;) {
      if (ld_volatile(ent_tail) == head) {  // wait for the scheduler
        const long long t0 = clock64();
        bool timed_out = false;
        while (ld_volatile(ent_tail) == head) {
          __nanosleep(32);
          if (clock64() - t0 > (1ll << 31)) {
            timed_out = true;
            break;
          }
        }
        if (timed_out) {
          flag_status(p.status, SEER_DEV_TIMEOUT);
          break;
        }
      }
      __threadfence_block();
      const int4 e = ent[head & (kEntries - 1)];
      __threadfence_block();
      st_volatile(ent_head, ++head);
      if (e.x < 0) break;
      // the newest block may hold a row appended by another CTA's gate row
      if constexpr (FUSED) if (f.gate.k_new != nullptr) fence_proxy_async_global();
      const int slot = issued % kStages;
      const uint32_t phase = (issued / kStages) & 1;
      if (!mbar_wait(&empty_bar[slot], phase ^ 1)) {
        flag_status(p.status, SEER_DEV_TIMEOUT);
        break;
      }
      const int h = (int)((uint32_t)e.y >> 16);
      const int t = ((e.y >> 8) & 0xff) * kTileTokens;
      stage_meta[slot] = make_int2(e.y & 0xff, (e.z << 1) | ((e.y >> 8) & 1));
      uint8_t* st = ring + slot * kStageBytes;
      mbar_arrive_expect_tx(&full_bar[slot], kStageBytes);
      const int c1 = p.token_inner ? t : h;
      const int c2 = p.token_inner ? h : t;
      tma_load_4d(st + 0 * kHalfTileBytes, &tm_k, 0, c1, c2, e.x, &full_bar[slot], policy);
      tma_load_4d(st + 1 * kHalfTileBytes, &tm_k, 64, c1, c2, e.x, &full_bar[slot], policy);
      tma_load_4d(st + 2 * kHalfTileBytes, &tm_v, 0, c1, c2, e.x, &full_bar[slot], policy);
      tma_load_4d(st + 3 * kHalfTileBytes, &tm_v, 64, c1, c2, e.x, &full_bar[slot], policy);
      ++issued;
    }
    // Let every copy this CTA started land before the CTA can retire.
    for (uint32_t k = 0; k < kStages && k < issued; ++k) {
      const uint32_t s_it = issued - 1 - k;
      mbar_wait(&full_bar[s_it % kStages], (s_it / kStages) & 1);
    }
    return;
  }

  // ================================================================== math
  const int group = warp >> 2;  // kMathWarps / 4 == kGroups
  const int wq = warp & 3;   // which 16 tokens of a stage
  const int r = lane >> 2;   // fragment row group
  const int c = lane & 3;    // fragment column pair
  const int mi = lane >> 3;  // ldmatrix sub-matrix this lane addresses
  uint32_t stage_base = 0;
  bool ok = true;
  int last_it = -1;

  for (int it_no = 0; ok; ++it_no) {
    const int islot = it_no % kItemSlots;
    const uint32_t iphase = (it_no / kItemSlots) & 1;
    if (!mbar_wait(&item_full[islot], iphase)) {
      flag_status(p.status, SEER_DEV_TIMEOUT);
      ok = false;
      break;
    }
    const int2 rec = item_rec[islot];
    if (rec.x < 0) break;  // end of items
    const int item = rec.x;
    const int nst = ok ? rec.y : 0;
    const int first_group = (int)(stage_base % Shape::kGroups);  // takes the item's stage 0
    const int ibh = item_bh(p, item);
    const int64_t mass_row0 = ((int64_t)(ibh / p.Hkv) * p.Hq + (int64_t)(ibh % p.Hkv) * G) *
                              p.max_blocks;  // first query head's block-mass row

    // q^T fragments (B operand of S^T = K q^T): n = head, k = dim.
    uint32_t qb[NT][8][2];
    {
      const uint32_t qs = smem_u32(qbuf + islot * kQSlotBytes);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int head = nt * 8 + (lane & 7);
        const bool live = nt * 8 + r < G;
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          // 4 matrices: 8 head rows x dim chunks 4kp .. 4kp+3 (two k-steps)
          const uint32_t addr = qs + head * (kHeadDim * 2) + (4 * kp + mi) * 16;
          uint32_t x0, x1, x2, x3;
          ldmatrix_x4(addr, x0, x1, x2, x3);
          qb[nt][2 * kp][0] = live ? x0 : 0u;
          qb[nt][2 * kp][1] = live ? x1 : 0u;
          qb[nt][2 * kp + 1][0] = live ? x2 : 0u;
          qb[nt][2 * kp + 1][1] = live ? x3 : 0u;
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[islot]);

    float m[NT][2], l[NT][2];
    float o[8][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    }

    for (int k = 0; k < nst; ++k) {
      const uint32_t gi = stage_base + k;
      if ((int)(gi % Shape::kGroups) != group) continue;
      const int slot = gi % kStages;
      const uint32_t phase = (gi / kStages) & 1;
      if (ok && !mbar_wait(&full_bar[slot], phase)) {
        flag_status(p.status, SEER_DEV_TIMEOUT);
        ok = false;
      }
      if (!ok) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);
        continue;
      }
      const int2 smeta = stage_meta[slot];
      const int valid = smeta.x;
      const uint32_t k_base = smem_u32(ring + slot * kStageBytes);
      const uint32_t v_base = k_base + 2 * kHalfTileBytes;

      // ---- S^T = K q^T over this warp's 16 tokens (two chains of 4 k-steps)
      float sacc[NT][2][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int a = 0; a < 2; ++a)
          sacc[nt][a][0] = sacc[nt][a][1] = sacc[nt][a][2] = sacc[nt][a][3] = 0.f;
      {
        const int tok = wq * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int chunk = 2 * kk + (mi >> 1);  // 16-byte chunk of the 128 dims
          const uint32_t addr = k_base + (chunk >> 3) * kHalfTileBytes + tok * 128 +
                                (((chunk & 7) ^ (tok & 7)) << 4);
          uint32_t a[4];
          ldmatrix_x4(addr, a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_bf16_16816(sacc[nt][kk & 1], a, qb[nt][kk][0], qb[nt][kk][1]);
        }
      }
      // ---- V^T fragments (A operand of O^T += V^T P^T), then hand the stage back
      uint32_t va[8][4];
      {
        const int tok = wq * 16 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int chunk = 2 * mt + (mi & 1);
          const uint32_t addr = v_base + (chunk >> 3) * kHalfTileBytes + tok * 128 +
                                (((chunk & 7) ^ (tok & 7)) << 4);
          ldmatrix_x4_trans(addr, va[mt][0], va[mt][1], va[mt][2], va[mt][3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[slot]);

      // ---- tokens past the sequence end (only on the newest tile)
      const int t0 = wq * 16 + r;  // token of S^T rows r and r + 8
      const bool in0 = t0 < valid, in1 = t0 + 8 < valid;
      if (valid < kTileTokens) {
        const int u = wq * 16 + 2 * c;  // tokens of the V^T fragment columns
        const uint32_t mlo = (u < valid ? 0x0000ffffu : 0u) | (u + 1 < valid ? 0xffff0000u : 0u);
        const uint32_t mhi =
            (u + 8 < valid ? 0x0000ffffu : 0u) | (u + 9 < valid ? 0xffff0000u : 0u);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          va[mt][0] &= mlo;
          va[mt][1] &= mlo;
          va[mt][2] &= mhi;
          va[mt][3] &= mhi;
        }
      }

      // ---- online softmax per head column, P^T fragments via movmatrix
      uint32_t pb[NT][4];  // hi b0, hi b1, lo b0, lo b1
      float mass_sum[NT][2], mass_mu[NT][2];  // per head column: this lane's e^(x - mu) sum, mu
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = sacc[nt][0][e] + sacc[nt][1][e];
        x[0] = in0 ? x[0] * p.scale_log2 : -INFINITY;
        x[1] = in0 ? x[1] * p.scale_log2 : -INFINITY;
        x[2] = in1 ? x[2] * p.scale_log2 : -INFINITY;
        x[3] = in1 ? x[3] * p.scale_log2 : -INFINITY;
        float pr[4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mx = fmaxf(x[e], x[2 + e]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float mn = fmaxf(m[nt][e], mx);
          const float mu = (mn == -INFINITY) ? 0.f : mn;
          const float alpha = fast_exp2(m[nt][e] - mu);
          m[nt][e] = mn;
          pr[e] = fast_exp2(x[e] - mu);
          pr[2 + e] = fast_exp2(x[2 + e] - mu);
          l[nt][e] = l[nt][e] * alpha + (pr[e] + pr[2 + e]);
          if constexpr (MASS) {
            mass_sum[nt][e] = pr[e] + pr[2 + e];
            mass_mu[nt][e] = mu;
          }
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            o[mt][nt][e] *= alpha;
            o[mt][nt][2 + e] *= alpha;
          }
        }
        uint32_t h0, l0, h1, l1;
        split_bf16x2(pr[0], pr[1], h0, l0);  // token r     : heads 2c, 2c+1
        split_bf16x2(pr[2], pr[3], h1, l1);  // token r + 8 : heads 2c, 2c+1
        pb[nt][0] = movmatrix_trans(h0);
        pb[nt][1] = movmatrix_trans(h1);
        pb[nt][2] = movmatrix_trans(l0);
        pb[nt][3] = movmatrix_trans(l1);
      }

      // ---- O^T += V^T P^T (hi and lo halves of P)
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_bf16_16816(o[mt][nt], va[mt], pb[nt][0], pb[nt][1]);
          mma_bf16_16816(o[mt][nt], va[mt], pb[nt][2], pb[nt][3]);
        }
      }
      if constexpr (MASS) {
        // This warp's 16 tokens of the block: ln sum_t e^{x_t} (natural log of
        // the scaled scores), one piece of the block's attention mass.  Done
        // after the P.V issue so it overlaps the tensor pipe; one butterfly
        // reduces both head columns of a lane: after the first exchange
        // even-r lanes carry column 2c, odd-r lanes column 2c + 1.
        const int pieces = (p.bs / kTileTokens) * 4;
        const int64_t col = (int64_t)(smeta.y >> 1) * pieces + (smeta.y & 1) * 4 + wq;
        const bool odd = (r & 1) != 0;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float keep = odd ? mass_sum[nt][1] : mass_sum[nt][0];
          keep += __shfl_xor_sync(0xffffffffu, odd ? mass_sum[nt][0] : mass_sum[nt][1], 4);
          keep += __shfl_xor_sync(0xffffffffu, keep, 8);
          keep += __shfl_xor_sync(0xffffffffu, keep, 16);
          const int head = nt * 8 + 2 * c + (odd ? 1 : 0);
          if (r < 2 && head < G) {
            const float mu = odd ? mass_mu[nt][1] : mass_mu[nt][0];
            p.block_lse[(mass_row0 + (int64_t)head * p.max_blocks) * pieces + col] =
                keep > 0.f ? (mu + __log2f(keep)) * kLn2 : -INFINITY;
          }
        }
      }
    }
    stage_base += nst;

    // ---- hand this item's softmax state to the merge: the 8 warps' states
    // meet in a shared-memory slot; each warp then merges 1/8 of the
    // previous item, so no warp waits for another at item boundaries (with
    // two slots; one slot makes it a rendezvous per item)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = l[nt][e];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        l[nt][e] = v;
      }
    }
    if (!kMergeWarp && it_no > 0) merge_item(it_no - 1, warp * 32 + lane, kMathThreads, false, ok);
    {
      const int ms = it_no % MSLOTS;
      const uint32_t use = (uint32_t)(it_no / MSLOTS);
      if (ok && !mbar_wait(&state_empty[ms], (use & 1) ^ 1)) {
        flag_status(p.status, SEER_DEV_TIMEOUT);
        ok = false;
      }
      float* mw = ml_base + (size_t)ms * (Shape::kMLBytes / 4) + warp * 2 * kMaxGroup;
      if (r == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            mw[nt * 8 + 2 * c + e] = m[nt][e];
            mw[kMaxGroup + nt * 8 + 2 * c + e] = l[nt][e];
          }
        }
      }
      float* ow = o_base + (size_t)ms * o_slot + (size_t)warp * G * kOStride;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int head = nt * 8 + 2 * c + e;
          if (head < G) {
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
              ow[head * kOStride + mt * 16 + r] = o[mt][nt][e];
              ow[head * kOStride + mt * 16 + r + 8] = o[mt][nt][2 + e];
            }
          }
        }
      }
      if (warp == 0 && lane == 0) slot_item[ms] = (item << 1) | first_group;
      __syncwarp();
      if (lane == 0) mbar_arrive(&state_full[ms]);
    }
    last_it = it_no;
  }
  if constexpr (kMergeWarp) {
    // end-of-items mark for the merge warp, in the slot after the last item
    const int u = last_it + 1;
    const int ms = u % MSLOTS;
    if (ok && !mbar_wait(&state_empty[ms], ((u / MSLOTS) & 1) ^ 1)) {
      flag_status(p.status, SEER_DEV_TIMEOUT);
      ok = false;
    }
    if (warp == 0 && lane == 0) slot_item[ms] = -1;
    __syncwarp();
    if (lane == 0) mbar_arrive(&state_full[ms]);
  } else if (last_it >= 0) {
    merge_item(last_it, warp * 32 + lane, kMathThreads, false, ok);
  }

  // ---- single-launch step, phase C (math warps and merge warps)
  if constexpr (FUSED) phase_c();
}

// ------------------------------------------------------------------ launcher
template <int NT, int STAGES, int MSLOTS, bool MASS, bool FUSED, bool ROWFLAGS = false>
static cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv,
                                 const DecodeParams& p, const FusedParams& f, int num_sms,
                                 cudaStream_t stream, bool pdl) {
  using Shape = DecodeShape<NT, STAGES, MSLOTS, merge_warps(MSLOTS, FUSED)>;
  const size_t smem = FUSED ? Shape::smem_bytes_fused(p.G) : Shape::smem_bytes(p.G);
  auto kern = sparse_decode_kernel<NT, STAGES, MSLOTS, MASS, FUSED, ROWFLAGS>;
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem_limit(kern, smem_set);
  if (e != cudaSuccess) return e;
  // at most one CTA per SM and no more CTAs than items (there are never more
  // gate rows than items); the single-launch step's CTAs wait on one another,
  // so its grid must be co-resident: a cooperative launch fails rather than
  // start one that is not
  const int grid = p.num_items < num_sms ? p.num_items : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Shape::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (FUSED) {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  }
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tk, tv, p, f);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int NT_, int MSLOTS_>
struct ShapeTag {
  static constexpr int kNT = NT_;
  static constexpr int kMSlots = MSLOTS_;
};

// Two merge slots (no per-item rendezvous of the math warps) when shared
// memory allows, else one.
cudaError_t run_sparse_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                              int num_sms, cudaStream_t stream, bool pdl, uint32_t* ctl,
                              uint32_t* row_flag) {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    optin = 227 * 1024;
  const bool mass = p.block_lse != nullptr;
  FusedParams fl = {};  // row flags only (and the epoch word they count from)
  const bool flags = row_flag != nullptr && ctl != nullptr;
  if (flags) {
    fl.ctl = ctl;
    fl.row_flag = row_flag;
  }
  auto go = [&](auto shape_tag, auto mass_tag, auto flags_tag) {
    using T = decltype(shape_tag);
    return launch_decode<T::kNT, 4, T::kMSlots, decltype(mass_tag)::value, false,
                         decltype(flags_tag)::value>(tk, tv, p, fl, num_sms, stream, pdl);
  };
  auto pick = [&](auto shape_tag) {
    if (mass)
      return flags ? go(shape_tag, std::true_type{}, std::true_type{})
                   : go(shape_tag, std::true_type{}, std::false_type{});
    return flags ? go(shape_tag, std::false_type{}, std::true_type{})
                 : go(shape_tag, std::false_type{}, std::false_type{});
  };
  if (p.G <= 8) {
    if (DecodeShape<1, 4, 2>::smem_bytes(p.G) + 256 <= (size_t)optin)  // + static shared
      return pick(ShapeTag<1, 2>{});
    return pick(ShapeTag<1, 1>{});
  }
  return pick(ShapeTag<2, 1>{});
}

// The single-launch step (gate rows, decode, combine in one cooperative grid).
cudaError_t run_fused_step(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                           const FusedParams& f, int num_sms, cudaStream_t stream) {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    optin = 227 * 1024;
  if (p.G <= 8) {
    if (DecodeShape<1, 4, 2>::smem_bytes_fused(p.G) + 256 <= (size_t)optin)
      return launch_decode<1, 4, 2, false, true>(tk, tv, p, f, num_sms, stream, false);
    return launch_decode<1, 4, 1, false, true>(tk, tv, p, f, num_sms, stream, false);
  }
  return launch_decode<2, 4, 1, false, true>(tk, tv, p, f, num_sms, stream, false);
}

}  // namespace seer

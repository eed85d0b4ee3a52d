// Parameter blocks and launchers of the libseer kernels (internal).
#pragma once

#include "seer_common.cuh"

namespace seer {

struct PoolParams {
  const uint16_t* k_pool;
  const int32_t* page_table;
  const int32_t* seqlens;
  float* kbar;
  int32_t* status;
  int Hkv, bs, max_blocks, incremental;
  int64_t num_pages, stride_page, stride_token, stride_head;
};

struct GateParams {
  const uint16_t* q;
  const float* w_gate;
  const float* kbar;
  const int32_t* seqlens;
  float* scores;
  int32_t* status;
  int Hq, Hkv, G, bs, max_blocks, blocks_per_cta;
  float gate_scale;
};

struct SelectParams {
  const float* scores;
  const int32_t* seqlens;
  const int32_t* k_per_seq;
  int32_t* idx;
  int32_t* n_sel;
  int32_t* status;
  int Hkv, bs, max_blocks, k_max, force_newest;
};

struct GateSelectParams {
  const uint16_t* q;
  const float* w_gate;
  float* kbar;
  const int32_t* seqlens;
  const int32_t* k_per_seq;
  float* scores;
  int32_t* idx;
  int32_t* n_sel;
  int32_t* status;
  const uint16_t* k_pool;     // for the incremental pooled-key refresh
  uint16_t* k_pool_w;         // the same pools, written by the KV append
  uint16_t* v_pool_w;
  const uint16_t* k_new;      // optional [B][Hkv][D]: the token appended at L - 1
  const uint16_t* v_new;
  const int32_t* page_table;
  int incremental;
  int64_t num_pages, stride_page, stride_token, stride_head;
  int Hq, Hkv, G, bs, max_blocks, k_max, force_newest;
  float gate_scale;
  int scores_only;          // 1: stop after the scores (the unified select follows)
  uint32_t* work_counter;  // optional: zeroed for the decode grid that follows
  int B;
  uint32_t* row_counter;   // the row-claiming gate grid's counter (zero before it starts)
  uint32_t* row_done;      // its CTAs done; the last one puts both back to zero
  // optional: q is then host memory mapped into the device's address space,
  // and each gate row copies its group's query rows into q_copy (device) for
  // the decode grid
  uint16_t* q_copy;
  // optional: each row publishes row_flag[bh] = epoch[0] + 1 once its
  // selection, appended K/V row and query copy are out (the decode grid that
  // follows then waits per row, not for the whole gate grid)
  uint32_t* row_flag;
  const uint32_t* epoch;
};

struct DecodeParams {
  const uint16_t* q;
  const int32_t* page_table;
  const int32_t* seqlens;
  const int32_t* idx;
  const int32_t* n_sel;
  float* o_part;
  float* lse_part;
  int32_t* status;
  int B, Hq, Hkv, G, bs, max_blocks, k_max, S;
  int num_items;
  int token_inner;  // tensor map dims are (D, token, head, page), not (D, head, token, page)
  int64_t num_pages;
  float scale_log2;  // softmax_scale * log2(e)
  // optional: per (b, query head, block, piece) ln sum_t e^{x_t}, piece =
  // sub-tile * 4 + warp (16 tokens each); nullptr: not written
  float* block_lse;
  // optional: 2 words (next item, CTAs done); items are then handed out by
  // atomicAdd and the last CTA zeroes both; nullptr = round-robin items
  uint32_t* work_counter;
};

// Prefill with query pooling: query block i (bs tokens) is gated with the
// mean of its queries over tokens and the group's heads against the pooled
// keys of blocks 0..i, block i is always selected, and every query token
// attends causally over its block's selection.
struct PrefillParams {
  const uint16_t* q;        // [B][Lq][Hq][D], Lq = max_blocks * bs
  const float* w_gate;      // [Hkv][D][D]
  const float* kbar;        // [B][Hkv][max_blocks][D] pooled keys
  const int32_t* page_table;
  const int32_t* seqlens;
  float* scores;            // optional [B][Hkv][max_blocks][max_blocks]
  int32_t* idx;             // [B][Hkv][max_blocks][k_max]
  int32_t* n_sel;           // [B][Hkv][max_blocks]
  uint16_t* out;            // [B][Lq][Hq][D]
  float* lse;               // optional [B][Hq][Lq]
  int32_t* status;
  int B, Hq, Hkv, G, bs, max_blocks, k_max;
  int sparsity_permille, budget_tokens;  // k_i from a budget when budget_tokens > 0
  int token_inner;
  int64_t num_pages;
  float gate_scale, scale_log2;
};

cudaError_t run_prefill_gate_select(const PrefillParams& p, cudaStream_t stream);
cudaError_t run_prefill_attention(const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const PrefillParams& p,
                                  cudaStream_t stream);

// The single-launch step: the decode kernel with the gate rows before it and
// the combine after it, in one cooperative grid.  Control words of a step
// workspace (zero before the first launch; every completed launch leaves
// them ready for the next):
//   ctl[0] next item, ctl[1] schedulers done (the decode's item counter),
//   ctl[2] launch epoch, ctl[3] CTAs done decoding, ctl[4] CTAs done
//   combining, ctl[5] next row and ctl[6] CTAs done of the row-claiming gate
//   grid; row_flag[bh] = epoch + 1 once row bh's selection is out (this
//   step, or a per-stage step whose gate grid publishes rows).
struct FusedParams {
  GateSelectParams gate;
  uint32_t* ctl;
  uint32_t* row_flag;
  uint16_t* out;
  float* lse_out;
};

struct MassParams {
  const int32_t* idx;
  const int32_t* n_sel;
  const int32_t* seqlens;
  const float* block_lse;
  const float* lse;
  float* mass;
  int Hq, Hkv, G, bs, max_blocks, k_max;
};

struct CombineParams {
  const float* o_part;
  const float* lse_part;
  uint16_t* out;
  float* lse_out;
  int S;
  uint16_t* out_host;  // optional: host memory mapped into the device, written besides out
};

cudaError_t run_pool_keys(const PoolParams& p, int B, cudaStream_t stream);
cudaError_t run_gate_scores(const GateParams& p, int B, cudaStream_t stream);
cudaError_t run_block_select(const SelectParams& p, int B, cudaStream_t stream);
cudaError_t run_gate_select(const GateSelectParams& p, int B, cudaStream_t stream, bool pdl);
cudaError_t run_gate_select_rows(const GateSelectParams& p, int num_sms, cudaStream_t stream,
                                 bool pdl);
cudaError_t run_unified_select(const SelectParams& p, int B, cudaStream_t stream, bool pdl);
cudaError_t run_fill_k(const int32_t* seqlens, int B, int bs, int permille, int budget,
                       int32_t* k_out, cudaStream_t stream);
cudaError_t run_fused_step(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                           const FusedParams& f, int num_sms, cudaStream_t stream);
// ctl / row_flag (optional): the step workspace's control words and row
// flags published by the gate grid before it; nullptr: wait for the whole
// preceding grid.
cudaError_t run_sparse_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                              int num_sms, cudaStream_t stream, bool pdl,
                              uint32_t* ctl = nullptr, uint32_t* row_flag = nullptr);
cudaError_t run_combine(const CombineParams& p, int B, int Hq, cudaStream_t stream, bool pdl);
// one warp per row; o_part on 16-byte boundaries; packed: out (and out_host)
// on 8-byte boundaries, written 8 bytes per lane
cudaError_t run_combine_rows(const CombineParams& p, int B, int Hq, cudaStream_t stream,
                             bool pdl, bool packed);
cudaError_t run_block_mass(const MassParams& p, int B, cudaStream_t stream);

}  // namespace seer

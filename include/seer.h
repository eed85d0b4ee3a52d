/*
 * seer.h -- C ABI of the block-sparse decode attention step (SeerAttention-R)
 * for NVIDIA B200 (sm_100a).
 *
 * What the step computes (one decode token per sequence, one attention layer):
 *
 *   kbar[b,h,j]  = mean of the keys of block j of sequence b, KV head h
 *   g[b,h]       = W[h] . mean over the GQA group's query heads of q
 *   score[b,h,j] = gate_scale * g[b,h] . kbar[b,h,j]
 *   idx[b,h,:]   = the top-k blocks by score (ties to the lower block index,
 *                  the newest block optionally forced in), ascending
 *   out[b,qh]    = softmax(q[b,qh] . K^T * softmax_scale) V over the tokens of
 *                  the selected blocks only (t < seqlen), computed as S
 *                  split-KV partials merged by a log-sum-exp combine.
 *
 * Sources, by page and section:
 *   - "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning",
 *     Abstract: a self-distilled gate chooses KV blocks for each decode query,
 *     query pooling removed for decoding, block sizes 64/128, a 4K-token
 *     budget, a sparse decoding kernel run at 90% sparsity behind a
 *     FlashAttention-style interface (paged cache, cache_seqlens, num_splits,
 *     softmax_scale, out + lse).
 *   - "Sparse Attention Reasoning" (Agent Skill page), Step 1: top-k over gate
 *     scores, k from a sparsity ratio; Step 4: sparse attention is softmax
 *     attention with unselected keys filled with -inf, scale 1/sqrt(head_dim).
 *
 * Conventions for every entry point:
 *   - Pointers named *_host are host memory; every other pointer is device
 *     memory on the current device.  The caller owns every buffer; the library
 *     never allocates, frees or synchronises, and keeps no state between calls
 *     besides what it sets up once: the driver entry point of the tensor-map
 *     encoder, each kernel's shared-memory limit, and the fixed device scratch
 *     array of seer_decode_step_noalloc.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Host-side checks return an error before anything is enqueued.
 *     SEER_ERR_CUDA reports a launch error (cudaGetLastError()).
 *   - Conditions only the device can see are OR-ed into the optional
 *     `dev_status` word (device int32, may be NULL): see SEER_DEV_*.
 *     Kernels never trap, assert or spin without a bound.
 *
 * Shapes (row-major, innermost last):
 *   q          [B][Hq][D] bf16; query head qh belongs to KV head qh / (Hq/Hkv)
 *   k_pool,
 *   v_pool     [num_pages][block_size][Hkv][D] bf16 by default, or any layout
 *              given by (stride_page, stride_token, stride_head) in elements
 *              with the D elements of one row contiguous; all strides and the
 *              base address 16-byte aligned.  One page holds one KV block.
 *   page_table [B][max_blocks] int32: page of logical block j of sequence b;
 *              may be NULL for the identity table page = b * max_blocks + j
 *              (a contiguous [B][max_blocks * block_size][Hkv][D] cache).
 *              Entries at j >= NB_b are never read.
 *   seqlens    [B] int32: tokens in the cache, the current token's K/V
 *              already appended at position seqlen - 1; 0 <= seqlen <=
 *              max_blocks * block_size.  NB_b = ceil(seqlen_b / block_size).
 *   w_gate     [Hkv][D][D] fp32, g[i] = sum_j W[h][i][j] qbar[j]
 *   kbar       [B][Hkv][max_blocks][D] fp32
 *   scores     [B][Hkv][max_blocks] fp32 (-inf at j >= NB_b)
 *   idx        [B][Hkv][k_max] int32, ascending, -1 after the n_sel entries
 *   n_sel      [B][Hkv] int32
 *   o_part     [B][Hq][num_splits][D] fp32 (16-byte aligned),
 *              lse_part [B][Hq][num_splits] fp32
 *   out        [B][Hq][D] bf16 (round-to-nearest-even), lse_out [B][Hq] fp32
 *              natural-log log-sum-exp of the scaled scores (-inf if empty)
 */
#ifndef SEER_H_
#define SEER_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SEER_API __attribute__((visibility("default")))
#else
#define SEER_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *seer_stream;

typedef enum seer_status {
  SEER_OK = 0,
  SEER_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size */
  SEER_ERR_UNSUPPORTED = 2, /* D != 128, block_size not 64/128, Hq/Hkv > 16,
                               misaligned pointer or stride, too many blocks */
  SEER_ERR_CUDA = 3,        /* a CUDA call or kernel launch failed */
  SEER_ERR_WORKSPACE = 4    /* workspace missing or smaller than required */
} seer_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define SEER_DEV_NONFINITE_SCORE 1 /* a gate score was NaN or +-inf */
#define SEER_DEV_BAD_INDEX 2       /* an idx entry outside [0, NB_b): skipped */
#define SEER_DEV_BAD_PAGE 4        /* page outside [0, num_pages): page 0 used */
#define SEER_DEV_K_CLAMPED 8       /* k_per_seq[b] > k_max: clamped to k_max */
#define SEER_DEV_TIMEOUT 16        /* a pipeline wait gave up after ~1 s */

typedef struct seer_dims {
  int32_t batch;        /* B >= 1 */
  int32_t num_q_heads;  /* Hq, a multiple of Hkv, Hq / Hkv <= 16 */
  int32_t num_kv_heads; /* Hkv >= 1 */
  int32_t head_dim;     /* D, must be 128 */
  int32_t block_size;   /* bs, 64 or 128; equal to the page size */
  int32_t max_blocks;   /* NBmax >= 1: row length of page_table, kbar, scores;
                           at most 4096 */
  int64_t num_pages;    /* pages in each pool (>= B * NBmax if table NULL) */
  int64_t stride_page;  /* element strides of k_pool and v_pool */
  int64_t stride_token;
  int64_t stride_head;
} seer_dims;

/* Library version, as 10000 * major + 100 * minor + patch. */
SEER_API int32_t seer_version(void);

/* Static text for a status code. */
SEER_API const char *seer_status_string(seer_status s);

/* The CUDA runtime's message for the error behind the last SEER_ERR_CUDA
 * returned on the calling host thread ("no error" if there was none); a
 * static string, owned by the runtime. */
SEER_API const char *seer_last_cuda_error(void);

/* Fill a seer_dims for the default pool layout [P][bs][Hkv][D]. */
SEER_API seer_status seer_dims_default(int32_t batch, int32_t num_q_heads,
                              int32_t num_kv_heads, int32_t head_dim,
                              int32_t block_size, int32_t max_blocks,
                              int64_t num_pages, seer_dims *out);

/* ---------------------------------------------------------------- helpers
 * k from a sparsity in permille (0..1000): max(1, ceil((1000 - s) * nb / 1000))
 * -- "keep the top (1 - sparsity) fraction" (Agent Skill page, Step 1),
 * rounded up.  k from a token budget: max(1, min(nb, budget / block_size))
 * (paper summary page, Abstract: 4K token budget).  Both in exact integers. */
SEER_API seer_status seer_k_from_sparsity(int32_t nb, int32_t sparsity_permille,
                                 int32_t *k);
SEER_API seer_status seer_k_from_budget(int32_t nb, int32_t budget_tokens,
                               int32_t block_size, int32_t *k);

/* Device version of the two rules above, one k per sequence from seqlens:
 * budget mode when budget_tokens > 0, else sparsity mode. */
SEER_API seer_status seer_fill_k(const seer_dims *d, const int32_t *seqlens,
                        int32_t sparsity_permille, int32_t budget_tokens,
                        int32_t *k_per_seq, seer_stream stream);

/* Splits that keep every SM busy for k_max selected blocks per KV head:
 * enough (b, h, split) items for about four per SM, at least 2 blocks per
 * split, between 1 and 64. */
SEER_API int32_t seer_default_splits(const seer_dims *d, int32_t k_max,
                            int32_t num_sms);

/* Bytes of caller workspace seer_decode_step needs (scores, idx, n_sel,
 * o_part, lse_part, then the control words: the decode grid's item counter,
 * the row flags' epoch, the single-launch step's phase counters, the
 * row-claiming gate grid's counters, and the [B][Hkv] u32 row flags;
 * each part 256-byte aligned).  seer_decode_step and seer_decode_step_fused
 * need seer_step_workspace_init once before a workspace's first use. */
SEER_API size_t seer_step_workspace_bytes(const seer_dims *d, int32_t k_max,
                                 int32_t num_splits);

/* ------------------------------------------------------------- the steps */

/* a0. Mean-pooled block keys.  incremental = 0 rebuilds every block (blocks
 * j >= NB_b are written as zeros); incremental = 1 recomputes only the
 * newest block NB_b - 1 of every (b, h), the one the appended token changed.
 * Pooling keys but not queries follows the Abstract ("removing query
 * pooling").  fp32 sums in a fixed order. */
SEER_API seer_status seer_pool_keys(const seer_dims *d, const uint16_t *k_pool,
                           const int32_t *page_table, const int32_t *seqlens,
                           int32_t incremental, float *kbar,
                           int32_t *dev_status, seer_stream stream);

/* a1. Gate scores, fp32: score[b,h,j] = gate_scale * (W[h] qbar) . kbar[j]
 * with qbar the mean of the G query heads of KV head h (the mean of the
 * per-head scores, by linearity).  j >= NB_b gets -inf.  Non-finite scores
 * of valid blocks set SEER_DEV_NONFINITE_SCORE. */
SEER_API seer_status seer_gate_scores(const seer_dims *d, const uint16_t *q,
                             const float *w_gate, const float *kbar,
                             const int32_t *seqlens, float gate_scale,
                             float *scores, int32_t *dev_status,
                             seer_stream stream);

/* a2. Top-k block selection per (b, h) (Agent Skill page, Step 1).  k_b =
 * k_per_seq[b] (values < 1 count as 1, values > k_max are clamped and flag
 * SEER_DEV_K_CLAMPED), n_sel = min(k_b, NB_b).  Order: score descending,
 * then lower index; NaN below -inf; -0.0 == +0.0.  force_newest != 0 takes
 * block NB_b - 1 first, counting toward k.  idx rows are ascending and padded
 * with -1 to k_max.  Exact: the result depends only on the scores. */
SEER_API seer_status seer_block_select(const seer_dims *d, const float *scores,
                              const int32_t *seqlens,
                              const int32_t *k_per_seq, int32_t force_newest,
                              int32_t k_max, int32_t *idx, int32_t *n_sel,
                              int32_t *dev_status, seer_stream stream);

/* a2, unified variant (next to the per-head selection): one block set per
 * sequence shared by every KV head, after the unified cross-head ranking of
 * the LessIsMore abstract on the author page.  A block's aggregate is the sum
 * of its scores over the KV heads, added in head order in fp32; the top-k of
 * the aggregate follows the same order, k, forced block, padding and flag
 * rules as seer_block_select, and the one index row (and n_sel) is written to
 * every head's row, so seer_sparse_decode needs no change.  Arguments as for
 * seer_block_select; scores of all KV heads must be present. */
SEER_API seer_status seer_block_select_unified(const seer_dims *d, const float *scores,
                              const int32_t *seqlens,
                              const int32_t *k_per_seq, int32_t force_newest,
                              int32_t k_max, int32_t *idx, int32_t *n_sel,
                              int32_t *dev_status, seer_stream stream);

/* a3. Split-KV sparse flash-decoding (Agent Skill page, Step 4: masked
 * softmax attention, scale softmax_scale).  For each (b, h, split s) the
 * selected blocks idx[b,h, floor(s*n/S) .. floor((s+1)*n/S)) are staged by
 * TMA into shared memory; all G query heads of the group attend them with an
 * online softmax, so each K/V byte is read from HBM once.  Tokens t >=
 * seqlen_b never enter the math; unselected blocks are never read.  Writes
 * o_part (normalised per split) and lse_part (natural log); an empty split
 * writes o = 0, lse = -inf.  1 <= num_splits <= 64.
 *
 * work_counter (optional, may be NULL): two uint32 words of device memory,
 * 8-byte aligned, zero before the first launch that uses them.  The
 * persistent grid then hands out its (b, h, split) items through them, so
 * CTAs that stream faster take more items and the grid finishes together;
 * the last CTA puts both words back to zero, so a launch that completes
 * without SEER_DEV_TIMEOUT leaves them ready for the next one.  Launches that
 * share the words must not overlap.  NULL: items round-robin over the CTAs.
 * The results do not depend on the choice. */
SEER_API seer_status seer_sparse_decode(const seer_dims *d, const uint16_t *q,
                               const uint16_t *k_pool, const uint16_t *v_pool,
                               const int32_t *page_table,
                               const int32_t *seqlens, const int32_t *idx,
                               const int32_t *n_sel, int32_t k_max,
                               int32_t num_splits, float softmax_scale,
                               float *o_part, float *lse_part,
                               uint32_t *work_counter,
                               int32_t *dev_status, seer_stream stream);

/* a4. Log-sum-exp combine of the split partials: lse = log sum_s e^{lse_s},
 * out = sum_s e^{lse_s - lse} o_s, rounded to bf16.  lse_out may be NULL. */
SEER_API seer_status seer_combine(const seer_dims *d, const float *o_part,
                         const float *lse_part, int32_t num_splits,
                         uint16_t *out, float *lse_out, seer_stream stream);

/* The whole step, a0 (optional) .. a4, enqueued back to back on `stream`.
 * Needs no host synchronisation and can be captured in a CUDA graph. */
typedef struct seer_step_args {
  const uint16_t *q;
  const uint16_t *k_pool;
  const uint16_t *v_pool;
  const int32_t *page_table; /* may be NULL (identity) */
  const int32_t *seqlens;
  const float *w_gate;
  float *kbar;               /* read by the gate; written when update_kbar */
  const int32_t *k_per_seq;
  int32_t update_kbar;       /* 0: use kbar as is, 1: incremental, 2: full */
  int32_t force_newest;
  int32_t k_max;
  int32_t num_splits;
  float gate_scale;          /* 1/sqrt(D) */
  float softmax_scale;       /* 1/sqrt(D) */
  void *workspace;           /* seer_step_workspace_bytes() bytes, 256-aligned */
  size_t workspace_bytes;
  uint16_t *out;
  float *lse_out;            /* may be NULL, unless block_mass is set */
  int32_t *dev_status;       /* may be NULL */
  /* Optional per-block attention mass of this step (see seer_block_mass):
   * both NULL, or block_lse (seer_block_lse_elems() floats) and block_mass
   * ([B][Hq][max_blocks] fp32) together with lse_out. */
  float *block_lse;
  float *block_mass;
  /* 0: each KV head selects its own blocks (seer_block_select); 1: one block
   * set per sequence shared by all its KV heads (seer_block_select_unified). */
  int32_t unified_heads;
  /* Optional KV append (both NULL, or both [B][Hkv][D] bf16, 8-byte aligned):
   * the step first writes the new token's K and V rows at position
   * seqlens[b] - 1 of k_pool and v_pool (through the page table), then pools,
   * gates and attends with them.  seqlens already counts the new token.  The
   * pools are written only in this case. */
  const uint16_t *k_new;
  const uint16_t *v_new;
} seer_step_args;

/* The step: a0 (incremental when update_kbar = 1) + a1 + a2 in one gate grid
 * (or a gate grid and the unified select), a3, a4.
 *   - The workspace's control words must be zero before the first call:
 *     seer_step_workspace_init once after allocating it (and again after a
 *     call that flagged SEER_DEV_TIMEOUT).  Every completed call leaves them
 *     ready for the next; calls that share a workspace must not overlap.
 *   - With more (b, KV head) rows than SMs the gate grid is persistent and
 *     claims rows one after another; then (without unified_heads) each row
 *     publishes a flag in the workspace once its selection and KV append are
 *     out, and the decode grid starts on that row at once instead of
 *     waiting for the whole gate grid (bounded waits; SEER_DEV_TIMEOUT when
 *     one runs out). */
SEER_API seer_status seer_decode_step(const seer_dims *d, const seer_step_args *a,
                             seer_stream stream);

/* End-to-end form for callers holding q and out in host memory: the step with
 * a->q replaced by q_dev, q taken from q_host (B*Hq*D bf16) and the output
 * delivered to out_host (B*Hq*D bf16) as well as a->out.  A host buffer that
 * is pinned and mapped into the device's address space (cudaHostAlloc /
 * cudaMallocHost memory, or cudaHostRegister'ed with the mapped flag; see
 * seer_host_ptr_mapped) is accessed by the step's kernels directly: the gate
 * reads q_host (when it is also 16-byte aligned) and fills q_dev, the combine
 * writes out_host, and no copy is enqueued.  Any other host buffer goes through cudaMemcpyAsync on `stream`
 * (before the step for q, after it for out).  Asynchronous either way: q_host
 * must stay unchanged and out_host is valid only once the stream is
 * synchronised. */
SEER_API seer_status seer_decode_step_host(const seer_dims *d, const seer_step_args *a,
                                  const uint16_t *q_host, uint16_t *q_dev,
                                  uint16_t *out_host, seer_stream stream);

/* 1 if seer_decode_step_host reads or writes this host buffer directly
 * (pinned and mapped into the device's address space), else 0. */
SEER_API int32_t seer_host_ptr_mapped(const void *host_ptr);

/* ------------------------------------------------- per-block attention mass
 * The dense model's block-level attention distribution is what the
 * self-distilled gate is trained toward (SeerAttention-R, Abstract:
 * "learning attention sparsity through a self-distilled gating mechanism";
 * Agent Skill page, Step 2: the full model is the teacher).  With every block
 * selected (k = NB, e.g. sparsity 0) these calls give that target for one
 * decode step; with a sparse selection they give the mass of each selected
 * block.  mass[b,qh,j] = sum over the tokens t < seqlen of block j of query
 * head qh's softmax weight; the mass of a KV head's group is the mean over
 * its G query heads.
 *
 * seer_sparse_decode_mass is seer_sparse_decode (same arguments, same
 * outputs, bit for bit) that also writes block_lse [B][Hq][max_blocks][P],
 * P = 4 * block_size / 64: per 16-token piece of each processed block, the
 * natural log of sum_t e^{scaled score}.  Only the selected blocks' pieces
 * are written.  seer_block_mass turns them into mass [B][Hq][max_blocks] fp32
 * with the merged lse of each row (seer_combine's lse_out): selected blocks
 * e^{piece - lse} summed, every other block 0. */
SEER_API size_t seer_block_lse_elems(const seer_dims *d);

SEER_API seer_status seer_sparse_decode_mass(
    const seer_dims *d, const uint16_t *q, const uint16_t *k_pool,
    const uint16_t *v_pool, const int32_t *page_table, const int32_t *seqlens,
    const int32_t *idx, const int32_t *n_sel, int32_t k_max,
    int32_t num_splits, float softmax_scale, float *o_part, float *lse_part,
    float *block_lse, uint32_t *work_counter, int32_t *dev_status,
    seer_stream stream);

SEER_API seer_status seer_block_mass(const seer_dims *d, const int32_t *idx,
                                     const int32_t *n_sel, int32_t k_max,
                                     const int32_t *seqlens,
                                     const float *block_lse, const float *lse,
                                     float *mass, seer_stream stream);

/* ------------------------------------------------------ no-allocation step
 * No counterpart in the paper: this entry point exists for callers that
 * cannot allocate device memory themselves -- a host framework or serving
 * runtime that owns every byte of GPU memory through its own pool (a
 * separate allocation would escape its accounting, or fail), or a decode loop
 * that must never enter the CUDA allocator (cudaMalloc can serialise against
 * other work and can fail under memory pressure mid-generation).
 *
 * It runs exactly seer_decode_step (its control words zeroed on the stream
 * first), but its workspace is a file-scope device
 * array of SEER_NOALLOC_SCRATCH_BYTES (16 MiB) inside this library: every GPU
 * that loads the library holds those 16 MiB until the process exits.
 * a->workspace and a->workspace_bytes are ignored; the caller still passes
 * every input and output.  Nothing is allocated or freed, by this call or by
 * anything it calls.
 *   - Limit: when seer_step_workspace_bytes(d, a->k_max, a->num_splits)
 *     exceeds SEER_NOALLOC_SCRATCH_BYTES the call returns SEER_ERR_WORKSPACE
 *     before anything is enqueued.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current and caches it
 *     for the rest of the process; make that first call before any stream
 *     capture begins.  The cached address belongs to the device's primary
 *     context: after cudaDeviceReset (or from a caller that made another
 *     context current) it no longer points at the array, so do not call
 *     this entry point again after a reset.
 *   - Sharing: all calls on a device use the same array, which keeps the last
 *     call's contents.  Nothing in it has to start at zero (every byte the
 *     step reads there is written earlier by the same call), but calls whose
 *     work can overlap on the GPU -- two streams, or two host threads -- race
 *     on it: order them on one stream or serialise them. */
#define SEER_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

SEER_API seer_status seer_decode_step_noalloc(const seer_dims *d,
                                              const seer_step_args *a,
                                              seer_stream stream);

/* ------------------------------------------------ prefill with query pooling
 * The SeerAttention form that SeerAttention-R drops to decode token by token
 * (paper summary page, Abstract), for a whole prompt: query block i (the
 * query tokens [i*bs, (i+1)*bs)) is gated with its pooled query -- the mean
 * over its tokens and the group's G heads -- against the pooled keys of the
 * blocks j <= i (gate_scale * (W qbar_i) . kbar_j); block i is always chosen
 * and counts toward k_i (k_i from the sparsity over i + 1 candidates, or
 * min(i + 1, budget / bs)); every query token then attends causally over the
 * tokens of its block's chosen blocks up to itself.  q and out are
 * [B][max_blocks * block_size][Hq][D] bf16 (16-byte aligned); K/V come from
 * the paged pools; lse_out is [B][Hq][max_blocks * block_size] fp32 or NULL;
 * scores_out, if not NULL, receives the block gate scores
 * [B][Hkv][max_blocks][max_blocks] (-inf above the diagonal).  The workspace
 * (seer_prefill_workspace_bytes) receives the chosen indices
 * [B][Hkv][max_blocks][k_max] (ascending, -1 padded) and their counts
 * [B][Hkv][max_blocks] int32.  pool_keys != 0 rebuilds kbar first. */
typedef struct seer_prefill_args {
  const uint16_t *q;
  const uint16_t *k_pool;
  const uint16_t *v_pool;
  const int32_t *page_table; /* may be NULL (identity) */
  const int32_t *seqlens;
  const float *w_gate;
  float *kbar;
  int32_t pool_keys;
  int32_t sparsity_permille;
  int32_t budget_tokens;     /* > 0: budget rule */
  int32_t k_max;             /* >= every k_i: seer_prefill_k_max */
  float gate_scale;
  float softmax_scale;
  void *workspace;
  size_t workspace_bytes;
  uint16_t *out;
  float *lse_out;
  float *scores_out;
  int32_t *dev_status;
} seer_prefill_args;

/* k of the last query block, which bounds every k_i (0 on bad dims). */
SEER_API int32_t seer_prefill_k_max(const seer_dims *d, int32_t sparsity_permille,
                                    int32_t budget_tokens);
SEER_API size_t seer_prefill_workspace_bytes(const seer_dims *d, int32_t k_max);
SEER_API seer_status seer_prefill(const seer_dims *d, const seer_prefill_args *a,
                                  seer_stream stream);

/* The attention stage of seer_prefill alone, over a selection the caller
 * gives (the causal masked softmax of the "Sparse Attention Reasoning" page,
 * Step 4, per query block): idx [B][Hkv][max_blocks][a->k_max] ascending
 * block indices (-1 padded) and n_sel [B][Hkv][max_blocks] their counts, the
 * layout seer_prefill leaves in its workspace.  Every query token t of query
 * block i attends the tokens s <= t (s < seqlens[b]) of the blocks listed for
 * i; blocks after i, out of range, or on pages outside the pool are skipped
 * and flagged (SEER_DEV_BAD_INDEX / SEER_DEV_BAD_PAGE).  Uses a->q, k_pool,
 * v_pool, page_table, seqlens, k_max, softmax_scale, out, lse_out and
 * dev_status; the gate fields and the workspace are not read.  Same kernel,
 * same bits as the attention inside seer_prefill. */
SEER_API seer_status seer_prefill_attention(const seer_dims *d, const seer_prefill_args *a,
                                            const int32_t *idx, const int32_t *n_sel,
                                            seer_stream stream);

/* ------------------------------------------------------ single-launch step
 * The whole step in one cooperative launch (the persistent decode grid runs
 * the gate rows first and the LSE combine last; next to the per-stage path,
 * it removes the launch boundaries between gate + select, decode and
 * combine): same arguments, same results bit for bit as seer_decode_step --
 * including the optional KV append -- except that unified_heads and the block
 * mass are not offered here (SEER_ERR_UNSUPPORTED; use seer_decode_step).
 *   - The grid holds one CTA per SM and every CTA must be resident at once:
 *     the launch fails with SEER_ERR_CUDA if they cannot be (other work
 *     holding SMs).  CTAs wait on each other only through bounded waits on
 *     flags in the workspace (SEER_DEV_TIMEOUT when one runs out).
 *   - The workspace's control words must be zero before the first call:
 *     seer_step_workspace_init once after allocating it (and again after a
 *     call that flagged SEER_DEV_TIMEOUT).  Every completed call leaves them
 *     ready for the next; calls that share a workspace must not overlap.
 *   - update_kbar = 2 runs the full key pooling as its own launch first. */
SEER_API seer_status seer_decode_step_fused(const seer_dims *d,
                                            const seer_step_args *a,
                                            seer_stream stream);

/* Zeroes the control words of a step workspace (bytes from
 * seer_step_workspace_bytes with the same k_max and num_splits); enqueued on
 * `stream`.  Needed once before seer_decode_step or seer_decode_step_fused
 * uses the workspace. */
SEER_API seer_status seer_step_workspace_init(const seer_dims *d, int32_t k_max,
                                              int32_t num_splits, void *workspace,
                                              size_t workspace_bytes,
                                              seer_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SEER_H_ */

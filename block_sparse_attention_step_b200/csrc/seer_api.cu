// C ABI of libseer: argument checks, launch geometry, tensor maps and the
// fused step.  Declared in include/seer.h.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <climits>
#include <cstdlib>
#include <mutex>

#include "seer_kernels.cuh"

using namespace seer;

namespace {

constexpr int kMaxDevices = 64;

// NVTX ranges around each step and each stage it enqueues, for profilers
// (ncu --nvtx-include, nsys): compiled in, off unless the environment has
// SEER_NVTX=1 when the library first checks (a host-side push/pop only).
bool nvtx_on() {
  static const bool on = [] {
    const char* v = std::getenv("SEER_NVTX");
    return v != nullptr && v[0] == '1';
  }();
  return on;
}

struct NvtxRange {
  const bool on;
  explicit NvtxRange(const char* name) : on(nvtx_on()) {
    if (on) nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (on) nvtxRangePop();
  }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

int num_sms_current() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < kMaxDevices) {
    const int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Pool tensor map: dims (D, head, token, page) or (D, token, head, page),
// whichever lists the smaller stride first; box = 64 dims x 64 tokens,
// 128-byte swizzle (conflict-free ldmatrix rows).
seer_status make_kv_map(const uint16_t* base, const seer_dims* d, int token_inner, CUtensorMap* map) {
  auto enc = tensor_map_encoder();
  if (!enc) return SEER_ERR_CUDA;
  cuuint64_t dims[4];
  cuuint64_t strides[3];
  cuuint32_t box[4];
  const cuuint32_t elem[4] = {1, 1, 1, 1};
  dims[0] = (cuuint64_t)d->head_dim;
  box[0] = 64;
  if (token_inner) {
    dims[1] = (cuuint64_t)d->block_size;
    dims[2] = (cuuint64_t)d->num_kv_heads;
    strides[0] = (cuuint64_t)d->stride_token * 2;
    strides[1] = (cuuint64_t)d->stride_head * 2;
    box[1] = kTileTokens;
    box[2] = 1;
  } else {
    dims[1] = (cuuint64_t)d->num_kv_heads;
    dims[2] = (cuuint64_t)d->block_size;
    strides[0] = (cuuint64_t)d->stride_head * 2;
    strides[1] = (cuuint64_t)d->stride_token * 2;
    box[1] = 1;
    box[2] = kTileTokens;
  }
  dims[3] = (cuuint64_t)d->num_pages;
  strides[2] = (cuuint64_t)d->stride_page * 2;
  box[3] = 1;
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(base), dims,
                         strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SEER_OK : SEER_ERR_UNSUPPORTED;
}

// Prompt-query tensor map over q [B][Lq][Hq][D] (Lq = max_blocks * bs): dims
// (D, head, token, batch); box = 64 dims x 1 head x 64 tokens, 128-byte swizzle.
seer_status make_q_map(const uint16_t* q, const seer_dims* d, CUtensorMap* map) {
  auto enc = tensor_map_encoder();
  if (!enc) return SEER_ERR_CUDA;
  const cuuint64_t lq = (cuuint64_t)d->max_blocks * d->block_size;
  const cuuint64_t row = (cuuint64_t)d->head_dim * 2;
  const cuuint64_t dims[4] = {(cuuint64_t)d->head_dim, (cuuint64_t)d->num_q_heads, lq,
                              (cuuint64_t)d->batch};
  const cuuint64_t strides[3] = {row, row * d->num_q_heads, row * d->num_q_heads * lq};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)kTileTokens, 1};
  const cuuint32_t elem[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(q), dims,
                         strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SEER_OK : SEER_ERR_UNSUPPORTED;
}

seer_status check_dims(const seer_dims* d) {
  if (d == nullptr) return SEER_ERR_INVALID_ARG;
  if (d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 || d->max_blocks < 1 ||
      d->num_pages < 1)
    return SEER_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return SEER_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim) return SEER_ERR_UNSUPPORTED;
  if (d->num_q_heads / d->num_kv_heads > kMaxGroup) return SEER_ERR_UNSUPPORTED;
  if (d->block_size != 64 && d->block_size != 128) return SEER_ERR_UNSUPPORTED;
  if (d->max_blocks > kMaxBlocks) return SEER_ERR_UNSUPPORTED;
  if (d->batch > 65535 || d->num_kv_heads > 65535 || d->num_q_heads > 65535)
    return SEER_ERR_UNSUPPORTED;
  if (d->num_pages > INT_MAX) return SEER_ERR_UNSUPPORTED;
  return SEER_OK;
}

seer_status check_pool(const seer_dims* d, const uint16_t* pool) {
  if (pool == nullptr) return SEER_ERR_INVALID_ARG;
  if (d->stride_page < 1 || d->stride_token < 1 || d->stride_head < 1) return SEER_ERR_INVALID_ARG;
  if (!aligned(pool, 16) || d->stride_page % 8 || d->stride_token % 8 || d->stride_head % 8)
    return SEER_ERR_UNSUPPORTED;
  return SEER_OK;
}

#define SEER_TRY(expr)                     \
  do {                                     \
    const seer_status st_ = (expr);        \
    if (st_ != SEER_OK) return st_;        \
  } while (0)

// the CUDA error behind this host thread's last SEER_ERR_CUDA
static thread_local cudaError_t g_last_cuda_error = cudaSuccess;

#define SEER_CUDA(expr)                   \
  do {                                    \
    const cudaError_t seer_e_ = (expr);   \
    if (seer_e_ != cudaSuccess) {         \
      g_last_cuda_error = seer_e_;        \
      return SEER_ERR_CUDA;               \
    }                                     \
  } while (0)

struct Workspace {
  float* scores;
  int32_t* idx;
  int32_t* n_sel;
  float* o_part;
  float* lse_part;
  uint32_t* work_counter;  // control words: decode item counter (2), epoch, phase counters
  uint32_t* row_flag;      // [B][Hkv] single-launch step: row selection published
  size_t ctl_bytes;        // from work_counter to the end of row_flag
  size_t bytes;
};

Workspace carve(const seer_dims* d, int32_t k_max, int32_t S, void* base) {
  const size_t bh = (size_t)d->batch * d->num_kv_heads;
  const size_t bq = (size_t)d->batch * d->num_q_heads;
  size_t off = 0;
  Workspace w{};
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? static_cast<uint8_t*>(base) + off : nullptr;
    off += round256(bytes);
    return p;
  };
  w.scores = reinterpret_cast<float*>(take(bh * d->max_blocks * sizeof(float)));
  w.idx = reinterpret_cast<int32_t*>(take(bh * k_max * sizeof(int32_t)));
  w.n_sel = reinterpret_cast<int32_t*>(take(bh * sizeof(int32_t)));
  w.o_part = reinterpret_cast<float*>(take(bq * S * kHeadDim * sizeof(float)));
  w.lse_part = reinterpret_cast<float*>(take(bq * S * sizeof(float)));
  w.work_counter = reinterpret_cast<uint32_t*>(take(8 * sizeof(uint32_t)));
  w.row_flag = reinterpret_cast<uint32_t*>(take(bh * sizeof(uint32_t)));
  w.ctl_bytes = round256(8 * sizeof(uint32_t)) + round256(bh * sizeof(uint32_t));
  w.bytes = off;
  return w;
}

}  // namespace

struct DecodeLaunch {
  CUtensorMap tk, tv;
  DecodeParams p;
};

// Checks and tensor maps of a decode launch (nothing is enqueued).
static seer_status decode_prepare(const seer_dims* d, const uint16_t* q, const uint16_t* k_pool,
                                  const uint16_t* v_pool, const int32_t* page_table,
                                  const int32_t* seqlens, const int32_t* idx,
                                  const int32_t* n_sel, int32_t k_max, int32_t num_splits,
                                  float softmax_scale, float* o_part, float* lse_part,
                                  uint32_t* work_counter, int32_t* dev_status, DecodeLaunch* L) {
  SEER_TRY(check_dims(d));
  SEER_TRY(check_pool(d, k_pool));
  SEER_TRY(check_pool(d, v_pool));
  if (!q || !seqlens || !idx || !n_sel || !o_part || !lse_part) return SEER_ERR_INVALID_ARG;
  if (k_max < 1 || k_max > d->max_blocks || num_splits < 1 || num_splits > kMaxSplits)
    return SEER_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(o_part, 16) || !aligned(work_counter, 8))
    return SEER_ERR_UNSUPPORTED;
  const int64_t items = (int64_t)d->batch * d->num_kv_heads * num_splits;
  if (items > INT_MAX / 2) return SEER_ERR_UNSUPPORTED;  // item ids carry a flag bit
  const int token_inner = d->stride_token < d->stride_head ? 1 : 0;
  SEER_TRY(make_kv_map(k_pool, d, token_inner, &L->tk));
  SEER_TRY(make_kv_map(v_pool, d, token_inner, &L->tv));
  DecodeParams& p = L->p;
  p.q = q;
  p.page_table = page_table;
  p.seqlens = seqlens;
  p.idx = idx;
  p.n_sel = n_sel;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.status = dev_status;
  p.B = d->batch;
  p.Hq = d->num_q_heads;
  p.Hkv = d->num_kv_heads;
  p.G = d->num_q_heads / d->num_kv_heads;
  p.bs = d->block_size;
  p.max_blocks = d->max_blocks;
  p.k_max = k_max;
  p.S = num_splits;
  p.num_items = (int)items;
  p.token_inner = token_inner;
  p.num_pages = d->num_pages;
  p.scale_log2 = softmax_scale * kLog2e;
  p.block_lse = nullptr;
  p.work_counter = work_counter;
  return SEER_OK;
}

extern "C" {

int32_t seer_version(void) { return 10000; }

const char* seer_last_cuda_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

const char* seer_status_string(seer_status s) {
  switch (s) {
    case SEER_OK: return "ok";
    case SEER_ERR_INVALID_ARG: return "invalid argument";
    case SEER_ERR_UNSUPPORTED: return "unsupported shape, layout or alignment";
    case SEER_ERR_CUDA: return "CUDA error";
    case SEER_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

seer_status seer_dims_default(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, int32_t max_blocks,
                              int64_t num_pages, seer_dims* out) {
  if (out == nullptr) return SEER_ERR_INVALID_ARG;
  seer_dims d;
  d.batch = batch;
  d.num_q_heads = num_q_heads;
  d.num_kv_heads = num_kv_heads;
  d.head_dim = head_dim;
  d.block_size = block_size;
  d.max_blocks = max_blocks;
  d.num_pages = num_pages;
  d.stride_head = head_dim;
  d.stride_token = (int64_t)num_kv_heads * head_dim;
  d.stride_page = (int64_t)block_size * num_kv_heads * head_dim;
  SEER_TRY(check_dims(&d));
  *out = d;
  return SEER_OK;
}

seer_status seer_k_from_sparsity(int32_t nb, int32_t sparsity_permille, int32_t* k) {
  if (k == nullptr || nb < 0 || sparsity_permille < 0 || sparsity_permille > 1000)
    return SEER_ERR_INVALID_ARG;
  const int64_t kept = ((int64_t)(1000 - sparsity_permille) * nb + 999) / 1000;
  *k = (int32_t)(kept < 1 ? 1 : kept);
  return SEER_OK;
}

seer_status seer_k_from_budget(int32_t nb, int32_t budget_tokens, int32_t block_size, int32_t* k) {
  if (k == nullptr || nb < 0 || budget_tokens < 0 || block_size < 1) return SEER_ERR_INVALID_ARG;
  int64_t v = budget_tokens / block_size;
  if (v > nb) v = nb;
  *k = (int32_t)(v < 1 ? 1 : v);
  return SEER_OK;
}

seer_status seer_fill_k(const seer_dims* d, const int32_t* seqlens, int32_t sparsity_permille,
                        int32_t budget_tokens, int32_t* k_per_seq, seer_stream stream) {
  SEER_TRY(check_dims(d));
  if (!seqlens || !k_per_seq || budget_tokens < 0 || sparsity_permille < 0 ||
      sparsity_permille > 1000)
    return SEER_ERR_INVALID_ARG;
  SEER_CUDA(run_fill_k(seqlens, d->batch, d->block_size, sparsity_permille, budget_tokens,
                       k_per_seq, stream));
  return SEER_OK;
}

int32_t seer_default_splits(const seer_dims* d, int32_t k_max, int32_t num_sms) {
  if (check_dims(d) != SEER_OK || k_max < 1) return 1;
  if (num_sms < 1) num_sms = num_sms_current();
  const int64_t bh = (int64_t)d->batch * d->num_kv_heads;
  int64_t s = (4 * (int64_t)num_sms + bh - 1) / bh;
  int64_t cap = k_max / 2;
  if (cap < 1) cap = 1;
  if (cap > kMaxSplits) cap = kMaxSplits;
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  return (int32_t)s;
}

size_t seer_step_workspace_bytes(const seer_dims* d, int32_t k_max, int32_t num_splits) {
  if (check_dims(d) != SEER_OK || k_max < 1 || num_splits < 1) return 0;
  return carve(d, k_max, num_splits, nullptr).bytes;
}

seer_status seer_pool_keys(const seer_dims* d, const uint16_t* k_pool, const int32_t* page_table,
                           const int32_t* seqlens, int32_t incremental, float* kbar,
                           int32_t* dev_status, seer_stream stream) {
  SEER_TRY(check_dims(d));
  SEER_TRY(check_pool(d, k_pool));
  if (!seqlens || !kbar || (incremental != 0 && incremental != 1)) return SEER_ERR_INVALID_ARG;
  if (!aligned(kbar, 16)) return SEER_ERR_UNSUPPORTED;
  PoolParams p;
  p.k_pool = k_pool;
  p.page_table = page_table;
  p.seqlens = seqlens;
  p.kbar = kbar;
  p.status = dev_status;
  p.Hkv = d->num_kv_heads;
  p.bs = d->block_size;
  p.max_blocks = d->max_blocks;
  p.incremental = incremental;
  p.num_pages = d->num_pages;
  p.stride_page = d->stride_page;
  p.stride_token = d->stride_token;
  p.stride_head = d->stride_head;
  SEER_CUDA(run_pool_keys(p, d->batch, stream));
  return SEER_OK;
}

seer_status seer_gate_scores(const seer_dims* d, const uint16_t* q, const float* w_gate,
                             const float* kbar, const int32_t* seqlens, float gate_scale,
                             float* scores, int32_t* dev_status, seer_stream stream) {
  SEER_TRY(check_dims(d));
  if (!q || !w_gate || !kbar || !seqlens || !scores) return SEER_ERR_INVALID_ARG;
  if (!aligned(w_gate, 16) || !aligned(kbar, 16) || !aligned(q, 4)) return SEER_ERR_UNSUPPORTED;
  GateParams p;
  p.q = q;
  p.w_gate = w_gate;
  p.kbar = kbar;
  p.seqlens = seqlens;
  p.scores = scores;
  p.status = dev_status;
  p.Hq = d->num_q_heads;
  p.Hkv = d->num_kv_heads;
  p.G = d->num_q_heads / d->num_kv_heads;
  p.bs = d->block_size;
  p.max_blocks = d->max_blocks;
  p.gate_scale = gate_scale;
  // about two CTAs per SM, each with a whole number of 32-row sweeps
  const int64_t bh = (int64_t)d->batch * d->num_kv_heads;
  int64_t chunks = (2 * (int64_t)num_sms_current() + bh - 1) / bh;
  if (chunks < 1) chunks = 1;
  int64_t per = (d->max_blocks + chunks - 1) / chunks;
  per = ((per + 31) / 32) * 32;
  p.blocks_per_cta = (int)per;
  SEER_CUDA(run_gate_scores(p, d->batch, stream));
  return SEER_OK;
}

seer_status seer_block_select(const seer_dims* d, const float* scores, const int32_t* seqlens,
                              const int32_t* k_per_seq, int32_t force_newest, int32_t k_max,
                              int32_t* idx, int32_t* n_sel, int32_t* dev_status,
                              seer_stream stream) {
  SEER_TRY(check_dims(d));
  if (!scores || !seqlens || !k_per_seq || !idx || !n_sel) return SEER_ERR_INVALID_ARG;
  if (k_max < 1 || k_max > d->max_blocks) return SEER_ERR_INVALID_ARG;
  SelectParams p;
  p.scores = scores;
  p.seqlens = seqlens;
  p.k_per_seq = k_per_seq;
  p.idx = idx;
  p.n_sel = n_sel;
  p.status = dev_status;
  p.Hkv = d->num_kv_heads;
  p.bs = d->block_size;
  p.max_blocks = d->max_blocks;
  p.k_max = k_max;
  p.force_newest = force_newest ? 1 : 0;
  SEER_CUDA(run_block_select(p, d->batch, stream));
  return SEER_OK;
}

seer_status seer_block_select_unified(const seer_dims* d, const float* scores, const int32_t* seqlens,
                                      const int32_t* k_per_seq, int32_t force_newest, int32_t k_max,
                                      int32_t* idx, int32_t* n_sel, int32_t* dev_status,
                                      seer_stream stream) {
  SEER_TRY(check_dims(d));
  if (!scores || !seqlens || !k_per_seq || !idx || !n_sel) return SEER_ERR_INVALID_ARG;
  if (k_max < 1 || k_max > d->max_blocks) return SEER_ERR_INVALID_ARG;
  SelectParams p;
  p.scores = scores;
  p.seqlens = seqlens;
  p.k_per_seq = k_per_seq;
  p.idx = idx;
  p.n_sel = n_sel;
  p.status = dev_status;
  p.Hkv = d->num_kv_heads;
  p.bs = d->block_size;
  p.max_blocks = d->max_blocks;
  p.k_max = k_max;
  p.force_newest = force_newest ? 1 : 0;
  SEER_CUDA(run_unified_select(p, d->batch, stream, false));
  return SEER_OK;
}

seer_status seer_sparse_decode(const seer_dims* d, const uint16_t* q, const uint16_t* k_pool,
                               const uint16_t* v_pool, const int32_t* page_table,
                               const int32_t* seqlens, const int32_t* idx, const int32_t* n_sel,
                               int32_t k_max, int32_t num_splits, float softmax_scale,
                               float* o_part, float* lse_part, uint32_t* work_counter,
                               int32_t* dev_status, seer_stream stream) {
  DecodeLaunch L;
  SEER_TRY(decode_prepare(d, q, k_pool, v_pool, page_table, seqlens, idx, n_sel, k_max,
                          num_splits, softmax_scale, o_part, lse_part, work_counter, dev_status,
                          &L));
  SEER_CUDA(run_sparse_decode(L.tk, L.tv, L.p, num_sms_current(), stream, false));
  return SEER_OK;
}

size_t seer_block_lse_elems(const seer_dims* d) {
  if (check_dims(d) != SEER_OK) return 0;
  return (size_t)d->batch * d->num_q_heads * d->max_blocks * (d->block_size / kTileTokens) * 4;
}

seer_status seer_sparse_decode_mass(const seer_dims* d, const uint16_t* q, const uint16_t* k_pool,
                                    const uint16_t* v_pool, const int32_t* page_table,
                                    const int32_t* seqlens, const int32_t* idx,
                                    const int32_t* n_sel, int32_t k_max, int32_t num_splits,
                                    float softmax_scale, float* o_part, float* lse_part,
                                    float* block_lse, uint32_t* work_counter, int32_t* dev_status,
                                    seer_stream stream) {
  if (block_lse == nullptr) return SEER_ERR_INVALID_ARG;
  DecodeLaunch L;
  SEER_TRY(decode_prepare(d, q, k_pool, v_pool, page_table, seqlens, idx, n_sel, k_max,
                          num_splits, softmax_scale, o_part, lse_part, work_counter, dev_status,
                          &L));
  L.p.block_lse = block_lse;
  SEER_CUDA(run_sparse_decode(L.tk, L.tv, L.p, num_sms_current(), stream, false));
  return SEER_OK;
}

seer_status seer_block_mass(const seer_dims* d, const int32_t* idx, const int32_t* n_sel,
                            int32_t k_max, const int32_t* seqlens, const float* block_lse,
                            const float* lse, float* mass, seer_stream stream) {
  SEER_TRY(check_dims(d));
  if (!idx || !n_sel || !seqlens || !block_lse || !lse || !mass) return SEER_ERR_INVALID_ARG;
  if (k_max < 1 || k_max > d->max_blocks) return SEER_ERR_INVALID_ARG;
  MassParams p;
  p.idx = idx;
  p.n_sel = n_sel;
  p.seqlens = seqlens;
  p.block_lse = block_lse;
  p.lse = lse;
  p.mass = mass;
  p.Hq = d->num_q_heads;
  p.Hkv = d->num_kv_heads;
  p.G = d->num_q_heads / d->num_kv_heads;
  p.bs = d->block_size;
  p.max_blocks = d->max_blocks;
  p.k_max = k_max;
  SEER_CUDA(run_block_mass(p, d->batch, stream));
  return SEER_OK;
}

seer_status seer_combine(const seer_dims* d, const float* o_part, const float* lse_part,
                         int32_t num_splits, uint16_t* out, float* lse_out, seer_stream stream) {
  SEER_TRY(check_dims(d));
  if (!o_part || !lse_part || !out) return SEER_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > kMaxSplits) return SEER_ERR_INVALID_ARG;
  CombineParams p = {};
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.out = out;
  p.lse_out = lse_out;
  p.S = num_splits;
  SEER_CUDA(run_combine(p, d->batch, d->num_q_heads, stream, false));
  return SEER_OK;
}

// What an entry point adds around the step's kernels, enqueued only once
// every check has passed.
struct StepExtras {
  const uint16_t* q_mapped = nullptr;     // host q mapped into the device: the gate reads
                                          // it and fills a->q for the decode
  uint16_t* out_mapped = nullptr;         // host out mapped into the device: the combine
                                          // writes it besides a->out
  const uint16_t* q_host_copy = nullptr;  // host q copied into a->q before the kernels
  bool zero_ctl = false;                  // control words and row flags zeroed first
};

static seer_status decode_step_impl(const seer_dims* d, const seer_step_args* a,
                                    seer_stream stream, const StepExtras& x) {
  const uint16_t* q_mapped = x.q_mapped;
  uint16_t* out_mapped = x.out_mapped;
  NvtxRange step_range("seer_decode_step");
  SEER_TRY(check_dims(d));
  if (a == nullptr || a->k_per_seq == nullptr || a->kbar == nullptr) return SEER_ERR_INVALID_ARG;
  if (a->update_kbar < 0 || a->update_kbar > 2) return SEER_ERR_INVALID_ARG;
  if (a->unified_heads != 0 && a->unified_heads != 1) return SEER_ERR_INVALID_ARG;
  if ((a->k_new == nullptr) != (a->v_new == nullptr)) return SEER_ERR_INVALID_ARG;
  if (a->k_new && (!aligned(a->k_new, 8) || !aligned(a->v_new, 8))) return SEER_ERR_UNSUPPORTED;
  if (a->k_max < 1 || a->num_splits < 1) return SEER_ERR_INVALID_ARG;
  if (a->workspace == nullptr || !aligned(a->workspace, 256)) return SEER_ERR_WORKSPACE;
  const Workspace w = carve(d, a->k_max, a->num_splits, a->workspace);
  if (a->workspace_bytes < w.bytes) return SEER_ERR_WORKSPACE;
  // every check (and the decode tensor maps) before anything is enqueued
  if (!a->q || !a->w_gate || !a->seqlens || !a->out) return SEER_ERR_INVALID_ARG;
  if (!aligned(a->w_gate, 16) || !aligned(a->kbar, 16)) return SEER_ERR_UNSUPPORTED;
  DecodeLaunch L;
  SEER_TRY(decode_prepare(d, a->q, a->k_pool, a->v_pool, a->page_table, a->seqlens, w.idx,
                          w.n_sel, a->k_max, a->num_splits, a->softmax_scale, w.o_part,
                          w.lse_part, w.work_counter, a->dev_status, &L));
  const bool mass = a->block_mass != nullptr || a->block_lse != nullptr;
  if (mass && (!a->block_mass || !a->block_lse || !a->lse_out)) return SEER_ERR_INVALID_ARG;
  L.p.block_lse = mass ? a->block_lse : nullptr;

  if (x.zero_ctl) SEER_CUDA(cudaMemsetAsync(w.work_counter, 0, w.ctl_bytes, stream));
  if (x.q_host_copy != nullptr)
    SEER_CUDA(cudaMemcpyAsync(const_cast<uint16_t*>(a->q), x.q_host_copy,
                              (size_t)d->batch * d->num_q_heads * kHeadDim * sizeof(uint16_t),
                              cudaMemcpyHostToDevice, stream));
  if (a->update_kbar == 2) {
    NvtxRange r("pool_keys (full rebuild)");
    SEER_TRY(seer_pool_keys(d, a->k_pool, a->page_table, a->seqlens, 0, a->kbar, a->dev_status,
                            stream));
  }
  // a0 (incremental) + a1 + a2 in one kernel; same results as the three calls
  GateSelectParams g = {};
  g.q = q_mapped != nullptr ? q_mapped : a->q;
  g.q_copy = q_mapped != nullptr ? const_cast<uint16_t*>(a->q) : nullptr;
  g.w_gate = a->w_gate;
  g.kbar = a->kbar;
  g.seqlens = a->seqlens;
  g.k_per_seq = a->k_per_seq;
  g.scores = w.scores;
  g.idx = w.idx;
  g.n_sel = w.n_sel;
  g.status = a->dev_status;
  g.k_pool = a->k_pool;
  // the KV append writes the caller's pools (their own buffers, given as const
  // because nothing else in the step writes them)
  g.k_pool_w = const_cast<uint16_t*>(a->k_pool);
  g.v_pool_w = const_cast<uint16_t*>(a->v_pool);
  g.k_new = a->k_new;
  g.v_new = a->v_new;
  g.page_table = a->page_table;
  g.incremental = a->update_kbar == 1 ? 1 : 0;
  g.num_pages = d->num_pages;
  g.stride_page = d->stride_page;
  g.stride_token = d->stride_token;
  g.stride_head = d->stride_head;
  g.Hq = d->num_q_heads;
  g.Hkv = d->num_kv_heads;
  g.G = d->num_q_heads / d->num_kv_heads;
  g.bs = d->block_size;
  g.max_blocks = d->max_blocks;
  g.k_max = a->k_max;
  g.force_newest = a->force_newest ? 1 : 0;
  g.gate_scale = a->gate_scale;
  g.scores_only = a->unified_heads ? 1 : 0;
  g.B = d->batch;
  const int num_sms = num_sms_current();
  // More rows than SMs: a persistent row-claiming gate grid, whose rows finish
  // one after another over the whole gate phase.  Each row then publishes a
  // flag and the decode grid starts on it at once instead of waiting for the
  // whole gate grid (the unified select, a grid of its own, keeps the wait).
  // With one row per CTA the rows finish within a few microseconds of each
  // other and the grid-wide wait is cheaper than the per-row protocol.
  const bool rows_grid = (int64_t)d->batch * d->num_kv_heads > num_sms;
  const bool row_flags = rows_grid && !a->unified_heads;
  // the decode's item counter: at rest from the last launch (or
  // seer_step_workspace_init); without row flags the gate grid also zeroes
  // it, before the decode grid reads it
  g.work_counter = row_flags ? nullptr : w.work_counter;
  g.row_flag = row_flags ? w.row_flag : nullptr;
  g.epoch = w.work_counter + 2;
  g.row_counter = w.work_counter + 5;  // the row-claiming grid's counter and
  g.row_done = w.work_counter + 6;     // its CTAs done (the last resets both)
  {
    NvtxRange r("gate_select");
    if (rows_grid) {
      SEER_CUDA(run_gate_select_rows(g, num_sms, stream, true));
    } else {
      SEER_CUDA(run_gate_select(g, d->batch, stream, true));
    }
  }
  if (a->unified_heads) {  // one block set per sequence, shared by its KV heads
    SelectParams u;
    u.scores = w.scores;
    u.seqlens = a->seqlens;
    u.k_per_seq = a->k_per_seq;
    u.idx = w.idx;
    u.n_sel = w.n_sel;
    u.status = a->dev_status;
    u.Hkv = d->num_kv_heads;
    u.bs = d->block_size;
    u.max_blocks = d->max_blocks;
    u.k_max = a->k_max;
    u.force_newest = a->force_newest ? 1 : 0;
    NvtxRange r("unified_select");
    SEER_CUDA(run_unified_select(u, d->batch, stream, true));
  }
  // a3, then a4; each grid launches early and waits for its predecessor
  {
    NvtxRange r("sparse_decode");
    SEER_CUDA(run_sparse_decode(L.tk, L.tv, L.p, num_sms_current(), stream, true,
                                row_flags ? w.work_counter : nullptr,
                                row_flags ? w.row_flag : nullptr));
  }
  CombineParams c = {};
  c.o_part = w.o_part;
  c.lse_part = w.lse_part;
  c.out = a->out;
  c.lse_out = a->lse_out;
  c.S = a->num_splits;
  c.out_host = out_mapped;
  {
    NvtxRange r("combine");
    // One CTA of 128 threads per (b, query head) row while those fit on the
    // GPU at once (2048 resident threads per SM); past that, one warp per row
    // (the same bits), which needs a quarter of the threads.
    // Output in mapped host memory: one warp per row with 8-byte stores when
    // both outputs allow them, so each row crosses PCIe as one 256-byte write.
    const int64_t rows = (int64_t)d->batch * d->num_q_heads;
    const bool packed = aligned(a->out, 8) && (out_mapped == nullptr || aligned(out_mapped, 8));
    if (rows * kHeadDim > (int64_t)num_sms * 2048 || (out_mapped != nullptr && packed))
      SEER_CUDA(run_combine_rows(c, d->batch, d->num_q_heads, stream, true, packed));
    else
      SEER_CUDA(run_combine(c, d->batch, d->num_q_heads, stream, true));
  }
  if (mass) {
    MassParams m;
    m.idx = w.idx;
    m.n_sel = w.n_sel;
    m.seqlens = a->seqlens;
    m.block_lse = a->block_lse;
    m.lse = a->lse_out;
    m.mass = a->block_mass;
    m.Hq = d->num_q_heads;
    m.Hkv = d->num_kv_heads;
    m.G = d->num_q_heads / d->num_kv_heads;
    m.bs = d->block_size;
    m.max_blocks = d->max_blocks;
    m.k_max = a->k_max;
    NvtxRange r("block_mass");
    SEER_CUDA(run_block_mass(m, d->batch, stream));
  }
  return SEER_OK;
}

seer_status seer_decode_step(const seer_dims* d, const seer_step_args* a, seer_stream stream) {
  return decode_step_impl(d, a, stream, StepExtras{});
}

// The step with its control words zeroed on the stream first, after every
// check (the no-allocation entry point, whose workspace is shared by calls
// of any shape).
seer_status decode_step_zeroed_ctl(const seer_dims* d, const seer_step_args* a,
                                   seer_stream stream) {
  StepExtras x;
  x.zero_ctl = true;
  return decode_step_impl(d, a, stream, x);
}

seer_status seer_step_workspace_init(const seer_dims* d, int32_t k_max, int32_t num_splits,
                                     void* workspace, size_t workspace_bytes,
                                     seer_stream stream) {
  SEER_TRY(check_dims(d));
  if (k_max < 1 || num_splits < 1) return SEER_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned(workspace, 256)) return SEER_ERR_WORKSPACE;
  const Workspace w = carve(d, k_max, num_splits, workspace);
  if (workspace_bytes < w.bytes) return SEER_ERR_WORKSPACE;
  SEER_CUDA(cudaMemsetAsync(w.work_counter, 0, w.ctl_bytes, stream));
  return SEER_OK;
}

seer_status seer_decode_step_fused(const seer_dims* d, const seer_step_args* a,
                                   seer_stream stream) {
  NvtxRange step_range("seer_decode_step_fused");
  SEER_TRY(check_dims(d));
  if (a == nullptr || a->k_per_seq == nullptr || a->kbar == nullptr) return SEER_ERR_INVALID_ARG;
  if (a->update_kbar < 0 || a->update_kbar > 2) return SEER_ERR_INVALID_ARG;
  if (a->k_max < 1 || a->num_splits < 1) return SEER_ERR_INVALID_ARG;
  if ((a->k_new == nullptr) != (a->v_new == nullptr)) return SEER_ERR_INVALID_ARG;
  if (a->unified_heads != 0 || a->block_lse != nullptr || a->block_mass != nullptr)
    return SEER_ERR_UNSUPPORTED;  // those run through seer_decode_step
  if (a->workspace == nullptr || !aligned(a->workspace, 256)) return SEER_ERR_WORKSPACE;
  const Workspace w = carve(d, a->k_max, a->num_splits, a->workspace);
  if (a->workspace_bytes < w.bytes) return SEER_ERR_WORKSPACE;
  if (!a->q || !a->w_gate || !a->seqlens || !a->out) return SEER_ERR_INVALID_ARG;
  if (!aligned(a->w_gate, 16) || !aligned(a->kbar, 16)) return SEER_ERR_UNSUPPORTED;
  if (a->k_new && (!aligned(a->k_new, 8) || !aligned(a->v_new, 8))) return SEER_ERR_UNSUPPORTED;
  DecodeLaunch L;
  SEER_TRY(decode_prepare(d, a->q, a->k_pool, a->v_pool, a->page_table, a->seqlens, w.idx,
                          w.n_sel, a->k_max, a->num_splits, a->softmax_scale, w.o_part,
                          w.lse_part, w.work_counter, a->dev_status, &L));
  if (a->update_kbar == 2)  // a full rebuild is its own pass over K (prefill time)
    SEER_TRY(seer_pool_keys(d, a->k_pool, a->page_table, a->seqlens, 0, a->kbar, a->dev_status,
                            stream));
  FusedParams f = {};
  GateSelectParams& g = f.gate;
  g.q = a->q;
  g.w_gate = a->w_gate;
  g.kbar = a->kbar;
  g.seqlens = a->seqlens;
  g.k_per_seq = a->k_per_seq;
  g.scores = w.scores;
  g.idx = w.idx;
  g.n_sel = w.n_sel;
  g.status = a->dev_status;
  g.k_pool = a->k_pool;
  g.k_pool_w = const_cast<uint16_t*>(a->k_pool);
  g.v_pool_w = const_cast<uint16_t*>(a->v_pool);
  g.k_new = a->k_new;
  g.v_new = a->v_new;
  g.page_table = a->page_table;
  g.incremental = a->update_kbar == 1 ? 1 : 0;
  g.num_pages = d->num_pages;
  g.stride_page = d->stride_page;
  g.stride_token = d->stride_token;
  g.stride_head = d->stride_head;
  g.Hq = d->num_q_heads;
  g.Hkv = d->num_kv_heads;
  g.G = d->num_q_heads / d->num_kv_heads;
  g.bs = d->block_size;
  g.max_blocks = d->max_blocks;
  g.k_max = a->k_max;
  g.force_newest = a->force_newest ? 1 : 0;
  g.gate_scale = a->gate_scale;
  f.ctl = w.work_counter;
  f.row_flag = w.row_flag;
  f.out = a->out;
  f.lse_out = a->lse_out;
  SEER_CUDA(run_fused_step(L.tk, L.tv, L.p, f, num_sms_current(), stream));
  return SEER_OK;
}

int32_t seer_prefill_k_max(const seer_dims* d, int32_t sparsity_permille, int32_t budget_tokens) {
  if (check_dims(d) != SEER_OK) return 0;
  int32_t k = 0;
  const seer_status st = budget_tokens > 0
                             ? seer_k_from_budget(d->max_blocks, budget_tokens, d->block_size, &k)
                             : seer_k_from_sparsity(d->max_blocks, sparsity_permille, &k);
  return st == SEER_OK ? k : 0;
}

size_t seer_prefill_workspace_bytes(const seer_dims* d, int32_t k_max) {
  if (check_dims(d) != SEER_OK || k_max < 1) return 0;
  const size_t rows = (size_t)d->batch * d->num_kv_heads * d->max_blocks;
  return round256(rows * k_max * sizeof(int32_t)) + round256(rows * sizeof(int32_t));
}

// Checks, tensor maps and parameters shared by the whole prefill and its
// attention stage (nothing is enqueued).  `gate`: the gate fields are used.
static seer_status prefill_prepare(const seer_dims* d, const seer_prefill_args* a, bool gate,
                                   PrefillParams* p, CUtensorMap* tq, CUtensorMap* tk,
                                   CUtensorMap* tv) {
  SEER_TRY(check_dims(d));
  if (a == nullptr || !a->q || !a->k_pool || !a->v_pool || !a->seqlens || !a->out)
    return SEER_ERR_INVALID_ARG;
  if (a->k_max < 1 || a->k_max > d->max_blocks) return SEER_ERR_INVALID_ARG;
  if (!aligned(a->q, 16) || !aligned(a->out, 16)) return SEER_ERR_UNSUPPORTED;
  if (gate) {
    if (!a->w_gate || !a->kbar) return SEER_ERR_INVALID_ARG;
    if (a->sparsity_permille < 0 || a->sparsity_permille > 1000 || a->budget_tokens < 0)
      return SEER_ERR_INVALID_ARG;
    if (a->workspace == nullptr || !aligned(a->workspace, 256) ||
        a->workspace_bytes < seer_prefill_workspace_bytes(d, a->k_max))
      return SEER_ERR_WORKSPACE;
    if (!aligned(a->w_gate, 16) || !aligned(a->kbar, 16)) return SEER_ERR_UNSUPPORTED;
  }
  SEER_TRY(check_pool(d, a->k_pool));
  SEER_TRY(check_pool(d, a->v_pool));
  const int token_inner = d->stride_token < d->stride_head ? 1 : 0;
  SEER_TRY(make_q_map(a->q, d, tq));
  SEER_TRY(make_kv_map(a->k_pool, d, token_inner, tk));
  SEER_TRY(make_kv_map(a->v_pool, d, token_inner, tv));
  *p = PrefillParams{};
  p->q = a->q;
  p->w_gate = a->w_gate;
  p->kbar = a->kbar;
  p->page_table = a->page_table;
  p->seqlens = a->seqlens;
  p->scores = a->scores_out;
  p->out = a->out;
  p->lse = a->lse_out;
  p->status = a->dev_status;
  p->B = d->batch;
  p->Hq = d->num_q_heads;
  p->Hkv = d->num_kv_heads;
  p->G = d->num_q_heads / d->num_kv_heads;
  p->bs = d->block_size;
  p->max_blocks = d->max_blocks;
  p->k_max = a->k_max;
  p->sparsity_permille = a->sparsity_permille;
  p->budget_tokens = a->budget_tokens;
  p->token_inner = token_inner;
  p->num_pages = d->num_pages;
  p->gate_scale = a->gate_scale;
  p->scale_log2 = a->softmax_scale * kLog2e;
  return SEER_OK;
}

seer_status seer_prefill(const seer_dims* d, const seer_prefill_args* a, seer_stream stream) {
  NvtxRange prefill_range("seer_prefill");
  PrefillParams p;
  CUtensorMap tq, tk, tv;
  SEER_TRY(prefill_prepare(d, a, true, &p, &tq, &tk, &tv));
  const size_t rows = (size_t)d->batch * d->num_kv_heads * d->max_blocks;
  p.idx = reinterpret_cast<int32_t*>(a->workspace);
  p.n_sel = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(a->workspace) +
                                       round256(rows * a->k_max * sizeof(int32_t)));
  if (a->pool_keys)
    SEER_TRY(seer_pool_keys(d, a->k_pool, a->page_table, a->seqlens, 0, a->kbar, a->dev_status,
                            stream));
  {
    NvtxRange r("prefill_gate_select");
    SEER_CUDA(run_prefill_gate_select(p, stream));
  }
  NvtxRange r("prefill_attention");
  SEER_CUDA(run_prefill_attention(tq, tk, tv, p, stream));
  return SEER_OK;
}

seer_status seer_prefill_attention(const seer_dims* d, const seer_prefill_args* a,
                                   const int32_t* idx, const int32_t* n_sel,
                                   seer_stream stream) {
  NvtxRange r("seer_prefill_attention");
  if (idx == nullptr || n_sel == nullptr) return SEER_ERR_INVALID_ARG;
  PrefillParams p;
  CUtensorMap tq, tk, tv;
  SEER_TRY(prefill_prepare(d, a, false, &p, &tq, &tk, &tv));
  p.idx = const_cast<int32_t*>(idx);
  p.n_sel = const_cast<int32_t*>(n_sel);
  SEER_CUDA(run_prefill_attention(tq, tk, tv, p, stream));
  return SEER_OK;
}

// Device address of host memory that is pinned and mapped into the device's
// address space, else NULL (pageable memory, or not a host pointer).
static void* mapped_host_ptr(const void* host) {
  cudaPointerAttributes at;
  if (host == nullptr || cudaPointerGetAttributes(&at, host) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

int32_t seer_host_ptr_mapped(const void* host_ptr) {
  return mapped_host_ptr(host_ptr) != nullptr ? 1 : 0;
}

seer_status seer_decode_step_host(const seer_dims* d, const seer_step_args* a,
                                  const uint16_t* q_host, uint16_t* q_dev, uint16_t* out_host,
                                  seer_stream stream) {
  SEER_TRY(check_dims(d));
  if (a == nullptr || q_host == nullptr || q_dev == nullptr || out_host == nullptr ||
      a->out == nullptr)
    return SEER_ERR_INVALID_ARG;
  const size_t bytes = (size_t)d->batch * d->num_q_heads * d->head_dim * sizeof(uint16_t);
  // mapped buffers are read and written by the step's own kernels; others
  // go through a copy on the stream
  // (the gate reads mapped q as 16-byte words: a q_host off that boundary is copied)
  StepExtras x;
  x.q_mapped = static_cast<const uint16_t*>(mapped_host_ptr(q_host));
  if (x.q_mapped != nullptr && !aligned(x.q_mapped, 16)) x.q_mapped = nullptr;
  x.out_mapped = static_cast<uint16_t*>(mapped_host_ptr(out_host));
  if (x.q_mapped == nullptr) x.q_host_copy = q_host;  // copied after the step's checks
  seer_step_args b = *a;
  b.q = q_dev;
  SEER_TRY(decode_step_impl(d, &b, stream, x));
  if (x.out_mapped == nullptr)
    SEER_CUDA(cudaMemcpyAsync(out_host, a->out, bytes, cudaMemcpyDeviceToHost, stream));
  return SEER_OK;
}

}  // extern "C"

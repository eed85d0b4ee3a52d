// seer_decode_step_noalloc: the per-stage decode step (seer_decode_step) for
// callers that cannot allocate device memory.  Its workspace (scores,
// indices, counts, split partials) lives in one file-scope device array owned
// by this library instead of a caller buffer.
#include <mutex>

#include "seer_kernels.cuh"

namespace {

constexpr size_t kScratchBytes = SEER_NOALLOC_SCRATCH_BYTES;  // per device
constexpr int kMaxDevices = 64;

// Held by every GPU that loads the library, until the process exits.
static __device__ __align__(256) uint8_t g_step_scratch[kScratchBytes];

// Device address of g_step_scratch, looked up once per device with that
// device current and kept for the process (valid while the device's primary
// context lives).  In host code the symbol itself is only a host-side
// handle, never a device pointer.
void* scratch_address(int device) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  if (device < 0 || device >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[device] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_step_scratch) != cudaSuccess) return nullptr;
    addr[device] = p;
  }
  return addr[device];
}

}  // namespace

// seer_decode_step with the control words and row flags zeroed on the stream
// after every check and before the kernels (defined with the other step
// entry points; C linkage, hidden like every symbol outside the header).
extern "C" seer_status decode_step_zeroed_ctl(const seer_dims* d, const seer_step_args* a,
                                              seer_stream stream);

extern "C" {

seer_status seer_decode_step_noalloc(const seer_dims* d, const seer_step_args* a,
                                     seer_stream stream) {
  if (a == nullptr) return SEER_ERR_INVALID_ARG;
  const size_t need = seer_step_workspace_bytes(d, a->k_max, a->num_splits);
  if (need == 0) return SEER_ERR_INVALID_ARG;
  if (need > kScratchBytes) return SEER_ERR_WORKSPACE;  // beyond the fixed array
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess) return SEER_ERR_CUDA;
  void* scratch = scratch_address(device);
  if (scratch == nullptr) return SEER_ERR_CUDA;
  seer_step_args b = *a;
  b.workspace = scratch;
  b.workspace_bytes = kScratchBytes;
  // The control words sit at an offset that depends on the shape, k_max and
  // split count, so a call after a differently shaped one would find other
  // data there: the step zeroes them on the stream first.
  return decode_step_zeroed_ctl(d, &b, stream);
}

}  // extern "C"

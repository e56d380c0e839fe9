// Forward entry point whose scratch lives in a fixed, statically sized device array of this
// module instead of a caller-supplied workspace. It runs the same tensor-core forward as
// etp_forward; only the origin of the scratch differs.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>

#include "etp_internal.h"

namespace etp {
namespace {

constexpr size_t kScratchBytes = 256 * 1024;
constexpr int kMaxDevices = 64;

// Pre-split weights and the pipeline status word of the tensor-core forward. One copy per
// device (a __device__ variable is instantiated in every context that loads the module).
__device__ __align__(256) unsigned char g_fixed_scratch[kScratchBytes];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_fixed_scratch on the current device, looked up once per device.
etp_status fixed_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "etp_forward_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("etp_forward_noalloc: device ordinal " + std::to_string(dev) + " beyond the supported " +
              std::to_string(kMaxDevices));
    return ETP_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fixed_scratch);
    if (e != cudaSuccess) return cuda_status(e, "etp_forward_noalloc: cudaGetSymbolAddress");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ETP_OK;
}

}  // namespace
}  // namespace etp

using etp::set_error;

extern "C" etp_status etp_forward_noalloc(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                                          const int* sender, const float* edge_vec, const float* x,
                                          const float* W, float* out, void* stream) {
  const etp::Ctx* c = etp::ctx_of(h);
  if (!c) {
    set_error("etp_forward_noalloc: NULL handle");
    return ETP_ERR_INVALID_ARG;
  }
  if (n_nodes < 0 || n_edges < 0) {
    set_error("etp_forward_noalloc: negative size");
    return ETP_ERR_INVALID_ARG;
  }
  if (static_cast<long long>(n_nodes) * c->dim >= (1LL << 31)) {
    set_error("etp_forward_noalloc: n_nodes * dim must stay below 2^31");
    return ETP_ERR_UNSUPPORTED;
  }
  if (!row_ptr || !out || (n_edges > 0 && (!sender || !edge_vec || !x || !W))) {
    set_error("etp_forward_noalloc: NULL array");
    return ETP_ERR_INVALID_ARG;
  }
  if (!etp::aligned16(out) || (x && !etp::aligned16(x)) || (W && !etp::aligned16(W))) {
    set_error("etp_forward_noalloc: x, W and out must be 16-byte aligned");
    return ETP_ERR_INVALID_ARG;
  }
  if (c->general) {   // the general kernels need no scratch at all
    if (static_cast<long long>(n_nodes) * c->gen.dim_out >= (1LL << 31)) {
      set_error("etp_forward_noalloc: n_nodes * dim must stay below 2^31");
      return ETP_ERR_UNSUPPORTED;
    }
    return etp::launch_general_forward(c->gen, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out,
                                       static_cast<cudaStream_t>(stream));
  }
  const size_t need = etp::tc::forward_tc_workspace_bytes(*c, n_nodes);
  if (need > etp::kScratchBytes) {
    set_error("etp_forward_noalloc: this handle needs " + std::to_string(need) +
              " bytes of scratch, above the fixed " + std::to_string(etp::kScratchBytes) +
              "; use etp_forward with a workspace");
    return ETP_ERR_CAPACITY;
  }
  if (n_nodes == 0) return ETP_OK;
  void* scratch = nullptr;
  etp_status st = etp::fixed_scratch(&scratch);
  if (st != ETP_OK) return st;
  // The status word inside the scratch is cleared by the first kernel of the launch sequence and
  // the pre-split weights are rewritten in full on every call, so nothing depends on its contents
  // from an earlier call.
  return etp::tc::launch_forward_tc(*c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, scratch,
                                    static_cast<cudaStream_t>(stream));
}

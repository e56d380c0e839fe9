// Forward entry point whose scratch lives in a fixed, statically sized device array of this
// module instead of a caller-supplied workspace. For uniform handles it always runs the
// edge-major tensor-core forward (whatever ETP_FORWARD says); general handles run the
// general forward, which needs no scratch (its tensor-core form builds its split weights in
// shared memory).
#include <cuda_runtime.h>

#include <cstdint>
#include <string>

#include "etp_internal.h"

namespace etp {
namespace {

constexpr size_t kScratchBytes = 256 * 1024;

// Pre-split weights of the tensor-core forward. One copy per device (a __device__ variable is
// instantiated in every context that loads the module).
__device__ __align__(256) unsigned char g_fixed_scratch[kScratchBytes];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of g_fixed_scratch in the current device's context. Looked up on every call (a
// host-side query, cheap next to the launches), so a context that was torn down and re-created,
// which may load the module at another address, never sees a stale pointer.
etp_status fixed_scratch(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_fixed_scratch);
  if (e != cudaSuccess) return cuda_status(e, "etp_forward_noalloc: cudaGetSymbolAddress");
  *out = p;
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
  if (etp::gate(h, "etp_forward_noalloc") != ETP_OK) return ETP_ERR_CUDA;
  if (c->general) {   // the general forward needs no scratch at all
    if (static_cast<long long>(n_nodes) * c->gen.dim_out >= (1LL << 31)) {
      set_error("etp_forward_noalloc: n_nodes * dim must stay below 2^31");
      return ETP_ERR_UNSUPPORTED;
    }
    return etp::launch_general_forward(c->gen, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out,
                                       static_cast<cudaStream_t>(stream), c->status_dev);
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
  // The pre-split weights are rewritten in full on every call, so nothing depends on the array's
  // contents from an earlier call. A bounded wait that gives up stores its code in the handle's
  // status word (pinned host memory), which etp_get_status and every later call report.
  return etp::tc::launch_forward_tc(*c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, scratch,
                                    static_cast<cudaStream_t>(stream));
}

// Internal declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "etp.h"

namespace etp {

constexpr int kNumBasis = 8;     // radial basis functions (fixed at compile time)
constexpr int kBatch = 4;        // channels per register batch (one float4 per component)
constexpr int kMaxL = 3;

// General irreps (any multiplicities and parities, rank <= 4): the path table the kernels read
// from their parameter block. Path p couples input block component rows starting at in_off with
// the harmonics of rank l2 into the output block at out_off, over mul channels, with weight
// columns woff .. woff + mul - 1; tri is the coupling index of (l1, l2, l3). The paths are also
// listed grouped by output block (forward work units) and by input block (backward work units),
// each group keeping the lexicographic path order.
constexpr int kGenMaxPaths = 128;
constexpr int kGenMaxBlocks = 16;
struct GenPath {
  int in_off, out_off, woff, mul, tri;
};
struct GenGroup {
  int off, size;      // the block's row segment: offset and mul (2l + 1) floats
  int beg, end;       // its paths: order[beg .. end - 1]
};
// Tensor-core forward plan: the paths' channels cut into slices of 32 (path, first channel),
// dealt to the four TMEM lane quadrants; MMA block b holds slice b of every quadrant (128 weight
// columns as the rows of the A operand). n_blocks = 0: the plan does not fit and the FP32
// forward serves the handle.
constexpr int kGenTcMaxBlocks = 16;
struct GenTcPlan {
  int n_blocks = 0;
  short path[kGenTcMaxBlocks][4] = {};   // path of quadrant q's slice in block b (-1: none)
  short u0[kGenTcMaxBlocks][4] = {};     // its first channel
};
struct GenParams {
  int n_paths = 0;
  int dim_in = 0;
  int dim_out = 0;
  int cols = 0;        // weight columns per basis function (sum of the paths' multiplicities)
  int sh_lmax = 0;
  float inv_rc = 0.f;
  int n_out_groups = 0;
  int n_in_groups = 0;
  int max_out_size = 0;
  int max_in_size = 0;
  GenPath p[kGenMaxPaths];
  GenGroup out_grp[kGenMaxBlocks];
  GenGroup in_grp[kGenMaxBlocks];
  unsigned char order_out[kGenMaxPaths];
  unsigned char order_in[kGenMaxPaths];
  GenTcPlan tcp;
};
static_assert(sizeof(GenParams) <= 3900, "the path table travels as a kernel parameter");

struct Ctx {
  int lmax = 0;
  int channels = 0;    // the common multiplicity (0 for a general handle whose blocks differ)
  int dim = 0;         // dim_in (= dim_out for the uniform kernels)
  int n_paths = 0;
  int cg_nnz = 0;
  int sum_2l3p1 = 0;
  float r_cut = 0.f;
  int flop_fwd = 0;       // FP32 flop per edge of the forward / backward contraction
  int flop_bwd = 0;
  bool general = false;   // true: the table-driven kernels of etp_general.cu serve this handle
  // Sticky pipeline status word: pinned host memory mapped into the device address space (status
  // for the host, status_dev for kernels; the same address under unified addressing). A kernel
  // whose bounded wait gives up stores its code there; every later call on the handle reports it.
  int* status = nullptr;
  int* status_dev = nullptr;
  bool status_mapped = false;
  GenParams gen;
  short path_blocks[kGenMaxPaths][3] = {};   // host copy of the path list: (input block, l2, output block)
};

// Configuration behind a handle (NULL for a NULL handle).
const Ctx* ctx_of(etp_handle h);

// Error message of the last failing call on this host thread.
void set_error(const std::string& msg);
etp_status cuda_status(cudaError_t e, const char* what);
// Synchronises s, then reads the handle's status word: ETP_ERR_CUDA (word left set) if nonzero.
etp_status read_status(const Ctx& c, cudaStream_t s, const char* who);
// ETP_ERR_CUDA (message set) while the handle's status word holds a code, else ETP_OK.
etp_status gate(etp_handle h, const char* who);

// ---- conv kernels (etp_conv.cu)
etp_status launch_forward(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr,
                          const int* sender, const float* edge_vec, const float* x,
                          const float* W, float* out, cudaStream_t s);
etp_status launch_backward(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr,
                           const int* sender, const float* edge_vec, const int* t_row_ptr,
                           const int* t_perm, const float* x, const float* W,
                           const float* grad_out, float* grad_x, float* grad_edge_vec,
                           int* recv_map, cudaStream_t s);
etp_status launch_radial_weights(const Ctx& c, int n_edges, const float* edge_vec,
                                 const float* W, float* w_out, cudaStream_t s);
etp_status launch_forces(int n_nodes, int n_edges, const int* row_ptr, const int* t_row_ptr,
                         const int* t_perm, const float* grad_edge_vec, float* forces,
                         cudaStream_t s);
// Returns ETP_OK or ETP_ERR_BAD_GRAPH (synchronises s). scratch: >= n_edges ints + 1.
etp_status validate_graph(int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                          const int* t_row_ptr, const int* t_perm, int* scratch, cudaStream_t s);

namespace tc {
// ---- forward with the radial projection on tcgen05 tensor cores (etp_fwd_tc.cu)
size_t forward_tc_workspace_bytes(const Ctx& c, int n_nodes);
etp_status forward_tc_status(const Ctx& c, const void* ws, cudaStream_t s);
// path_mask: per canonical edge, bit p set = path p contributes (null: every path)
etp_status launch_forward_tc(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                             const float* edge_vec, const float* x, const float* W, float* out, void* ws,
                             cudaStream_t s, const uint32_t* path_mask = nullptr);

// ---- backward with the radial projections on tcgen05 tensor cores (etp_bwd_tc.cu)
size_t backward_tc_workspace_bytes(const Ctx& c, int n_edges);
etp_status backward_tc_status(const Ctx& c, const void* ws, cudaStream_t s);
// recv: n_edges ints of scratch (filled with the receiver of every edge)
etp_status launch_backward_tc(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const float* edge_vec,
                              const int* t_row_ptr, const int* t_perm, const float* x, const float* W,
                              const float* grad_out, float* grad_x, float* grad_edge_vec, int* recv, void* ws,
                              cudaStream_t s, const uint32_t* path_mask = nullptr);
}  // namespace tc

// ---- the full product ladder (etp_ladder_full.cu)
namespace lad {
bool supported(int lmax, int channels);
size_t workspace_bytes(int lmax, int channels, int n_nodes);
size_t step_weight_floats(int lmax, int channels);
etp_status launch(int lmax, int channels, int order, int n_nodes, const float* A, const float* W, float* out,
                  void* ws, cudaStream_t s, int** status_dev);
}  // namespace lad

// ---- channel-major forward with path subsets (etp_fwd_cx.cu): l_max <= 2, 4 <= C <= 64, C % 4 == 0
namespace cx {
bool supported(const Ctx& c);
size_t workspace_bytes(const Ctx& c);
etp_status launch(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                  const float* edge_vec, const float* x, const float* W, float* out, void* ws, cudaStream_t s);
etp_status status(const Ctx& c, const void* ws, cudaStream_t s);
}  // namespace cx

// receiver of every canonical edge, recv[e] (etp_bwd_tc.cu)
etp_status launch_recv_of_edge(const int* row_ptr, int n_nodes, int n_edges, int* recv, cudaStream_t s);

// ---- weight gradient dL/dW (etp_dw.cu); recv: n_edges ints of scratch
size_t weight_grad_workspace_bytes(const Ctx& c, int n_edges);
etp_status launch_weight_grad(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                              const float* edge_vec, const float* x, const float* grad_out, float* grad_W,
                              int* recv, void* ws, cudaStream_t s);

// ---- general irreps (etp_general.cu); recv: n_edges ints of scratch; part: the per-input-block
// edge-gradient partials (general_backward_partials_bytes)
constexpr int kGenMaxDim = 4096;   // floats per node row
size_t general_backward_partials_bytes(const GenParams& g, int n_edges);
size_t general_weight_grad_bytes(const GenParams& g, int n_edges);
etp_status launch_general_weight_grad(const GenParams& g, int n_nodes, int n_edges, const int* row_ptr,
                                      const int* sender, const float* edge_vec, const float* x,
                                      const float* grad_out, float* grad_W, int* recv, float* part,
                                      cudaStream_t s);
// Runs the tensor-core forward (etp_general_tc.cu) when the handle has a plan, no mask is given and
// ETP_GEN_FORWARD is not "fp32"; err: the handle's status word (bounded waits of that kernel).
etp_status launch_general_forward(const GenParams& g, int n_nodes, int n_edges, const int* row_ptr,
                                  const int* sender, const float* edge_vec, const float* x, const float* W,
                                  float* out, cudaStream_t s, int* err, const uint32_t* path_mask = nullptr);
// Fills g.tcp (n_blocks = 0 when the plan does not fit) from the path table.
void plan_general_tc(GenParams& g);
bool general_tc_selected(const GenParams& g, const uint32_t* path_mask);
etp_status launch_general_forward_tc(const GenParams& g, int n_nodes, const int* row_ptr, const int* sender,
                                     const float* edge_vec, const float* x, const float* W, float* out,
                                     cudaStream_t s, int* err);
etp_status launch_general_backward(const GenParams& g, int n_nodes, int n_edges, const int* row_ptr,
                                   const float* edge_vec, const int* t_row_ptr, const int* t_perm,
                                   const float* x, const float* W, const float* grad_out, float* grad_x,
                                   float* grad_edge_vec, int* recv, float* part, cudaStream_t s,
                                   const uint32_t* path_mask = nullptr);

// ---- node-local product ladder (etp_product.cu)
etp_status launch_node_ladder(int lmax, int channels, int n_nodes, int nu, const float* A, const float* W,
                              float* out, cudaStream_t s);

// ---- graph kernels (etp_graph.cu)
size_t graph_workspace_bytes(int n_nodes, int max_edges);
etp_status neighbors(const float* pos, int n_nodes, const double* cell, const int* pbc,
                     float r_cut, int max_edges, int* n_edges, int* row_ptr, int* sender,
                     float* edge_vec, int* shift, int* t_row_ptr, int* t_perm, void* ws,
                     size_t ws_bytes, cudaStream_t s);
etp_status build_csr(int n_nodes, int n_edges, const int* receiver, const int* sender_in,
                     const float* edge_vec_in, int* row_ptr, int* sender, float* edge_vec,
                     int* perm, int* t_row_ptr, int* t_perm, void* ws, size_t ws_bytes,
                     cudaStream_t s);

inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace etp

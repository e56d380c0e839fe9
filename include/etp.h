/*
 * etp.h -- C ABI of the B200 equivariant edge tensor-product convolution library (libetp.so).
 *
 * The operation (see "Fast and Accurate Foundation Models for Equivariant MLIPs", section VII,
 * and "FlashCart", Fig. 3 caption, Table C1 and Fig. D1, for the pages that name it; the
 * formulas are the textbook ones):
 *
 *   for each receiver i and each edge e = (i <- j, S) of its CSR row:
 *     r_e = pos[j] - pos[i] + S . cell        (receiver -> sender),  d = |r_e|,  n = r_e / d
 *     Y_l2(n)  real spherical harmonics, component normalisation (sum_m Y_lm^2 = 2l+1), z polar
 *     R_b(d)   = (2/r_c) sin(b pi d / r_c) / d * u(d / r_c),  b = 1..n_basis,
 *     u(t)     = 1 - 28 t^6 + 48 t^7 - 21 t^8 for t < 1, else 0          (p = 6 envelope)
 *     w_{e,p,u} = sum_b R_b(d) W[b, p, u]                                 (radial projection)
 *     out[i, l3, m3, u] += w_{e,p,u} sum_{m1,m2} C^{l1 l2 l3}_{m1 m2 m3} x[j, l1, m1, u] Y_{l2 m2}(n)
 *
 *   with C the real-basis Clebsch-Gordan coefficients, paths p = (l1, l2, l3) enumerated
 *   lexicographically over (input block, l2 = 0..sh_lmax, output block) with the triangle rule
 *   and parity p1 (-1)^l2 = p3, and "uvu" channel pairing (output channel = input channel, so a
 *   path joins blocks of equal multiplicity only; see etp_create for general irreps).
 *
 * Layouts (all row-major, 32-bit):
 *   node features x, out, grad_x, grad_out : [n_nodes][dim], dim = C (L+1)^2; the row holds the
 *       blocks l = 0..L in order, block l is [m = -l..l][u = 0..C-1] (channels contiguous):
 *       element (l, m, u) sits at (l*l + l + m) * C + u. General irreps handles: the blocks in
 *       irreps-string order, block b as [m][u] with its own multiplicity (dim_in / dim_out in
 *       etp_info_t).
 *   W           : [n_basis][n_paths][C]; general irreps handles: [n_basis][cols], path p's mul_p
 *                 columns after the earlier paths' (etp_get_paths gives the order)
 *   edge arrays : receiver-sorted CSR. row_ptr [n_nodes+1], sender [n_edges], edge_vec [n_edges][3]
 *                 (float32 r_e). Canonical edge order: (receiver, sender, S0, S1, S2).
 *   transposed  : t_row_ptr [n_nodes+1] (edges per sender), t_perm [n_edges]: the edge ids in
 *                 (sender, receiver, S) order.
 *
 * Conventions.
 *   Pointers: every array argument is a CUDA DEVICE pointer owned by the caller unless the
 *   comment says "host". The library allocates no device memory; scratch comes from the caller
 *   through `workspace` (size from the matching *_workspace_bytes query, 256-byte aligned),
 *   except for etp_forward_noalloc, which uses a fixed array of the library's device module.
 *   Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Calls are
 *   asynchronous on that stream unless documented otherwise.
 *   Outputs are overwritten, never accumulated into.
 *   Errors: every call returns an etp_status; no call throws or traps. ETP_ERR_CUDA reports a
 *   launch error (no implicit synchronisation). etp_last_error() returns a thread-local message
 *   for the last failing call on the calling host thread.
 *   Pipeline status: every wait inside the tensor-core kernels is bounded (about 2 s). A kernel
 *   whose wait gives up stores a nonzero code in its handle's status word, pinned host memory
 *   mapped into the device address space, and exits early, so that call's outputs are
 *   incomplete. Kernels run after the call has returned, so the call itself still returned
 *   ETP_OK; from then on every compute call on the handle returns ETP_ERR_CUDA until
 *   etp_get_status reads and clears the code (etp_get_status synchronises; with ETP_VALIDATE=1
 *   the forward and backward also synchronise and report the code of their own launch).
 *   Thread safety: a handle is immutable after etp_create; concurrent calls on different
 *   streams with distinct output and workspace buffers are safe.
 *   Graph validation: with the environment variable ETP_VALIDATE=1, etp_forward and etp_backward
 *   first check the CSR arrays on the device (monotone row pointers, indices in range, t_perm a
 *   permutation) and return ETP_ERR_BAD_GRAPH without touching the outputs; this synchronises
 *   the stream.
 */
#ifndef ETP_H
#define ETP_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct etp_ctx* etp_handle;

typedef enum {
  ETP_OK = 0,
  ETP_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer, workspace too small */
  ETP_ERR_IRREPS = 2,        /* malformed irreps string */
  ETP_ERR_UNSUPPORTED = 3,   /* well-formed but outside what the kernels implement */
  ETP_ERR_BAD_GRAPH = 4,     /* CSR arrays failed validation (ETP_VALIDATE=1) */
  ETP_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
  ETP_ERR_CAPACITY = 6       /* an output buffer or fixed scratch is smaller than needed (n_edges reported) */
} etp_status;

typedef struct {
  int lmax;          /* L: irreps_in = irreps_out = C x (0e + 1o + ... ), SH lmax = L */
  int channels;      /* C */
  int dim_in;        /* C (L+1)^2 */
  int dim_out;       /* C (L+1)^2 */
  int n_paths;       /* P */
  int n_basis;
  int weight_numel;  /* n_basis * P * C */
  int cg_nnz;        /* real-CG nonzeros summed over the path set */
  int sum_2l3p1;     /* sum over paths of 2 l3 + 1 */
  float r_cut;
  int general;       /* 1: general irreps handle (table-driven kernels), 0: uniform kernels */
  int flop_fwd;      /* FP32 flop per edge of the forward contraction: sum_p 2 (nnz_p + 2 l3 + 1) mul_p */
  int flop_bwd;      /* the same for the backward: sum_p 2 (3 nnz_p + 2 (2 l3 + 1)) mul_p */
} etp_info_t;

/* Create a convolution handle. Host-only, synchronous; allocates host memory only: the handle,
 * and its 64-byte status word in pinned host memory mapped for the device (plain host memory when
 * no CUDA device is present). Fails with ETP_ERR_CUDA if a device is present but the pinned word
 * cannot be allocated.
 * irreps_in / irreps_out: "mulxLp+mulxLp+..." strings, e.g. "64x0e+64x1o+64x2e".
 * Two kinds of handle, chosen here:
 *  - uniform (the tensor-core kernels): every block has the same multiplicity C (C % 4 == 0,
 *    4 <= C <= 256), blocks are l = 0..L in order with parity (-1)^l, irreps_out == irreps_in,
 *    sh_lmax == L, L in {1,2,3};
 *  - general (table-driven kernels, info.general = 1): any blocks with 0 <= l <= 4 and
 *    1 <= mul <= 1024 in any order and either parity, sh_lmax <= 4, node rows of at most 4096
 *    floats, 1 to 128 paths, at most 16 blocks a side. Paths join blocks of EQUAL multiplicity only (uvu: channel u to
 *    channel u), so irreps like NequIP's 128x0e+64x1o+32x2e+32x3o couple 2e with 3o but not 1o
 *    with 2e. Paths with l1 + l2 + l3 odd use the real antisymmetric coupling (the imaginary
 *    part of the complex-to-real transformed Clebsch-Gordan tensor; the cross product for
 *    1 x 1 -> 1). W is [n_basis][cols] with path p's mul_p columns after the earlier paths'
 *    (the same as [n_basis][n_paths][C] when all blocks have C channels); node rows hold the
 *    blocks in string order, block b as [m][u] with mul_b channels. General handles support
 *    etp_forward, etp_forward_noalloc (no scratch needed), etp_backward, etp_backward_weights and,
 *    for handles with at most 32 paths (the mask has 32 bits), etp_forward_masked and
 *    etp_backward_masked (more paths: ETP_ERR_UNSUPPORTED); etp_radial_weights returns
 *    ETP_ERR_UNSUPPORTED for them. Their forward computes the radial weights on the tensor cores
 *    (kind::tf32, three products of the tf32 split) when the handle's plan fits (the paths' 32-channel
 *    slices fill at most 16 blocks of 128 weight columns, and the split weights, the output row
 *    copies and the staging fit 227 KB of shared memory); masked calls, handles outside that plan
 *    and ETP_GEN_FORWARD=fp32 run the FP32 kernel (the two agree with the float64 reference within
 *    the same tolerance, not bit for bit). The backward and the weight gradient are FP32 kernels.
 * Both need n_basis == 8 and r_cut > 0. Malformed strings -> ETP_ERR_IRREPS; anything else
 * outside these sets -> ETP_ERR_UNSUPPORTED. The path list is the enumeration described above. */
etp_status etp_create(const char* irreps_in, int sh_lmax, const char* irreps_out, int n_basis,
                      float r_cut, etp_handle* out);

/* Release a handle and its status word. NULL is accepted. */
etp_status etp_destroy(etp_handle h);

/* Pipeline status of a handle: synchronises `stream`, stores the handle's status word in *code
 * (host pointer, may be NULL) and clears it. ETP_OK when the word was 0; ETP_ERR_CUDA (with a
 * message naming the code) when a kernel of an earlier call on the handle gave up a bounded
 * wait, in which case the outputs of the calls since the previous check may be incomplete.
 * Without a CUDA device nothing is synchronised. */
etp_status etp_get_status(etp_handle h, void* stream, int* code);

/* Host address of the handle's status word (NULL for a NULL handle), for callers that poll it
 * without synchronising: nonzero means a kernel gave up a bounded wait. Writing 0 clears it. */
int* etp_status_word(etp_handle h);

/* Dimensions and path statistics of a handle (info: host pointer). */
etp_status etp_get_info(etp_handle h, etp_info_t* info);

/* The handle's path list, in the order W's columns use: paths[3 p + 0..2] = (input block index,
 * l2, output block index) of path p, block indices counting from 0 in irreps-string order.
 * paths: host array of at least 3 * capacity ints; capacity < n_paths -> ETP_ERR_CAPACITY. */
etp_status etp_get_paths(etp_handle h, int* paths, int capacity);

/* Static text for a status code, and the last detailed error message of this host thread. */
const char* etp_status_string(etp_status s);
const char* etp_last_error(void);

/* Bytes of device workspace etp_forward / etp_backward / etp_backward_weights need for a graph of
 * this size. */
size_t etp_workspace_bytes(etp_handle h, int n_nodes, int n_edges);

/* Fused forward: out[n_nodes][dim_out] = convolution of x[n_nodes][dim_in] over the CSR graph.
 * Spherical harmonics, radial basis, radial projection, Clebsch-Gordan contraction and the
 * per-receiver segmented sum run in one kernel pass; receivers without edges get zero rows.
 * Edges with d >= r_cut contribute zero (u = 0). workspace may be NULL when
 * etp_workspace_bytes returns 0. Kernel: for uniform handles with L <= 2 and 4 <= C <= 64 the
 * channel-major path-subset kernel (the CTAs take equal contiguous ranges of canonical edges;
 * a receiver whose edges cross a range boundary is summed by the CTA that adds its last part,
 * in CTA order, so the result is still bitwise reproducible), else the edge-major tensor-core
 * kernel; the environment variable ETP_FORWARD=edge or generic selects another kernel (all
 * agree with the float64 reference within the same tolerance). */
etp_status etp_forward(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                       const int* sender, const float* edge_vec, const float* x, const float* W,
                       float* out, void* workspace, size_t workspace_bytes, void* stream);

/* Forward without a workspace argument: the same computation as etp_forward, but its scratch
 * (the tf32-split radial weight matrix) sits in a fixed 256 KiB array inside libetp's device
 * module, one per device, so the call allocates no memory and takes nothing from the caller but
 * the tensors. For uniform handles it always runs the edge-major tensor-core forward and ignores
 * ETP_FORWARD, so its bits can differ from etp_forward's default kernel (both agree with the
 * float64 reference within the same tolerance); general handles run the same kernel as their
 * etp_forward, which needs no scratch (the tensor-core form splits its weights in shared memory).
 * The method has no such call; it is an interface convenience. It is for callers that cannot
 * provide device scratch: for instance a host program that reaches the model through a fixed
 * plugin interface that hands over only the input and output tensors, with no allocator of its
 * own and nowhere to keep a workspace alive between calls.
 * Limit: a handle whose scratch would exceed the 256 KiB (lmax 3 with more than 160 channels)
 * is refused with ETP_ERR_CAPACITY and a message naming both sizes; use etp_forward for it.
 * Every call looks up the array's device address in the current device's context
 * (cudaGetSymbolAddress, a host-side query that does not synchronise); the first call in a
 * context also loads the module there, so make a first call before beginning any stream
 * capture. Nothing in the array needs to start at zero: each call rewrites the weights in full.
 * A bounded wait that gives up is reported through the handle's status word (etp_get_status).
 * Overlapping calls on one device (different streams or host threads) share the array and race
 * with each other; order them (one stream, or events). The ETP_VALIDATE graph checks are not run. */
etp_status etp_forward_noalloc(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                               const int* sender, const float* edge_vec, const float* x,
                               const float* W, float* out, void* stream);

/* Fused backward (vector-Jacobian product of etp_forward for the cotangent grad_out):
 *   grad_x[n_nodes][dim_in]        = dL/dx,        L = <grad_out, out>
 *   grad_edge_vec[n_edges][3]      = dL/dr_e       (indexed by canonical edge id)
 * Runs over the transposed (sender-sorted) order so grad_x is a segmented sum per sender.
 * grad_x or grad_edge_vec may be NULL to skip that output (not both). */
etp_status etp_backward(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                        const int* sender, const float* edge_vec, const int* t_row_ptr,
                        const int* t_perm, const float* x, const float* W, const float* grad_out,
                        float* grad_x, float* grad_edge_vec, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Node-local product ladder of correlation order nu (FlashCart Fig. 3b and Fig. E1, path-reduced):
 *   B_1 = A,  B_{q+1}[l3, m3, u] = sum_{p=(l1,l2,l3)} W[q-1][p][u] sum_{m1,m2} C B_q[l1, m1, u] A[l2, m2, u],
 *   out = B_1 + ... + B_nu,
 * with the real Clebsch-Gordan coefficients and the path set of the convolution for in = SH = out
 * = lmax (4, 11, 23 paths for lmax 1, 2, 3), no edges and no radial part. A, out: [n_nodes][dim]
 * node rows (layout as for the convolution, dim = channels (lmax + 1)^2); W: [nu - 1][n_paths]
 * [channels] (unused when nu == 1). channels: a multiple of 4 in [4, 256]; 1 <= nu <= 8. Device
 * pointers, 16-byte aligned; asynchronous on stream; no workspace. */
etp_status etp_node_ladder(int lmax, int channels, int n_nodes, int nu, const float* A, const float* W,
                           float* out, void* stream);

/* The full node-local product ladder of correlation order nu (FlashCart Fig. 3b dashed curves and
 * Fig. E1 (b): the products of the retained coupling paths are compressed by W^(q) to the channel
 * width per retained rank, mixing paths and channels):
 *   T_p[m3, u] = sum_{m1,m2} C B_q[l1, m1, u] A[l2, m2, u]   for every path p = (l1, l2, l3),
 *   B_{q+1}[l3, m3, v] = sum_{p of rank l3} sum_u W_q,l3[v][p' C + u] T_p[m3, u],
 *   B_1 = A,  out = B_1 + ... + B_nu,
 * p' = the index of p among the paths of rank l3 in path order (the order of etp_node_ladder).
 * W: the nu - 1 steps one after another; a step holds the matrices W_q,l3 for l3 = 0..lmax one
 * after another, each [C][P_l3 C] row-major (P_l3 = the number of paths of rank l3; a step has
 * etp_node_ladder_full_step_floats(lmax, channels) floats). The mixing runs on the tensor cores
 * (3xTF32, fp32 accumulation): one GEMM per output component, rows = nodes, K = P_l3 C, N = C.
 * lmax 1..3; channels 32, 64, 96 or 128; 1 <= nu <= 8. A, W, out: device pointers, 16-byte
 * aligned; workspace: etp_node_ladder_full_workspace_bytes(lmax, channels, n_nodes) bytes, 256-byte
 * aligned. Asynchronous on stream; with ETP_VALIDATE=1 the call synchronises and returns
 * ETP_ERR_CUDA if a bounded pipeline wait gave up. */
size_t etp_node_ladder_full_step_floats(int lmax, int channels);
size_t etp_node_ladder_full_workspace_bytes(int lmax, int channels, int n_nodes);
etp_status etp_node_ladder_full(int lmax, int channels, int n_nodes, int nu, const float* A, const float* W,
                                float* out, void* workspace, size_t workspace_bytes, void* stream);

/* Per-edge path selection (adaptive computation: an edge may use only some of the paths).
 * path_mask[n_edges] (device, canonical edge order): bit p set = path p contributes for that edge;
 * a clear bit is the same as w_{e,p,u} = 0 for every u. Paths that no edge of a 32-edge tile needs
 * are skipped, so masks that switch paths off for whole neighbourhoods also save time. Otherwise as
 * etp_forward / etp_backward (always the tensor-core kernels; the backward is the VJP of the masked
 * forward). */
etp_status etp_forward_masked(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                              const int* sender, const float* edge_vec, const float* x, const float* W,
                              const unsigned int* path_mask, float* out, void* workspace,
                              size_t workspace_bytes, void* stream);
etp_status etp_backward_masked(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                               const int* sender, const float* edge_vec, const int* t_row_ptr,
                               const int* t_perm, const float* x, const float* W,
                               const unsigned int* path_mask, const float* grad_out, float* grad_x,
                               float* grad_edge_vec, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Weight gradient of the convolution for the cotangent grad_out (the training path):
 *   grad_W[n_basis][n_paths][C] = dL/dW,  L = <grad_out, out>,
 *   dL/dW[b][p][u] = sum_e R_b(d_e) sum_{m1,m3} x[send, l1, m1, u] (sum_m2 C Y_{l2 m2}) g[recv, l3, m3, u].
 * Runs over the canonical (receiver-sorted) order, with the channels on the lanes; partial sums
 * per range of edges are added in range order, so repeated calls give identical bits.
 * grad_W is overwritten (zero for a graph without edges). Uses the etp_workspace_bytes workspace.
 * For a general irreps handle grad_W has the W layout [n_basis][cols]; the kernel stages the
 * geometry of 128 canonical edges at a time, runs each path's channels over them and writes one
 * partial column per range; the ranges are added in order (also bit-reproducible). */
etp_status etp_backward_weights(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                                const int* sender, const float* edge_vec, const float* x,
                                const float* grad_out, float* grad_W, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Radial projection alone: w_out[n_edges][n_paths][C] = sum_b R_b(|r_e|) W[b][p][u]. */
etp_status etp_radial_weights(etp_handle h, int n_edges, const float* edge_vec, const float* W,
                              float* w_out, void* stream);

/* Forces from edge-vector gradients, F = -dL/dpos with r_e = pos[sender] - pos[receiver] + S:
 *   F[k] = sum_{e: receiver(e)=k} grad_edge_vec[e] - sum_{e: sender(e)=k} grad_edge_vec[e],
 * summed in canonical (row) order and transposed (t_perm) order respectively. */
etp_status etp_forces(int n_nodes, int n_edges, const int* row_ptr, const int* t_row_ptr,
                      const int* t_perm, const float* grad_edge_vec, float* forces, void* stream);

/* ---- graph construction (integer outputs are bit-exact against a float64 brute force) ----
 * Defined by the pages' force workloads, which build the neighbour graph of periodic cells with
 * ghost images ("Fast and Accurate Foundation Models...", section V). */

/* Device workspace for etp_neighbors / etp_build_csr with up to max_edges edges. */
size_t etp_graph_workspace_bytes(int n_nodes, int max_edges);

/* Neighbour list and canonical CSR. pos: [n_nodes][3] float32 (device). cell: 9 doubles,
 * rows = lattice vectors (HOST pointer; NULL for no cell). pbc: 3 ints (HOST pointer; NULL = none
 * periodic). An edge (i <- j, S) is kept iff, in float64 without fused multiply-add,
 *     s = (S0 cell[0] + S1 cell[1]) + S2 cell[2];  r = (pos[j] - pos[i]) + s;
 *     (r_x r_x + r_y r_y) + r_z r_z < r_cut^2,  and not (i == j and S == 0),
 * scanning every image with |S_a| <= ceil(r_cut / plane spacing_a) on periodic axes.
 * Outputs (device, capacity max_edges): row_ptr, sender, edge_vec (= float32(r)), shift
 * [max_edges][3] (may be NULL), t_row_ptr, t_perm. *n_edges (HOST) receives the edge count;
 * this call synchronises `stream` once to read it (twice if it falls back, below). If the count
 * exceeds max_edges the call returns ETP_ERR_CAPACITY after filling row_ptr only.
 * Search: from 2048 atoms (and, on a fully periodic cell, at least 4 x 4 x 4 bins of width >=
 * r_cut), atoms are binned by fractional coordinate and each receiver tests only the atoms of its
 * neighbouring bins; otherwise every pair is tested. Both apply the test above to the same
 * candidate images and produce identical outputs. Environment variable ETP_NEIGHBORS = "bins" or
 * "all-pairs" forces one; coordinates beyond about 1e8 cell lengths (or 1e6 r_cut on a
 * non-periodic axis) fall back to all pairs. */
etp_status etp_neighbors(const float* pos, int n_nodes, const double* cell, const int* pbc,
                         float r_cut, int max_edges, int* n_edges, int* row_ptr, int* sender,
                         float* edge_vec, int* shift, int* t_row_ptr, int* t_perm,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Canonical CSR from a given edge list in any order (receiver[e], sender[e], edge_vec_in[e]):
 * stable sort by (receiver, sender); perm[k] = input index of canonical edge k (may be NULL). */
etp_status etp_build_csr(int n_nodes, int n_edges, const int* receiver, const int* sender_in,
                         const float* edge_vec_in, int* row_ptr, int* sender, float* edge_vec,
                         int* perm, int* t_row_ptr, int* t_perm, void* workspace,
                         size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ETP_H */

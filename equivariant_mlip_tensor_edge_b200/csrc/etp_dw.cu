// Gradient of the edge convolution with respect to the radial weight matrix W:
//
//   dL/dW[b][p][u] = sum_e R_b(d_e) gw_{e,p,u},
//   gw_{e,p,u}     = sum_{m1,m3} x[send(e), l1, m1, u] (sum_m2 C[m1,m2,m3] Y_{l2 m2}(e)) g[recv(e), l3, m3, u].
//
// A reduction over all edges for every (b, p, u), so the lanes hold channels, not edges: a warp
// takes a contiguous range of canonical edges and a slice of 32 channels, walks the edges in
// order with the per-channel factors gw in registers (generated per-path code), and keeps the
// 8 x P sums of its channel in registers. The per-edge geometry (Y, R, indices) of 32 edges at a
// time is computed one edge per lane and shared through shared memory. Receiver rows of the
// cotangent change only at receiver boundaries (canonical order) and stay in registers.
// Each warp writes its partial sums; a second kernel adds the edge ranges in a fixed order, so
// the result does not depend on scheduling.
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"

namespace etp {
namespace {

constexpr int kWarpsPerBlock = 8;

// basis functions summed per sweep over the edges (registers: NB x P sums per lane)
template <int L>
struct DwCfg {
  static constexpr int D = Gen<L>::D;
  static constexpr int P = Gen<L>::P;
  static constexpr int NB = L >= 3 ? 4 : kNumBasis;
  static constexpr int SWEEPS = kNumBasis / NB;
};

#define ETP_GW_BIND(LL)                                                                            \
  template <class GS>                                                                              \
  __device__ __forceinline__ void tp_gw(IntL<LL>, const float* Y, const float (&x)[Gen<LL>::D][1], \
                                        const float (&g)[Gen<LL>::D][1], GS&& gs) {                \
    etp_gen::tp_gw_##LL<1>(Y, x, g, gs);                                                           \
  }
template <int L> struct IntL {};
ETP_GW_BIND(1)
ETP_GW_BIND(2)
ETP_GW_BIND(3)
#undef ETP_GW_BIND

// Warp task t: edge range r = t / n_slices ([r * chunk, (r + 1) * chunk) of the canonical order)
// and channel slice t % n_slices. part[r][b][p][u] = sum over the range (basis b0 .. b0 + NB - 1).
template <int L>
__global__ void __launch_bounds__(32 * kWarpsPerBlock) k_dw(int n_edges, int C, int dim, float inv_rc,
                                                              int chunk, int n_slices, int n_tasks, int b0,
                                                              const int* __restrict__ recv,
                                                              const int* __restrict__ sender,
                                                              const float* __restrict__ edge_vec,
                                                              const float* __restrict__ x,
                                                              const float* __restrict__ g,
                                                              float* __restrict__ part) {
  using G = DwCfg<L>;
  constexpr int D = G::D, P = G::P, NB = G::NB;
  __shared__ float sY[kWarpsPerBlock][32][D + 1];
  __shared__ float sR[kWarpsPerBlock][32][NB + 1];
  __shared__ int sI[kWarpsPerBlock][32];
  __shared__ int sJ[kWarpsPerBlock][32];
  const int lane = threadIdx.x & 31;
  const int wb = threadIdx.x >> 5;
  const int t = blockIdx.x * kWarpsPerBlock + wb;
  if (t >= n_tasks) return;
  const int r = t / n_slices;
  const int u = (t - r * n_slices) * 32 + lane;
  const bool cu = u < C;
  const int e_beg = r * chunk;
  const int e_end = e_beg + chunk < n_edges ? e_beg + chunk : n_edges;

  float acc[NB][P];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int p = 0; p < P; ++p) acc[b][p] = 0.0f;
  float gv[D][1];
  int cur_i = -1;

  for (int e0 = e_beg; e0 < e_end; e0 += 32) {
    // geometry of 32 edges, one per lane
    {
      const int e = e0 + lane;
      float Y[D], R[kNumBasis], dR[kNumBasis];
#pragma unroll
      for (int c = 0; c < D; ++c) Y[c] = 0.0f;
      int i = -1, j = 0;
      if (e < e_end) {
        const float vx = edge_vec[3 * e], vy = edge_vec[3 * e + 1], vz = edge_vec[3 * e + 2];
        const float dd = sqrtf(vx * vx + vy * vy + vz * vz);
        const float inv_d = dd > 0.0f ? 1.0f / dd : 0.0f;
        Gen<L>::sh(vx * inv_d, vy * inv_d, vz * inv_d, Y);
        radial_basis<false>(dd, inv_rc, R, dR);
        i = recv[e];
        j = sender[e];
      } else {
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) R[b] = 0.0f;
      }
#pragma unroll
      for (int c = 0; c < D; ++c) sY[wb][lane][c] = Y[c];
#pragma unroll
      for (int b = 0; b < NB; ++b) sR[wb][lane][b] = R[b0 + b];
      sI[wb][lane] = i;
      sJ[wb][lane] = j;
    }
    __syncwarp();
    const int n = e_end - e0 < 32 ? e_end - e0 : 32;
    // the sender row of edge k + 1 is requested before edge k's contraction (one edge ahead)
    float xn[D];
#pragma unroll
    for (int c = 0; c < D; ++c) xn[c] = cu ? __ldg(x + static_cast<size_t>(sJ[wb][0]) * dim + c * C + u) : 0.0f;
    for (int k = 0; k < n; ++k) {
      const int i = sI[wb][k];
      if (i != cur_i) {
        cur_i = i;
#pragma unroll
        for (int c = 0; c < D; ++c) gv[c][0] = cu ? __ldg(g + static_cast<size_t>(i) * dim + c * C + u) : 0.0f;
      }
      float xv[D][1];
#pragma unroll
      for (int c = 0; c < D; ++c) xv[c][0] = xn[c];
      if (k + 1 < n) {
        const int jn = sJ[wb][k + 1];
#pragma unroll
        for (int c = 0; c < D; ++c) xn[c] = cu ? __ldg(x + static_cast<size_t>(jn) * dim + c * C + u) : 0.0f;
      }
      float Y[D], R[NB];
#pragma unroll
      for (int c = 0; c < D; ++c) Y[c] = sY[wb][k][c];
#pragma unroll
      for (int b = 0; b < NB; ++b) R[b] = sR[wb][k][b];
      tp_gw(IntL<L>{}, Y, xv, gv, [&](auto pc, const float (&gw)[1]) {
        constexpr int p = decltype(pc)::value;
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b][p] = fmaf(R[b], gw[0], acc[b][p]);
      });
    }
    __syncwarp();
  }
  if (cu) {
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int p = 0; p < P; ++p) part[((static_cast<size_t>(r) * kNumBasis + b0 + b) * P + p) * C + u] = acc[b][p];
  }
}

// dW[b][p][u] = sum over edge ranges: a block per 32 outputs, warp w adds the ranges w, w + 8, ...
// in order, then warp 0 adds the 8 warp sums in order (a fixed summation tree: deterministic).
__global__ void __launch_bounds__(256) k_dw_sum(const float* __restrict__ part, int n_ranges, int n_out,
                                                float* __restrict__ dW) {
  __shared__ float ws[8][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int o = blockIdx.x * 32 + lane;
  float s = 0.0f;
  if (o < n_out)
    for (int r = w; r < n_ranges; r += 8) s += part[static_cast<size_t>(r) * n_out + o];
  ws[w][lane] = s;
  __syncthreads();
  if (w == 0 && o < n_out) {
    float t = ws[0][lane];
#pragma unroll
    for (int k = 1; k < 8; ++k) t += ws[k][lane];
    dW[o] = t;
  }
}

// Edge ranges: about 16 warps per SM in total, ranges a multiple of 32 edges.
void dw_split(const Ctx& c, int n_edges, int* n_ranges, int* chunk) {
  const int n_slices = (c.channels + 31) / 32;
  const long long want = 16LL * 148 / n_slices;   // device-independent: the partial buffer size is queried up front
  long long ch = (n_edges + want - 1) / (want > 0 ? want : 1);
  ch = (ch + 31) / 32 * 32;
  if (ch < 32) ch = 32;
  *chunk = static_cast<int>(ch);
  *n_ranges = n_edges > 0 ? static_cast<int>((n_edges + ch - 1) / ch) : 0;
}

template <int L>
etp_status dw_launch(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                     const float* edge_vec, const float* x, const float* g, float* dW, int* recv, float* part,
                     cudaStream_t s) {
  using G = DwCfg<L>;
  const int n_out = kNumBasis * G::P * c.channels;
  if (n_edges == 0) {
    cudaError_t e = cudaMemsetAsync(dW, 0, sizeof(float) * n_out, s);
    return e == cudaSuccess ? ETP_OK : cuda_status(e, "weight gradient memset");
  }
  etp_status st = launch_recv_of_edge(row_ptr, n_nodes, n_edges, recv, s);
  if (st != ETP_OK) return st;
  int n_ranges = 0, chunk = 0;
  dw_split(c, n_edges, &n_ranges, &chunk);
  const int n_slices = (c.channels + 31) / 32;
  const int n_tasks = n_ranges * n_slices;
  const int blocks = (n_tasks + kWarpsPerBlock - 1) / kWarpsPerBlock;
  for (int sw = 0; sw < G::SWEEPS; ++sw) {
    k_dw<L><<<blocks, 32 * kWarpsPerBlock, 0, s>>>(n_edges, c.channels, c.dim, 1.0f / c.r_cut, chunk, n_slices,
                                                   n_tasks, sw * G::NB, recv, sender, edge_vec, x, g, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e, "weight gradient launch");
  }
  k_dw_sum<<<(n_out + 31) / 32, 256, 0, s>>>(part, n_ranges, n_out, dW);
  return cuda_status(cudaGetLastError(), "weight gradient sum launch");
}

template <int L>
size_t dw_bytes(const Ctx& c, int n_edges) {
  int n_ranges = 0, chunk = 0;
  dw_split(c, n_edges, &n_ranges, &chunk);
  return align256(sizeof(float) * static_cast<size_t>(n_ranges > 0 ? n_ranges : 1) * kNumBasis * DwCfg<L>::P *
                  c.channels);
}

}  // namespace

size_t weight_grad_workspace_bytes(const Ctx& c, int n_edges) {
  switch (c.lmax) {
    case 1: return dw_bytes<1>(c, n_edges);
    case 2: return dw_bytes<2>(c, n_edges);
    default: return dw_bytes<3>(c, n_edges);
  }
}

etp_status launch_weight_grad(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                              const float* edge_vec, const float* x, const float* grad_out, float* grad_W,
                              int* recv, void* ws, cudaStream_t s) {
  float* part = static_cast<float*>(ws);
  switch (c.lmax) {
    case 1: return dw_launch<1>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, grad_out, grad_W, recv, part, s);
    case 2: return dw_launch<2>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, grad_out, grad_W, recv, part, s);
    case 3: return dw_launch<3>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, grad_out, grad_W, recv, part, s);
  }
  set_error("weight gradient: unsupported lmax");
  return ETP_ERR_UNSUPPORTED;
}

}  // namespace etp

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
// the result does not depend on scheduling. For l_max <= 2, k_dw_pair runs the same reduction in
// packed f32x2 arithmetic (two edges, or two basis functions, per instruction).
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

// Packed (f32x2) form for l_max <= 2, the same task split and partial sums as k_dw. The geometry
// of 32 edges is computed one edge per lane: R, and the per-edge coefficients M[m3][m1] =
// sum_m2 C Y of both path subsets (deduplicated up to sign, the set the forward uses), stored with
// the two edges of a pair interleaved. Edges are then taken in pairs: gw of both edges comes from
// one packed contraction (.x the first edge, .y the second), and the eight basis sums of a path
// are four packed basis pairs, (acc_2c, acc_2c+1) += (R_2c, R_2c+1) * (gw, gw), edge by edge.
constexpr int kPairWarps = 4;

template <int L>
struct DwPairCfg {
  using S0 = etp_gen::CxSub<L, 0>;
  using S1 = etp_gen::CxSub<L, 1>;
  static constexpr int D = Gen<L>::D;
  static constexpr int P = Gen<L>::P;
  static constexpr int CW0 = S0::NC, CW1 = S1::NC;
  static constexpr int PW = 2 * (CW0 + CW1) + (4 - (2 * (CW0 + CW1)) % 32 + 32) % 32;   // pair row, floats
  static_assert(kNumBasis == 8, "four basis pairs");
};

template <int L>
__global__ void __launch_bounds__(32 * kPairWarps) k_dw_pair(int n_edges, int C, int dim, float inv_rc, int chunk,
                                                               int n_slices, int n_tasks,
                                                               const int* __restrict__ recv,
                                                               const int* __restrict__ sender,
                                                               const float* __restrict__ edge_vec,
                                                               const float* __restrict__ x,
                                                               const float* __restrict__ g,
                                                               float* __restrict__ part) {
  using G = DwPairCfg<L>;
  using S0 = typename G::S0;
  using S1 = typename G::S1;
  constexpr int D = G::D, P = G::P, PW = G::PW;
  __shared__ __align__(16) float sC[kPairWarps][16][PW];
  __shared__ __align__(16) float sR[kPairWarps][32][kNumBasis];
  __shared__ int sI[kPairWarps][32];
  __shared__ int sJ[kPairWarps][32];
  const int lane = threadIdx.x & 31;
  const int wb = threadIdx.x >> 5;
  const int t = blockIdx.x * kPairWarps + wb;
  if (t >= n_tasks) return;
  const int r = t / n_slices;
  const int u = (t - r * n_slices) * 32 + lane;
  const bool cu = u < C;
  const int e_beg = r * chunk;
  const int e_end = e_beg + chunk < n_edges ? e_beg + chunk : n_edges;

  float2 acc[kNumBasis / 2][P];
#pragma unroll
  for (int b = 0; b < kNumBasis / 2; ++b)
#pragma unroll
    for (int p = 0; p < P; ++p) acc[b][p] = make_float2(0.0f, 0.0f);
  float2 gp[D];   // cotangent rows of the current pair's receivers (.x first edge, .y second)
  int gi0 = -1, gi1 = -1;
  // launched as a programmatic dependent of k_recv_of_edge, whose output (recv) is read below
  asm volatile("griddepcontrol.wait;" ::: "memory");
  auto node = [&](const float* a, int i, int c) { return cu ? __ldg(a + static_cast<size_t>(i) * dim + c * C + u) : 0.0f; };

  for (int e0 = e_beg; e0 < e_end; e0 += 32) {
    {
      const int e = e0 + lane;
      float Y[D], R[kNumBasis], dR[kNumBasis];
#pragma unroll
      for (int c = 0; c < D; ++c) Y[c] = 0.0f;
#pragma unroll
      for (int b = 0; b < kNumBasis; ++b) R[b] = 0.0f;
      int i = -1, j = 0;
      if (e < e_end) {
        const float vx = edge_vec[3 * e], vy = edge_vec[3 * e + 1], vz = edge_vec[3 * e + 2];
        const float dd = sqrtf(vx * vx + vy * vy + vz * vz);
        const float inv_d = dd > 0.0f ? 1.0f / dd : 0.0f;
        Gen<L>::sh(vx * inv_d, vy * inv_d, vz * inv_d, Y);
        radial_basis<false>(dd, inv_rc, R, dR);
        i = recv[e];
        j = sender[e];
      }
      float c0[G::CW0], c1[G::CW1];
      S0::coef(Y, c0);
      S1::coef(Y, c1);
      // lane 2 q + h holds edge h of pair q: one exchange per two coefficients gives the 8-byte
      // pieces (c_k of edge 0, c_k of edge 1)
      const int h = lane & 1;
      float* prow = &sC[wb][lane >> 1][2 * h];
#pragma unroll
      for (int k = 0; k < G::CW0 / 2; ++k) {
        const float got = __shfl_xor_sync(0xffffffffu, h == 0 ? c0[2 * k + 1] : c0[2 * k], 1);
        *reinterpret_cast<float2*>(prow + 4 * k) = h == 0 ? make_float2(c0[2 * k], got) : make_float2(got, c0[2 * k + 1]);
      }
#pragma unroll
      for (int k = 0; k < G::CW1 / 2; ++k) {
        const float got = __shfl_xor_sync(0xffffffffu, h == 0 ? c1[2 * k + 1] : c1[2 * k], 1);
        *reinterpret_cast<float2*>(prow + 2 * G::CW0 + 4 * k) =
            h == 0 ? make_float2(c1[2 * k], got) : make_float2(got, c1[2 * k + 1]);
      }
      *reinterpret_cast<float4*>(&sR[wb][lane][0]) = make_float4(R[0], R[1], R[2], R[3]);
      *reinterpret_cast<float4*>(&sR[wb][lane][4]) = make_float4(R[4], R[5], R[6], R[7]);
      sI[wb][lane] = i;
      sJ[wb][lane] = j;
    }
    __syncwarp();
    const int n = e_end - e0 < 32 ? e_end - e0 : 32;
    for (int k = 0; k < n; k += 2) {
      const bool two = k + 1 < n;   // a lone last edge: the second half runs with x = R = 0
      const int i0 = sI[wb][k], i1 = two ? sI[wb][k + 1] : i0;
      const int j0 = sJ[wb][k], j1 = two ? sJ[wb][k + 1] : j0;
      if (i0 != gi0 || i1 != gi1) {
        gi0 = i0;
        gi1 = i1;
#pragma unroll
        for (int c = 0; c < D; ++c) {
          const float a0 = node(g, i0, c);
          gp[c] = make_float2(a0, i1 == i0 ? a0 : node(g, i1, c));
        }
      }
      float2 xp[D];
#pragma unroll
      for (int c = 0; c < D; ++c) xp[c] = make_float2(node(x, j0, c), two ? node(x, j1, c) : 0.0f);
      float2 rA[kNumBasis / 2], rB[kNumBasis / 2];
      {
        const float4 a0 = *reinterpret_cast<const float4*>(&sR[wb][k][0]);
        const float4 a1 = *reinterpret_cast<const float4*>(&sR[wb][k][4]);
        rA[0] = make_float2(a0.x, a0.y);
        rA[1] = make_float2(a0.z, a0.w);
        rA[2] = make_float2(a1.x, a1.y);
        rA[3] = make_float2(a1.z, a1.w);
        const float4 b0 = two ? *reinterpret_cast<const float4*>(&sR[wb][k + 1][0]) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 b1 = two ? *reinterpret_cast<const float4*>(&sR[wb][k + 1][4]) : make_float4(0.f, 0.f, 0.f, 0.f);
        rB[0] = make_float2(b0.x, b0.y);
        rB[1] = make_float2(b0.z, b0.w);
        rB[2] = make_float2(b1.x, b1.y);
        rB[3] = make_float2(b1.z, b1.w);
      }
      auto sink = [&](auto pc, float2 gw) {
        constexpr int p = decltype(pc)::value;
        const float2 wa = make_float2(gw.x, gw.x), wbb = make_float2(gw.y, gw.y);
#pragma unroll
        for (int b = 0; b < kNumBasis / 2; ++b) acc[b][p] = __ffma2_rn(rA[b], wa, acc[b][p]);
#pragma unroll
        for (int b = 0; b < kNumBasis / 2; ++b) acc[b][p] = __ffma2_rn(rB[b], wbb, acc[b][p]);
      };
      {
        float2 xs[S0::NX], gs[S0::NO];
#pragma unroll
        for (int q = 0; q < S0::NX; ++q) xs[q] = xp[S0::xcomp(q)];
#pragma unroll
        for (int q = 0; q < S0::NO; ++q) gs[q] = gp[S0::ocomp(q)];
        S0::gw2(reinterpret_cast<const float4*>(&sC[wb][k >> 1][0]), xs, gs, sink);
      }
      {
        float2 xs[S1::NX], gs[S1::NO];
#pragma unroll
        for (int q = 0; q < S1::NX; ++q) xs[q] = xp[S1::xcomp(q)];
#pragma unroll
        for (int q = 0; q < S1::NO; ++q) gs[q] = gp[S1::ocomp(q)];
        S1::gw2(reinterpret_cast<const float4*>(&sC[wb][k >> 1][2 * G::CW0]), xs, gs, sink);
      }
    }
    __syncwarp();
  }
  if (cu) {
#pragma unroll
    for (int b = 0; b < kNumBasis / 2; ++b)
#pragma unroll
      for (int p = 0; p < P; ++p) {
        part[((static_cast<size_t>(r) * kNumBasis + 2 * b) * P + p) * C + u] = acc[b][p].x;
        part[((static_cast<size_t>(r) * kNumBasis + 2 * b + 1) * P + p) * C + u] = acc[b][p].y;
      }
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

// Edge ranges. k_dw: about 16 warps per SM in total, ranges a multiple of 32 edges. k_dw_pair
// (l_max <= 2): one warp task per resident warp slot (two blocks of kPairWarps per SM at its
// register count), so the whole grid runs as one wave; ranges an even number of edges. The split
// uses a fixed 148 SMs: the partial buffer size is queried before the launch, independently of
// the device.
void dw_split(const Ctx& c, int n_edges, int* n_ranges, int* chunk) {
  const int n_slices = (c.channels + 31) / 32;
  const bool pair = c.lmax <= 2;
  const long long want = (pair ? 2LL * kPairWarps : 16LL) * 148 / n_slices;
  long long ch = (n_edges + want - 1) / (want > 0 ? want : 1);
  ch = pair ? (ch + 1) / 2 * 2 : (ch + 31) / 32 * 32;
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
  if (L <= 2) {
    const int pblocks = (n_tasks + kPairWarps - 1) / kPairWarps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pblocks);
    cfg.blockDim = dim3(32 * kPairWarps);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_dw_pair<L <= 2 ? L : 2>, n_edges, c.channels, c.dim, 1.0f / c.r_cut,
                                       chunk, n_slices, n_tasks, static_cast<const int*>(recv), sender, edge_vec, x,
                                       g, part);
    if (e != cudaSuccess) return cuda_status(e, "weight gradient launch");
    k_dw_sum<<<(n_out + 31) / 32, 256, 0, s>>>(part, n_ranges, n_out, dW);
    return cuda_status(cudaGetLastError(), "weight gradient sum launch");
  }
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

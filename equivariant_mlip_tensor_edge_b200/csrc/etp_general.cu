// Edge convolution for general irreps: any multiplicity per block, both parities, rank <= 4,
// paths with l1 + l2 + l3 odd (real antisymmetric couplings) included.
//
// The path list is data (a parameter block of the kernels), the couplings are generated code,
// one forward and one backward contraction per (l1, l2, l3) with CG immediates, dispatched by a
// warp-uniform coupling index. Lanes hold channels: a path with mul channels runs its channel
// u on lane u % 32, so every node-row access of a warp is one coalesced row segment.
//
//   forward : a warp per receiver, its output row accumulated in shared memory (each element
//             belongs to one lane), edges in CSR order, paths in order: deterministic.
//   backward: a warp per sender over the transposed order; grad_x accumulated like the forward
//             output; per edge, dL/dY and dL/dR_b summed over the lanes in a fixed butterfly
//             and turned into dL/dr_e by lane 0 (chain through the harmonics' gradient and dR/dd).
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"

namespace etp {
namespace {

constexpr int kGenWarps = 4;     // warps per block, one node row each in shared memory
constexpr int kY = 25;           // harmonics up to l = 4

__device__ __forceinline__ void gen_sh(int sh_lmax, float nx, float ny, float nz, float (&Y)[kY]) {
#pragma unroll
  for (int i = 0; i < kY; ++i) Y[i] = 0.0f;
  switch (sh_lmax) {
    case 0: Y[0] = 1.0f; break;
    case 1: etp_gen::sh_eval_1(nx, ny, nz, Y); break;
    case 2: etp_gen::sh_eval_2(nx, ny, nz, Y); break;
    case 3: etp_gen::sh_eval_3(nx, ny, nz, Y); break;
    default: etp_gen::sh_eval_4(nx, ny, nz, Y); break;
  }
}

__device__ __forceinline__ void gen_sh_grad(int sh_lmax, float nx, float ny, float nz, const float (&gY)[kY],
                                            float& Gx, float& Gy, float& Gz, float& S) {
  Gx = Gy = Gz = S = 0.0f;
  switch (sh_lmax) {
    case 0: break;
    case 1: etp_gen::sh_grad_1(nx, ny, nz, gY, Gx, Gy, Gz, S); break;
    case 2: etp_gen::sh_grad_2(nx, ny, nz, gY, Gx, Gy, Gz, S); break;
    case 3: etp_gen::sh_grad_3(nx, ny, nz, gY, Gx, Gy, Gz, S); break;
    default: etp_gen::sh_grad_4(nx, ny, nz, gY, Gx, Gy, Gz, S); break;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(32 * kGenWarps) k_gen_fwd(const __grid_constant__ GenParams g, int n_nodes,
                                                            const int* __restrict__ row_ptr,
                                                            const int* __restrict__ sender,
                                                            const float* __restrict__ edge_vec,
                                                            const float* __restrict__ x,
                                                            const float* __restrict__ W,
                                                            float* __restrict__ out) {
  extern __shared__ float sacc[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* acc = sacc + wib * g.dim_out;
  const int stride = gridDim.x * kGenWarps;
  for (int i = blockIdx.x * kGenWarps + wib; i < n_nodes; i += stride) {
    for (int v = lane; v < g.dim_out; v += 32) acc[v] = 0.0f;
    __syncwarp();
    const int e1 = row_ptr[i + 1];
    for (int e = row_ptr[i]; e < e1; ++e) {
      const float vx = edge_vec[3 * e], vy = edge_vec[3 * e + 1], vz = edge_vec[3 * e + 2];
      const float d = sqrtf(vx * vx + vy * vy + vz * vz);
      const float inv_d = d > 0.0f ? 1.0f / d : 0.0f;
      float Y[kY], R[kNumBasis], dR[kNumBasis];
      gen_sh(g.sh_lmax, vx * inv_d, vy * inv_d, vz * inv_d, Y);
      radial_basis<false>(d, g.inv_rc, R, dR);
      const float* xj = x + static_cast<size_t>(sender[e]) * g.dim_in;
      for (int p = 0; p < g.n_paths; ++p) {
        const GenPath& P = g.p[p];
        for (int u = lane; u < P.mul; u += 32) {
          float w = 0.0f;
#pragma unroll
          for (int b = 0; b < kNumBasis; ++b) w = fmaf(R[b], __ldg(W + static_cast<size_t>(b) * g.cols + P.woff + u), w);
          etp_gen::gen_fwd(P.tri, xj + P.in_off + u, P.mul, Y, w, acc + P.out_off + u);
        }
      }
    }
    __syncwarp();
    float* orow = out + static_cast<size_t>(i) * g.dim_out;
    for (int v = lane; v < g.dim_out; v += 32) orow[v] = acc[v];
    __syncwarp();
  }
}

__global__ void __launch_bounds__(32 * kGenWarps) k_gen_bwd(const __grid_constant__ GenParams g, int n_nodes,
                                                            const int* __restrict__ t_row_ptr,
                                                            const int* __restrict__ t_perm,
                                                            const int* __restrict__ recv,
                                                            const float* __restrict__ edge_vec,
                                                            const float* __restrict__ x,
                                                            const float* __restrict__ W,
                                                            const float* __restrict__ gout,
                                                            float* __restrict__ grad_x,
                                                            float* __restrict__ grad_vec) {
  extern __shared__ float sgx[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* gx = sgx + wib * g.dim_in;
  const int stride = gridDim.x * kGenWarps;
  for (int j = blockIdx.x * kGenWarps + wib; j < n_nodes; j += stride) {
    for (int v = lane; v < g.dim_in; v += 32) gx[v] = 0.0f;
    __syncwarp();
    const float* xj = x + static_cast<size_t>(j) * g.dim_in;
    const int t1 = t_row_ptr[j + 1];
    for (int t = t_row_ptr[j]; t < t1; ++t) {
      const int e = t_perm[t];
      const int i = recv[e];
      const float vx = edge_vec[3 * e], vy = edge_vec[3 * e + 1], vz = edge_vec[3 * e + 2];
      const float d = sqrtf(vx * vx + vy * vy + vz * vz);
      const float inv_d = d > 0.0f ? 1.0f / d : 0.0f;
      const float nx = vx * inv_d, ny = vy * inv_d, nz = vz * inv_d;
      float Y[kY], R[kNumBasis], dR[kNumBasis];
      gen_sh(g.sh_lmax, nx, ny, nz, Y);
      radial_basis<true>(d, g.inv_rc, R, dR);
      float gY[kY], gR[kNumBasis];
#pragma unroll
      for (int k = 0; k < kY; ++k) gY[k] = 0.0f;
#pragma unroll
      for (int b = 0; b < kNumBasis; ++b) gR[b] = 0.0f;
      const float* gi = gout + static_cast<size_t>(i) * g.dim_out;
      for (int p = 0; p < g.n_paths; ++p) {
        const GenPath& P = g.p[p];
        for (int u = lane; u < P.mul; u += 32) {
          float wb[kNumBasis];
          float w = 0.0f;
#pragma unroll
          for (int b = 0; b < kNumBasis; ++b) {
            wb[b] = __ldg(W + static_cast<size_t>(b) * g.cols + P.woff + u);
            w = fmaf(R[b], wb[b], w);
          }
          float gw = 0.0f;
          etp_gen::gen_bwd(P.tri, xj + P.in_off + u, gi + P.out_off + u, P.mul, Y, w, gx + P.in_off + u, gY, gw);
#pragma unroll
          for (int b = 0; b < kNumBasis; ++b) gR[b] = fmaf(wb[b], gw, gR[b]);
        }
      }
      if (grad_vec) {
#pragma unroll
        for (int k = 0; k < kY; ++k) gY[k] = warp_sum(gY[k]);
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) gR[b] = warp_sum(gR[b]);
        if (lane == 0) {
          float gd = 0.0f;
#pragma unroll
          for (int b = 0; b < kNumBasis; ++b) gd = fmaf(gR[b], dR[b], gd);
          float Gx, Gy, Gz, S;
          gen_sh_grad(g.sh_lmax, nx, ny, nz, gY, Gx, Gy, Gz, S);
          // dL/dr = gd n + (G - S n) / d
          grad_vec[3 * e + 0] = fmaf(gd, nx, (Gx - S * nx) * inv_d);
          grad_vec[3 * e + 1] = fmaf(gd, ny, (Gy - S * ny) * inv_d);
          grad_vec[3 * e + 2] = fmaf(gd, nz, (Gz - S * nz) * inv_d);
        }
      }
    }
    __syncwarp();
    if (grad_x) {
      float* row = grad_x + static_cast<size_t>(j) * g.dim_in;
      for (int v = lane; v < g.dim_in; v += 32) row[v] = gx[v];
    }
    __syncwarp();
  }
}

int gen_blocks(int n_nodes) {
  static int n_sms = 0;
  if (n_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev);
    if (n_sms <= 0) n_sms = 148;
  }
  long long b = (static_cast<long long>(n_nodes) + kGenWarps - 1) / kGenWarps;
  const long long cap = 16LL * n_sms;
  if (b > cap) b = cap;
  return b < 1 ? 1 : static_cast<int>(b);
}

}  // namespace

etp_status launch_general_forward(const GenParams& g, int n_nodes, int n_edges, const int* row_ptr,
                                  const int* sender, const float* edge_vec, const float* x, const float* W,
                                  float* out, cudaStream_t s) {
  (void)n_edges;
  if (n_nodes == 0) return ETP_OK;
  const size_t smem = sizeof(float) * kGenWarps * static_cast<size_t>(g.dim_out);
  cudaError_t e = cudaFuncSetAttribute(k_gen_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_status(e, "general forward smem attribute");
  k_gen_fwd<<<gen_blocks(n_nodes), 32 * kGenWarps, smem, s>>>(g, n_nodes, row_ptr, sender, edge_vec, x, W, out);
  return cuda_status(cudaGetLastError(), "general forward launch");
}

etp_status launch_general_backward(const GenParams& g, int n_nodes, int n_edges, const int* row_ptr,
                                   const float* edge_vec, const int* t_row_ptr, const int* t_perm,
                                   const float* x, const float* W, const float* grad_out, float* grad_x,
                                   float* grad_edge_vec, int* recv, cudaStream_t s) {
  if (n_nodes == 0) return ETP_OK;
  if (n_edges > 0) {
    etp_status st = launch_recv_of_edge(row_ptr, n_nodes, n_edges, recv, s);
    if (st != ETP_OK) return st;
  }
  const size_t smem = sizeof(float) * kGenWarps * static_cast<size_t>(g.dim_in);
  cudaError_t e = cudaFuncSetAttribute(k_gen_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_status(e, "general backward smem attribute");
  k_gen_bwd<<<gen_blocks(n_nodes), 32 * kGenWarps, smem, s>>>(g, n_nodes, t_row_ptr, t_perm, recv, edge_vec, x, W,
                                                               grad_out, grad_x, grad_edge_vec);
  return cuda_status(cudaGetLastError(), "general backward launch");
}

}  // namespace etp

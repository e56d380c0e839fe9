// Edge convolution for general irreps: any multiplicity per block, both parities, rank <= 4,
// paths with l1 + l2 + l3 odd (real antisymmetric couplings) included.
//
// The path list is data (a parameter block of the kernels), the couplings are generated code,
// one forward and one backward contraction per (l1, l2, l3) with CG immediates, dispatched by a
// warp-uniform coupling index. Lanes hold channels: a path with mul channels runs its channel
// u on lane u % 32, so every node-row access of a warp is one coalesced row segment.
//
//   forward : a warp per (receiver, output block): the block's row segment accumulated in shared
//             memory (each element belongs to one lane). The geometry of 32 edges at a time
//             (harmonics, radial basis) is computed one edge per lane and staged in shared memory;
//             then, path by path, each lane runs its channel over the 32 edges with the path's W
//             column and sums in registers. Fixed order (chunks, paths, edges): deterministic.
//   backward: a warp per (sender, input block) over the transposed order; grad_x accumulated like
//             the forward output; per edge, dL/dY and dL/dR_b summed over the lanes by a fixed
//             scatter-reduction, and once per 32 edges lane k turns edge k's sums into the block's
//             share of dL/dr_e (chain through the harmonics' gradient and dR/dd); the shares are
//             added over the blocks in order.
//   dL/dW   : a warp per (range of 128 edges, output block): per path and channel, the sum over
//             the range of R_b gw; the ranges' partial columns are added in order.
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

// Per-edge geometry staged in shared memory, one edge per lane, read back by every lane.
constexpr int kGeoF = etp_gen::kGenGeoF;                   // forward: Y, R (odd stride: no bank conflicts)
static_assert(kGeoF == kY + kNumBasis, "staged forward geometry");
constexpr int kRun = 32;                                   // forward: edges per path-major run (the whole chunk)
constexpr int kGeoB = kY + 2 * kNumBasis + 4;              // backward: Y, R, dR, n, 1/d

__device__ __forceinline__ void edge_geometry(const float* __restrict__ edge_vec, int e, int sh_lmax, float inv_rc,
                                              float (&Y)[kY], float (&R)[kNumBasis], float (&dR)[kNumBasis],
                                              float (&n)[3], float& inv_d, bool deriv) {
  const float vx = edge_vec[3 * e], vy = edge_vec[3 * e + 1], vz = edge_vec[3 * e + 2];
  const float d = sqrtf(vx * vx + vy * vy + vz * vz);
  inv_d = d > 0.0f ? 1.0f / d : 0.0f;
  n[0] = vx * inv_d;
  n[1] = vy * inv_d;
  n[2] = vz * inv_d;
  gen_sh(sh_lmax, n[0], n[1], n[2], Y);
  if (deriv) radial_basis<true>(d, inv_rc, R, dR);
  else radial_basis<false>(d, inv_rc, R, dR);
}

// Work unit: (receiver i, output block q). The warp sums, over i's edges and the paths into q,
// the block's row segment in shared memory (element (m3, u) belongs to lane u % 32).
__global__ void __launch_bounds__(32 * kGenWarps) k_gen_fwd(const __grid_constant__ GenParams g, int n_nodes,
                                                            const int* __restrict__ row_ptr,
                                                            const int* __restrict__ sender,
                                                            const float* __restrict__ edge_vec,
                                                            const float* __restrict__ x,
                                                            const float* __restrict__ W,
                                                            const uint32_t* __restrict__ mask,
                                                            float* __restrict__ out) {
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* acc = smem + wib * (g.max_out_size + 32 * kGeoF + 64);
  float* geo = acc + g.max_out_size;
  int* sj = reinterpret_cast<int*>(geo + 32 * kGeoF);
  unsigned* sm = reinterpret_cast<unsigned*>(sj + 32);
  const int n_items = n_nodes * g.n_out_groups;
  const int stride = gridDim.x * kGenWarps;
  for (int it = blockIdx.x * kGenWarps + wib; it < n_items; it += stride) {
    const int i = it / g.n_out_groups;
    const GenGroup& G = g.out_grp[it - i * g.n_out_groups];
    for (int v = lane; v < G.size; v += 32) acc[v] = 0.0f;
    const int e1 = row_ptr[i + 1];
    for (int c0 = row_ptr[i]; c0 < e1; c0 += 32) {
      __syncwarp();   // the previous chunk's geometry has been read
      if (c0 + lane < e1) {
        float Y[kY], R[kNumBasis], dR[kNumBasis], nv[3], inv_d;
        edge_geometry(edge_vec, c0 + lane, g.sh_lmax, g.inv_rc, Y, R, dR, nv, inv_d, false);
#pragma unroll
        for (int c = 0; c < kY; ++c) geo[lane * kGeoF + c] = Y[c];
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) geo[lane * kGeoF + kY + b] = R[b];
        sj[lane] = sender[c0 + lane];
        if (mask) sm[lane] = mask[c0 + lane];
      }
      __syncwarp();
      const int cnt = e1 - c0 < 32 ? e1 - c0 : 32;
      // path-major over runs of kRun edges: the channel's W column and path sums stay in
      // registers, and the run's sender rows stay in L1 across the paths
      for (int r0 = 0; r0 < cnt; r0 += kRun) {
        const int rc = cnt - r0 < kRun ? cnt - r0 : kRun;
        for (int pi = G.beg; pi < G.end; ++pi) {
          const GenPath& P = g.p[g.order_out[pi]];
          for (int u = lane; u < P.mul; u += 32) {
            float wb[kNumBasis];
#pragma unroll
            for (int b = 0; b < kNumBasis; ++b) wb[b] = __ldg(W + static_cast<size_t>(b) * g.cols + P.woff + u);
            etp_gen::gen_fwd_chunk(P.tri, geo + r0 * kGeoF, sj + r0, rc, x + P.in_off + u, g.dim_in, P.mul, wb,
                                   acc + (P.out_off - G.off) + u, mask ? sm + r0 : nullptr,
                                   1u << (g.order_out[pi] & 31));
          }
        }
      }
    }
    __syncwarp();
    float* orow = out + static_cast<size_t>(i) * g.dim_out + G.off;
    for (int v = lane; v < G.size; v += 32) orow[v] = acc[v];
  }
}

// Sum of v[k] over the warp for k = 0..31, scattered: lane L returns the sum of v[L]. Recursive
// halving (16 + 8 + 4 + 2 + 1 shuffles), a fixed order.
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float send = up ? v[k] : v[k + o];
      const float keep = up ? v[k + o] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

constexpr int kRed = 33;   // per-edge reduced values: dL/dY (up to 25) and dL/dR (8), padded row

// Work unit: (sender j, input block q) over the transposed order. grad_x of the block's row
// segment as in the forward. Per edge the lanes'
// dL/dY and dL/dR_b are summed by one scatter-reduction into a shared row; once per 32 edges,
// lane k turns edge k's row into the group's share of dL/dr_e (chain through the harmonics'
// gradient and dR/dd) at vec_out + 3 e: grad_edge_vec itself when there is one group, else the
// group's partial array, summed over the groups in order afterwards.
__global__ void __launch_bounds__(32 * kGenWarps, 3) k_gen_bwd(const __grid_constant__ GenParams g, int n_nodes,
                                                            int n_edges,
                                                            const int* __restrict__ t_row_ptr,
                                                            const int* __restrict__ t_perm,
                                                            const int* __restrict__ recv,
                                                            const float* __restrict__ edge_vec,
                                                            const float* __restrict__ x,
                                                            const float* __restrict__ W,
                                                            const float* __restrict__ gout,
                                                            const uint32_t* __restrict__ mask,
                                                            float* __restrict__ grad_x,
                                                            float* __restrict__ vec_out) {
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* gx = smem + wib * (g.max_in_size + 32 * kGeoB + 32 * kRed + 96);
  float* geo = gx + g.max_in_size;
  float* red = geo + 32 * kGeoB;
  int* si = reinterpret_cast<int*>(red + 32 * kRed);
  int* se = si + 32;
  unsigned* sm = reinterpret_cast<unsigned*>(se + 32);
  const bool wide = g.sh_lmax > 3;   // 25 + 8 values: one more than the scatter-reduction holds
  const int n_items = n_nodes * g.n_in_groups;
  const int stride = gridDim.x * kGenWarps;
  for (int it = blockIdx.x * kGenWarps + wib; it < n_items; it += stride) {
    const int j = it / g.n_in_groups;
    const int q = it - j * g.n_in_groups;
    const GenGroup& G = g.in_grp[q];
    float* vq = vec_out ? vec_out + (g.n_in_groups > 1 ? static_cast<size_t>(q) * 3 * n_edges : 0) : nullptr;
    for (int v = lane; v < G.size; v += 32) gx[v] = 0.0f;
    const float* xj = x + static_cast<size_t>(j) * g.dim_in;
    const int t1 = t_row_ptr[j + 1];
    for (int c0 = t_row_ptr[j]; c0 < t1; c0 += 32) {
      __syncwarp();
      if (c0 + lane < t1) {
        const int e = t_perm[c0 + lane];
        float Y[kY], R[kNumBasis], dR[kNumBasis], nv[3], inv_d;
        edge_geometry(edge_vec, e, g.sh_lmax, g.inv_rc, Y, R, dR, nv, inv_d, true);
        float* o = geo + lane * kGeoB;
#pragma unroll
        for (int c = 0; c < kY; ++c) o[c] = Y[c];
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) {
          o[kY + b] = R[b];
          o[kY + kNumBasis + b] = dR[b];
        }
        o[kY + 2 * kNumBasis + 0] = nv[0];
        o[kY + 2 * kNumBasis + 1] = nv[1];
        o[kY + 2 * kNumBasis + 2] = nv[2];
        o[kY + 2 * kNumBasis + 3] = inv_d;
        si[lane] = recv[e];
        se[lane] = e;
        sm[lane] = mask ? mask[e] : ~0u;
      }
      __syncwarp();
      const int cnt = t1 - c0 < 32 ? t1 - c0 : 32;
      for (int k = 0; k < cnt; ++k) {
        const float* o = geo + k * kGeoB;
        const float* Y = o;   // harmonics of edge k, read where the coupling uses them
        float R[kNumBasis];
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) R[b] = o[kY + b];
        float gY[kY], gR[kNumBasis];
#pragma unroll
        for (int c = 0; c < kY; ++c) gY[c] = 0.0f;
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) gR[b] = 0.0f;
        const float* gi = gout + static_cast<size_t>(si[k]) * g.dim_out;
        for (int pi = G.beg; pi < G.end; ++pi) {
          if (!(sm[k] & (1u << (g.order_in[pi] & 31)))) continue;   // path off for this edge
          const GenPath& P = g.p[g.order_in[pi]];
          for (int u = lane; u < P.mul; u += 32) {
            float wb[kNumBasis];
            float w = 0.0f;
#pragma unroll
            for (int b = 0; b < kNumBasis; ++b) {
              wb[b] = __ldg(W + static_cast<size_t>(b) * g.cols + P.woff + u);
              w = fmaf(R[b], wb[b], w);
            }
            float gw = 0.0f;
            etp_gen::gen_bwd(P.tri, xj + P.in_off + u, gi + P.out_off + u, P.mul, Y, w, gx + (P.in_off - G.off) + u,
                             gY, gw);
#pragma unroll
            for (int b = 0; b < kNumBasis; ++b) gR[b] = fmaf(wb[b], gw, gR[b]);
          }
        }
        if (vq) {
          // row layout: harmonics to l = 3 -> [gY 0..15][gR 0..7]; to l = 4 -> [gY 0..24][gR 0..7]
          float v[32];
          if (!wide) {
#pragma unroll
            for (int c = 0; c < 16; ++c) v[c] = gY[c];
#pragma unroll
            for (int b = 0; b < kNumBasis; ++b) v[16 + b] = gR[b];
#pragma unroll
            for (int c = 24; c < 32; ++c) v[c] = 0.0f;
          } else {
#pragma unroll
            for (int c = 0; c < kY; ++c) v[c] = gY[c];
#pragma unroll
            for (int b = 0; b < 7; ++b) v[kY + b] = gR[b];
          }
          const float r = reduce_scatter32(v, lane);
          red[k * kRed + lane] = r;
          if (wide) {
            const float r7 = warp_sum(gR[7]);
            if (lane == 0) red[k * kRed + 32] = r7;
          }
        }
      }
      if (vq) {
        __syncwarp();
        if (lane < cnt) {
          const float* rr = red + lane * kRed;
          const float* o = geo + lane * kGeoB;
          float gY[kY], gR[kNumBasis];
          if (!wide) {
#pragma unroll
            for (int c = 0; c < kY; ++c) gY[c] = c < 16 ? rr[c] : 0.0f;
#pragma unroll
            for (int b = 0; b < kNumBasis; ++b) gR[b] = rr[16 + b];
          } else {
#pragma unroll
            for (int c = 0; c < kY; ++c) gY[c] = rr[c];
#pragma unroll
            for (int b = 0; b < kNumBasis; ++b) gR[b] = rr[kY + b];
          }
          float gd = 0.0f;
#pragma unroll
          for (int b = 0; b < kNumBasis; ++b) gd = fmaf(gR[b], o[kY + kNumBasis + b], gd);
          const float nx = o[kY + 2 * kNumBasis], ny = o[kY + 2 * kNumBasis + 1], nz = o[kY + 2 * kNumBasis + 2];
          const float inv_d = o[kY + 2 * kNumBasis + 3];
          float Gx, Gy, Gz, S;
          gen_sh_grad(g.sh_lmax, nx, ny, nz, gY, Gx, Gy, Gz, S);
          // dL/dr = gd n + (G - S n) / d
          const int e = se[lane];
          vq[3 * e + 0] = fmaf(gd, nx, (Gx - S * nx) * inv_d);
          vq[3 * e + 1] = fmaf(gd, ny, (Gy - S * ny) * inv_d);
          vq[3 * e + 2] = fmaf(gd, nz, (Gz - S * nz) * inv_d);
        }
      }
    }
    __syncwarp();
    if (grad_x) {
      float* row = grad_x + static_cast<size_t>(j) * g.dim_in + G.off;
      for (int v = lane; v < G.size; v += 32) row[v] = gx[v];
    }
  }
}

// dL/dW for general irreps: work unit (canonical edge range r of kDwRange edges, output block q).
// The range's geometry (harmonics, radial basis, sender, receiver) is staged once; then path by
// path each lane runs its channel u over the range (gdwc_t: gw = g . sum C Y x per edge, and
// sum_e R_b gw for the 8 basis functions) and writes its column of the range's partial sums,
// part[r][b][column]. k_gen_dw_sum adds the ranges in a fixed order.
constexpr int kDwRange = 128;

__global__ void __launch_bounds__(32 * kGenWarps) k_gen_dw(const __grid_constant__ GenParams g, int n_edges,
                                                           int n_ranges, const int* __restrict__ recv,
                                                           const int* __restrict__ sender,
                                                           const float* __restrict__ edge_vec,
                                                           const float* __restrict__ x,
                                                           const float* __restrict__ gout,
                                                           float* __restrict__ part) {
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* geo = smem + wib * (kDwRange * kGeoF + 2 * kDwRange);
  int* sj = reinterpret_cast<int*>(geo + kDwRange * kGeoF);
  int* si = sj + kDwRange;
  const int n_items = n_ranges * g.n_out_groups;
  const int stride = gridDim.x * kGenWarps;
  for (int it = blockIdx.x * kGenWarps + wib; it < n_items; it += stride) {
    const int r = it / g.n_out_groups;
    const GenGroup& G = g.out_grp[it - r * g.n_out_groups];
    const int e0 = r * kDwRange;
    const int cnt = n_edges - e0 < kDwRange ? n_edges - e0 : kDwRange;
    __syncwarp();   // the previous unit's staged rows have been read
    for (int k = lane; k < cnt; k += 32) {
      float Y[kY], R[kNumBasis], dR[kNumBasis], nv[3], inv_d;
      edge_geometry(edge_vec, e0 + k, g.sh_lmax, g.inv_rc, Y, R, dR, nv, inv_d, false);
#pragma unroll
      for (int c = 0; c < kY; ++c) geo[k * kGeoF + c] = Y[c];
#pragma unroll
      for (int b = 0; b < kNumBasis; ++b) geo[k * kGeoF + kY + b] = R[b];
      sj[k] = sender[e0 + k];
      si[k] = recv[e0 + k];
    }
    __syncwarp();
    float* pr = part + static_cast<size_t>(r) * kNumBasis * g.cols;
    for (int pi = G.beg; pi < G.end; ++pi) {
      const GenPath& P = g.p[g.order_out[pi]];
      for (int u = lane; u < P.mul; u += 32) {
        float acc8[kNumBasis];
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) acc8[b] = 0.0f;
        etp_gen::gen_dw_chunk(P.tri, geo, sj, si, cnt, x + P.in_off + u, gout + P.out_off + u, g.dim_in, g.dim_out,
                              P.mul, acc8);
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) pr[static_cast<size_t>(b) * g.cols + P.woff + u] = acc8[b];
      }
    }
  }
}

// dW[o] = sum over ranges of part[r][o]: a block per 32 outputs, warp w adds the ranges w, w + 8,
// ... in order, then warp 0 adds the 8 warp sums in order.
__global__ void __launch_bounds__(256) k_gen_dw_sum(const float* __restrict__ part, int n_ranges, int n_out,
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

// grad_edge_vec = sum of the input blocks' partials, in block order.
__global__ void k_gen_sum_parts(const float* __restrict__ part, int n_groups, int n, float* __restrict__ out) {
  for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < n; v += gridDim.x * blockDim.x) {
    float s = part[v];
    for (int q = 1; q < n_groups; ++q) s += part[static_cast<size_t>(q) * n + v];
    out[v] = s;
  }
}

// Input blocks that no path reads get zero grad_x rows.
__global__ void k_gen_zero_unread(const __grid_constant__ GenParams g, int n_nodes, float* __restrict__ grad_x) {
  const long long total = static_cast<long long>(n_nodes) * g.dim_in;
  for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < total;
       v += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(v % g.dim_in);
    bool read = false;
    for (int q = 0; q < g.n_in_groups; ++q) read |= c >= g.in_grp[q].off && c < g.in_grp[q].off + g.in_grp[q].size;
    if (!read) grad_x[v] = 0.0f;
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

size_t general_backward_partials_bytes(const GenParams& g, int n_edges) {
  return g.n_in_groups > 1 ? align256(sizeof(float) * 3 * static_cast<size_t>(n_edges) * g.n_in_groups) : 0;
}

size_t general_weight_grad_bytes(const GenParams& g, int n_edges) {
  const long long n_ranges = (static_cast<long long>(n_edges) + kDwRange - 1) / kDwRange;
  return align256(sizeof(float) * static_cast<size_t>(n_ranges > 0 ? n_ranges : 1) * kNumBasis * g.cols);
}

etp_status launch_general_weight_grad(const GenParams& g, int n_nodes, int n_edges, const int* row_ptr,
                                      const int* sender, const float* edge_vec, const float* x,
                                      const float* grad_out, float* grad_W, int* recv, float* part,
                                      cudaStream_t s) {
  const int n_out = kNumBasis * g.cols;
  if (n_edges == 0) {
    cudaError_t e = cudaMemsetAsync(grad_W, 0, sizeof(float) * n_out, s);
    return e == cudaSuccess ? ETP_OK : cuda_status(e, "general weight gradient memset");
  }
  etp_status st = launch_recv_of_edge(row_ptr, n_nodes, n_edges, recv, s);
  if (st != ETP_OK) return st;
  const int n_ranges = (n_edges + kDwRange - 1) / kDwRange;
  const size_t smem = sizeof(float) * kGenWarps * static_cast<size_t>(kDwRange * kGeoF + 2 * kDwRange);
  cudaError_t e = cudaFuncSetAttribute(k_gen_dw, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_status(e, "general weight gradient smem attribute");
  k_gen_dw<<<gen_blocks(n_ranges * g.n_out_groups), 32 * kGenWarps, smem, s>>>(g, n_edges, n_ranges, recv, sender,
                                                                                edge_vec, x, grad_out, part);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "general weight gradient launch");
  k_gen_dw_sum<<<(n_out + 31) / 32, 256, 0, s>>>(part, n_ranges, n_out, grad_W);
  return cuda_status(cudaGetLastError(), "general weight gradient sum launch");
}

etp_status launch_general_forward(const GenParams& g, int n_nodes, int n_edges, const int* row_ptr,
                                  const int* sender, const float* edge_vec, const float* x, const float* W,
                                  float* out, cudaStream_t s, int* err, const uint32_t* path_mask) {
  (void)n_edges;
  if (n_nodes == 0) return ETP_OK;
  if (general_tc_selected(g, path_mask))
    return launch_general_forward_tc(g, n_nodes, row_ptr, sender, edge_vec, x, W, out, s, err);
  int covered = 0;
  for (int q = 0; q < g.n_out_groups; ++q) covered += g.out_grp[q].size;
  if (covered < g.dim_out) {
    // output blocks that no path writes are zero
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * static_cast<size_t>(n_nodes) * g.dim_out, s);
    if (e != cudaSuccess) return cuda_status(e, "general forward memset");
  }
  const size_t smem = sizeof(float) * kGenWarps * static_cast<size_t>(g.max_out_size + 32 * kGeoF + 64);
  cudaError_t e = cudaFuncSetAttribute(k_gen_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_status(e, "general forward smem attribute");
  k_gen_fwd<<<gen_blocks(n_nodes * g.n_out_groups), 32 * kGenWarps, smem, s>>>(g, n_nodes, row_ptr, sender, edge_vec,
                                                                                x, W, path_mask, out);
  return cuda_status(cudaGetLastError(), "general forward launch");
}

etp_status launch_general_backward(const GenParams& g, int n_nodes, int n_edges, const int* row_ptr,
                                   const float* edge_vec, const int* t_row_ptr, const int* t_perm,
                                   const float* x, const float* W, const float* grad_out, float* grad_x,
                                   float* grad_edge_vec, int* recv, float* part, cudaStream_t s,
                                   const uint32_t* path_mask) {
  if (n_nodes == 0) return ETP_OK;
  if (n_edges > 0) {
    etp_status st = launch_recv_of_edge(row_ptr, n_nodes, n_edges, recv, s);
    if (st != ETP_OK) return st;
  }
  int covered = 0;
  for (int q = 0; q < g.n_in_groups; ++q) covered += g.in_grp[q].size;
  if (grad_x && covered < g.dim_in) {
    k_gen_zero_unread<<<gen_blocks(n_nodes), 256, 0, s>>>(g, n_nodes, grad_x);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e, "general backward zero launch");
  }
  const bool split = grad_edge_vec && g.n_in_groups > 1 && n_edges > 0;
  float* vec_out = split ? part : grad_edge_vec;
  const size_t smem = sizeof(float) * kGenWarps * static_cast<size_t>(g.max_in_size + 32 * kGeoB + 32 * kRed + 96);
  cudaError_t e = cudaFuncSetAttribute(k_gen_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_status(e, "general backward smem attribute");
  k_gen_bwd<<<gen_blocks(n_nodes * g.n_in_groups), 32 * kGenWarps, smem, s>>>(g, n_nodes, n_edges, t_row_ptr, t_perm,
                                                                               recv, edge_vec, x, W, grad_out, path_mask,
                                                                               grad_x, vec_out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "general backward launch");
  if (split) {
    k_gen_sum_parts<<<gen_blocks(3 * n_edges), 256, 0, s>>>(part, g.n_in_groups, 3 * n_edges, grad_edge_vec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e, "general backward sum launch");
  }
  return ETP_OK;
}

}  // namespace etp

// Fused edge tensor-product convolution kernels (forward, backward) and small helpers.
//
// Work decomposition ("edge-major"): every warp owns a contiguous range of whole receivers
// (forward) or senders (backward) of the CSR order, split so that warps get about the same
// number of edges. A warp walks its range 32 edges at a time, one edge per lane. Each lane
// evaluates its edge's harmonics, radial basis and radial weights, and contracts the gathered
// sender row with the unrolled per-path Clebsch-Gordan code, four channels (one float4 per
// component) at a time. The per-receiver sum is a segmented shuffle reduction across the
// lanes of the same receiver; segment heads store (first piece of a row) or add (later
// pieces) into the output row, which only the owning warp ever touches: no atomics, fixed
// summation order, bitwise reproducible.
#include <cstdio>

#include "etp_internal.h"
#include "etp_device.h"

namespace etp {
namespace {

// Sorted-array searches on the CSR pointers.
__device__ __forceinline__ int lower_bound_ptr(const int* __restrict__ ptr, int n, long long v) {
  int lo = 0, hi = n;   // first index in [0, n) with ptr[idx] >= v, or n
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<long long>(ptr[mid]) < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Rows [r_lo, r_hi) of warp gw out of nw, splitting the edges evenly at row boundaries.
__device__ __forceinline__ void warp_rows(const int* __restrict__ ptr, int n_rows, int n_edges, int gw,
                                          int nw, int* r_lo, int* r_hi) {
  const long long e = n_edges;
  *r_lo = lower_bound_ptr(ptr, n_rows + 1, e * gw / nw);
  *r_hi = (gw == nw - 1) ? n_rows : lower_bound_ptr(ptr, n_rows + 1, e * (gw + 1) / nw);
  if (*r_lo > n_rows) *r_lo = n_rows;
  if (*r_hi > n_rows) *r_hi = n_rows;
}

__device__ __forceinline__ void zero_empty_rows(const int* __restrict__ ptr, int r_lo, int r_hi, int dim,
                                                float* __restrict__ dst, int lane) {
  for (int r = r_lo; r < r_hi; ++r) {
    if (ptr[r] == ptr[r + 1]) {
      float4* row = reinterpret_cast<float4*>(dst + static_cast<size_t>(r) * dim);
      for (int q = lane; q < dim / 4; q += 32) row[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// Segment masks: bit s set when lane + 2^s belongs to the same segment (same key, valid).
__device__ __forceinline__ unsigned segment_merge_mask(int key, bool valid, int lane) {
  unsigned m = 0;
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int off = 1 << s;
    const int other = __shfl_down_sync(kFull, key, off);
    if (valid && lane + off < 32 && other == key) m |= 1u << s;
  }
  return m;
}

template <int D, int K>
__device__ __forceinline__ void segmented_reduce(float (&v)[D][K], unsigned merge) {
#pragma unroll
  for (int c = 0; c < D; ++c) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      float a = v[c][k];
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const float t = __shfl_down_sync(kFull, a, 1 << s);
        if ((merge >> s) & 1u) a += t;
      }
      v[c][k] = a;
    }
  }
}

// ---------------------------------------------------------------- forward

template <int L>
__global__ void __launch_bounds__(128) k_conv_fwd(int n_nodes, int n_edges, int C, float inv_rc,
                                                  const int* __restrict__ row_ptr,
                                                  const int* __restrict__ sender,
                                                  const float* __restrict__ edge_vec,
                                                  const float* __restrict__ x,
                                                  const float* __restrict__ W,
                                                  float* __restrict__ out) {
  using G = Gen<L>;
  constexpr int D = G::D, P = G::P, K = kBatch;
  extern __shared__ float4 smem4[];
  float* Ws = reinterpret_cast<float*>(smem4);
  const int wn = kNumBasis * P * C;
  for (int i = threadIdx.x; i < wn / 4; i += blockDim.x)
    smem4[i] = __ldg(reinterpret_cast<const float4*>(W) + i);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int dim = C * D;
  int r_lo, r_hi;
  warp_rows(row_ptr, n_nodes, n_edges, gw, nw, &r_lo, &r_hi);
  zero_empty_rows(row_ptr, r_lo, r_hi, dim, out, lane);
  if (r_lo >= r_hi) return;
  const int e_beg = row_ptr[r_lo], e_end = row_ptr[r_hi];

  for (int e0 = e_beg; e0 < e_end; e0 += 32) {
    const int e = e0 + lane;
    const bool valid = e < e_end;
    int rr = -1;
    if (valid) {  // last row r in [r_lo, r_hi) with row_ptr[r] <= e
      int lo = r_lo, hi = r_hi - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
      }
      rr = lo;
    }
    const int rr_up = __shfl_up_sync(kFull, rr, 1);
    const bool head = valid && (lane == 0 || rr_up != rr);
    const bool row_start = valid && e == row_ptr[rr];
    const unsigned merge = segment_merge_mask(rr, valid, lane);

    float Y[D];
    float R[kNumBasis], dRunused[kNumBasis];
    int j = 0;
#pragma unroll
    for (int c = 0; c < D; ++c) Y[c] = 0.0f;
    if (valid) {
      const float vx = edge_vec[3 * e + 0], vy = edge_vec[3 * e + 1], vz = edge_vec[3 * e + 2];
      j = sender[e];
      const float d = sqrtf(vx * vx + vy * vy + vz * vz);
      const float inv_d = d > 0.0f ? 1.0f / d : 0.0f;
      G::sh(vx * inv_d, vy * inv_d, vz * inv_d, Y);
      radial_basis<false>(d, inv_rc, R, dRunused);
    } else {
#pragma unroll
      for (int b = 0; b < kNumBasis; ++b) R[b] = 0.0f;
    }
    const float* xrow = x + static_cast<size_t>(j) * dim;
    float* orow = out + static_cast<size_t>(rr < 0 ? 0 : rr) * dim;

    for (int cb = 0; cb < C; cb += K) {
      float xv[D][K];
#pragma unroll
      for (int c = 0; c < D; ++c) {
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) t = __ldg(reinterpret_cast<const float4*>(xrow + c * C + cb));
        xv[c][0] = t.x; xv[c][1] = t.y; xv[c][2] = t.z; xv[c][3] = t.w;
      }
      float acc[D][K];
#pragma unroll
      for (int c = 0; c < D; ++c)
#pragma unroll
        for (int k = 0; k < K; ++k) acc[c][k] = 0.0f;
      auto wf = [&](int p, float (&wp)[K]) {
        const float* wcol = Ws + p * C + cb;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) {
          const float4 wb = *reinterpret_cast<const float4*>(wcol + b * P * C);
          a.x = fmaf(R[b], wb.x, a.x);
          a.y = fmaf(R[b], wb.y, a.y);
          a.z = fmaf(R[b], wb.z, a.z);
          a.w = fmaf(R[b], wb.w, a.w);
        }
        wp[0] = a.x; wp[1] = a.y; wp[2] = a.z; wp[3] = a.w;
      };
      G::template fwd<K>(Y, wf, xv, acc);
      segmented_reduce<D, K>(acc, merge);
      if (head) {
#pragma unroll
        for (int c = 0; c < D; ++c) {
          float4* op = reinterpret_cast<float4*>(orow + c * C + cb);
          float4 o = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
          if (!row_start) {
            const float4 old = *op;
            o.x += old.x; o.y += old.y; o.z += old.z; o.w += old.w;
          }
          *op = o;
        }
      }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------- backward

__global__ void k_recv_map(const int* __restrict__ row_ptr, int n_nodes, int* __restrict__ recv_map) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < n_nodes; r += gridDim.x * blockDim.x) {
    const int a = row_ptr[r], b = row_ptr[r + 1];
    for (int e = a; e < b; ++e) recv_map[e] = r;
  }
}

template <int L, bool kGX, bool kGE>
__global__ void __launch_bounds__(128) k_conv_bwd(int n_nodes, int n_edges, int C, float inv_rc,
                                                  const int* __restrict__ sender,
                                                  const float* __restrict__ edge_vec,
                                                  const int* __restrict__ t_row_ptr,
                                                  const int* __restrict__ t_perm,
                                                  const int* __restrict__ recv_map,
                                                  const float* __restrict__ x,
                                                  const float* __restrict__ W,
                                                  const float* __restrict__ g,
                                                  float* __restrict__ grad_x,
                                                  float* __restrict__ grad_vec) {
  using G = Gen<L>;
  constexpr int D = G::D, P = G::P, K = kBatch;
  extern __shared__ float4 smem4[];
  float* Ws = reinterpret_cast<float*>(smem4);
  const int wn = kNumBasis * P * C;
  for (int i = threadIdx.x; i < wn / 4; i += blockDim.x)
    smem4[i] = __ldg(reinterpret_cast<const float4*>(W) + i);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int dim = C * D;
  int s_lo, s_hi;
  warp_rows(t_row_ptr, n_nodes, n_edges, gw, nw, &s_lo, &s_hi);
  if (kGX) zero_empty_rows(t_row_ptr, s_lo, s_hi, dim, grad_x, lane);
  if (s_lo >= s_hi) return;
  const int k_beg = t_row_ptr[s_lo], k_end = t_row_ptr[s_hi];

  for (int k0 = k_beg; k0 < k_end; k0 += 32) {
    const int kk = k0 + lane;
    const bool valid = kk < k_end;
    int e = 0, ss = -1, rr = 0;
    if (valid) {
      e = t_perm[kk];
      ss = sender[e];
      rr = recv_map[e];
    }
    const int ss_up = __shfl_up_sync(kFull, ss, 1);
    const bool head = valid && (lane == 0 || ss_up != ss);
    const bool row_start = valid && kk == t_row_ptr[ss];
    const unsigned merge = segment_merge_mask(ss, valid, lane);

    float Y[D], gY[D];
    float R[kNumBasis], dR[kNumBasis];
    float nx = 0.f, ny = 0.f, nz = 0.f, inv_d = 0.f;
#pragma unroll
    for (int c = 0; c < D; ++c) {
      Y[c] = 0.0f;
      gY[c] = 0.0f;
    }
    if (valid) {
      const float vx = edge_vec[3 * e + 0], vy = edge_vec[3 * e + 1], vz = edge_vec[3 * e + 2];
      const float d = sqrtf(vx * vx + vy * vy + vz * vz);
      inv_d = d > 0.0f ? 1.0f / d : 0.0f;
      nx = vx * inv_d;
      ny = vy * inv_d;
      nz = vz * inv_d;
      G::sh(nx, ny, nz, Y);
      radial_basis<true>(d, inv_rc, R, dR);
    } else {
#pragma unroll
      for (int b = 0; b < kNumBasis; ++b) {
        R[b] = 0.0f;
        dR[b] = 0.0f;
      }
    }
    float accd = 0.0f;
    const float* xrow = x + static_cast<size_t>(ss < 0 ? 0 : ss) * dim;
    const float* grow = g + static_cast<size_t>(rr) * dim;
    float* gxrow = kGX ? grad_x + static_cast<size_t>(ss < 0 ? 0 : ss) * dim : nullptr;

    for (int cb = 0; cb < C; cb += K) {
      float xv[D][K], gv[D][K], gx[D][K];
#pragma unroll
      for (int c = 0; c < D; ++c) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (valid) {
          a = __ldg(reinterpret_cast<const float4*>(xrow + c * C + cb));
          b = __ldg(reinterpret_cast<const float4*>(grow + c * C + cb));
        }
        xv[c][0] = a.x; xv[c][1] = a.y; xv[c][2] = a.z; xv[c][3] = a.w;
        gv[c][0] = b.x; gv[c][1] = b.y; gv[c][2] = b.z; gv[c][3] = b.w;
#pragma unroll
        for (int q = 0; q < K; ++q) gx[c][q] = 0.0f;
      }
      auto wf = [&](int p, float (&wp)[K], float (&wdp)[K]) {
        const float* wcol = Ws + p * C + cb;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
#pragma unroll
        for (int q = 0; q < kNumBasis; ++q) {
          const float4 wb = *reinterpret_cast<const float4*>(wcol + q * P * C);
          a.x = fmaf(R[q], wb.x, a.x);
          a.y = fmaf(R[q], wb.y, a.y);
          a.z = fmaf(R[q], wb.z, a.z);
          a.w = fmaf(R[q], wb.w, a.w);
          b.x = fmaf(dR[q], wb.x, b.x);
          b.y = fmaf(dR[q], wb.y, b.y);
          b.z = fmaf(dR[q], wb.z, b.z);
          b.w = fmaf(dR[q], wb.w, b.w);
        }
        wp[0] = a.x; wp[1] = a.y; wp[2] = a.z; wp[3] = a.w;
        wdp[0] = b.x; wdp[1] = b.y; wdp[2] = b.z; wdp[3] = b.w;
      };
      G::template bwd<K>(Y, wf, xv, gv, gx, gY, accd);
      if (kGX) {
        segmented_reduce<D, K>(gx, merge);
        if (head) {
#pragma unroll
          for (int c = 0; c < D; ++c) {
            float4* op = reinterpret_cast<float4*>(gxrow + c * C + cb);
            float4 o = make_float4(gx[c][0], gx[c][1], gx[c][2], gx[c][3]);
            if (!row_start) {
              const float4 old = *op;
              o.x += old.x; o.y += old.y; o.z += old.z; o.w += old.w;
            }
            *op = o;
          }
        }
      }
    }
    if (kGE && valid) {
      float Gx, Gy, Gz, S;
      G::sh_grad(nx, ny, nz, gY, Gx, Gy, Gz, S);
      // dL/dr = accd n + (G - S n) / d
      grad_vec[3 * e + 0] = fmaf(accd, nx, (Gx - S * nx) * inv_d);
      grad_vec[3 * e + 1] = fmaf(accd, ny, (Gy - S * ny) * inv_d);
      grad_vec[3 * e + 2] = fmaf(accd, nz, (Gz - S * nz) * inv_d);
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------- helpers

template <int L>
__global__ void k_radial_weights(int n_edges, int C, float inv_rc, const float* __restrict__ edge_vec,
                                 const float* __restrict__ W, float* __restrict__ w_out) {
  constexpr int P = Gen<L>::P;
  const int lane = threadIdx.x & 31;
  const int pc = P * C;
  for (int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); e < n_edges;
       e += gridDim.x * (blockDim.x >> 5)) {
    const float vx = edge_vec[3 * e], vy = edge_vec[3 * e + 1], vz = edge_vec[3 * e + 2];
    float R[kNumBasis], dR[kNumBasis];
    radial_basis<false>(sqrtf(vx * vx + vy * vy + vz * vz), inv_rc, R, dR);
    for (int q = lane; q < pc; q += 32) {
      float a = 0.0f;
#pragma unroll
      for (int b = 0; b < kNumBasis; ++b) a = fmaf(R[b], W[b * pc + q], a);
      w_out[static_cast<size_t>(e) * pc + q] = a;
    }
  }
}

// One warp per node: F_k = sum over edges received minus sum over edges sent, lane-strided over
// the two rows, then a fixed-order warp sum.
__global__ void k_forces(int n_nodes, const int* __restrict__ row_ptr, const int* __restrict__ t_row_ptr,
                         const int* __restrict__ t_perm, const float* __restrict__ gv,
                         float* __restrict__ f) {
  const int lane = threadIdx.x & 31;
  const int n_warps = gridDim.x * (blockDim.x >> 5);
  for (int k = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); k < n_nodes; k += n_warps) {
    float fx = 0.f, fy = 0.f, fz = 0.f;
    for (int e = row_ptr[k] + lane; e < row_ptr[k + 1]; e += 32) {
      fx += gv[3 * e];
      fy += gv[3 * e + 1];
      fz += gv[3 * e + 2];
    }
    for (int q = t_row_ptr[k] + lane; q < t_row_ptr[k + 1]; q += 32) {
      const int e = t_perm[q];
      fx -= gv[3 * e];
      fy -= gv[3 * e + 1];
      fz -= gv[3 * e + 2];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      fx += __shfl_xor_sync(kFull, fx, o);
      fy += __shfl_xor_sync(kFull, fy, o);
      fz += __shfl_xor_sync(kFull, fz, o);
    }
    if (lane == 0) {
      f[3 * k] = fx;
      f[3 * k + 1] = fy;
      f[3 * k + 2] = fz;
    }
  }
}

// flag bits: 1 row_ptr, 2 sender, 4 t_row_ptr, 8 t_perm range, 16 t_perm bucket, 32 t_perm not a permutation
__global__ void k_validate_ptr(const int* __restrict__ ptr, int n_nodes, int n_edges, int bit, int* flag) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r <= n_nodes; r += gridDim.x * blockDim.x) {
    const int v = ptr[r];
    bool bad = v < 0 || v > n_edges || (r == 0 && v != 0) || (r == n_nodes && v != n_edges);
    if (r < n_nodes && ptr[r + 1] < v) bad = true;
    if (bad) atomicOr(flag, bit);
  }
}

__global__ void k_validate_edges(const int* __restrict__ sender, const int* __restrict__ t_row_ptr,
                                 const int* __restrict__ t_perm, int n_nodes, int n_edges,
                                 int* __restrict__ marks, int* flag) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n_edges; k += gridDim.x * blockDim.x) {
    const int s = sender[k];
    if (s < 0 || s >= n_nodes) atomicOr(flag, 2);
    if (t_perm) {
      const int e = t_perm[k];
      if (e < 0 || e >= n_edges) {
        atomicOr(flag, 8);
        continue;
      }
      atomicAdd(marks + e, 1);
      const int se = sender[e];
      if (se >= 0 && se < n_nodes && !(t_row_ptr[se] <= k && k < t_row_ptr[se + 1])) atomicOr(flag, 16);
    }
  }
}

__global__ void k_validate_marks(const int* __restrict__ marks, int n_edges, int* flag) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n_edges; k += gridDim.x * blockDim.x)
    if (marks[k] != 1) atomicOr(flag, 32);
}

int blocks_for(long long n, int threads, int cap) {
  long long b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > cap) b = cap;
  return static_cast<int>(b);
}

int g_num_sms = 0;
int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

// Warps for an edge range: about 96 edges per warp, at most 16 warps per SM.
int conv_blocks(int n_edges) {
  long long warps = (static_cast<long long>(n_edges) + 95) / 96;
  const long long cap = 16LL * num_sms();
  if (warps > cap) warps = cap;
  if (warps < 1) warps = 1;
  return static_cast<int>((warps + 3) / 4);
}

template <int L>
etp_status fwd_impl(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                    const float* edge_vec, const float* x, const float* W, float* out, cudaStream_t s) {
  const size_t smem = sizeof(float) * kNumBasis * Gen<L>::P * c.channels;
  cudaError_t e = cudaFuncSetAttribute(k_conv_fwd<L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_status(e, "forward smem attribute");
  k_conv_fwd<L><<<conv_blocks(n_edges), 128, smem, s>>>(n_nodes, n_edges, c.channels, 1.0f / c.r_cut,
                                                        row_ptr, sender, edge_vec, x, W, out);
  return cuda_status(cudaGetLastError(), "forward launch");
}

template <int L, bool kGX, bool kGE>
etp_status bwd_impl2(const Ctx& c, int n_nodes, int n_edges, const int* sender, const float* edge_vec,
                     const int* t_row_ptr, const int* t_perm, const int* recv_map, const float* x,
                     const float* W, const float* g, float* grad_x, float* grad_vec, cudaStream_t s) {
  const size_t smem = sizeof(float) * kNumBasis * Gen<L>::P * c.channels;
  cudaError_t e = cudaFuncSetAttribute(k_conv_bwd<L, kGX, kGE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_status(e, "backward smem attribute");
  k_conv_bwd<L, kGX, kGE><<<conv_blocks(n_edges), 128, smem, s>>>(
      n_nodes, n_edges, c.channels, 1.0f / c.r_cut, sender, edge_vec, t_row_ptr, t_perm, recv_map, x, W,
      g, grad_x, grad_vec);
  return cuda_status(cudaGetLastError(), "backward launch");
}

template <int L>
etp_status bwd_impl(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                    const float* edge_vec, const int* t_row_ptr, const int* t_perm, const float* x,
                    const float* W, const float* g, float* grad_x, float* grad_vec, int* recv_map,
                    cudaStream_t s) {
  if (n_edges > 0) {
    k_recv_map<<<blocks_for(n_nodes, 128, 4096), 128, 0, s>>>(row_ptr, n_nodes, recv_map);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e, "receiver map");
  }
  if (grad_x && grad_vec)
    return bwd_impl2<L, true, true>(c, n_nodes, n_edges, sender, edge_vec, t_row_ptr, t_perm, recv_map, x, W, g,
                                    grad_x, grad_vec, s);
  if (grad_x)
    return bwd_impl2<L, true, false>(c, n_nodes, n_edges, sender, edge_vec, t_row_ptr, t_perm, recv_map, x, W, g,
                                     grad_x, grad_vec, s);
  return bwd_impl2<L, false, true>(c, n_nodes, n_edges, sender, edge_vec, t_row_ptr, t_perm, recv_map, x, W, g,
                                   grad_x, grad_vec, s);
}

}  // namespace

etp_status launch_forward(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                          const float* edge_vec, const float* x, const float* W, float* out, cudaStream_t s) {
  switch (c.lmax) {
    case 1: return fwd_impl<1>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, s);
    case 2: return fwd_impl<2>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, s);
    case 3: return fwd_impl<3>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, s);
  }
  set_error("launch_forward: unsupported lmax");
  return ETP_ERR_UNSUPPORTED;
}

etp_status launch_backward(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                           const float* edge_vec, const int* t_row_ptr, const int* t_perm, const float* x,
                           const float* W, const float* grad_out, float* grad_x, float* grad_edge_vec,
                           int* recv_map, cudaStream_t s) {
  switch (c.lmax) {
    case 1: return bwd_impl<1>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, t_row_ptr, t_perm, x, W, grad_out,
                               grad_x, grad_edge_vec, recv_map, s);
    case 2: return bwd_impl<2>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, t_row_ptr, t_perm, x, W, grad_out,
                               grad_x, grad_edge_vec, recv_map, s);
    case 3: return bwd_impl<3>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, t_row_ptr, t_perm, x, W, grad_out,
                               grad_x, grad_edge_vec, recv_map, s);
  }
  set_error("launch_backward: unsupported lmax");
  return ETP_ERR_UNSUPPORTED;
}

etp_status launch_radial_weights(const Ctx& c, int n_edges, const float* edge_vec, const float* W, float* w_out,
                                 cudaStream_t s) {
  const int blocks = blocks_for(n_edges, 4, 8 * 148);
  const float inv_rc = 1.0f / c.r_cut;
  switch (c.lmax) {
    case 1: k_radial_weights<1><<<blocks, 128, 0, s>>>(n_edges, c.channels, inv_rc, edge_vec, W, w_out); break;
    case 2: k_radial_weights<2><<<blocks, 128, 0, s>>>(n_edges, c.channels, inv_rc, edge_vec, W, w_out); break;
    case 3: k_radial_weights<3><<<blocks, 128, 0, s>>>(n_edges, c.channels, inv_rc, edge_vec, W, w_out); break;
    default: set_error("radial weights: unsupported lmax"); return ETP_ERR_UNSUPPORTED;
  }
  return cuda_status(cudaGetLastError(), "radial weights launch");
}

etp_status launch_forces(int n_nodes, int n_edges, const int* row_ptr, const int* t_row_ptr, const int* t_perm,
                         const float* grad_edge_vec, float* forces, cudaStream_t s) {
  (void)n_edges;
  k_forces<<<blocks_for(static_cast<long long>(n_nodes) * 32, 128, 4096), 128, 0, s>>>(n_nodes, row_ptr, t_row_ptr,
                                                                                       t_perm, grad_edge_vec, forces);
  return cuda_status(cudaGetLastError(), "forces launch");
}

etp_status validate_graph(int n_nodes, int n_edges, const int* row_ptr, const int* sender, const int* t_row_ptr,
                          const int* t_perm, int* scratch, cudaStream_t s) {
  int* flag = scratch + n_edges;
  cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(int) * (static_cast<size_t>(n_edges) + 1), s);
  if (e != cudaSuccess) return cuda_status(e, "validate memset");
  k_validate_ptr<<<blocks_for(n_nodes + 1, 256, 4096), 256, 0, s>>>(row_ptr, n_nodes, n_edges, 1, flag);
  if (t_row_ptr) k_validate_ptr<<<blocks_for(n_nodes + 1, 256, 4096), 256, 0, s>>>(t_row_ptr, n_nodes, n_edges, 4, flag);
  if (n_edges > 0) {
    k_validate_edges<<<blocks_for(n_edges, 256, 4096), 256, 0, s>>>(sender, t_row_ptr, t_perm, n_nodes, n_edges,
                                                                  scratch, flag);
    if (t_perm) k_validate_marks<<<blocks_for(n_edges, 256, 4096), 256, 0, s>>>(scratch, n_edges, flag);
  }
  int bad = 0;
  if ((e = cudaMemcpyAsync(&bad, flag, sizeof(int), cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_status(e, "validate read");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_status(e, "validate sync");
  if (bad) {
    char buf[96];
    snprintf(buf, sizeof buf, "graph validation failed (flags 0x%x)", bad);
    set_error(buf);
    return ETP_ERR_BAD_GRAPH;
  }
  return ETP_OK;
}

}  // namespace etp

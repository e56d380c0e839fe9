// Edge convolution forward for general irreps with the radial projection on the tensor cores.
//
// The weights of a round of up to 32 edges of one receiver, w[e][(p, u)] = sum_b R_b(d_e)
// W[b][(p, u)], are one kind::tf32 MMA per block of 128 weight columns: D[column][edge] = W^T R^T
// (M = 128 columns as the rows of the A operand, N = 32 edges, K = 8 basis functions), as three
// products hi*hi + hi*lo + lo*hi of the tf32 split with fp32 accumulation. TMEM lane = weight
// column, so warp q, which reads lane quadrant q, finds on its lane t the weights of channel
// u0 + t of its slice (p, u0) along the columns, edge after edge: the lanes-hold-channels layout
// of the FP32 general forward, without its eight FMAs per edge, path and channel.
//
// A CTA of four warps takes one receiver at a time (receivers strided over the grid). Per round of
// <= 32 edges (padded to whole quads with edges of zero weight and zero harmonics that read a real
// sender's row): warp 0 stages the harmonics, warp 1 the radial basis as the B operand (tf32 hi /
// lo rows), warp 2 the senders; thread 0 issues the MMAs; then every warp runs its slices over the
// round's edges with the generated coupling code (gfwdw_t: quads of edges with their loads ahead
// of the arithmetic), each slice's message summed in registers and added once per round into the
// warp's own copy of the output row in shared memory. Per receiver the four copies are added in
// warp order and the row is stored. Fixed order throughout: bitwise reproducible.
//
// The split W^T tiles of all blocks are built once per CTA in shared memory. Several CTAs share an
// SM and overlap their phases; the dynamic shared memory is padded so that the CTAs an SM can hold
// never ask for more than its 512 TMEM columns. The MMA wait is bounded: a timeout stores code 81
// in the status word and the CTA stops; a batch that never completes (code 82) keeps its TMEM.
#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "etp_device.h"
#include "etp_internal.h"
#include "etp_tc_common.h"

namespace etp {
namespace {

using tc::canon;

constexpr int kNE = 32;                    // edges per round: the MMA's N
constexpr int kThr = 128;                  // four warps, one per TMEM lane quadrant
constexpr int kYS = etp_gen::kGenYS;       // staged harmonics per edge
constexpr int kTile = 128 * 8;             // floats of one [128 x 8] operand tile

// Shared memory map (bytes) for nb MMA blocks and output rows of dim_out floats.
struct GSmem {
  static constexpr int OFF_B = 1024;                       // [hl][kNE x 8 canonical]
  static constexpr int OFF_W = OFF_B + 2 * kNE * 8 * 4;    // [block][hl][128 x 8 canonical]
  __host__ __device__ static constexpr int off_y(int nb) { return OFF_W + nb * 2 * kTile * 4; }
  __host__ __device__ static constexpr int off_j(int nb) { return off_y(nb) + kNE * kYS * 4; }
  __host__ __device__ static constexpr int off_acc(int nb) { return off_j(nb) + kNE * 4; }
  __host__ __device__ static constexpr int bytes(int nb, int dim_out) { return off_acc(nb) + 4 * 4 * dim_out; }
};
static_assert(GSmem::OFF_W % 1024 == 0 && (kNE * kYS * 4) % 16 == 0, "operand and row alignment");

__host__ __device__ constexpr int tmem_cols_for(int nb) {
  int n = 32;
  while (n < nb * kNE) n <<= 1;
  return n;
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
  uint32_t r0, r1, r2, r3;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(taddr)
               : "memory");
  v[0] = __uint_as_float(r0);
  v[1] = __uint_as_float(r1);
  v[2] = __uint_as_float(r2);
  v[3] = __uint_as_float(r3);
}

__device__ __forceinline__ void sh_upto(int sh_lmax, float nx, float ny, float nz, float (&Y)[kYS]) {
#pragma unroll
  for (int i = 0; i < kYS; ++i) Y[i] = 0.0f;
  switch (sh_lmax) {
    case 0: Y[0] = 1.0f; break;
    case 1: etp_gen::sh_eval_1(nx, ny, nz, Y); break;
    case 2: etp_gen::sh_eval_2(nx, ny, nz, Y); break;
    case 3: etp_gen::sh_eval_3(nx, ny, nz, Y); break;
    default: etp_gen::sh_eval_4(nx, ny, nz, Y); break;
  }
}

__global__ void __launch_bounds__(kThr) k_gen_fwd_tc(const __grid_constant__ GenParams g, int n_nodes,
                                                     const int* __restrict__ row_ptr,
                                                     const int* __restrict__ sender,
                                                     const float* __restrict__ edge_vec,
                                                     const float* __restrict__ x,
                                                     const float* __restrict__ W, float* __restrict__ out,
                                                     int* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* mma_done = reinterpret_cast<uint64_t*>(smem);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 12);
  volatile int* undrained = reinterpret_cast<volatile int*>(smem + 16);
  const int nb = g.tcp.n_blocks;
  float* Bt = reinterpret_cast<float*>(smem + GSmem::OFF_B);
  float* Wt = reinterpret_cast<float*>(smem + GSmem::OFF_W);
  float* Ys = reinterpret_cast<float*>(smem + GSmem::off_y(nb));
  int* sj = reinterpret_cast<int*>(smem + GSmem::off_j(nb));
  float* acc = reinterpret_cast<float*>(smem + GSmem::off_acc(nb));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dim_out = g.dim_out;
  const uint32_t ncols = static_cast<uint32_t>(tmem_cols_for(nb));

  if (threadIdx.x == 0) {
    tc::mbar_init(mma_done, 1);
    *abort_flag = 0;
    *undrained = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc::sptr(tmem_holder)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // W^T tiles: row r = 32 q + t of block b is weight column woff + u0 + t of quadrant q's slice
  for (int i = threadIdx.x; i < nb * kTile; i += kThr) {
    const int b = i >> 10, r = (i >> 3) & 127, k = i & 7;
    const int q = r >> 5, t = r & 31;
    const int p = g.tcp.path[b][q];
    float v = 0.0f;
    if (p >= 0) {
      const int u = g.tcp.u0[b][q] + t;
      if (u < g.p[p].mul) v = __ldg(W + static_cast<size_t>(k) * g.cols + g.p[p].woff + u);
    }
    float hi, lo;
    tc::split_tf32(v, &hi, &lo);
    Wt[(2 * b) * kTile + canon(r, k)] = hi;
    Wt[(2 * b + 1) * kTile + canon(r, k)] = lo;
  }
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  constexpr uint32_t idesc = tc::idesc_tf32(kNE);
  uint32_t phase = 0;
  bool pending = false;   // thread 0: a committed batch whose completion nobody observed
  bool ok = true;         // CTA-uniform: changes only right after a barrier

  for (int i = blockIdx.x; i < n_nodes && ok; i += gridDim.x) {
    for (int v = threadIdx.x; v < 4 * dim_out; v += kThr) acc[v] = 0.0f;
    const int e0 = row_ptr[i], e1 = row_ptr[i + 1];
    for (int c0 = e0; c0 < e1; c0 += kNE) {
      const int cnt = e1 - c0 < kNE ? e1 - c0 : kNE;
      tc::tc_fence_before();
      __syncthreads();   // the previous round's TMEM columns and staged rows have been read
      if (*abort_flag) {
        ok = false;
        break;
      }
      const int nk = (cnt + 3) & ~3;   // whole quads: the padding edges have w = 0 and Y = 0
      const bool valid = lane < cnt;
      const int e = c0 + lane;
      if (warp == 2) {
        if (lane < nk) sj[lane] = sender[valid ? e : c0];   // a padding edge reads a real sender's row
      } else if (warp < 2) {
        float vx = 0.0f, vy = 0.0f, vz = 0.0f;
        if (valid) {
          vx = edge_vec[3 * static_cast<size_t>(e)];
          vy = edge_vec[3 * static_cast<size_t>(e) + 1];
          vz = edge_vec[3 * static_cast<size_t>(e) + 2];
        }
        const float d = sqrtf(vx * vx + vy * vy + vz * vz);
        if (warp == 0) {
          if (lane < nk) {
            const float inv_d = d > 0.0f ? 1.0f / d : 0.0f;
            float Y[kYS];
            sh_upto(g.sh_lmax, vx * inv_d, vy * inv_d, vz * inv_d, Y);
#pragma unroll
            for (int c = 0; c < kYS; ++c) Ys[lane * kYS + c] = valid ? Y[c] : 0.0f;
          }
        } else {
          float R[kNumBasis], dR[kNumBasis];
          if (valid) {
            radial_basis<false>(d, g.inv_rc, R, dR);
          } else {
#pragma unroll
            for (int b = 0; b < kNumBasis; ++b) R[b] = 0.0f;
          }
#pragma unroll
          for (int b = 0; b < kNumBasis; ++b) {
            float hi, lo;
            tc::split_tf32(R[b], &hi, &lo);
            Bt[canon(lane, b)] = hi;
            Bt[kNE * 8 + canon(lane, b)] = lo;
          }
        }
      }
      tc::fence_proxy_async();
      __syncthreads();
      if (threadIdx.x == 0) {
        tc::tc_fence_after();
        const uint64_t bh = tc::smem_desc(tc::sptr(Bt)), bl = tc::smem_desc(tc::sptr(Bt + kNE * 8));
        for (int b = 0; b < nb; ++b) {
          const uint32_t d = tmem + static_cast<uint32_t>(b * kNE);
          const uint64_t ah = tc::smem_desc(tc::sptr(Wt + (2 * b) * kTile));
          const uint64_t al = tc::smem_desc(tc::sptr(Wt + (2 * b + 1) * kTile));
          tc::mma_tf32(d, ah, bh, idesc, 0u);
          tc::mma_tf32(d, ah, bl, idesc, 1u);
          tc::mma_tf32(d, al, bh, idesc, 1u);
        }
        tc::mma_commit(mma_done);
        pending = true;
      }
      const bool got = tc::warp_wait(mma_done, phase, abort_flag, err, 81);
      phase ^= 1u;
      if (!got) continue;   // the abort flag is up: the next barrier ends the CTA's work
      if (threadIdx.x == 0) pending = false;
      tc::tc_fence_after();
      float* accw = acc + warp * dim_out;
      for (int b = 0; b < nb; ++b) {
        const int p = g.tcp.path[b][warp];
        if (p < 0) continue;
        const GenPath& P = g.p[p];
        const int u = g.tcp.u0[b][warp] + lane;
        const bool act = u < P.mul;
        const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(b * kNE);
        auto wl = [&](int k0, float (&w)[4]) {
          tmem_ld4(taddr + static_cast<uint32_t>(k0), w);
          tc::tmem_wait_ld();
        };
        etp_gen::gen_fwd_w(P.tri, Ys, sj, nk, x + P.in_off + u, g.dim_in, P.mul, wl, act,
                           accw + (P.out_off + u));
      }
    }
    __syncthreads();   // every warp's copy of the row is complete
    if (*abort_flag) ok = false;
    if (ok) {
      float* orow = out + static_cast<size_t>(i) * dim_out;
      for (int c = threadIdx.x; c < dim_out; c += kThr)
        orow[c] = ((acc[c] + acc[dim_out + c]) + acc[2 * dim_out + c]) + acc[3 * dim_out + c];
    }
    __syncthreads();   // read before the next receiver clears the copies
  }

  // teardown: every thread reaches these barriers exactly once
  tc::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && pending) {
    // an aborted wait left the last batch unobserved: wait for it (ignoring the abort flag) before
    // the columns are released
    if (!tc::mbar_wait_drain(mma_done, phase ^ 1u)) {
      tc::report_code(err, 82);
      *undrained = 1;
    }
  }
  __syncthreads();
  if (warp == 0 && !*undrained) {
    tc::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
}

int coupling_cost(int tri) {
  for (int a = 0; a <= etp_gen::kGenLmax; ++a)
    for (int b = 0; b <= etp_gen::kGenLmax; ++b)
      for (int c = 0; c <= etp_gen::kGenLmax; ++c)
        if (etp_gen::kGenTriId[(a * 5 + b) * 5 + c] == tri)
          return etp_gen::kGenTriNnz[tri] + (2 * a + 1) + 2 * (2 * c + 1) + 6;
  return 1;
}

}  // namespace

void plan_general_tc(GenParams& g) {
  g.tcp = GenTcPlan{};
  struct Slice {
    int p, u0, cost;
  };
  std::vector<Slice> sl;
  for (int p = 0; p < g.n_paths; ++p) {
    const int cost = coupling_cost(g.p[p].tri);
    for (int u0 = 0; u0 < g.p[p].mul; u0 += 32) sl.push_back(Slice{p, u0, cost});
  }
  // longest first onto the least loaded quadrant (ties: the lower quadrant), then each quadrant's
  // slices in path order: the order in which its warp adds them into its copy of the row
  std::stable_sort(sl.begin(), sl.end(), [](const Slice& a, const Slice& b) { return a.cost > b.cost; });
  std::vector<Slice> list[4];
  long long load[4] = {0, 0, 0, 0};
  for (const Slice& s : sl) {
    int q = 0;
    for (int k = 1; k < 4; ++k)
      if (load[k] < load[q]) q = k;
    list[q].push_back(s);
    load[q] += s.cost;
  }
  size_t nb = 0;
  for (auto& l : list) {
    std::stable_sort(l.begin(), l.end(), [](const Slice& a, const Slice& b) {
      return a.p != b.p ? a.p < b.p : a.u0 < b.u0;
    });
    nb = std::max(nb, l.size());
  }
  if (nb == 0 || nb > static_cast<size_t>(kGenTcMaxBlocks)) return;
  if (GSmem::bytes(static_cast<int>(nb), g.dim_out) > 227 * 1024) return;
  for (size_t b = 0; b < nb; ++b)
    for (int q = 0; q < 4; ++q) {
      g.tcp.path[b][q] = static_cast<short>(b < list[q].size() ? list[q][b].p : -1);
      g.tcp.u0[b][q] = static_cast<short>(b < list[q].size() ? list[q][b].u0 : 0);
    }
  g.tcp.n_blocks = static_cast<int>(nb);
}

bool general_tc_selected(const GenParams& g, const uint32_t* path_mask) {
  if (path_mask || g.tcp.n_blocks == 0) return false;
  const char* v = std::getenv("ETP_GEN_FORWARD");
  return !(v && std::strcmp(v, "fp32") == 0);
}

etp_status launch_general_forward_tc(const GenParams& g, int n_nodes, const int* row_ptr, const int* sender,
                                     const float* edge_vec, const float* x, const float* W, float* out,
                                     cudaStream_t s, int* err) {
  if (n_nodes == 0) return ETP_OK;
  const int nb = g.tcp.n_blocks;
  int dev = 0, smem_sm = 0, reserved = 0, n_sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_status(e, "general tensor-core forward: device attributes");
  // pad so that one more CTA than the TMEM columns allow never fits an SM
  const int per_sm = tc::kTmemCols / tmem_cols_for(nb);
  int smem = GSmem::bytes(nb, g.dim_out);
  const int floor_bytes = smem_sm / (per_sm + 1) - reserved + 1;
  if (smem < floor_bytes) smem = (floor_bytes + 127) & ~127;
  if (smem > 227 * 1024) {
    set_error("general tensor-core forward: shared memory plan above 227 KB");
    return ETP_ERR_UNSUPPORTED;
  }
  e = cudaFuncSetAttribute(k_gen_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_status(e, "general tensor-core forward smem attribute");
  long long grid = 4LL * per_sm * (n_sms > 0 ? n_sms : 148);
  if (grid > n_nodes) grid = n_nodes;
  k_gen_fwd_tc<<<static_cast<int>(grid), kThr, smem, s>>>(g, n_nodes, row_ptr, sender, edge_vec, x, W, out, err);
  return cuda_status(cudaGetLastError(), "general tensor-core forward launch");
}

}  // namespace etp

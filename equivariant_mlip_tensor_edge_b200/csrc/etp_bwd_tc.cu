// Fused backward (vector-Jacobian product) of the edge convolution with the radial projections
// on the 5th-generation tensor cores.
//
// The backward runs over the transposed (sender-sorted) edge order, so grad_x[j] is a sum over
// the edges that j sends: a work unit ("group") is four senders times a range of 16 channels, a
// persistent CTA per SM walks a contiguous block of groups.
//
// For edge e = (i <- j) and path p = (l1, l2, l3), with w = R W, w' = R' W (R' = dR/dd):
//   v[m1]       = sum_{m2,m3} C Y_{m2} g[i, l3, m3]        (per channel)
//   grad_x[j]  += w v
//   grad_w      = sum_m1 x[j, l1, m1] v[m1];   accd += w' grad_w      (distance term)
//   grad_Y[m2] += w sum_{m1,m3} C x[j, l1, m1] g[i, l3, m3]
//   grad_r      = accd n + (sum_m2 grad_Y dY/dn - (sum_m2 l2 grad_Y Y) n) / d
//
//   producer warp 4 (lane 0): per item (channel pass, 32-edge tile), w and w' for the 128 edges
//     as six kind::tf32 MMAs (hi*hi + hi*lo + lo*hi each; M = 128 edges, N = K P rounded up to
//     32, K = 8 basis functions) into the two halves of a TMEM slot, and the unit's pre-split
//     W^T slices by cp.async.bulk.
//   consumer warps 0..3: warp q owns sender q of the group (TMEM lane quadrant q), one edge per
//     lane. Setup per sender round: edge id, receiver, direction, Y, R and R' (tf32 hi/lo rows
//     of the two A tiles). Per item: the lane's receiver row of grad_out for the pass arrives by
//     cp.async one item ahead; x[j] of the pass is one broadcast load per pass; w, w' from TMEM;
//     the unrolled VJP code accumulates grad_x (per sender, across tiles) and grad_Y, the
//     distance term (per edge, across passes, in shared memory). Per pass: one fixed-order
//     cross-lane sum of grad_x. Per group: each lane writes its edges' gradient contributions
//     of the unit's channels; a final pass sums the units in a fixed order.
//
// Synchronisation as in the forward: bounded mbarrier waits, warp-uniform outcomes, clean abort.
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"
#include "etp_tc_common.h"

namespace etp {
namespace tc {
namespace {

constexpr int kQuads = 4;
constexpr int kThreads = 32 * (kQuads + 1);
constexpr int kUnitC = 16;
constexpr int kStages = 2;

template <int L>
struct BCfg {
  static constexpr int D = Gen<L>::D;
  static constexpr int P = Gen<L>::P;
  static constexpr int K = L == 1 ? 8 : (L == 2 ? 4 : 2);     // channels per pass
  static constexpr int SMAX = L >= 3 ? 2 : 4;                  // tiles per sender round
  static constexpr int NPASS = kUnitC / K;
  static constexpr int NCOL = ((K * P + 31) / 32) * 32;        // MMA N (w); w' follows
  static constexpr int SLOTC = 2 * NCOL;                       // TMEM columns per slot
  static constexpr int NSLOT = kTmemCols / SLOTC;
  static constexpr int PPC = 16 / K;                           // paths per 16-column chunk
  static constexpr int ROWB = D * K * 4;                       // gathered bytes per edge and pass
  static constexpr int SLOTB = ROWB + 16;
  static constexpr int STAGEB = 32 * SLOTB;
  static constexpr int V = D * K;
  static constexpr int VS = 4 * ((V / 4) | 1);
  static constexpr int EW = 2 * D + 5;                         // per-edge words: Y, gY, accd, n, 1/d
  static constexpr int WSLICE = 2 * NCOL * 32;
  static constexpr int WBUF = NPASS * WSLICE;
  static constexpr int MAXRG = 64;
  static constexpr int OFF_G = 1024;
  static constexpr int OFF_A = OFF_G + 2048;                   // [tile][R hi, R lo, R' hi, R' lo]
  static constexpr int OFF_W = OFF_A + SMAX * 4 * 4096;
  static constexpr int OFF_E = OFF_W + 2 * WBUF;               // [quad][tile][EW][32]
  static constexpr int OFF_J = OFF_E + kQuads * SMAX * EW * 32 * 4;   // receivers [quad][tile][32]
  static constexpr int OFF_I = OFF_J + kQuads * SMAX * 32 * 4;        // edge ids   [quad][tile][32]
  static constexpr int OFF_K = OFF_I + kQuads * SMAX * 32 * 4;        // path masks [quad][tile][32]
  static constexpr int OFF_X = OFF_K + kQuads * SMAX * 32 * 4;
  static constexpr int OFF_R = OFF_X + kQuads * kStages * STAGEB;
  static constexpr int END = OFF_R + kQuads * 32 * VS * 4;
  static constexpr int SMEM = END < 118 * 1024 ? 118 * 1024 : END;
  static_assert(END <= 227 * 1024, "shared memory budget");
  static_assert(NSLOT >= 2, "TMEM slot ring");
  static_assert(K == 2 || K % 4 == 0, "pass width");
  static_assert((MAXRG * kQuads + 8) * 4 <= 2048, "row-pointer cache");
};

struct BArgs {
  int n_nodes;
  int C;
  int dim;
  int n_units;
  int n_groups;
  float inv_rc;
  const int* t_row_ptr;
  const int* t_perm;
  const int* recv;        // receiver of each canonical edge
  const float* edge_vec;
  const float* x;
  const float* g;         // grad_out
  const float* wt;
  const uint32_t* mask;   // per-edge path mask (bit p: path p on), or null
  float* grad_x;          // may be null
  float* gpart;           // [unit][E][3] partial edge gradients, or grad_edge_vec when n_units == 1; may be null
  int n_edges;
  int* err;
};

struct BGroup {
  int rg, unit, rounds, nbatch;
  int deg[kQuads];
  int beg[kQuads];
};

template <int SMAX>
__device__ __forceinline__ int btiles_of(int deg, int round) {
  const int rem = deg - round * 32 * SMAX;
  if (rem <= 0) return 0;
  const int t = (rem + 31) / 32;
  return t < SMAX ? t : SMAX;
}

template <int SMAX>
__device__ __forceinline__ void bgroup_info(const BArgs& a, const int* rp, int rg_beg, int g, BGroup* gi) {
  gi->rg = g / a.n_units;
  gi->unit = g - gi->rg * a.n_units;
  int rounds = 1;
#pragma unroll
  for (int q = 0; q < kQuads; ++q) {
    const int r = gi->rg * kQuads + q;
    int b = 0, d = 0;
    if (r < a.n_nodes) {
      const int o = r - rg_beg * kQuads;
      b = rp[o];
      d = rp[o + 1] - b;
    }
    gi->beg[q] = b;
    gi->deg[q] = d;
    const int rr = (d + 32 * SMAX - 1) / (32 * SMAX);
    rounds = rr > rounds ? rr : rounds;
  }
  gi->rounds = rounds;
  const int left = a.C - gi->unit * kUnitC;
  gi->nbatch = (left >= kUnitC ? kUnitC : left) / 4;
}

template <int SMAX>
__device__ __forceinline__ int bgroup_tiles(const BGroup& gi, int round) {
  int S = 0;
#pragma unroll
  for (int q = 0; q < kQuads; ++q) {
    const int t = btiles_of<SMAX>(gi.deg[q], round);
    S = t > S ? t : S;
  }
  return S;
}

__device__ __forceinline__ void tmem_ld16x(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Pre-split weights for the backward's pass width: wt[unit][pass][hl][canonical NCOL x 8].
template <int L>
__global__ void k_bprep(const float* __restrict__ W, int C, int n_units, float* __restrict__ wt) {
  using G = BCfg<L>;
  constexpr int K = G::K;
  const int per_pass = 2 * G::NCOL * 8;
  const int total = n_units * G::NPASS * per_pass;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int slab = i / per_pass;
    const int rem = i - slab * per_pass;
    const int hl = rem / (G::NCOL * 8);
    const int e = rem - hl * (G::NCOL * 8);
    const int n = e / 8, kb = e % 8;
    const int p = n / K, k = n % K;
    const int u = slab * K + k;
    float v = 0.0f;
    if (p < G::P && u < C) v = W[(kb * G::P + p) * C + u];
    float hi, lo;
    split_tf32(v, &hi, &lo);
    wt[slab * per_pass + hl * G::NCOL * 8 + canon(n, kb)] = hl ? lo : hi;
  }
}

// receiver of every canonical edge. A kernel launched as its programmatic dependent may start at once
// and waits for this grid (griddepcontrol.wait) before reading recv.
__global__ void k_recv_of_edge(const int* __restrict__ row_ptr, int n_nodes, int n_edges, int* __restrict__ recv) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n_edges; e += gridDim.x * blockDim.x) {
    int lo = 0, hi = n_nodes - 1;   // last r with row_ptr[r] <= e
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
    }
    recv[e] = lo;
  }
}

// grad_edge_vec[e] = sum over channel units of the partial contributions, in unit order
__global__ void k_sum_units(const float* __restrict__ part, int n_units, int n_edges, float* __restrict__ out) {
  const long long n3 = 3LL * n_edges;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n3;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float s = part[i];
    for (int u = 1; u < n_units; ++u) s += part[u * n3 + i];
    out[i] = s;
  }
}

// MASKED: as in the forward, a path whose bit is clear in an edge's mask contributes nothing for
// that edge (w = w' = 0), and a path no edge of the item needs is skipped.
template <int L, bool MASKED>
__global__ void __launch_bounds__(kThreads, 1) k_bwd_tc(BArgs a) {
  using G = BCfg<L>;
  using Gn = Gen<L>;
  constexpr int D = G::D, K = G::K, V = G::V, VS = G::VS, NCOL = G::NCOL, NSLOT = G::NSLOT;
  constexpr int SMAX = G::SMAX, EW = G::EW;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* tfull = reinterpret_cast<uint64_t*>(smem);
  uint64_t* tempty = tfull + NSLOT;
  uint64_t* rready = tempty + NSLOT;
  uint64_t* sfree = rready + 1;
  uint64_t* wload = sfree + 1;
  uint64_t* wfree = wload + 2;
  uint64_t* drainb = wfree + 2;   // final commit of the producer (abort-safe drain)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drainb + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* rp = reinterpret_cast<int*>(smem + G::OFF_G);
  float* Atile = reinterpret_cast<float*>(smem + G::OFF_A);   // [tile][4][128 x 8]
  float* Wbuf = reinterpret_cast<float*>(smem + G::OFF_W);
  float* Ebuf = reinterpret_cast<float*>(smem + G::OFF_E);    // [quad][tile][EW][32]
  int* Jbuf = reinterpret_cast<int*>(smem + G::OFF_J);        // receivers
  int* Ibuf = reinterpret_cast<int*>(smem + G::OFF_I);        // canonical edge ids
  uint32_t* Kbuf = reinterpret_cast<uint32_t*>(smem + G::OFF_K);
  unsigned char* Xbuf = smem + G::OFF_X;
  float* Red = reinterpret_cast<float*>(smem + G::OFF_R);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g_beg = static_cast<int>(static_cast<long long>(a.n_groups) * blockIdx.x / gridDim.x);
  const int g_end = static_cast<int>(static_cast<long long>(a.n_groups) * (blockIdx.x + 1) / gridDim.x);
  const int rg_beg = g_beg / a.n_units;
  const int rg_end = g_end > g_beg ? (g_end - 1) / a.n_units + 1 : rg_beg;
  const int n_rp = (rg_end - rg_beg) * kQuads + 1;
  for (int i = threadIdx.x; i < n_rp; i += blockDim.x) {
    const int r = rg_beg * kQuads + i;
    rp[i] = a.t_row_ptr[r < a.n_nodes ? r : a.n_nodes];
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(tfull + i, 1);
      mbar_init(tempty + i, kQuads);
    }
    mbar_init(rready, kQuads);
    mbar_init(sfree, kQuads);
    mbar_init(wload + 0, 1);
    mbar_init(wload + 1, 1);
    mbar_init(wfree + 0, 1);
    mbar_init(wfree + 1, 1);
    mbar_init(drainb, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kQuads) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sptr(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  bool drained = true;   // false: issued tensor-core work did not finish; TMEM is then not released
  // launched as a programmatic dependent of k_recv_of_edge: the setup above overlaps it, the work
  // below reads its output (the pre-split weights come from k_bprep, complete before it began)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kQuads) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32(NCOL);
      uint32_t titem = 0, n_setup = 0, n_loads = 0, n_issued = 0;
      int cached_rg = -1, cached_round = -1;
      bool ok = true;
      auto load_w = [&](int g, uint32_t n) -> bool {
        const int unit = g % a.n_units;
        const int wb = n & 1;
        if (n >= 2 && !mbar_wait(wfree + wb, ((n >> 1) - 1) & 1, abort_flag, a.err, 31)) return false;
        mbar_expect_tx(wload + wb, G::WBUF);
        bulk_g2s(Wbuf + wb * (G::WBUF / 4), a.wt + static_cast<size_t>(unit) * (G::WBUF / 4), G::WBUF, wload + wb);
        ++n_issued;
        return true;
      };
      if (g_beg < g_end) ok = load_w(g_beg, 0);
      for (int g = g_beg; g < g_end && ok; ++g) {
        BGroup gi;
        bgroup_info<SMAX>(a, rp, rg_beg, g, &gi);
        const int wb = n_loads & 1;
        const int npass = (gi.nbatch * 4 + K - 1) / K;
        ok = mbar_wait(wload + wb, (n_loads >> 1) & 1, abort_flag, a.err, 32);
        ++n_loads;
        for (int round = 0; round < gi.rounds && ok; ++round) {
          const int S = bgroup_tiles<SMAX>(gi, round);
          if (gi.rg != cached_rg || round != cached_round) {
            ok = mbar_wait(rready, n_setup & 1, abort_flag, a.err, 33);
            ++n_setup;
            cached_rg = gi.rg;
            cached_round = round;
            if (!ok) break;
          }
          tc_fence_after();
          for (int pass = 0; pass < npass && ok; ++pass) {
            for (int s = 0; s < S; ++s) {
              const int slot = titem % NSLOT;
              ok = mbar_wait(tempty + slot, ((titem / NSLOT) & 1) ^ 1, abort_flag, a.err, 34);
              if (!ok) break;
              tc_fence_after();
              const uint32_t d = tmem + slot * G::SLOTC;
              const float* at = Atile + s * 4 * 1024;
              const uint64_t rh = smem_desc(sptr(at)), rl = smem_desc(sptr(at + 1024));
              const uint64_t dh = smem_desc(sptr(at + 2048)), dl = smem_desc(sptr(at + 3072));
              const float* wsl = Wbuf + wb * (G::WBUF / 4) + pass * (G::WSLICE / 4);
              const uint64_t bh = smem_desc(sptr(wsl)), bl = smem_desc(sptr(wsl + NCOL * 8));
              mma_tf32(d, rh, bh, idesc, 0u);
              mma_tf32(d, rh, bl, idesc, 1u);
              mma_tf32(d, rl, bh, idesc, 1u);
              mma_tf32(d + NCOL, dh, bh, idesc, 0u);
              mma_tf32(d + NCOL, dh, bl, idesc, 1u);
              mma_tf32(d + NCOL, dl, bh, idesc, 1u);
              mma_commit(tfull + slot);
              ++titem;
            }
          }
        }
        mma_commit(wfree + wb);
        if (ok && g + 1 < g_end) ok = load_w(g + 1, n_loads);
      }
      // drain, ignoring the abort flag: one more commit tracks every MMA issued so far, and the
      // weight load issued for a group that was never consumed may still be in flight
      mma_commit(drainb);
      bool dr = mbar_wait_drain(drainb, 0);
      if (dr && n_issued > n_loads)
        dr = mbar_wait_drain(wload + ((n_issued - 1) & 1), ((n_issued - 1) >> 1) & 1);
      if (!dr) {
        report_code(a.err, 35);
        *abort_flag = 1;
        drained = false;
      }
    }
    drained = __shfl_sync(kFull, drained ? 1 : 0, 0) != 0;
  } else {
    // ---------------------------------------------------------------- consumers
    const int q = warp;
    float* Eq = Ebuf + q * (SMAX * EW * 32);
    int* Jq = Jbuf + q * (SMAX * 32);
    int* Iq = Ibuf + q * (SMAX * 32);
    uint32_t* Kq = Kbuf + q * (SMAX * 32);
    float* Rw = Red + q * (32 * VS);
    unsigned char* Xw = Xbuf + q * kStages * G::STAGEB + lane * G::SLOTB;
    uint32_t titem = 0, n_setup = 0;
    int cached_rg = -1, cached_round = -1;
    bool ok = true;
    for (int g = g_beg; g < g_end && ok; ++g) {
      BGroup gi;
      bgroup_info<SMAX>(a, rp, rg_beg, g, &gi);
      const int j = gi.rg * kQuads + q;     // this warp's sender
      const int deg = gi.deg[q];
      const int npass = (gi.nbatch * 4 + K - 1) / K;
      const int cbase = gi.unit * kUnitC;
      for (int round = 0; round < gi.rounds && ok; ++round) {
        const int S = bgroup_tiles<SMAX>(gi, round);
        const int Sq = btiles_of<SMAX>(deg, round);
        if (gi.rg != cached_rg || round != cached_round) {
          if (n_setup > 0) {
            mbar_arrive_lane0(sfree, lane);
            ok = warp_wait(sfree, (n_setup - 1) & 1, abort_flag, a.err, 41);
            if (!ok) break;
          }
          for (int s = 0; s < Sq; ++s) {
            const int le = round * 32 * SMAX + s * 32 + lane;
            float Y[D];
            float R[kNumBasis], dR[kNumBasis];
#pragma unroll
            for (int c = 0; c < D; ++c) Y[c] = 0.0f;
#pragma unroll
            for (int bb = 0; bb < kNumBasis; ++bb) {
              R[bb] = 0.0f;
              dR[bb] = 0.0f;
            }
            int recv = -1, e = -1;
            float nx = 0.f, ny = 0.f, nz = 0.f, inv_d = 0.f;
            if (le < deg) {
              e = a.t_perm[gi.beg[q] + le];
              recv = a.recv[e];
              const float vx = a.edge_vec[3 * e], vy = a.edge_vec[3 * e + 1], vz = a.edge_vec[3 * e + 2];
              const float dd = sqrtf(vx * vx + vy * vy + vz * vz);
              inv_d = dd > 0.0f ? 1.0f / dd : 0.0f;
              nx = vx * inv_d;
              ny = vy * inv_d;
              nz = vz * inv_d;
              Gn::sh(nx, ny, nz, Y);
              radial_basis<true>(dd, a.inv_rc, R, dR);
            }
            Jq[s * 32 + lane] = recv;
            Iq[s * 32 + lane] = e;
            if constexpr (MASKED) Kq[s * 32 + lane] = e >= 0 ? a.mask[e] : 0u;
            float* E = Eq + s * EW * 32 + lane;
#pragma unroll
            for (int c = 0; c < D; ++c) E[c * 32] = Y[c];
            E[(2 * D + 1) * 32] = nx;
            E[(2 * D + 2) * 32] = ny;
            E[(2 * D + 3) * 32] = nz;
            E[(2 * D + 4) * 32] = inv_d;
            const int row = 32 * q + lane;
            float h[kNumBasis], l[kNumBasis];
            float* at = Atile + s * 4 * 1024;
#pragma unroll
            for (int bb = 0; bb < kNumBasis; ++bb) split_tf32(R[bb], &h[bb], &l[bb]);
            *reinterpret_cast<float4*>(at + canon(row, 0)) = make_float4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<float4*>(at + canon(row, 4)) = make_float4(h[4], h[5], h[6], h[7]);
            *reinterpret_cast<float4*>(at + 1024 + canon(row, 0)) = make_float4(l[0], l[1], l[2], l[3]);
            *reinterpret_cast<float4*>(at + 1024 + canon(row, 4)) = make_float4(l[4], l[5], l[6], l[7]);
#pragma unroll
            for (int bb = 0; bb < kNumBasis; ++bb) split_tf32(dR[bb], &h[bb], &l[bb]);
            *reinterpret_cast<float4*>(at + 2048 + canon(row, 0)) = make_float4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<float4*>(at + 2048 + canon(row, 4)) = make_float4(h[4], h[5], h[6], h[7]);
            *reinterpret_cast<float4*>(at + 3072 + canon(row, 0)) = make_float4(l[0], l[1], l[2], l[3]);
            *reinterpret_cast<float4*>(at + 3072 + canon(row, 4)) = make_float4(l[4], l[5], l[6], l[7]);
          }
          fence_proxy_async();
          __syncwarp();
          mbar_arrive_lane0(rready, lane);
          ok = warp_wait(rready, n_setup & 1, abort_flag, a.err, 42);
          ++n_setup;
          cached_rg = gi.rg;
          cached_round = round;
          if (!ok) break;
        }
        // per-edge accumulators of this unit start at zero
        for (int s = 0; s < Sq; ++s) {
          float* E = Eq + s * EW * 32 + lane;
#pragma unroll
          for (int c = 0; c <= D; ++c) E[(D + c) * 32] = 0.0f;
        }
        auto prefetch = [&](int pass, int s, int st) {
          const int ii = Jq[s * 32 + lane];
          const int ch = cbase + pass * K;
          const float* src = a.g + static_cast<size_t>(ii < 0 ? 0 : ii) * a.dim + ch;
          unsigned char* dst = Xw + st * G::STAGEB;
          const int nvalid = a.C - ch;
#pragma unroll
          for (int c = 0; c < D; ++c) {
            if constexpr (K >= 4) {
#pragma unroll
              for (int k4 = 0; k4 < K / 4; ++k4) {
                const bool in = ii >= 0 && 4 * k4 < nvalid;
                cp_async16(dst + (c * K + 4 * k4) * 4, src + c * a.C + 4 * k4, in ? 16u : 0u);
              }
            } else {
              cp_async8(dst + c * K * 4, src + c * a.C, ii >= 0 ? 8u : 0u);
            }
          }
          cp_async_commit();
        };
        int stage = 0;
        if (Sq > 0) prefetch(0, 0, 0);
        for (int pass = 0; pass < npass && ok; ++pass) {
          const int ch0 = cbase + pass * K;
          // x of this warp's sender for the pass: one broadcast load per component
          float xv[D][K];
          {
            const float* xs = a.x + static_cast<size_t>(j < a.n_nodes ? j : 0) * a.dim + ch0;
#pragma unroll
            for (int c = 0; c < D; ++c)
#pragma unroll
              for (int k = 0; k < K; ++k) xv[c][k] = (j < a.n_nodes && ch0 + k < a.C) ? __ldg(xs + c * a.C + k) : 0.0f;
          }
          float gx[D][K];
#pragma unroll
          for (int c = 0; c < D; ++c)
#pragma unroll
            for (int k = 0; k < K; ++k) gx[c][k] = 0.0f;
          for (int s = 0; s < S; ++s) {
            const int slot = titem % NSLOT;
            const bool mine = s < Sq;
            float gv[D][K];
            if (mine) {
              cp_async_wait<0>();
              const float* gs = reinterpret_cast<const float*>(Xw + stage * G::STAGEB);
#pragma unroll
              for (int c = 0; c < D; ++c)
#pragma unroll
                for (int k = 0; k < K; ++k) gv[c][k] = gs[c * K + k];
              int np = pass, ns = s + 1;
              if (ns >= Sq) {
                ns = 0;
                ++np;
              }
              if (np < npass) prefetch(np, ns, stage ^ 1);
              stage ^= 1;
            }
            ok = warp_wait(tfull + slot, (titem / NSLOT) & 1, abort_flag, a.err, 43);
            if (!ok) break;
            tc_fence_after();
            if (mine) {
              float* E = Eq + s * EW * 32 + lane;
              float Y[D], gY[D];
#pragma unroll
              for (int c = 0; c < D; ++c) {
                Y[c] = E[c * 32];
                gY[c] = E[(D + c) * 32];
              }
              float accd = E[(2 * D) * 32];
              const uint32_t tb = tmem + (static_cast<uint32_t>(32 * q) << 16) + slot * G::SLOTC;
              float wch[16], dch[16];
              // (array bounds spelled G::K: see the forward kernel)
              [[maybe_unused]] const uint32_t mbits = MASKED ? Kq[s * 32 + lane] : ~0u;
              auto wf = [&](auto pc, float (&wp)[G::K], float (&wdp)[G::K]) {
                constexpr int p = decltype(pc)::value;
                if constexpr (p % G::PPC == 0) {
                  tmem_ld16x(tb + 16 * (p / G::PPC), wch);
                  tmem_ld16x(tb + G::NCOL + 16 * (p / G::PPC), dch);
                  tmem_wait_ld();
                }
                constexpr int o = (p % G::PPC) * G::K;
                if constexpr (MASKED) {
                  const bool on = (mbits >> p) & 1u;
#pragma unroll
                  for (int k = 0; k < G::K; ++k) {
                    wp[k] = on ? wch[o + k] : 0.0f;
                    wdp[k] = on ? dch[o + k] : 0.0f;
                  }
                  return __any_sync(kFull, on);
                } else {
#pragma unroll
                  for (int k = 0; k < G::K; ++k) {
                    wp[k] = wch[o + k];
                    wdp[k] = dch[o + k];
                  }
                }
              };
              Gn::template bwd<K>(Y, wf, xv, gv, gx, gY, accd);
#pragma unroll
              for (int c = 1; c < D; ++c) E[(D + c) * 32] = gY[c];
              E[(2 * D) * 32] = accd;
            }
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(tempty + slot, lane);
            ++titem;
          }
          if (!ok) break;
          // grad_x of the sender: cross-lane sum, then store (round 0) or add
          if (a.grad_x && (Sq > 0 || round == 0)) {
#pragma unroll
            for (int c = 0; c < D; ++c)
#pragma unroll
              for (int k4 = 0; k4 < (K + 3) / 4; ++k4) {
                if (K >= 4) {
                  *reinterpret_cast<float4*>(Rw + lane * VS + c * K + 4 * k4) =
                      make_float4(gx[c][4 * k4], gx[c][4 * k4 + 1], gx[c][4 * k4 + 2], gx[c][4 * k4 + 3]);
                } else {
#pragma unroll
                  for (int k = 0; k < K; ++k) Rw[lane * VS + c * K + k] = gx[c][k];
                }
              }
            __syncwarp();
            if (j < a.n_nodes) {
              for (int v = lane; v < V; v += 32) {
                const int c = v / K, k = v % K;
                const int ch = ch0 + k;
                if (ch < a.C) {
                  float col[32];
#pragma unroll
                  for (int l2 = 0; l2 < 32; ++l2) col[l2] = Rw[l2 * VS + v];
#pragma unroll
                  for (int w2 = 16; w2 > 0; w2 >>= 1)
#pragma unroll
                    for (int l2 = 0; l2 < w2; ++l2) col[l2] += col[l2 + w2];
                  float* op = a.grad_x + static_cast<size_t>(j) * a.dim + c * a.C + ch;
                  if (round == 0) *op = col[0]; else *op += col[0];
                }
              }
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        // this unit's contribution to each edge's gradient
        if (a.gpart) {
          for (int s = 0; s < Sq; ++s) {
            const int e = Iq[s * 32 + lane];
            if (e >= 0) {
              const float* E = Eq + s * EW * 32 + lane;
              float gY[D];
#pragma unroll
              for (int c = 0; c < D; ++c) gY[c] = E[(D + c) * 32];
              gY[0] = 0.0f;
              const float accd = E[(2 * D) * 32];
              const float nx = E[(2 * D + 1) * 32], ny = E[(2 * D + 2) * 32], nz = E[(2 * D + 3) * 32];
              const float inv_d = E[(2 * D + 4) * 32];
              float Gx, Gy, Gz, Ss;
              Gn::sh_grad(nx, ny, nz, gY, Gx, Gy, Gz, Ss);
              float* out = a.gpart + (static_cast<size_t>(gi.unit) * a.n_edges + e) * 3;
              out[0] = fmaf(accd, nx, (Gx - Ss * nx) * inv_d);
              out[1] = fmaf(accd, ny, (Gy - Ss * ny) * inv_d);
              out[2] = fmaf(accd, nz, (Gz - Ss * nz) * inv_d);
            }
          }
        }
      }
    }
    cp_async_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kQuads && drained) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

int g_bsms = 0;
int bnum_sms() {
  if (g_bsms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_bsms, cudaDevAttrMultiProcessorCount, dev);
    if (g_bsms <= 0) g_bsms = 148;
  }
  return g_bsms;
}

// Workspace: [wt][status][partials: units x E x 3 floats, when units > 1]
template <int L>
size_t bws_bytes(int channels, int n_edges) {
  const int n_units = (channels + kUnitC - 1) / kUnitC;
  size_t b = align256(static_cast<size_t>(n_units) * BCfg<L>::WBUF);
  if (n_units > 1) b += align256(sizeof(float) * 3 * static_cast<size_t>(n_units) * n_edges);
  return b;
}

template <int L>
etp_status blaunch(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const float* edge_vec,
                   const int* t_row_ptr, const int* t_perm, const float* x, const float* W, const float* g,
                   float* grad_x, float* grad_vec, int* recv, void* ws, cudaStream_t s, const uint32_t* mask) {
  using G = BCfg<L>;
  const int n_units = (c.channels + kUnitC - 1) / kUnitC;
  char* p = static_cast<char*>(ws);
  float* wt = reinterpret_cast<float*>(p);
  p += align256(static_cast<size_t>(n_units) * G::WBUF);
  float* part = n_units > 1 ? reinterpret_cast<float*>(p) : grad_vec;
  k_bprep<L><<<32, 256, 0, s>>>(W, c.channels, n_units, wt);
  if (n_edges > 0) {
    int blocks = (n_edges + 255) / 256;
    if (blocks > 8 * bnum_sms()) blocks = 8 * bnum_sms();
    k_recv_of_edge<<<blocks, 256, 0, s>>>(row_ptr, n_nodes, n_edges, recv);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "backward prep");
  e = mask ? cudaFuncSetAttribute(k_bwd_tc<L, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM)
           : cudaFuncSetAttribute(k_bwd_tc<L, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return cuda_status(e, "tc backward smem attribute");
  BArgs a;
  a.n_nodes = n_nodes;
  a.C = c.channels;
  a.dim = c.dim;
  a.n_units = n_units;
  a.n_groups = ((n_nodes + kQuads - 1) / kQuads) * n_units;
  a.inv_rc = 1.0f / c.r_cut;
  a.t_row_ptr = t_row_ptr;
  a.t_perm = t_perm;
  a.recv = recv;
  a.edge_vec = edge_vec;
  a.x = x;
  a.g = g;
  a.wt = wt;
  a.mask = mask;
  a.grad_x = grad_x;
  a.gpart = grad_vec ? part : nullptr;
  a.n_edges = n_edges;
  a.err = c.status_dev;
  long long grid = bnum_sms();
  const long long n_rg = (n_nodes + kQuads - 1) / kQuads;
  const long long min_grid = (n_rg + G::MAXRG - 3) / (G::MAXRG - 2);
  if (grid < min_grid) grid = min_grid;
  if (grid > a.n_groups) grid = a.n_groups;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = mask ? cudaLaunchKernelEx(&cfg, k_bwd_tc<L, true>, a) : cudaLaunchKernelEx(&cfg, k_bwd_tc<L, false>, a);
  if (e != cudaSuccess) return cuda_status(e, "tc backward launch");
  if (grad_vec && n_units > 1 && n_edges > 0) {
    long long blocks = (3LL * n_edges + 255) / 256;
    if (blocks > 8LL * bnum_sms()) blocks = 8LL * bnum_sms();
    k_sum_units<<<static_cast<int>(blocks), 256, 0, s>>>(part, n_units, n_edges, grad_vec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e, "edge-gradient sum launch");
  }
  return ETP_OK;
}

}  // namespace

size_t backward_tc_workspace_bytes(const Ctx& c, int n_edges) {
  switch (c.lmax) {
    case 1: return bws_bytes<1>(c.channels, n_edges);
    case 2: return bws_bytes<2>(c.channels, n_edges);
    default: return bws_bytes<3>(c.channels, n_edges);
  }
}

etp_status backward_tc_status(const Ctx& c, const void* ws, cudaStream_t s) {
  (void)ws;
  return read_status(c, s, "tensor-core backward");
}

etp_status launch_backward_tc(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const float* edge_vec,
                              const int* t_row_ptr, const int* t_perm, const float* x, const float* W,
                              const float* grad_out, float* grad_x, float* grad_edge_vec, int* recv, void* ws,
                              cudaStream_t s, const uint32_t* path_mask) {
  switch (c.lmax) {
    case 1: return blaunch<1>(c, n_nodes, n_edges, row_ptr, edge_vec, t_row_ptr, t_perm, x, W, grad_out, grad_x,
                              grad_edge_vec, recv, ws, s, path_mask);
    case 2: return blaunch<2>(c, n_nodes, n_edges, row_ptr, edge_vec, t_row_ptr, t_perm, x, W, grad_out, grad_x,
                              grad_edge_vec, recv, ws, s, path_mask);
    case 3: return blaunch<3>(c, n_nodes, n_edges, row_ptr, edge_vec, t_row_ptr, t_perm, x, W, grad_out, grad_x,
                              grad_edge_vec, recv, ws, s, path_mask);
  }
  set_error("tc backward: unsupported lmax");
  return ETP_ERR_UNSUPPORTED;
}

}  // namespace tc

etp_status launch_recv_of_edge(const int* row_ptr, int n_nodes, int n_edges, int* recv, cudaStream_t s) {
  if (n_edges <= 0) return ETP_OK;
  int blocks = (n_edges + 255) / 256;
  if (blocks > 8 * tc::bnum_sms()) blocks = 8 * tc::bnum_sms();
  tc::k_recv_of_edge<<<blocks, 256, 0, s>>>(row_ptr, n_nodes, n_edges, recv);
  return cuda_status(cudaGetLastError(), "edge receivers");
}

}  // namespace etp

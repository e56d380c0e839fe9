// Fused forward, channel-major: lanes hold channels, warps walk the edges in canonical order.
// (An alternative to the edge-major kernel of etp_fwd_tc.cu, selected by ETP_FORWARD=channel: no
// per-lane gathers and no cross-lane sums, but one channel per lane leaves less reuse of the
// per-edge coefficients; it wins on irregular degrees and loses on regular ones.)
//
// For C in {32, 64, 128} and l_max <= 2. Each CTA owns a contiguous range of receivers (cut by
// edge count) and streams its edges in batches of 16:
//   setup warp 4: per 32 edges (one per lane): direction, Y, radial basis R_b(d) (as the tf32
//     hi/lo rows of the MMA B operand), and the per-edge coefficients M_p[m3][m1] = sum_m2 C Y
//     for every path, stored once per edge in shared memory; lane 0 then issues, per batch,
//     w^T = W^T R^T on the tensor cores: D[(path, channel)][edge] for 16 edges, M = 128 rows per
//     block of paths, three kind::tf32 MMAs (hi*hi + hi*lo + lo*hi) per block, into a TMEM ring.
//   consumer warps 0..3: warp q reads TMEM lane quadrant q, i.e. a fixed 32-channel slice and a
//     fixed subset of the paths (the C / 32 slices x 128 / C subsets tile the 128 rows). Per edge:
//     the sender's 32-channel row slice (coalesced loads, prefetched one group of 4 edges ahead),
//     the edge's coefficients (broadcast shared-memory reads), w from TMEM, and the generated
//     contraction accumulate the receiver's message in registers. At a receiver boundary the
//     warps that share a channel slice add their path subsets in a fixed order and one stores.
// No cross-lane reduction and no atomics; the result is bitwise reproducible. Every mbarrier wait
// is bounded; on timeout the kernel records an error code and exits cleanly.
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"
#include "etp_tc_common.h"

namespace etp {
namespace cm {
namespace {

using tc::canon;
using tc::fence_proxy_async;
using tc::idesc_tf32;
using tc::kTmemCols;
using tc::mbar_arrive_lane0;
using tc::mbar_init;
using tc::mbar_wait;
using tc::mma_commit;
using tc::mma_tf32;
using tc::smem_desc;
using tc::split_tf32;
using tc::sptr;
using tc::tc_fence_after;
using tc::tc_fence_before;
using tc::warp_wait;

constexpr int kCons = 4;                 // consumer warps = TMEM lane quadrants
constexpr int kSetup = kCons;            // setup + MMA warp
constexpr int kLoader = kCons + 1;       // sender-row loader warp
constexpr int kThreads = 32 * (kCons + 2);
constexpr int kNXS = 3;                  // sender-row stages (one MMA batch each)
constexpr int kNB = 16;                  // edges per MMA batch (N)
constexpr int kNPS = 4;                  // setup ring depth (rounds of 32 edges)

template <int L, int C>
struct CmCfg {
  static constexpr int D = Gen<L>::D;
  static constexpr int P = Gen<L>::P;
  static constexpr int NSL = C / 32;     // channel slices
  static constexpr int G = 4 / NSL;      // path subsets
  using Lay = etp_gen::CmLayout<L, G>;
  static constexpr int NBLK = Lay::NBLK;
  static constexpr int MW = Lay::MW;
  static constexpr int BCOLS = NBLK * kNB;
  static constexpr int NS = (kTmemCols / BCOLS) < 4 ? (kTmemCols / BCOLS) : 4;   // TMEM batch ring
  static constexpr int OFF_A = 1024;                               // [blk][hl][128 x 8]
  static constexpr int OFF_B = OFF_A + NBLK * 2 * 4096;            // [round][half][hl][16 x 8]
  static constexpr int OFF_M = OFF_B + kNPS * 2 * 2 * 512;         // [round][32][MW]
  static constexpr int OFF_J = OFF_M + kNPS * 32 * MW * 4;         // [round][32] senders
  static constexpr int OFF_I = OFF_J + kNPS * 32 * 4;              // [round][32] receivers
  static constexpr int OFF_C = OFF_I + kNPS * 32 * 4;              // [slice][subset][D][32] combine
  static constexpr int OFF_X = ((OFF_C + NSL * G * D * 32 * 4) + 127) / 128 * 128;   // [stage][16][row]
  static constexpr int ROWB = D * C * 4;                           // one sender row (bytes)
  // sender rows staged in shared memory by bulk copies when they fit, else loaded by the consumers
  static constexpr bool XSTAGE = OFF_X + kNXS * kNB * ROWB <= 227 * 1024;
  static constexpr int END = XSTAGE ? OFF_X + kNXS * kNB * ROWB : OFF_X;
  static constexpr int SMEM = END < 118 * 1024 ? 118 * 1024 : END;  // one CTA per SM (all TMEM)
  static_assert(NS >= 2, "TMEM ring");
  static_assert(END <= 227 * 1024, "shared memory budget");
  static_assert((MW / 4) % 2 == 1, "coefficient rows: odd float4 stride (conflict-free stores)");
};

struct CmArgs {
  int n_nodes;
  int dim;
  int n_edges;
  float inv_rc;
  const int* row_ptr;
  const int* sender;
  const float* edge_vec;
  const float* x;
  const float* wa;     // pre-split W^T blocks [blk][hl][128 x 8 canonical]
  float* out;
  int* err;
};

// W^T blocks: row r of block blk is (path Lay::path[g][blk], channel 32 sl + r % 32) with
// quadrant r / 32 = NSL g + sl; tf32 hi / lo in canonical K-major order. Clears the status word.
template <int L, int C>
__global__ void k_cm_prep(const float* __restrict__ W, float* __restrict__ wa) {
  using G = CmCfg<L, C>;
  const int total = G::NBLK * 2 * 128 * 8;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int blk = i / (2 * 1024);
    const int rem = i - blk * 2 * 1024;
    const int hl = rem / 1024;
    const int e = rem - hl * 1024;
    const int r = e / 8, b = e % 8;
    const int qq = r / 32;
    const int g = qq / G::NSL, sl = qq % G::NSL;
    const int p = G::Lay::path_at(g, blk);
    const int u = sl * 32 + (r % 32);
    const float v = p >= 0 ? W[(b * G::P + p) * C + u] : 0.0f;
    float hi, lo;
    split_tf32(v, &hi, &lo);
    wa[(blk * 2 + hl) * 1024 + canon(r, b)] = hl ? lo : hi;
  }
}

__device__ __forceinline__ int lower_bound_ptr(const int* __restrict__ ptr, int n, int key) {
  int lo = 0, hi = n;   // first r in [0, n] with ptr[r] >= key
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (ptr[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}

template <int L, int C>
__global__ void __launch_bounds__(kThreads, 1) k_fwd_cm(CmArgs a) {
  using G = CmCfg<L, C>;
  using Lay = typename G::Lay;
  constexpr int D = G::D, NBLK = G::NBLK, MW = G::MW, NS = G::NS, BCOLS = G::BCOLS;
  constexpr int NSL = G::NSL, NG = G::G;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* mready = reinterpret_cast<uint64_t*>(smem);    // [kNPS] setup round written
  uint64_t* sfree = mready + kNPS;                          // [kNPS] round consumed
  uint64_t* tfull = sfree + kNPS;                           // [NS] batch MMAs done
  uint64_t* tempty = tfull + NS;                            // [NS] batch consumed
  uint64_t* aload = tempty + NS;                            // W^T blocks landed
  uint64_t* cready = aload + 1;                             // [NSL] subset partials written
  uint64_t* cdone = cready + NSL;                           // [NSL] partials consumed
  uint64_t* xfull = cdone + NSL;                            // [kNXS] sender rows landed
  uint64_t* xfree = xfull + kNXS;                           // [kNXS] sender rows consumed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(xfree + kNXS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* Ab = reinterpret_cast<float*>(smem + G::OFF_A);
  float* Bb = reinterpret_cast<float*>(smem + G::OFF_B);
  float* Mb = reinterpret_cast<float*>(smem + G::OFF_M);
  int* Jb = reinterpret_cast<int*>(smem + G::OFF_J);
  int* Ib = reinterpret_cast<int*>(smem + G::OFF_I);
  float* Cb = reinterpret_cast<float*>(smem + G::OFF_C);
  float* Xb = reinterpret_cast<float*>(smem + G::OFF_X);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // receivers [r0, r1) of this CTA, cut by edge count
  const long long E = a.n_edges;
  const int r0 = blockIdx.x == 0 ? 0 : lower_bound_ptr(a.row_ptr, a.n_nodes, static_cast<int>(E * blockIdx.x / gridDim.x));
  const int r1 = blockIdx.x + 1 == gridDim.x
                     ? a.n_nodes
                     : lower_bound_ptr(a.row_ptr, a.n_nodes, static_cast<int>(E * (blockIdx.x + 1) / gridDim.x));
  const int e0 = a.row_ptr[r0];
  const int e1 = a.row_ptr[r1 > r0 ? r1 : r0];
  const int n_e = e1 - e0;
  const int n_batches = (n_e + kNB - 1) / kNB;
  const int n_rounds = (n_e + 31) / 32;

  if constexpr (G::XSTAGE)
    for (int i = threadIdx.x; i < kNXS * kNB * G::ROWB / 16; i += blockDim.x)
      reinterpret_cast<float4*>(Xb)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNPS; ++i) {
      mbar_init(mready + i, 1);
      mbar_init(sfree + i, kCons);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(tfull + i, 1);
      mbar_init(tempty + i, kCons);
    }
    mbar_init(aload, 1);
    for (int i = 0; i < NSL; ++i) {
      mbar_init(cready + i, NG > 1 ? NG - 1 : 1);
      mbar_init(cdone + i, 1);
    }
    for (int i = 0; i < kNXS; ++i) {
      mbar_init(xfull + i, 1);
      mbar_init(xfree + i, kCons);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kSetup) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sptr(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kLoader) {
    // ---------------------------------------------------------------- sender-row loader warp
    // per batch: the 16 senders' rows (ROWB contiguous bytes each) by cp.async.bulk into a
    // stage of the ring, completion counted in bytes on the stage's mbarrier
    if constexpr (G::XSTAGE) {
      bool ok = true;
      for (int b = 0; b < n_batches && ok; ++b) {
        const int t = b >> 1, h = b & 1, s = t % kNPS, xs = b % kNXS;
        if (h == 0) ok = warp_wait(mready + s, (t / kNPS) & 1, abort_flag, a.err, 71);
        if (ok && b >= kNXS) ok = warp_wait(xfree + xs, ((b / kNXS) - 1) & 1, abort_flag, a.err, 72);
        if (!ok) break;
        const int j = lane < 16 ? Jb[s * 32 + 16 * h + lane] : -1;
        const unsigned valid = __ballot_sync(kFull, j >= 0);
        if (lane == 0) tc::mbar_expect_tx(xfull + xs, __popc(valid) * G::ROWB);
        __syncwarp();
        if (j >= 0)
          tc::bulk_g2s(Xb + (xs * kNB + lane) * (G::ROWB / 4), a.x + static_cast<size_t>(j) * a.dim, G::ROWB,
                       xfull + xs);
      }
    }
    __syncwarp();
  } else if (warp == kSetup) {
    // ---------------------------------------------------------------- setup + MMA warp
    bool ok = true;
    if (lane == 0 && n_batches > 0) {
      tc::mbar_expect_tx(aload, NBLK * 2 * 4096);
      tc::bulk_g2s(Ab, a.wa, NBLK * 2 * 4096, aload);
      ok = mbar_wait(aload, 0, abort_flag, a.err, 51);
    }
    ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    constexpr uint32_t idesc = idesc_tf32(kNB);
    // the next round's edge vectors and senders are loaded one round ahead
    float nvx = 0.f, nvy = 0.f, nvz = 0.f;
    int nj = -1;
    auto load_raw = [&](int t) {
      const int e = e0 + 32 * t + lane;
      nj = -1;
      if (e < e1) {
        nvx = a.edge_vec[3 * e];
        nvy = a.edge_vec[3 * e + 1];
        nvz = a.edge_vec[3 * e + 2];
        nj = a.sender[e];
      }
    };
    if (n_rounds > 0) load_raw(0);
    int rbase = r0;   // receiver of an edge at or before the round's first edge
    for (int t = 0; t < n_rounds && ok; ++t) {
      const int s = t % kNPS;
      if (t >= kNPS) {
        ok = warp_wait(sfree + s, ((t / kNPS) - 1) & 1, abort_flag, a.err, 52);
        if (!ok) break;
      }
      const int e = e0 + 32 * t + lane;
      const bool valid = e < e1;
      const float vx = nvx, vy = nvy, vz = nvz;
      const int j = nj;
      if (t + 1 < n_rounds) load_raw(t + 1);
      // receiver of edge e = the last r with row_ptr[r] <= e: count the row pointers after rbase,
      // 32 per window (one per lane), that do not exceed e; row_ptr[r1] = e1 ends every search
      int i = -1;
      {
        int base = rbase;
        bool done = !valid;
        while (__any_sync(kFull, !done)) {
          const int idx = base + 1 + lane;
          const int rp = a.row_ptr[idx < r1 ? idx : r1];
          int cnt = 0;
#pragma unroll
          for (int k = 0; k < 32; ++k) cnt += __shfl_sync(kFull, rp, k) <= e ? 1 : 0;
          if (!done && cnt < 32) {
            i = base + cnt;
            done = true;
          }
          base += 32;
        }
        const int n_valid = e1 - (e0 + 32 * t) < 32 ? e1 - (e0 + 32 * t) : 32;
        rbase = __shfl_sync(kFull, i, n_valid - 1);
      }
      float R[kNumBasis], dR[kNumBasis];
      float row[MW];
      if (valid) {
        const float dd = sqrtf(vx * vx + vy * vy + vz * vz);
        const float inv_d = dd > 0.0f ? 1.0f / dd : 0.0f;
        float Y[D];
        Gen<L>::sh(vx * inv_d, vy * inv_d, vz * inv_d, Y);
        radial_basis<false>(dd, a.inv_rc, R, dR);
        if constexpr (L == 1 && NG == 1) etp_gen::cm_coef_1_1(Y, row);
        if constexpr (L == 1 && NG == 2) etp_gen::cm_coef_1_2(Y, row);
        if constexpr (L == 1 && NG == 4) etp_gen::cm_coef_1_4(Y, row);
        if constexpr (L == 2 && NG == 1) etp_gen::cm_coef_2_1(Y, row);
        if constexpr (L == 2 && NG == 2) etp_gen::cm_coef_2_2(Y, row);
        if constexpr (L == 2 && NG == 4) etp_gen::cm_coef_2_4(Y, row);
      } else {
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) R[b] = 0.0f;
#pragma unroll
        for (int c = 0; c < MW; ++c) row[c] = 0.0f;
      }
      float4* mrow = reinterpret_cast<float4*>(Mb + (s * 32 + lane) * MW);
#pragma unroll
      for (int c4 = 0; c4 < MW / 4; ++c4)
        mrow[c4] = make_float4(row[4 * c4], row[4 * c4 + 1], row[4 * c4 + 2], row[4 * c4 + 3]);
      Jb[s * 32 + lane] = j;
      Ib[s * 32 + lane] = i;
      {
        float h[kNumBasis], l[kNumBasis];
#pragma unroll
        for (int b = 0; b < kNumBasis; ++b) split_tf32(R[b], &h[b], &l[b]);
        float* bt = Bb + ((s * 2 + (lane >> 4)) * 2) * 128;   // [round][half][hl][16 x 8]
        const int rr = lane & 15;
        *reinterpret_cast<float4*>(bt + canon(rr, 0)) = make_float4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<float4*>(bt + canon(rr, 4)) = make_float4(h[4], h[5], h[6], h[7]);
        *reinterpret_cast<float4*>(bt + 128 + canon(rr, 0)) = make_float4(l[0], l[1], l[2], l[3]);
        *reinterpret_cast<float4*>(bt + 128 + canon(rr, 4)) = make_float4(l[4], l[5], l[6], l[7]);
      }
      fence_proxy_async();
      __syncwarp();
      mbar_arrive_lane0(mready + s, lane);
      if (lane == 0) {
        for (int h = 0; h < 2 && ok; ++h) {
          const int b = 2 * t + h;
          if (b >= n_batches) break;
          const int ts = b % NS;
          if (b >= NS) ok = mbar_wait(tempty + ts, ((b / NS) - 1) & 1, abort_flag, a.err, 53);
          if (!ok) break;
          tc_fence_after();
          const float* bt = Bb + ((s * 2 + h) * 2) * 128;
          const uint64_t bh = smem_desc(sptr(bt)), bl = smem_desc(sptr(bt + 128));
#pragma unroll 1
          for (int blk = 0; blk < NBLK; ++blk) {
            const uint32_t d = tmem + ts * BCOLS + blk * kNB;
            const uint64_t ah = smem_desc(sptr(Ab + (blk * 2) * 1024)), al = smem_desc(sptr(Ab + (blk * 2 + 1) * 1024));
            mma_tf32(d, ah, bh, idesc, 0u);
            mma_tf32(d, ah, bl, idesc, 1u);
            mma_tf32(d, al, bh, idesc, 1u);
          }
          mma_commit(tfull + ts);
        }
      }
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers
    const int q = warp;
    const int sl = q % NSL, g = q / NSL;
    const int u = sl * 32 + lane;
    // the warp's path subset is a compile-time constant inside run()
    auto run = [&](auto sgc) {
      constexpr int SG = decltype(sgc)::value;
      constexpr int MOFF = Lay::off[SG];
      constexpr int MWID = Lay::width[SG];
      float acc[D];
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = 0.0f;
      int ri = -1;        // receiver held in acc
      int next_r = r0;    // first receiver not yet written
      [[maybe_unused]] uint32_t n_fl = 0;
      bool ok = true;

      // Receiver rr is complete with partial sums v: the subsets of this channel slice are added
      // in order (g = 0, 1, ...) and written by g == 0, after zeroing the rows without edges
      // that precede it. The hand-over between the warps of a slice goes through shared memory
      // with bounded mbarrier waits.
      auto finish = [&](float (&v)[D], int rr) -> bool {
        if constexpr (NG > 1) {
          if constexpr (SG > 0) {
            if (n_fl > 0 && !warp_wait(cdone + sl, (n_fl - 1) & 1, abort_flag, a.err, 63)) return false;
            float* cb = Cb + ((sl * NG + SG) * D) * 32 + lane;
#pragma unroll
            for (int c = 0; c < D; ++c) cb[c * 32] = v[c];
            __syncwarp();
            mbar_arrive_lane0(cready + sl, lane);
          } else {
            if (!warp_wait(cready + sl, n_fl & 1, abort_flag, a.err, 64)) return false;
            for (int hh = 1; hh < NG; ++hh) {
              const float* ch = Cb + ((sl * NG + hh) * D) * 32 + lane;
#pragma unroll
              for (int c = 0; c < D; ++c) v[c] += ch[c * 32];
            }
            __syncwarp();
            mbar_arrive_lane0(cdone + sl, lane);
          }
          ++n_fl;
        }
        if constexpr (SG == 0) {
          for (int z = next_r; z < rr; ++z) {
            float* op = a.out + static_cast<size_t>(z) * a.dim + u;
#pragma unroll
            for (int c = 0; c < D; ++c) op[c * C] = 0.0f;
          }
          float* op = a.out + static_cast<size_t>(rr) * a.dim + u;
#pragma unroll
          for (int c = 0; c < D; ++c) op[c * C] = v[c];
        }
        next_r = rr + 1;
        return true;
      };

      for (int t = 0; t < n_rounds && ok; ++t) {
        const int s = t % kNPS;
        ok = warp_wait(mready + s, (t / kNPS) & 1, abort_flag, a.err, 61);
        if (!ok) break;
        const int* Jr = Jb + s * 32;
        const int* Ir = Ib + s * 32;
        const float* Mr = Mb + s * 32 * MW + MOFF;
        const int n_round = n_e - 32 * t < 32 ? n_e - 32 * t : 32;
        // x of the round's edges: staged rows (XSTAGE) or, else, loaded one group of 4 edges ahead
        float xn[4][D];
        auto load_group = [&](int k0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int k = k0 + kk;
            const int jj = k < n_round ? Jr[k] : -1;
            const float* xs = a.x + static_cast<size_t>(jj < 0 ? 0 : jj) * a.dim + u;
#pragma unroll
            for (int c = 0; c < D; ++c) xn[kk][c] = jj >= 0 ? __ldg(xs + c * C) : 0.0f;
          }
        };
        if constexpr (!G::XSTAGE) load_group(0);
        for (int h = 0; h < 2 && ok; ++h) {
          const int b = 2 * t + h;
          if (b >= n_batches) break;
          const int ts = b % NS;
          const int xs = b % kNXS;
          ok = warp_wait(tfull + ts, (b / NS) & 1, abort_flag, a.err, 62);
          if (ok && G::XSTAGE) ok = warp_wait(xfull + xs, (b / kNXS) & 1, abort_flag, a.err, 65);
          if (!ok) break;
          tc_fence_after();
          const int nb = n_round - 16 * h < 16 ? n_round - 16 * h : 16;
          for (int k4 = 0; k4 < 4 && ok; ++k4) {
            if (4 * k4 >= nb) break;
            const int kb = 16 * h + 4 * k4;       // first edge of the group within the round
            // edges past the end of the range in the group carry w = 0 (zero radial rows) and
            // finite x (zeroed or older rows), so they add nothing
            float xc[4][D];
            if constexpr (G::XSTAGE) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const float* xr = Xb + (xs * kNB + 4 * k4 + kk) * (G::ROWB / 4) + u;
#pragma unroll
                for (int c = 0; c < D; ++c) xc[kk][c] = xr[c * C];
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int c = 0; c < D; ++c) xc[kk][c] = xn[kk][c];
              if (kb + 4 < n_round) load_group(kb + 4);
            }
            uint32_t wv[NBLK][4];
            const uint32_t tb = tmem + (static_cast<uint32_t>(32 * q) << 16) + ts * BCOLS + 4 * k4;
#pragma unroll
            for (int blk = 0; blk < NBLK; ++blk) tmem_ld4(tb + blk * kNB, wv[blk]);
            tc::tmem_wait_ld();
            float pend[4][D];
            int pend_r[4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int k = kb + kk;
              const int i = Ir[k];
              pend_r[kk] = -1;
              if (i >= 0 && i != ri) {   // a new receiver starts: the previous one is complete
                if (ri >= 0) {
#pragma unroll
                  for (int c = 0; c < D; ++c) pend[kk][c] = acc[c];
                  pend_r[kk] = ri;
                }
#pragma unroll
                for (int c = 0; c < D; ++c) acc[c] = 0.0f;
                ri = i;
              }
              float mv[MWID];
              const float4* m4 = reinterpret_cast<const float4*>(Mr + k * MW);
#pragma unroll
              for (int c4 = 0; c4 < MWID / 4; ++c4) {
                const float4 v = m4[c4];
                mv[4 * c4] = v.x; mv[4 * c4 + 1] = v.y; mv[4 * c4 + 2] = v.z; mv[4 * c4 + 3] = v.w;
              }
              auto wf = [&](auto pc) -> float {
                constexpr int slot = decltype(pc)::value;
                return __uint_as_float(wv[slot][kk]);
              };
              if constexpr (L == 1 && NG == 1) etp_gen::cm_fwd_1_1_0(mv, wf, xc[kk], acc);
              if constexpr (L == 1 && NG == 2 && SG == 0) etp_gen::cm_fwd_1_2_0(mv, wf, xc[kk], acc);
              if constexpr (L == 1 && NG == 2 && SG == 1) etp_gen::cm_fwd_1_2_1(mv, wf, xc[kk], acc);
              if constexpr (L == 1 && NG == 4 && SG == 0) etp_gen::cm_fwd_1_4_0(mv, wf, xc[kk], acc);
              if constexpr (L == 1 && NG == 4 && SG == 1) etp_gen::cm_fwd_1_4_1(mv, wf, xc[kk], acc);
              if constexpr (L == 1 && NG == 4 && SG == 2) etp_gen::cm_fwd_1_4_2(mv, wf, xc[kk], acc);
              if constexpr (L == 1 && NG == 4 && SG == 3) etp_gen::cm_fwd_1_4_3(mv, wf, xc[kk], acc);
              if constexpr (L == 2 && NG == 1) etp_gen::cm_fwd_2_1_0(mv, wf, xc[kk], acc);
              if constexpr (L == 2 && NG == 2 && SG == 0) etp_gen::cm_fwd_2_2_0(mv, wf, xc[kk], acc);
              if constexpr (L == 2 && NG == 2 && SG == 1) etp_gen::cm_fwd_2_2_1(mv, wf, xc[kk], acc);
              if constexpr (L == 2 && NG == 4 && SG == 0) etp_gen::cm_fwd_2_4_0(mv, wf, xc[kk], acc);
              if constexpr (L == 2 && NG == 4 && SG == 1) etp_gen::cm_fwd_2_4_1(mv, wf, xc[kk], acc);
              if constexpr (L == 2 && NG == 4 && SG == 2) etp_gen::cm_fwd_2_4_2(mv, wf, xc[kk], acc);
              if constexpr (L == 2 && NG == 4 && SG == 3) etp_gen::cm_fwd_2_4_3(mv, wf, xc[kk], acc);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              if (pend_r[kk] >= 0 && ok) ok = finish(pend[kk], pend_r[kk]);
          }
          if (!ok) break;
          tc_fence_before();
          __syncwarp();
          mbar_arrive_lane0(tempty + ts, lane);
          if constexpr (G::XSTAGE) mbar_arrive_lane0(xfree + xs, lane);
        }
        if (!ok) break;
        __syncwarp();
        mbar_arrive_lane0(sfree + s, lane);
      }
      if (ok && ri >= 0) ok = finish(acc, ri);
      if (ok && SG == 0)
        for (int z = next_r; z < r1; ++z) {
          float* op = a.out + static_cast<size_t>(z) * a.dim + u;
#pragma unroll
          for (int c = 0; c < D; ++c) op[c * C] = 0.0f;
        }
    };
    if (g == 0) run(etp_gen::IC<0>{});
    if constexpr (NG > 1) if (g == 1) run(etp_gen::IC<1>{});
    if constexpr (NG > 2) if (g == 2) run(etp_gen::IC<2>{});
    if constexpr (NG > 3) if (g == 3) run(etp_gen::IC<3>{});
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSetup) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

int g_cm_sms = 0;
int cm_num_sms() {
  if (g_cm_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_cm_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_cm_sms <= 0) g_cm_sms = 148;
  }
  return g_cm_sms;
}

// Workspace: [W^T blocks][status word]
template <int L, int C>
size_t cm_ws_bytes() {
  return align256(static_cast<size_t>(CmCfg<L, C>::NBLK) * 2 * 4096) + 256;
}

template <int L, int C>
etp_status cm_launch(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                     const float* edge_vec, const float* x, const float* W, float* out, void* ws, cudaStream_t s) {
  using G = CmCfg<L, C>;
  float* wa = static_cast<float*>(ws);
  k_cm_prep<L, C><<<16, 256, 0, s>>>(W, wa);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "channel-major forward prep");
  e = cudaFuncSetAttribute(k_fwd_cm<L, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return cuda_status(e, "channel-major forward smem attribute");
  CmArgs a;
  a.n_nodes = n_nodes;
  a.dim = c.dim;
  a.n_edges = n_edges;
  a.inv_rc = 1.0f / c.r_cut;
  a.row_ptr = row_ptr;
  a.sender = sender;
  a.edge_vec = edge_vec;
  a.x = x;
  a.wa = wa;
  a.out = out;
  a.err = c.status_dev;
  k_fwd_cm<L, C><<<cm_num_sms(), kThreads, G::SMEM, s>>>(a);
  return cuda_status(cudaGetLastError(), "channel-major forward launch");
}

template <int L>
etp_status cm_dispatch_c(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                         const float* edge_vec, const float* x, const float* W, float* out, void* ws,
                         cudaStream_t s) {
  switch (c.channels) {
    case 32: return cm_launch<L, 32>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
    case 64: return cm_launch<L, 64>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
    case 128: return cm_launch<L, 128>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
  }
  set_error("channel-major forward: unsupported channel count");
  return ETP_ERR_UNSUPPORTED;
}

template <int L>
size_t cm_ws_c(int channels) {
  switch (channels) {
    case 32: return cm_ws_bytes<L, 32>();
    case 64: return cm_ws_bytes<L, 64>();
    default: return cm_ws_bytes<L, 128>();
  }
}

}  // namespace

bool supported(const Ctx& c) {
  return (c.lmax == 1 || c.lmax == 2) && (c.channels == 32 || c.channels == 64 || c.channels == 128);
}

size_t workspace_bytes(const Ctx& c) {
  if (!supported(c)) return 0;
  return c.lmax == 1 ? cm_ws_c<1>(c.channels) : cm_ws_c<2>(c.channels);
}

etp_status launch(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                  const float* edge_vec, const float* x, const float* W, float* out, void* ws, cudaStream_t s) {
  if (c.lmax == 1) return cm_dispatch_c<1>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
  if (c.lmax == 2) return cm_dispatch_c<2>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
  set_error("channel-major forward: unsupported lmax");
  return ETP_ERR_UNSUPPORTED;
}

etp_status status(const Ctx& c, const void* ws, cudaStream_t s) {
  (void)ws;
  return read_status(c, s, "channel-major forward");
}

}  // namespace cm
}  // namespace etp

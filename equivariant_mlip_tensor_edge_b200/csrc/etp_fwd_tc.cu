// Fused forward edge convolution with the radial projection on the 5th-generation tensor cores.
//
// Work unit ("group"): four receivers times a range of 16 channels. A persistent CTA per SM walks
// a contiguous block of groups (receivers outer, channel ranges inner: the per-edge geometry of
// four receivers is computed once and reused for all their channel ranges).
//
// Per group, the work is cut into CTA-wide items (channel pass p of K channels, 32-edge tile s):
//   producer warp 4 (lane 0): issues w = R W for the item as three kind::tf32 MMAs (hi*hi +
//     hi*lo + lo*hi of the tf32 split, fp32 accumulation; M = 128 edges, N = K P rounded up to
//     16, K = 8 basis functions) into a ring of TMEM slots, and streams the unit's pre-split W^T
//     slices with cp.async.bulk.
//   consumer warps 0..3: warp q owns receiver q of the group (TMEM lane quadrant q), one edge
//   per lane. Per receiver round (<= 128 edges): setup of the direction, real spherical
//   harmonics Y (shared memory), radial basis R_b(d) as tf32 hi/lo rows of the MMA A tiles, and
//   the sender index. Per item: the lane's sender row of the pass (D components x K channels,
//   whole 32-byte sectors) arrives by cp.async one item ahead in a per-warp two-stage buffer;
//   w comes from TMEM via tcgen05.ld; unrolled Clebsch-Gordan code accumulates the message in
//   registers across the receiver's tiles. Per pass: one fixed-order cross-lane sum through
//   shared memory and a store.
//
// Synchronisation: mbarriers (TMEM slot full/empty, setup ready/free,
// weight slices loaded/free). Every wait is bounded; on timeout the kernel records an error code
// and aborts cleanly. A receiver's sums never leave its warp: no atomics, fixed order.
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"
#include "etp_tc_common.h"

namespace etp {
namespace tc {
namespace {

constexpr int kQuads = 4;                     // receivers per group (TMEM lane quadrants)
constexpr int kThreads = 32 * (kQuads + 1);
constexpr int kUnitC = 16;                    // channels per work unit
constexpr int kStages = 2;                    // gather stages per consumer warp

template <int L>
struct Cfg {
  static constexpr int D = Gen<L>::D;
  static constexpr int P = Gen<L>::P;
  static constexpr int K = L >= 3 ? 4 : 8;                     // channels per pass
  static constexpr int SMAX = 4;                               // 32-edge tiles per receiver round
  static constexpr int NPASS = kUnitC / K;
  static constexpr int PPC = 32 / K;                           // paths per 32-column TMEM chunk
  static constexpr int NCOL = ((K * P + 15) / 16) * 16;        // MMA N
  static constexpr int NSLOT = kTmemCols / NCOL;
  static constexpr int ROWB = D * K * 4;                       // gathered bytes per edge and pass
  static constexpr int SLOTB = ROWB + 16;                      // padded: conflict-free row reads
  static constexpr int STAGEB = 32 * SLOTB;                    // one warp's stage
  static constexpr int V = D * K;                              // values per lane per pass
  static constexpr int VS = 4 * ((V / 4) | 1);                 // reduction row stride (odd float4 count)
  static_assert(VS * 4 <= SLOTB, "the reduction rows fit a gather stage");
  static constexpr int WSLICE = 2 * NCOL * 32;                 // bytes: hi + lo of one pass
  static constexpr int WBUF = NPASS * WSLICE;                  // one unit
  static constexpr int MAXRG = 64;                             // receiver groups cached per CTA
  // shared memory map (bytes)
  static constexpr int OFF_G = 1024;                           // cached row pointers
  static constexpr int OFF_A = OFF_G + 2048;                  // row-pointer cache: <= 2048 B
  static constexpr int OFF_W = OFF_A + SMAX * 2 * 4096;
  static constexpr int OFF_Y = OFF_W + 2 * WBUF;
  static constexpr int OFF_J = OFF_Y + kQuads * SMAX * D * 32 * 4;
  static constexpr int OFF_K = OFF_J + kQuads * SMAX * 32 * 4;   // [quad][tile][32] path masks
  static constexpr int OFF_X = OFF_K + kQuads * SMAX * 32 * 4;
  static constexpr int END = OFF_X + kQuads * kStages * STAGEB;
  static constexpr int SMEM = END < 118 * 1024 ? 118 * 1024 : END;   // > half an SM: one CTA per SM
  static_assert(END <= 227 * 1024, "shared memory budget");
  static_assert(OFF_A % 1024 == 0, "A tiles alignment");
  static_assert((MAXRG * kQuads + 8) * 4 <= 2048, "row-pointer cache");
  static_assert(ROWB % 16 == 0 && SLOTB % 16 == 0, "bulk copy granularity");
};

struct Args {
  int n_nodes;
  int C;
  int dim;
  int n_units;        // ceil(C / 16)
  int n_groups;       // ceil(n_nodes / 4) * n_units
  float inv_rc;
  const int* row_ptr;
  const int* sender;
  const float* edge_vec;
  const float* x;
  const float* wt;    // pre-split weights, [unit][pass][hi/lo][NCOL x 8 canonical]
  const uint32_t* mask;   // per-edge path mask (bit p: path p on), or null
  float* out;
  int* err;
};

// Group geometry from the CTA's cached row pointers (rp[q'] = row_ptr[4 rg_beg + q']).
struct GroupInfo {
  int rg, unit, rounds, nbatch;   // nbatch: valid 4-channel batches of the unit
  int deg[kQuads];
  int beg[kQuads];
};

template <int SMAX>
__device__ __forceinline__ void group_info(const Args& a, const int* rp, int rg_beg, int g, GroupInfo* gi) {
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
__device__ __forceinline__ int tiles_of(int deg, int round) {
  const int rem = deg - round * 32 * SMAX;
  if (rem <= 0) return 0;
  const int t = (rem + 31) / 32;
  return t < SMAX ? t : SMAX;
}

template <int SMAX>
__device__ __forceinline__ int group_tiles(const GroupInfo& gi, int round) {
  int S = 0;
#pragma unroll
  for (int q = 0; q < kQuads; ++q) {
    const int t = tiles_of<SMAX>(gi.deg[q], round);
    S = t > S ? t : S;
  }
  return S;
}

// Per call: wt[unit][pass][hl][canonical NCOL x 8] (row n = K p' + k: W[b][p'][16 unit + K pass + k],
// tf32 hi / lo).
template <int L>
__global__ void k_prep(const float* __restrict__ W, int C, int n_units, float* __restrict__ wt) {
  using G = Cfg<L>;
  constexpr int K = G::K;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int nthr = gridDim.x * blockDim.x;
  const int per_pass = 2 * G::NCOL * 8;
  const int wtotal = n_units * G::NPASS * per_pass;
  for (int i = tid; i < wtotal; i += nthr) {
    const int slab = i / per_pass;            // unit * NPASS + pass
    const int rem = i - slab * per_pass;
    const int hl = rem / (G::NCOL * 8);
    const int e = rem - hl * (G::NCOL * 8);
    const int n = e / 8, kb = e % 8;
    const int p = n / K, k = n % K;
    const int u = slab * K + k;               // channel
    float v = 0.0f;
    if (p < G::P && u < C) v = W[(kb * G::P + p) * C + u];
    float hi, lo;
    split_tf32(v, &hi, &lo);
    wt[slab * per_pass + hl * G::NCOL * 8 + canon(n, kb)] = hl ? lo : hi;
  }
}

// MASKED: a path whose bit is clear in an edge's mask contributes nothing for that edge, and a
// path no edge of the item needs is skipped.
template <int L, bool MASKED>
__global__ void __launch_bounds__(kThreads, 1) k_fwd_tc(Args a) {
  using G = Cfg<L>;
  using Gn = Gen<L>;
  constexpr int D = G::D, K = G::K, V = G::V, VS = G::VS, NCOL = G::NCOL, NSLOT = G::NSLOT;
  constexpr int NPASS = G::NPASS, SMAX = G::SMAX;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* tfull = reinterpret_cast<uint64_t*>(smem);   // [NSLOT]
  uint64_t* tempty = tfull + NSLOT;                       // [NSLOT]
  uint64_t* rready = tempty + NSLOT;
  uint64_t* sfree = rready + 1;
  uint64_t* wload = sfree + 1;    // [2]
  uint64_t* wfree = wload + 2;    // [2]
  uint64_t* drainb = wfree + 2;   // final commit of the producer (abort-safe drain)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drainb + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* rp = reinterpret_cast<int*>(smem + G::OFF_G);
  float* Atile = reinterpret_cast<float*>(smem + G::OFF_A);     // [SMAX][hl][128 x 8 canonical]
  float* Wbuf = reinterpret_cast<float*>(smem + G::OFF_W);      // [2][pass][hl][NCOL x 8]
  float* Ybuf = reinterpret_cast<float*>(smem + G::OFF_Y);      // [quad][tile][D][32]
  int* Jbuf = reinterpret_cast<int*>(smem + G::OFF_J);          // [quad][tile][32]
  uint32_t* Kbuf = reinterpret_cast<uint32_t*>(smem + G::OFF_K); // [quad][tile][32]
  unsigned char* Xbuf = smem + G::OFF_X;                        // [quad][stage][lane][SLOTB]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g_beg = static_cast<int>(static_cast<long long>(a.n_groups) * blockIdx.x / gridDim.x);
  const int g_end = static_cast<int>(static_cast<long long>(a.n_groups) * (blockIdx.x + 1) / gridDim.x);
  const int rg_beg = g_beg / a.n_units;
  const int rg_end = g_end > g_beg ? (g_end - 1) / a.n_units + 1 : rg_beg;
  const int n_rp = (rg_end - rg_beg) * kQuads + 1;

  // cache the row pointers of this CTA's receivers (host guarantees at most MAXRG groups of them)
  for (int i = threadIdx.x; i < n_rp; i += blockDim.x) {
    const int r = rg_beg * kQuads + i;
    rp[i] = a.row_ptr[r < a.n_nodes ? r : a.n_nodes];
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
  if (warp == kQuads) {   // producer warp owns the TMEM allocation
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

  if (warp == kQuads) {
    // ---------------------------------------------------------------- producer warp
    constexpr uint32_t idesc = idesc_tf32(NCOL);
    uint32_t titem = 0, n_setup = 0, n_loads = 0, n_issued = 0;
    int cached_rg = -1, cached_round = -1;
    bool ok = true;
    // weight slices of the k-th group of this CTA go to buffer k & 1; the next group's load is
    // issued once this group's MMAs are issued and the MMAs of the group before (same buffer) ended
    auto load_w = [&](int g, uint32_t n) -> bool {
      if (lane == 0) {
        const int unit = g % a.n_units;
        const int wb = n & 1;
        if (n >= 2 && !mbar_wait(wfree + wb, ((n >> 1) - 1) & 1, abort_flag, a.err, 11)) return false;
        mbar_expect_tx(wload + wb, G::WBUF);
        bulk_g2s(Wbuf + wb * (G::WBUF / 4), a.wt + static_cast<size_t>(unit) * (G::WBUF / 4), G::WBUF, wload + wb);
        ++n_issued;
      }
      return true;
    };
    if (g_beg < g_end) ok = load_w(g_beg, 0);
    for (int g = g_beg; g < g_end && ok; ++g) {
      GroupInfo gi;
      group_info<SMAX>(a, rp, rg_beg, g, &gi);
      const int wb = n_loads & 1;
      const int npass = (gi.nbatch * 4 + K - 1) / K;
      if (lane == 0) ok = mbar_wait(wload + wb, (n_loads >> 1) & 1, abort_flag, a.err, 12);
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
      ++n_loads;
      for (int round = 0; round < gi.rounds && ok; ++round) {
        const int S = group_tiles<SMAX>(gi, round);
        if (gi.rg != cached_rg || round != cached_round) {
          ok = warp_wait(rready, n_setup & 1, abort_flag, a.err, 13);
          ++n_setup;
          cached_rg = gi.rg;
          cached_round = round;
          if (!ok) break;
        }
        tc_fence_after();
        for (int pass = 0; pass < npass && ok; ++pass) {
          for (int s = 0; s < S; ++s) {
            // TMEM ring: w = R W for (pass, s)
            if (lane == 0) {
              const int slot = titem % NSLOT;
              ok = mbar_wait(tempty + slot, ((titem / NSLOT) & 1) ^ 1, abort_flag, a.err, 14);
              if (ok) {
                tc_fence_after();
                const uint32_t d = tmem + slot * NCOL;
                const uint64_t ah = smem_desc(sptr(Atile + (s * 2 + 0) * 1024));
                const uint64_t al = smem_desc(sptr(Atile + (s * 2 + 1) * 1024));
                const float* wsl = Wbuf + wb * (G::WBUF / 4) + pass * (G::WSLICE / 4);
                const uint64_t bh = smem_desc(sptr(wsl));
                const uint64_t bl = smem_desc(sptr(wsl + NCOL * 8));
                mma_tf32(d, ah, bh, idesc, 0u);
                mma_tf32(d, ah, bl, idesc, 1u);
                mma_tf32(d, al, bh, idesc, 1u);
                mma_commit(tfull + slot);
              }
            }
            ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
            ++titem;
          }
        }
      }
      if (lane == 0) mma_commit(wfree + wb);   // completes once every MMA issued so far has finished
      if (ok && g + 1 < g_end) ok = load_w(g + 1, n_loads);
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    }
    // drain, ignoring the abort flag: one more commit tracks every MMA issued so far, and the weight
    // load issued for a group that was never consumed may still be in flight
    if (lane == 0) {
      mma_commit(drainb);
      bool dr = mbar_wait_drain(drainb, 0);
      if (dr && n_issued > n_loads)
        dr = mbar_wait_drain(wload + ((n_issued - 1) & 1), ((n_issued - 1) >> 1) & 1);
      if (!dr) {
        report_code(a.err, 15);
        *abort_flag = 1;
        drained = false;
      }
    }
    drained = __shfl_sync(kFull, drained ? 1 : 0, 0) != 0;
  } else {
    // ---------------------------------------------------------------- consumer warps
    const int q = warp;
    float* Yq = Ybuf + q * (SMAX * D * 32);
    int* Jq = Jbuf + q * (SMAX * 32);
    uint32_t* Kq = Kbuf + q * (SMAX * 32);
    unsigned char* Xw0 = Xbuf + q * kStages * G::STAGEB;
    unsigned char* Xw = Xw0 + lane * G::SLOTB;
    uint32_t titem = 0, n_setup = 0;
    int cached_rg = -1, cached_round = -1;
    bool ok = true;
    for (int g = g_beg; g < g_end && ok; ++g) {
      GroupInfo gi;
      group_info<SMAX>(a, rp, rg_beg, g, &gi);
      const int r = gi.rg * kQuads + q;
      const int deg = gi.deg[q];
      const int npass = (gi.nbatch * 4 + K - 1) / K;
      const int cbase = gi.unit * kUnitC;
      for (int round = 0; round < gi.rounds && ok; ++round) {
        const int S = group_tiles<SMAX>(gi, round);
        const int Sq = tiles_of<SMAX>(deg, round);
        if (gi.rg != cached_rg || round != cached_round) {
          // all consumers must be done with setup n-1 (its items consumed, hence the MMAs and
          // gathers that read the old tiles complete) before anyone overwrites it
          if (n_setup > 0) {
            mbar_arrive_lane0(sfree, lane);
            ok = warp_wait(sfree, (n_setup - 1) & 1, abort_flag, a.err, 22);
            if (!ok) break;
          }
          for (int s = 0; s < Sq; ++s) {
            const int le = round * 32 * SMAX + s * 32 + lane;
            float Y[D];
            float R[kNumBasis], dR[kNumBasis];
#pragma unroll
            for (int c = 0; c < D; ++c) Y[c] = 0.0f;
#pragma unroll
            for (int bb = 0; bb < kNumBasis; ++bb) R[bb] = 0.0f;
            int jj = -1;
            if (le < deg) {
              const int e = gi.beg[q] + le;
              const float vx = a.edge_vec[3 * e], vy = a.edge_vec[3 * e + 1], vz = a.edge_vec[3 * e + 2];
              jj = a.sender[e];
              const float dd = sqrtf(vx * vx + vy * vy + vz * vz);
              const float inv_d = dd > 0.0f ? 1.0f / dd : 0.0f;
              Gn::sh(vx * inv_d, vy * inv_d, vz * inv_d, Y);
              radial_basis<false>(dd, a.inv_rc, R, dR);
            }
            Jq[s * 32 + lane] = jj;
            if constexpr (MASKED) Kq[s * 32 + lane] = jj >= 0 ? a.mask[gi.beg[q] + le] : 0u;
#pragma unroll
            for (int c = 0; c < D; ++c) Yq[(s * D + c) * 32 + lane] = Y[c];
            const int row = 32 * q + lane;
            float h[kNumBasis], l[kNumBasis];
#pragma unroll
            for (int bb = 0; bb < kNumBasis; ++bb) split_tf32(R[bb], &h[bb], &l[bb]);
            float* th = Atile + (s * 2 + 0) * 1024;
            float* tl = Atile + (s * 2 + 1) * 1024;
            *reinterpret_cast<float4*>(th + canon(row, 0)) = make_float4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<float4*>(th + canon(row, 4)) = make_float4(h[4], h[5], h[6], h[7]);
            *reinterpret_cast<float4*>(tl + canon(row, 0)) = make_float4(l[0], l[1], l[2], l[3]);
            *reinterpret_cast<float4*>(tl + canon(row, 4)) = make_float4(l[4], l[5], l[6], l[7]);
          }
          fence_proxy_async();
          __syncwarp();
          mbar_arrive_lane0(rready, lane);
          ok = warp_wait(rready, n_setup & 1, abort_flag, a.err, 23);
          ++n_setup;
          cached_rg = gi.rg;
          cached_round = round;
          if (!ok) break;
        }
        // the sender rows of tile s for a pass, D components x K channels each, into a stage.
        // The K channels of a component are whole 32-byte sectors; the (K / 4) lanes that share an
        // edge fetch its sectors' 16-byte halves in one instruction, so a sector is requested once.
        auto prefetch = [&](int pass, int s, int st) {
          constexpr int PARTS = K / 4;                // 16-byte chunks per component
          constexpr int EPI = 32 / PARTS;             // edges per instruction
          const int jj = Jq[s * 32 + lane];
          const int ch = cbase + pass * K;
          const int part = lane % PARTS;
          const bool in_c = 4 * part < a.C - ch;      // chunk inside C (C is a multiple of 4)
          unsigned char* stage_base = Xw0 + st * G::STAGEB;
#pragma unroll
          for (int it = 0; it < PARTS; ++it) {
            const int e = it * EPI + lane / PARTS;
            const int js = __shfl_sync(kFull, jj, e);
            const float* src = a.x + static_cast<size_t>(js < 0 ? 0 : js) * a.dim + ch + 4 * part;
            unsigned char* dst = stage_base + e * G::SLOTB + part * 16;
            const uint32_t nb = (js >= 0 && in_c) ? 16u : 0u;
#pragma unroll
            for (int c = 0; c < D; ++c) cp_async16(dst + c * K * 4, src + c * a.C, nb);
          }
          cp_async_commit();
        };
        int stage = 0;
        if (Sq > 0) prefetch(0, 0, 0);
        for (int pass = 0; pass < npass && ok; ++pass) {
          float acc[D][K];
#pragma unroll
          for (int c = 0; c < D; ++c)
#pragma unroll
            for (int k = 0; k < K; ++k) acc[c][k] = 0.0f;
          for (int s = 0; s < S; ++s) {
            const int slot = titem % NSLOT;
            const bool mine = s < Sq;
            float xv[D][K];
            if (mine) {
              // this item's rows (the only copies in flight); the lanes that fetched this lane's
              // row are others, and the stage the next copies target was read by every lane before
              cp_async_wait<0>();
              __syncwarp();
              const float4* xs = reinterpret_cast<const float4*>(Xw + stage * G::STAGEB);
#pragma unroll
              for (int c = 0; c < D; ++c)
#pragma unroll
                for (int k4 = 0; k4 < K / 4; ++k4) {
                  const float4 t = xs[c * (K / 4) + k4];
                  xv[c][4 * k4 + 0] = t.x; xv[c][4 * k4 + 1] = t.y;
                  xv[c][4 * k4 + 2] = t.z; xv[c][4 * k4 + 3] = t.w;
                }
              // next item of this lane's receiver: gathered while this one computes
              int np = pass, ns = s + 1;
              if (ns >= Sq) {
                ns = 0;
                ++np;
              }
              if (np < npass) prefetch(np, ns, stage ^ 1);
              stage ^= 1;
            }
            ok = warp_wait(tfull + slot, (titem / NSLOT) & 1, abort_flag, a.err, 21);
            if (!ok) break;
            tc_fence_after();
            if (mine) {
              float Y[D];
#pragma unroll
              for (int c = 0; c < D; ++c) Y[c] = Yq[(s * D + c) * 32 + lane];
              const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16) + slot * NCOL;
              float wch[32];
              // (array bounds spelled G::K: a generic lambda whose parameter is sized by a local
              // constexpr of the kernel template crashes the CUDA 12.9 front end)
              [[maybe_unused]] const uint32_t mbits = MASKED ? Kq[s * 32 + lane] : ~0u;
              auto wf = [&](auto pc, float (&wp)[G::K]) {
                constexpr int p = decltype(pc)::value;
                if constexpr (p % G::PPC == 0) {
                  if constexpr (G::NCOL - 32 * (p / G::PPC) >= 32) tmem_ld32(tbase + 32 * (p / G::PPC), wch);
                  else tmem_ld16(tbase + 32 * (p / G::PPC), wch);
                  tmem_wait_ld();
                }
                constexpr int o = (p % G::PPC) * G::K;
                if constexpr (MASKED) {
                  const bool on = (mbits >> p) & 1u;
#pragma unroll
                  for (int k = 0; k < G::K; ++k) wp[k] = on ? wch[o + k] : 0.0f;
                  return __any_sync(kFull, on);
                } else {
#pragma unroll
                  for (int k = 0; k < G::K; ++k) wp[k] = wch[o + k];
                }
              };
              Gn::template fwd<K>(Y, wf, xv, acc);
            }
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(tempty + slot, lane);
            ++titem;
          }
          if (!ok) break;
          // cross-lane sum of acc through shared memory, then one store (or add, later rounds).
          // The rows go to the gather stage this warp consumed last (no copy targets it; the next
          // one is issued after this sum).
          if (Sq > 0 || round == 0) {
            float* Rw = reinterpret_cast<float*>(Xw0 + (stage ^ 1) * G::STAGEB);
#pragma unroll
            for (int c = 0; c < D; ++c)
#pragma unroll
              for (int k4 = 0; k4 < K / 4; ++k4)
                *reinterpret_cast<float4*>(Rw + lane * VS + c * K + 4 * k4) =
                    make_float4(acc[c][4 * k4], acc[c][4 * k4 + 1], acc[c][4 * k4 + 2], acc[c][4 * k4 + 3]);
            __syncwarp();
            if (r < a.n_nodes) {
              for (int v = lane; v < V; v += 32) {
                const int c = v / K, k = v % K;
                const int ch = cbase + pass * K + k;
                if (ch < a.C) {
                  float col[32];
#pragma unroll
                  for (int l2 = 0; l2 < 32; ++l2) col[l2] = Rw[l2 * VS + v];
#pragma unroll
                  for (int w2 = 16; w2 > 0; w2 >>= 1)
#pragma unroll
                    for (int l2 = 0; l2 < w2; ++l2) col[l2] += col[l2 + w2];
                  const float sum = col[0];
                  float* op = a.out + static_cast<size_t>(r) * a.dim + c * a.C + ch;
                  if (round == 0) *op = sum; else *op += sum;
                }
              }
            }
            __syncwarp();
          }
        }
      }
    }
    cp_async_wait<0>();   // no copy may be in flight past this point (abort paths included)
  }

  // teardown: every thread reaches this barrier exactly once
  tc_fence_before();
  __syncthreads();
  if (warp == kQuads && drained) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

int g_sms = 0;

int num_sms() {
  if (g_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_sms <= 0) g_sms = 148;
  }
  return g_sms;
}

// Workspace: [wt]
template <int L>
size_t wt_bytes(int channels) {
  const int n_units = (channels + kUnitC - 1) / kUnitC;
  return align256(static_cast<size_t>(n_units) * Cfg<L>::WBUF);
}

template <int L>
size_t ws_bytes(int channels, int n_nodes) {
  (void)n_nodes;
  return wt_bytes<L>(channels);
}

template <int L>
etp_status launch(const Ctx& c, int n_nodes, const int* row_ptr, const int* sender, const float* edge_vec,
                  const float* x, const float* W, const uint32_t* a_mask, float* out, void* ws, cudaStream_t s) {
  using G = Cfg<L>;
  const int n_units = (c.channels + kUnitC - 1) / kUnitC;
  float* wt = static_cast<float*>(ws);
  k_prep<L><<<32, 256, 0, s>>>(W, c.channels, n_units, wt);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "forward prep");
  e = a_mask ? cudaFuncSetAttribute(k_fwd_tc<L, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM)
             : cudaFuncSetAttribute(k_fwd_tc<L, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return cuda_status(e, "tc forward smem attribute");
  Args a;
  a.n_nodes = n_nodes;
  a.C = c.channels;
  a.dim = c.dim;
  a.n_units = n_units;
  a.n_groups = ((n_nodes + kQuads - 1) / kQuads) * n_units;
  a.inv_rc = 1.0f / c.r_cut;
  a.row_ptr = row_ptr;
  a.sender = sender;
  a.edge_vec = edge_vec;
  a.x = x;
  a.wt = wt;
  a.mask = a_mask;
  a.out = out;
  a.err = c.status_dev;
  // enough CTAs that no CTA spans more than MAXRG receiver groups (row-pointer cache size)
  long long grid = num_sms();
  const long long n_rg = (n_nodes + kQuads - 1) / kQuads;
  const long long min_grid = (n_rg + G::MAXRG - 3) / (G::MAXRG - 2);
  if (grid < min_grid) grid = min_grid;
  if (grid > a.n_groups) grid = a.n_groups;
  if (a_mask) k_fwd_tc<L, true><<<static_cast<int>(grid), kThreads, G::SMEM, s>>>(a);
  else k_fwd_tc<L, false><<<static_cast<int>(grid), kThreads, G::SMEM, s>>>(a);
  return cuda_status(cudaGetLastError(), "tc forward launch");
}

}  // namespace

size_t forward_tc_workspace_bytes(const Ctx& c, int n_nodes) {
  switch (c.lmax) {
    case 1: return ws_bytes<1>(c.channels, n_nodes);
    case 2: return ws_bytes<2>(c.channels, n_nodes);
    default: return ws_bytes<3>(c.channels, n_nodes);
  }
}

// Synchronises the stream and reads the handle's status word (nonzero: a bounded wait gave up).
etp_status forward_tc_status(const Ctx& c, const void* ws, cudaStream_t s) {
  (void)ws;
  return read_status(c, s, "tensor-core forward");
}

etp_status launch_forward_tc(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                             const float* edge_vec, const float* x, const float* W, float* out, void* ws,
                             cudaStream_t s, const uint32_t* path_mask) {
  (void)n_edges;
  switch (c.lmax) {
    case 1: return launch<1>(c, n_nodes, row_ptr, sender, edge_vec, x, W, path_mask, out, ws, s);
    case 2: return launch<2>(c, n_nodes, row_ptr, sender, edge_vec, x, W, path_mask, out, ws, s);
    case 3: return launch<3>(c, n_nodes, row_ptr, sender, edge_vec, x, W, path_mask, out, ws, s);
  }
  set_error("tc forward: unsupported lmax");
  return ETP_ERR_UNSUPPORTED;
}

}  // namespace tc
}  // namespace etp

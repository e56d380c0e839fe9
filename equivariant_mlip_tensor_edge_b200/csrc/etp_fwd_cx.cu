// Fused forward edge convolution, channel-major with path subsets ("cx"), for l_max <= 2 and at
// most 64 channels.
//
// The CTAs split the canonical (receiver-sorted) edge list into equal contiguous ranges; the warps
// of a CTA walk its range together in batches of N = 16 edges. Lanes hold channels: a receiver's
// message accumulates in registers of the lanes that own its channels, so no cross-lane sums are
// needed, and the sender rows of a batch are staged in shared memory by whole-row bulk copies.
//
// Roles (one persistent CTA per SM, 13 warps):
//   setup warps 8, 9 (even and odd MMA batches): one edge per lane, 32 edges (two batches) per
//     pass: the direction, real spherical harmonics, the radial basis R_b(d) as the tf32 hi/lo
//     rows of the MMA B operand, and the per-edge coefficients M[m3][m1] = sum_m2 C Y[l2 m2] of both
//     path subsets, deduplicated up to sign, stored with the two edges of a pair interleaved.
//   MMA warp 10 (one thread): w^T = W^T R^T on the tensor cores, D[(path, channel)][edge]: one
//     block of 128 rows per path item, three kind::tf32 MMAs (hi*hi + hi*lo + lo*hi) per block,
//     into a two-slot TMEM ring.
//   loader warp 12: one bulk copy per edge of the sender's whole row (dim floats, contiguous) into
//     a ring of batch slots.
//   consumer warps 0..7: warp w reads TMEM lane quadrant q = w % 4. Quadrants 0, 1 run path
//     subset 0 (l1 < l_max) on channels 0..31 and 32..63, quadrants 2, 3 subset 1 (l1 = l_max),
//     so the two subsets read disjoint components of a sender row. The two warps of a quadrant
//     take the two halves of each batch. Edges go in pairs through the packed (f32x2) form of the
//     generated contraction: the lane's sender-row components and the pair's coefficients from
//     shared memory, w from registers loaded by tcgen05.ld. When the receiver changes, the warp
//     hands its partial message to the combine warp through a ring of shared-memory slots.
//   combine warp 11: per receiver, adds the eight partials in a fixed order and stores the row.
//     A receiver whose edges span several CTAs is summed by the CTA that adds its last part (a
//     per-receiver arrival counter, zeroed by the prep kernel), again in a fixed order.
// Every result is bitwise reproducible. Every mbarrier wait is bounded; on timeout the kernel
// records an error code, aborts its loops, drains the tensor-core and copy work it issued, exits.
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"
#include "etp_tc_common.h"

namespace etp {
namespace cx {
namespace {

using tc::bulk_g2s;
using tc::canon;
using tc::fence_proxy_async;
using tc::idesc_tf32;
using tc::kTmemCols;
using tc::kWaitCycles;
using tc::mbar_arrive;
using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::mbar_test;
using tc::mbar_wait;
using tc::mbar_wait_drain;
using tc::mma_commit;
using tc::mma_tf32;
using tc::smem_desc;
using tc::split_tf32;
using tc::sptr;
using tc::tc_fence_after;
using tc::tc_fence_before;
using tc::warp_wait;

constexpr int kQ = 4;                    // TMEM lane quadrants
constexpr int kH = 2;                    // consumer warps per quadrant
constexpr int kCons = kQ * kH;           // consumer warps
constexpr int kSetup0 = kCons;           // geometry warps kSetup0, kSetup0 + 1 (even, odd batches)
constexpr int kMmaWarp = kCons + 2;
constexpr int kCombWarp = kCons + 3;
constexpr int kLoadWarp = kCons + 4;     // sender-row loader
constexpr int kThreads = 32 * (kCons + 5);
constexpr int kGS = 8;                   // geometry ring (batches): per-edge coefficients
constexpr int kRS = kGS / 2;             // B operand ring (MMA batches)
constexpr int kXS = 3;                   // sender-row ring (batches)
constexpr int kNR = 2;                   // receiver ring (partial messages)
constexpr int kN = 16;                   // edges per setup / consumer batch
constexpr int kNM = 2 * kN;              // edges per MMA batch (MMA N): two consecutive batches
constexpr int kEPW = kN / kH;            // edges per consumer warp and batch
constexpr int kMaxC = 64;                // channels: two 32-lane slices
constexpr int kMinEdgesPerCta = 64;

template <int L>
struct Cfg {
  using S0 = etp_gen::CxSub<L, 0>;
  using S1 = etp_gen::CxSub<L, 1>;
  static constexpr int D = (L + 1) * (L + 1);
  static constexpr int P = etp_gen::PathSet<L>::P;
  static constexpr int NB = S0::NP > S1::NP ? S0::NP : S1::NP;   // MMA blocks: one path item each
  static constexpr int SLOTC = NB * kNM;                         // TMEM columns per ring slot
  static constexpr int CW0 = S0::NC, CW1 = S1::NC;
  // coefficient row of an edge pair: both subsets, the two edges interleaved (coefficient k of edge t
  // at 2 k + t), padded to 4 mod 32 floats so that the setup warp's 8-byte stores hit distinct banks
  static constexpr int PW = 2 * (CW0 + CW1) + (4 - (2 * (CW0 + CW1)) % 32 + 32) % 32;
  static constexpr int NOMAX = S0::NO > S1::NO ? S0::NO : S1::NO;
  static constexpr int XROW = kMaxC * D;                         // floats of the largest sender row
  // shared memory map (bytes)
  static constexpr int OFF_WA = 1024;                            // [NB][hi|lo][128 x 8]
  static constexpr int OFF_CF = OFF_WA + NB * 8192;              // [kGS][kN / 2][PW]
  static constexpr int OFF_RB = OFF_CF + kGS * (kN / 2) * PW * 4; // [kRS][hi|lo][kNM x 8]: B operand per MMA batch
  static constexpr int OFF_X = OFF_RB + kRS * 2 * kNM * 32;      // [kXS][kN][dim]
  static constexpr int OFF_PT = OFF_X + kXS * kN * XROW * 4;     // [kNR][kCons][NOMAX][32]
  static constexpr int END = OFF_PT + kNR * kCons * NOMAX * 32 * 4;
  static constexpr int SMEM = END < 118 * 1024 ? 118 * 1024 : END;   // > half an SM: one CTA per SM
  static_assert(2 * SLOTC <= kTmemCols, "two TMEM slots");
  static_assert(PW % 32 == 4 && CW0 % 4 == 0 && CW1 % 4 == 0, "coefficient row layout");
  static_assert(END <= 227 * 1024, "shared memory budget");
  static_assert(OFF_RB % 128 == 0 && OFF_X % 128 == 0 && OFF_WA % 1024 == 0, "operand alignment");
};

struct Args {
  int n_nodes;
  int n_edges;
  int C;
  int dim;
  int G;             // CTAs (edge ranges)
  float inv_rc;
  const int* row_ptr;
  const int* sender;
  const float* edge_vec;
  const float* x;
  const float* W;
  float* out;
  float* gpart;      // [G][2][dim]: partial rows of receivers that span CTAs
  int* cnt;          // [G]: arrivals per spanning receiver (indexed by its first CTA)
  int* err;
};

__device__ __forceinline__ long long range_beg(long long E, int G, int c) { return E * c / G; }

// CTA whose edge range holds canonical edge e (0 <= e < E)
__device__ __forceinline__ int cta_of(long long E, int G, long long e) {
  return static_cast<int>(((e + 1) * G - 1) / E);
}

// receiver of canonical edge e: the r with row_ptr[r] <= e < row_ptr[r + 1]. Warp-wide: the 32
// lanes probe 32 evenly spaced entries per step, so the range shrinks 32-fold per dependent load.
__device__ __forceinline__ int recv_of_warp(const int* __restrict__ row_ptr, int n, int e) {
  const int lane = threadIdx.x & 31;
  // the first index i with row_ptr[i] > e lies in [lo, hi] (hi = n + 1: none yet seen); answer i - 1
  int lo = 0, hi = n + 1;
  while (hi - lo > 32) {
    const int step = (hi - lo + 31) / 32;
    const int idx = lo + lane * step;
    const bool gt = idx < hi && __ldg(row_ptr + idx) > e;
    const unsigned m = __ballot_sync(0xffffffffu, gt);
    if (m == 0) {   // every probe <= e: the first greater index lies after the last probe below hi
      const int lv = (hi - 1 - lo) / step < 31 ? (hi - 1 - lo) / step : 31;
      lo = lo + lv * step + 1;
    } else {
      const int f = __ffs(m) - 1;   // first probe above e: the answer lies in (previous probe, this one]
      const int nhi = lo + f * step;
      lo = f == 0 ? lo : lo + (f - 1) * step + 1;
      hi = nhi;
    }
  }
  const int idx = lo + lane;
  const bool gt = idx < hi && __ldg(row_ptr + idx) > e;
  const unsigned m = __ballot_sync(0xffffffffu, gt);
  const int first = m ? lo + __ffs(m) - 1 : hi;
  return first - 1;
}

__device__ __forceinline__ void tmem_ld2(uint32_t taddr, float (&v)[2]) {
  uint32_t r[2];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr) : "memory");
  v[0] = __uint_as_float(r[0]);
  v[1] = __uint_as_float(r[1]);
}

// Bounded wait for the roles whose latency is hidden (setup, loader, combine): only lane 0 polls,
// and it is suspended in hardware between polls (until the phase completes or the hint runs out),
// so the waiting warp takes no issue slots from the consumer warps on its scheduler.
__device__ __forceinline__ bool warp_wait_lazy(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* err,
                                               int code) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0 && !mbar_test(b, parity)) {
    const long long t0 = clock64();
    while (true) {
      if (tc::mbar_test_sleep(b, parity, 50000u)) break;
      if (*abort_flag) {
        ok = false;
        break;
      }
      if (clock64() - t0 > kWaitCycles) {
        tc::report_code(err, code);
        *abort_flag = 1;
        ok = false;
        break;
      }
    }
  }
  __syncwarp();
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

struct Bars {
  uint64_t tfull[2], tempty[2];
  uint64_t sfull[kGS], sfree[kGS];   // geometry ring: coefficients and B operand written / read
  uint64_t xfull[kXS], xfree[kXS];   // sender-row ring: rows landed / read
  uint64_t rfull[kNR], rempty[kNR];
  uint64_t drain;
  uint32_t tmem_holder;
  int abort_flag;
  int r_begin, r_end;
  int e_beg, e_end;
  int x_last[kXS];   // per slot: the last batch whose sender-row copies were issued into it
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

template <class SUB>
__host__ __device__ constexpr int oidx(int c) {
  for (int i = 0; i < SUB::NO; ++i)
    if (SUB::ocomp(i) == c) return i;
  return -1;
}

// ---------------------------------------------------------------- consumer warps

// Consumer warp of quadrant q (path subset SI = q / 2, channel (q % 2) * 32 + lane), batch half h.
// Edges are taken in pairs: the two edges of a pair run through one packed (f32x2) contraction,
// component .x the first edge, .y the second, each into its own half of the accumulator; the halves
// are added (x + y) when the receiver's message is handed on, so the order of every sum is fixed.
// CT: the channel count when it is a compile-time constant (64), else 0 (a.C at run time).
template <int L, int SI, int CT>
__device__ __forceinline__ bool consume(const Args& a, unsigned char* smem, Bars* bars, int q, int h, uint32_t tmem,
                                        int nb) {
  using G = Cfg<L>;
  using SUB = etp_gen::CxSub<L, SI>;
  constexpr int NX = SUB::NX, NO = SUB::NO, NP = SUB::NP;
  constexpr int PW = G::PW;
  constexpr int CFO = SI == 0 ? 0 : 2 * G::CW0;   // the subset's coefficients within a pair's row
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int C = CT > 0 ? CT : a.C;
  const int dim = CT > 0 ? CT * G::D : a.dim;
  const int ch0 = (q & 1) * 32 + lane;
  const bool chv = CT > 0 ? true : ch0 < C;
  volatile int* abort_flag = &bars->abort_flag;
  const int e_beg = bars->e_beg, e_end = bars->e_end;
  const int r_end = bars->r_end;
  const float* cfbase = reinterpret_cast<const float*>(smem + G::OFF_CF);
  const float* xbase = reinterpret_cast<const float*>(smem + G::OFF_X);
  float* part = reinterpret_cast<float*>(smem + G::OFF_PT);

  int xoff[NX];
#pragma unroll
  for (int i = 0; i < NX; ++i) xoff[i] = SUB::xcomp(i) * C + ch0;
  float2 acc[NO];
#pragma unroll
  for (int o = 0; o < NO; ++o) acc[o] = make_float2(0.0f, 0.0f);

  int cur = bars->r_begin;
  int nxt = __ldg(a.row_ptr + cur + 1);
  int kr = 0;   // index of cur within the CTA's receiver sequence
  // hand the partial message of receiver cur to the combine warp, move to the next receiver
  auto flush = [&]() -> bool {
    const int slot = kr % kNR;
    if (kr >= kNR && !warp_wait(&bars->rempty[slot], ((kr / kNR) - 1) & 1, abort_flag, a.err, 33)) return false;
    float* pp = part + static_cast<size_t>(slot * kCons + warp) * (G::NOMAX * 32);
#pragma unroll
    for (int o = 0; o < NO; ++o) {
      pp[o * 32 + lane] = acc[o].x + acc[o].y;
      acc[o] = make_float2(0.0f, 0.0f);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->rfull[slot]);
    ++kr;
    ++cur;
    nxt = cur < a.n_nodes ? __ldg(a.row_ptr + cur + 1) : 0x7fffffff;
    return true;
  };

  bool ok = true;
  for (int k = 0; k < nb && ok; ++k) {
    const int m = k >> 1, ts = m & 1, sl = k % kGS, xl = k % kXS;   // MMA batch m covers batches 2 m, 2 m + 1
    const int base = e_beg + k * kN + h * kEPW;
    const int nval = e_end - base;   // edges of this batch half (may exceed kEPW or be <= 0)
    ok = warp_wait(&bars->tfull[ts], (m >> 1) & 1, abort_flag, a.err, 31);
    if (ok) ok = warp_wait(&bars->sfull[sl], (k / kGS) & 1, abort_flag, a.err, 32);
    if (ok) ok = warp_wait(&bars->xfull[xl], (k / kXS) & 1, abort_flag, a.err, 38);
    if (!ok) break;
    tc_fence_after();
    // pair j of this half: coefficient row cfs + j * PW, sender rows xs + (2 j + t) * dim
    const float* cfs = cfbase + static_cast<size_t>(sl * (kN / 2) + h * (kEPW / 2)) * PW + CFO;
    const float* xs = xbase + static_cast<size_t>(xl * kN + h * kEPW) * dim;
    const uint32_t tb = tmem + (static_cast<uint32_t>(32 * q) << 16) + ts * G::SLOTC + (k & 1) * kN + h * kEPW;
    const bool last_of_mma = (k & 1) || k == nb - 1;   // the MMA batch's columns are all read after this
    // the batch half pair by pair: w of the pair's two columns per path item, then one packed
    // contraction when both edges are valid and belong to the current receiver; otherwise the
    // pair is taken edge by edge with the other edge masked (w = x = 0), flushing in between
#pragma unroll 1
    for (int pr = 0; pr < kEPW / 2 && ok; ++pr) {
      const int i = 2 * pr;
      float wv[NP][2];
#pragma unroll
      for (int b = 0; b < NP; ++b) tmem_ld2(tb + b * kNM + i, wv[b]);
      tc::tmem_wait_ld();
#pragma unroll
      for (int b = 0; b < NP; ++b) asm volatile("" : "+f"(wv[b][0]), "+f"(wv[b][1]));   // no read above the wait
      if (pr == kEPW / 2 - 1 && last_of_mma) {   // every column of the slot this warp needs is read
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->tempty[ts]);
      }
      const int nv = nval - i;   // valid edges from this pair on (may be <= 0)
      if (nv <= 0) continue;
      const bool vb = nv >= 2;
      const float* xa = xs + static_cast<size_t>(i) * dim;
      const float* xb = xa + dim;
      const float4* cf = reinterpret_cast<const float4*>(cfs + pr * PW);
      if (vb && base + i + 1 < nxt) {
        float2 xv[NX];
#pragma unroll
        for (int c = 0; c < NX; ++c) xv[c] = chv ? make_float2(xa[xoff[c]], xb[xoff[c]]) : make_float2(0.0f, 0.0f);
        float2 w[NP];
#pragma unroll
        for (int pi = 0; pi < NP; ++pi) w[pi] = make_float2(wv[pi][0], wv[pi][1]);
        SUB::fwd2(cf, xv, w, acc);
        continue;
      }
      const int want = vb ? 3 : 1;
      int done = 0;   // bit t: edge t of the pair accumulated
      while (done != want) {
        const int first = done & 1;   // the next edge still to take
        while (base + i + first >= nxt) {
          ok = flush();
          if (!ok) break;
        }
        if (!ok) break;
        const bool m0 = first == 0;
        const bool m1 = vb && base + i + 1 < nxt;
        float2 xv[NX];
#pragma unroll
        for (int c = 0; c < NX; ++c)
          xv[c] = make_float2(chv && m0 ? xa[xoff[c]] : 0.0f, chv && m1 ? xb[xoff[c]] : 0.0f);
        float2 w[NP];
#pragma unroll
        for (int pi = 0; pi < NP; ++pi) w[pi] = make_float2(m0 ? wv[pi][0] : 0.0f, m1 ? wv[pi][1] : 0.0f);
        SUB::fwd2(cf, xv, w, acc);
        done |= (m0 ? 1 : 0) | (m1 ? 2 : 0);
      }
    }
    if (!ok) break;
    __syncwarp();
    if (lane == 0) {   // coefficients and sender rows of the batch read
      mbar_arrive(&bars->sfree[sl]);
      mbar_arrive(&bars->xfree[xl]);
    }
  }
  // the receivers this CTA still owes: the current one and any edgeless ones up to r_end
  while (ok && cur <= r_end) ok = flush();
  return ok;
}

// ---------------------------------------------------------------- setup warps

// Geometry warp s handles the MMA batches m = s, s + 2, ..., one edge per lane (the 32 edges of
// batches 2 m and 2 m + 1): the coefficients of both subsets and the radial basis as the rows of
// the B operand of MMA batch m.
template <int L>
__device__ __forceinline__ bool setup(const Args& a, unsigned char* smem, Bars* bars, int nb, int s) {
  using G = Cfg<L>;
  constexpr int D = G::D;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  float* cfbase = reinterpret_cast<float*>(smem + G::OFF_CF);
  float* rbase = reinterpret_cast<float*>(smem + G::OFF_RB);
  const int e_beg = bars->e_beg, e_end = bars->e_end;
  const int nbm = (nb + 1) / 2;
  // the edge vectors of this warp's next MMA batch are loaded while the current one is set up
  auto load_edge = [&](int m, float& vx, float& vy, float& vz) {
    const int e = e_beg + m * kNM + lane;
    vx = vy = vz = 0.0f;
    if (m < nbm && e < e_end) {
      vx = __ldg(a.edge_vec + 3 * e);
      vy = __ldg(a.edge_vec + 3 * e + 1);
      vz = __ldg(a.edge_vec + 3 * e + 2);
    }
  };
  float nvx, nvy, nvz;
  load_edge(s, nvx, nvy, nvz);
  bool ok = true;
  for (int m = s; m < nbm; m += 2) {
    const int k = 2 * m + (lane >> 4);   // this lane's consumer batch
    const int sl = k % kGS;
    const int e = e_beg + m * kNM + lane;
    const float vx = nvx, vy = nvy, vz = nvz;
    load_edge(m + 2, nvx, nvy, nvz);
    // both slots of the MMA batch must have been released by every consumer
    if (2 * m >= kGS) {
      ok = warp_wait_lazy(&bars->sfree[(2 * m) % kGS], ((2 * m / kGS) - 1) & 1, abort_flag, a.err, 34);
      if (ok && 2 * m + 1 < nb)
        ok = warp_wait_lazy(&bars->sfree[(2 * m + 1) % kGS], (((2 * m + 1) / kGS) - 1) & 1, abort_flag, a.err, 34);
      if (!ok) break;
    }
    float Y[D];
    float R[kNumBasis], dR[kNumBasis];
#pragma unroll
    for (int c = 0; c < D; ++c) Y[c] = 0.0f;
#pragma unroll
    for (int b = 0; b < kNumBasis; ++b) R[b] = 0.0f;
    if (e < e_end) {
      const float dd = sqrtf(vx * vx + vy * vy + vz * vz);
      const float inv_d = dd > 0.0f ? 1.0f / dd : 0.0f;
      Gen<L>::sh(vx * inv_d, vy * inv_d, vz * inv_d, Y);
      radial_basis<false>(dd, a.inv_rc, R, dR);
    }
    {
      // coefficients of both subsets into the pair row of this edge: lane 2 j + t holds edge t of
      // pair j; one exchange with the partner lane per two coefficients makes 8-byte stores of
      // (c_k of edge 0, c_k of edge 1). The slot of a batch past the range is not written: it may
      // still be read for an earlier batch.
      float c0[G::CW0], c1[G::CW1];
      G::S0::coef(Y, c0);
      G::S1::coef(Y, c1);
      const int t = lane & 1;
      float* prow = cfbase + static_cast<size_t>(sl * (kN / 2) + ((lane & (kN - 1)) >> 1)) * G::PW + 2 * t;
#pragma unroll
      for (int i = 0; i < G::CW0 / 2; ++i) {
        const float give = t == 0 ? c0[2 * i + 1] : c0[2 * i];
        const float got = __shfl_xor_sync(kFull, give, 1);
        if (k < nb)
          *reinterpret_cast<float2*>(prow + 4 * i) = t == 0 ? make_float2(c0[2 * i], got) : make_float2(got, c0[2 * i + 1]);
      }
#pragma unroll
      for (int i = 0; i < G::CW1 / 2; ++i) {
        const float give = t == 0 ? c1[2 * i + 1] : c1[2 * i];
        const float got = __shfl_xor_sync(kFull, give, 1);
        if (k < nb)
          *reinterpret_cast<float2*>(prow + 2 * G::CW0 + 4 * i) =
              t == 0 ? make_float2(c1[2 * i], got) : make_float2(got, c1[2 * i + 1]);
      }
    }
    {
      float hh[kNumBasis], ll[kNumBasis];
#pragma unroll
      for (int b = 0; b < kNumBasis; ++b) split_tf32(R[b], &hh[b], &ll[b]);
      // row `lane` of the B operand of MMA batch m, slot m % kRS. That slot was last read by the
      // MMAs of batch m - kRS, which completed before the consumers finished its batches, whose
      // geometry slot release this warp waited for.
      float* th = rbase + static_cast<size_t>(m % kRS) * (2 * kNM * 8);
      float* tl = th + kNM * 8;
      *reinterpret_cast<float4*>(th + canon(lane, 0)) = make_float4(hh[0], hh[1], hh[2], hh[3]);
      *reinterpret_cast<float4*>(th + canon(lane, 4)) = make_float4(hh[4], hh[5], hh[6], hh[7]);
      *reinterpret_cast<float4*>(tl + canon(lane, 0)) = make_float4(ll[0], ll[1], ll[2], ll[3]);
      *reinterpret_cast<float4*>(tl + canon(lane, 4)) = make_float4(ll[4], ll[5], ll[6], ll[7]);
    }
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&bars->sfull[(2 * m) % kGS]);
      if (2 * m + 1 < nb) mbar_arrive(&bars->sfull[(2 * m + 1) % kGS]);
    }
  }
  return ok;
}

// ---------------------------------------------------------------- sender-row loader

// One bulk copy per edge (the sender's whole row, dim floats) into the batch's slot, completion on
// xfull; a slot is refilled once every consumer has read it (xfree).
__device__ __forceinline__ bool load_rows(const Args& a, unsigned char* smem, Bars* bars, int nb, int off_x) {
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  float* xbase = reinterpret_cast<float*>(smem + off_x);
  const int e_beg = bars->e_beg, e_end = bars->e_end;
  const uint32_t row_bytes = static_cast<uint32_t>(a.dim) * 4u;
  auto load_j = [&](int k) {
    const int e = e_beg + k * kN + lane;
    return (lane < kN && k < nb && e < e_end) ? __ldg(a.sender + e) : -1;
  };
  int nj = load_j(0);
  for (int k = 0; k < nb; ++k) {
    const int xl = k % kXS;
    const int j = nj;
    nj = load_j(k + 1);
    if (k >= kXS && !warp_wait_lazy(&bars->xfree[xl], ((k / kXS) - 1) & 1, abort_flag, a.err, 41)) return false;
    const unsigned valid = __ballot_sync(0xffffffffu, j >= 0);
    if (lane == 0) {
      mbar_expect_tx(&bars->xfull[xl], static_cast<uint32_t>(__popc(valid)) * row_bytes);
      bars->x_last[xl] = k;   // a slot is reused only after xfree, so these writes are ordered
    }
    __syncwarp();
    if (j >= 0)
      bulk_g2s(xbase + static_cast<size_t>(xl * kN + lane) * a.dim, a.x + static_cast<size_t>(j) * a.dim, row_bytes,
               &bars->xfull[xl]);
  }
  return true;
}

// ---------------------------------------------------------------- MMA thread

// Issues MMA batch after MMA batch (kNM edges: setup batches 2 m and 2 m + 1); returns the number of
// MMA batches committed.
template <int L>
__device__ __forceinline__ int issue_mma(const Args& a, unsigned char* smem, Bars* bars, uint32_t tmem, int nb) {
  using G = Cfg<L>;
  constexpr int NB = G::NB;
  constexpr uint32_t idesc = idesc_tf32(kNM);
  volatile int* abort_flag = &bars->abort_flag;
  const float* wa = reinterpret_cast<const float*>(smem + G::OFF_WA);
  const float* rbase = reinterpret_cast<const float*>(smem + G::OFF_RB);
  uint64_t wdesc[2 * NB];   // A operand descriptors (hi, lo) of every block, fixed for the launch
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    wdesc[2 * b] = smem_desc(sptr(wa + b * 2048));
    wdesc[2 * b + 1] = smem_desc(sptr(wa + b * 2048 + 1024));
  }
  const int nbm = (nb + 1) / 2;
  int issued = 0;
  for (int m = 0; m < nbm; ++m) {
    const int ts = m & 1;
    bool ok = true;
    for (int k = 2 * m; k < 2 * m + 2 && k < nb && ok; ++k)
      ok = mbar_wait(&bars->sfull[k % kGS], (k / kGS) & 1, abort_flag, a.err, 35);
    if (ok && m >= 2) ok = mbar_wait(&bars->tempty[ts], ((m >> 1) - 1) & 1, abort_flag, a.err, 36);
    if (!ok) break;
    tc_fence_after();
    const float* rb = rbase + static_cast<size_t>(m % kRS) * (2 * kNM * 8);
    const uint64_t bh = smem_desc(sptr(rb));
    const uint64_t bl = smem_desc(sptr(rb + kNM * 8));
    const uint32_t d0 = tmem + ts * G::SLOTC;
    // the three products of the tf32 split accumulate into the same columns: issued pass by pass
    // over the blocks (measured faster than block by block)
#pragma unroll
    for (int b = 0; b < NB; ++b) mma_tf32(d0 + b * kNM, wdesc[2 * b], bh, idesc, 0u);
#pragma unroll
    for (int b = 0; b < NB; ++b) mma_tf32(d0 + b * kNM, wdesc[2 * b], bl, idesc, 1u);
#pragma unroll
    for (int b = 0; b < NB; ++b) mma_tf32(d0 + b * kNM, wdesc[2 * b + 1], bh, idesc, 1u);
    mma_commit(&bars->tfull[ts]);
    issued = m + 1;
  }
  return issued;
}

// ---------------------------------------------------------------- combine warp

template <int L>
__device__ __forceinline__ bool combine(const Args& a, unsigned char* smem, Bars* bars) {
  using G = Cfg<L>;
  using S0 = typename G::S0;
  using S1 = typename G::S1;
  constexpr int D = G::D;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  const float* part = reinterpret_cast<const float*>(smem + G::OFF_PT);
  const int r_begin = bars->r_begin, r_end = bars->r_end;
  const long long E = a.n_edges;
  // the counters are zeroed by the preceding prep kernel (this kernel may start before it ends)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int kr = 0; kr <= r_end - r_begin; ++kr) {
    const int slot = kr % kNR;
    if (!warp_wait_lazy(&bars->rfull[slot], (kr / kNR) & 1, abort_flag, a.err, 37)) return false;
    const int r = r_begin + kr;
    // does this receiver's edge list cross a CTA boundary?
    bool span = false;
    int ca = blockIdx.x, cz = blockIdx.x;
    if (kr == 0 || r == r_end) {
      const int rb = __ldg(a.row_ptr + r), re = __ldg(a.row_ptr + r + 1);
      if (re > rb) {
        ca = cta_of(E, a.G, rb);
        cz = cta_of(E, a.G, re - 1);
        span = ca != cz;
      }
    }
    // the CTA's part: a row of out, or this CTA's slot of the spanning receiver
    float* dst = span ? a.gpart + (static_cast<size_t>(blockIdx.x) * 2 + (static_cast<int>(blockIdx.x) == ca ? 1 : 0)) * a.dim
                      : a.out + static_cast<size_t>(r) * a.dim;
    const float* ps = part + static_cast<size_t>(slot) * kCons * (G::NOMAX * 32);
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const int ch0 = g * 32 + lane;
      if (ch0 >= a.C) continue;
#pragma unroll
      for (int c = 0; c < D; ++c) {
        constexpr int kStride = G::NOMAX * 32;
        const int o0 = oidx<S0>(c), o1 = oidx<S1>(c);
        // fixed order: subset 0 (warps g, g + 4), then subset 1 (warps 2 + g, 6 + g)
        float v = 0.0f;
        if (o0 >= 0) {
          v = ps[g * kStride + o0 * 32 + lane];
          v += ps[(g + 4) * kStride + o0 * 32 + lane];
        }
        if (o1 >= 0) {
          v += ps[(g + 2) * kStride + o1 * 32 + lane];
          v += ps[(g + 6) * kStride + o1 * 32 + lane];
        }
        dst[c * a.C + ch0] = v;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->rempty[slot]);
    if (span) {
      // the CTA that adds the last part sums all parts in CTA order and stores the row
      __threadfence();
      __syncwarp();
      int old = 0;
      if (lane == 0) old = atomicAdd(a.cnt + ca, 1);
      old = __shfl_sync(kFull, old, 0);
      if (old == cz - ca) {
        __threadfence();
        float* orow = a.out + static_cast<size_t>(r) * a.dim;
        // the row in chunks of 32 x kChunk floats: every load of a chunk is issued before the adds
        constexpr int kChunk = 8;
        for (int i0 = 0; i0 < a.dim; i0 += 32 * kChunk) {
          float v[kChunk];
          const float* p0 = a.gpart + (static_cast<size_t>(ca) * 2 + 1) * a.dim + i0 + lane;
#pragma unroll
          for (int t = 0; t < kChunk; ++t) v[t] = i0 + lane + 32 * t < a.dim ? __ldcg(p0 + 32 * t) : 0.0f;
          for (int cc = ca + 1; cc <= cz; ++cc) {
            const float* pc = a.gpart + (static_cast<size_t>(cc) * 2) * a.dim + i0 + lane;
            float u[kChunk];
#pragma unroll
            for (int t = 0; t < kChunk; ++t) u[t] = i0 + lane + 32 * t < a.dim ? __ldcg(pc + 32 * t) : 0.0f;
#pragma unroll
            for (int t = 0; t < kChunk; ++t) v[t] += u[t];
          }
#pragma unroll
          for (int t = 0; t < kChunk; ++t)
            if (i0 + lane + 32 * t < a.dim) orow[i0 + lane + 32 * t] = v[t];
        }
      }
    }
  }
  return true;
}

// ---------------------------------------------------------------- the kernel

template <int L, int CT>
__global__ void __launch_bounds__(kThreads, 1) k_fwd_cx(Args a) {
  using G = Cfg<L>;
  using S0 = typename G::S0;
  using S1 = typename G::S1;
  extern __shared__ __align__(1024) unsigned char smem[];
  Bars* bars = reinterpret_cast<Bars*>(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->tfull[i], 1);
      mbar_init(&bars->tempty[i], kCons);
    }
    for (int i = 0; i < kGS; ++i) {
      mbar_init(&bars->sfull[i], 1);
      mbar_init(&bars->sfree[i], kCons);
    }
    for (int i = 0; i < kXS; ++i) {
      mbar_init(&bars->xfull[i], 1);
      mbar_init(&bars->xfree[i], kCons);
    }
    for (int i = 0; i < kNR; ++i) {
      mbar_init(&bars->rfull[i], kCons);
      mbar_init(&bars->rempty[i], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    for (int i = 0; i < kXS; ++i) bars->x_last[i] = -1;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the CTA's edge range and the receivers it owes: three independent binary searches over
  // row_ptr, run by lane 0 of three different warps at once
  const long long E = a.n_edges;
  const int eb = static_cast<int>(range_beg(E, a.G, blockIdx.x));
  const int ee = static_cast<int>(range_beg(E, a.G, blockIdx.x + 1));
  if (warp == 1) {
    const int r = blockIdx.x == 0 ? 0 : recv_of_warp(a.row_ptr, a.n_nodes, eb);
    if (lane == 0) bars->r_begin = r;
  } else if (warp == 2) {
    const int r = recv_of_warp(a.row_ptr, a.n_nodes, ee - 1);
    if (lane == 0) bars->e_beg = r;   // last receiver (for now)
  } else if (warp == 3) {
    const int r = ee < a.n_edges ? recv_of_warp(a.row_ptr, a.n_nodes, ee) - 1 : a.n_nodes - 1;
    if (lane == 0) bars->e_end = r;
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sptr(&bars->tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // the MMA A operands: one [128 x 8] block per path item, tf32 hi / lo; row 32 q + t of block b
  // is W[.][path b of quadrant q's subset][channel (q % 2) * 32 + t]
  {
    float* wa = reinterpret_cast<float*>(smem + G::OFF_WA);
    constexpr int PER = (G::NB * 1024 + kThreads - 1) / kThreads;
    float v[PER];
#pragma unroll
    for (int r = 0; r < PER; ++r) {   // all loads first, so they are in flight together
      const int i = threadIdx.x + r * kThreads;
      const int b = i >> 10, rem = i & 1023;
      const int row = rem >> 3, kb = rem & 7;
      const int qq = row >> 5, t = row & 31;
      const int sub = qq >> 1;
      v[r] = 0.0f;
      if (i < G::NB * 1024 && b < (sub ? S1::NP : S0::NP)) {
        const int p = sub ? S1::path(b) : S0::path(b);
        const int ch = (qq & 1) * 32 + t;
        if (ch < a.C) v[r] = __ldg(a.W + (static_cast<size_t>(kb) * G::P + p) * a.C + ch);
      }
    }
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int i = threadIdx.x + r * kThreads;
      if (i >= G::NB * 1024) break;
      const int b = i >> 10, rem = i & 1023;
      const int row = rem >> 3, kb = rem & 7;
      float hi, lo;
      split_tf32(v[r], &hi, &lo);
      wa[b * 2048 + canon(row, kb)] = hi;
      wa[b * 2048 + 1024 + canon(row, kb)] = lo;
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_holder;
  if (threadIdx.x == 0) {
    const int last = bars->e_beg, after = bars->e_end;
    bars->r_end = after > last ? after : last;
    bars->e_beg = eb;
    bars->e_end = ee;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int nb = (ee - eb + kN - 1) / kN;
  bool drained = true;

  if (warp < kCons) {
    const int q = warp & 3, h = warp >> 2;
    if (q < 2) consume<L, 0, CT>(a, smem, bars, q, h, tmem, nb);
    else consume<L, 1, CT>(a, smem, bars, q, h, tmem, nb);
  } else if (warp < kSetup0 + 2) {
    setup<L>(a, smem, bars, nb, warp - kSetup0);
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      issue_mma<L>(a, smem, bars, tmem, nb);
      // drain, ignoring the abort flag: one more commit tracks every MMA issued so far
      mma_commit(&bars->drain);
      if (!mbar_wait_drain(&bars->drain, 0)) {
        tc::report_code(a.err, 39);
        bars->abort_flag = 1;
        drained = false;
      }
    }
    drained = __shfl_sync(kFull, drained ? 1 : 0, 0) != 0;
  } else if (warp == kCombWarp) {
    combine<L>(a, smem, bars);
  } else if (warp == kLoadWarp) {
    load_rows(a, smem, bars, nb, G::OFF_X);
  }

  // teardown: every thread reaches this barrier exactly once. Then the sender-row copies that may
  // still be in flight (on abort no consumer waited for them) are drained before the CTA exits. A
  // slot is refilled only after every consumer waited for its previous copies, so only the last
  // batch issued into each slot can be outstanding.
  __syncthreads();
  if (warp == kCombWarp && lane == 0) {
    for (int sl = 0; sl < kXS; ++sl) {
      const int k = bars->x_last[sl];
      if (k >= 0 && !mbar_wait_drain(&bars->xfull[sl], (k / kXS) & 1)) {
        tc::report_code(a.err, 40);
        break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp && drained) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// Per call: zero the spanning-receiver counters. The forward kernel is launched as its programmatic
// dependent, so its prologue overlaps this kernel; only its combine warp, the one user of the
// counters, waits for this grid's completion (griddepcontrol.wait) before touching them.
__global__ void k_cx_prep(int* __restrict__ cnt, int n) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int i = threadIdx.x; i < n; i += blockDim.x) cnt[i] = 0;
}

constexpr int kMaxCtas = 512;

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

// Workspace: [counters: kMaxCtas ints][partial rows: kMaxCtas x 2 x dim floats]
size_t cnt_bytes() { return align256(sizeof(int) * kMaxCtas); }
float* gpart_ptr(void* ws) { return reinterpret_cast<float*>(static_cast<char*>(ws) + cnt_bytes()); }

template <int L, int CT>
etp_status launch_t(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                    const float* edge_vec, const float* x, const float* W, float* out, void* ws, cudaStream_t s) {
  using G = Cfg<L>;
  if (n_edges == 0) {
    return cuda_status(cudaMemsetAsync(out, 0, sizeof(float) * static_cast<size_t>(n_nodes) * c.dim, s),
                       "cx forward: zero output");
  }
  int grid = n_edges / kMinEdgesPerCta;
  const int sms = num_sms();
  if (grid > sms) grid = sms;
  if (grid > kMaxCtas) grid = kMaxCtas;
  if (grid < 1) grid = 1;
  int* cnt = static_cast<int*>(ws);
  k_cx_prep<<<1, 256, 0, s>>>(cnt, grid);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "cx forward prep");
  e = cudaFuncSetAttribute(k_fwd_cx<L, CT>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return cuda_status(e, "cx forward smem attribute");
  Args a;
  a.n_nodes = n_nodes;
  a.n_edges = n_edges;
  a.C = c.channels;
  a.dim = c.dim;
  a.G = grid;
  a.inv_rc = 1.0f / c.r_cut;
  a.row_ptr = row_ptr;
  a.sender = sender;
  a.edge_vec = edge_vec;
  a.x = x;
  a.W = W;
  a.out = out;
  a.gpart = gpart_ptr(ws);
  a.cnt = cnt;
  a.err = c.status_dev;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, k_fwd_cx<L, CT>, a), "cx forward launch");
}

}  // namespace

bool supported(const Ctx& c) {
  return !c.general && (c.lmax == 1 || c.lmax == 2) && c.channels >= 4 && c.channels <= kMaxC &&
         c.channels % 4 == 0;
}

size_t workspace_bytes(const Ctx& c) {
  if (!supported(c)) return 0;
  return cnt_bytes() + align256(sizeof(float) * static_cast<size_t>(kMaxCtas) * 2 * c.dim);
}

etp_status launch(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender, const float* edge_vec,
                  const float* x, const float* W, float* out, void* ws, cudaStream_t s) {
  const bool c64 = c.channels == 64;
  if (c.lmax == 1) {
    return c64 ? launch_t<1, 64>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s)
               : launch_t<1, 0>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
  }
  return c64 ? launch_t<2, 64>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s)
             : launch_t<2, 0>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
}

// Synchronises the stream and reads the handle's status word (left set if nonzero).
etp_status status(const Ctx& c, const void* ws, cudaStream_t s) {
  (void)ws;
  return read_status(c, s, "path-subset forward");
}

}  // namespace cx
}  // namespace etp

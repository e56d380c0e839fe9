// Fused forward edge convolution with the radial projection on the 5th-generation tensor cores.
//
// Work unit ("group"): four receivers (one per consumer warp, TMEM lane quadrant = warp) times a
// range of 16 channels. A persistent CTA per SM walks a contiguous block of groups.
//
//   consumer warps 0..3 (one receiver each, one edge per lane, <=128 edges per round):
//     - per edge: direction, real spherical harmonics Y (kept in shared memory), radial basis
//       R_b(d) split into tf32 hi + lo parts and written as rows of the MMA A tile;
//     - per channel batch of 4: for each 32-edge tile, the sender rows are gathered into shared
//       memory with cp.async (prefetched one tile ahead), the radial weights w_{e,p,k} are read
//       from TMEM with tcgen05.ld, and the unrolled Clebsch-Gordan code accumulates the message
//       in registers (per lane, over the receiver's tiles);
//     - one cross-lane reduction per receiver and batch through shared memory, one store.
//   producer warp 4 (one elected lane):
//     - streams the pre-split weight slices W^T (hi, lo) of the group's channel range into
//       shared memory with cp.async.bulk;
//     - issues w = R W for every (batch, tile) as three kind::tf32 MMAs (hi*hi + hi*lo + lo*hi,
//       float32 accumulation; about float32 accuracy) into a ring of TMEM slots
//       (M = 128 edges, N = 4 P columns rounded up to 16, K = 8 basis functions).
//
// Synchronisation: mbarriers (full / empty per TMEM slot, tile-ready, weight-slice loaded /
// free). Every wait is bounded; on timeout the kernel records an error code and aborts cleanly.
// Receivers never span CTAs or warps: no atomics, fixed summation order.
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"

namespace etp {
namespace tc {
namespace {

constexpr int kConsumers = 4;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kSMax = 4;          // tiles per receiver round (128 edges)
constexpr int kUnitC = 16;        // channels per work unit
constexpr int kTmemCols = 512;
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 2 GHz: bounded waits

template <int L>
struct Cfg {
  static constexpr int D = Gen<L>::D;
  static constexpr int P = Gen<L>::P;
  static constexpr int NCOL = ((4 * P + 15) / 16) * 16;     // MMA N: 4 channels per path
  static constexpr int NSLOT = kTmemCols / NCOL;
  static constexpr int V = 4 * D;                           // values per lane per batch
  static constexpr int VS = 4 * (D | 1);                    // reduction row stride (odd float4 count)
  static constexpr int WSLICE = 2 * NCOL * 32;              // bytes: hi + lo of one batch
  static constexpr int WBUF = (kUnitC / 4) * WSLICE;        // one unit's four batches
  // shared memory map (bytes)
  static constexpr int OFF_A = 1024;
  static constexpr int OFF_W = OFF_A + kSMax * 2 * 4096;
  static constexpr int OFF_Y = OFF_W + 2 * WBUF;
  static constexpr int OFF_X = OFF_Y + kConsumers * kSMax * D * 32 * 4;
  static constexpr int OFF_R = OFF_X + kConsumers * 2 * D * 512;
  static constexpr int END = OFF_R + kConsumers * 32 * VS * 4;
  static constexpr int SMEM = END < 118 * 1024 ? 118 * 1024 : END;   // > half an SM: one CTA per SM
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
  const float* wt;    // pre-split weights, [unit][batch][hi/lo][NCOL x 8 canonical]
  float* out;
  int* err;
};

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t sptr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sptr(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(sptr(b)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(sptr(b)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(sptr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on the phase of the given parity. Returns false (and raises the CTA abort flag and
// the global error code) when the limit is exceeded or another thread has aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* err,
                                          int code) {
  if (mbar_test(b, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_test(b, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      atomicExch(err, code);
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major, no swizzle: 8-row x 16-byte core matrices; 128 B to the next core matrix along K,
// 256 B to the next 8 rows.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>(256u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;   // descriptor version for sm_100
  return d;                                // base offset 0, swizzle none
}

// kind::tf32 instruction descriptor: D f32, A/B tf32, both K-major, M = 128, N given.
__host__ __device__ constexpr uint32_t idesc_tf32(int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(z), "r"(z), "r"(z), "r"(z)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(sptr(b))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[32]) {
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

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sptr(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   sptr(dst)),
               "l"(src), "r"(bytes), "r"(sptr(bar))
               : "memory");
}

// tf32 split: hi keeps the top 10 explicit mantissa bits, lo = v - hi exactly.
__device__ __forceinline__ void split_tf32(float v, float* hi, float* lo) {
  const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
  *hi = h;
  *lo = v - h;
}

// Canonical K-major no-swizzle offset (floats) of element (row, k) of an [rows x 8] tf32 matrix.
__host__ __device__ __forceinline__ int canon(int row, int k) {
  return (row >> 3) * 64 + (k >> 2) * 32 + (row & 7) * 4 + (k & 3);
}

// ------------------------------------------------------------------ group geometry

struct GroupInfo {
  int rg, unit, rounds, nbatch;
  int deg[kConsumers];
  int beg[kConsumers];
};

__device__ __forceinline__ void group_info(const Args& a, int g, GroupInfo* gi) {
  gi->rg = g / a.n_units;
  gi->unit = g - gi->rg * a.n_units;
  int rounds = 1;
#pragma unroll
  for (int q = 0; q < kConsumers; ++q) {
    const int r = gi->rg * kConsumers + q;
    int b = 0, d = 0;
    if (r < a.n_nodes) {
      b = a.row_ptr[r];
      d = a.row_ptr[r + 1] - b;
    }
    gi->beg[q] = b;
    gi->deg[q] = d;
    const int rr = (d + 32 * kSMax - 1) / (32 * kSMax);
    rounds = rr > rounds ? rr : rounds;
  }
  gi->rounds = rounds;
  const int left = a.C - gi->unit * kUnitC;
  gi->nbatch = (left >= kUnitC ? kUnitC : left) / 4;
}

__device__ __forceinline__ int tiles_of(int deg, int round) {
  int rem = deg - round * 32 * kSMax;
  if (rem <= 0) return 0;
  const int t = (rem + 31) / 32;
  return t < kSMax ? t : kSMax;
}

// ------------------------------------------------------------------ kernels

// wt[unit][batch][hl][canonical NCOL x 8]: row n = 4 p + k holds W[b][p][16 unit + 4 batch + k].
template <int L>
__global__ void k_prep_weights(const float* __restrict__ W, int C, int n_units, float* __restrict__ wt,
                               int* __restrict__ err) {
  using G = Cfg<L>;
  if (blockIdx.x == 0 && threadIdx.x == 0) *err = 0;
  const int per_batch = 2 * G::NCOL * 8;
  const int total = n_units * 4 * per_batch;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int slab = i / per_batch;            // unit * 4 + batch
    const int rem = i - slab * per_batch;
    const int hl = rem / (G::NCOL * 8);
    const int e = rem - hl * (G::NCOL * 8);
    const int n = e / 8, kb = e % 8;
    const int p = n >> 2, k = n & 3;
    const int u = slab * 4 + k;                // channel
    float v = 0.0f;
    if (p < G::P && u < C) v = W[(kb * G::P + p) * C + u];
    float hi, lo;
    split_tf32(v, &hi, &lo);
    wt[slab * per_batch + hl * G::NCOL * 8 + canon(n, kb)] = hl ? lo : hi;
  }
}

template <int L>
__global__ void __launch_bounds__(kThreads, 1) k_fwd_tc(Args a) {
  using G = Cfg<L>;
  using Gn = Gen<L>;
  constexpr int D = G::D, V = G::V, VS = G::VS, NCOL = G::NCOL, NSLOT = G::NSLOT;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + NSLOT;
  uint64_t* rready = empty + NSLOT;
  uint64_t* wload = rready + 1;   // [2]
  uint64_t* wfree = wload + 2;    // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(wfree + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* Atile = reinterpret_cast<float*>(smem + G::OFF_A);     // [kSMax][hl][128 x 8 canonical]
  float* Wbuf = reinterpret_cast<float*>(smem + G::OFF_W);      // [2][batch][hl][NCOL x 8]
  float* Ybuf = reinterpret_cast<float*>(smem + G::OFF_Y);      // [warp][tile][D][32]
  float4* Xst = reinterpret_cast<float4*>(smem + G::OFF_X);     // [warp][stage][D][32]
  float* Red = reinterpret_cast<float*>(smem + G::OFF_R);       // [warp][32][VS]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g_beg = static_cast<int>(static_cast<long long>(a.n_groups) * blockIdx.x / gridDim.x);
  const int g_end = static_cast<int>(static_cast<long long>(a.n_groups) * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kConsumers);
    }
    mbar_init(rready, kConsumers);
    mbar_init(wload + 0, 1);
    mbar_init(wload + 1, 1);
    mbar_init(wfree + 0, 1);
    mbar_init(wfree + 1, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kConsumers) {   // producer warp owns the TMEM allocation
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sptr(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32(NCOL);
      uint32_t item = 0, n_setup = 0, n_loads = 0;
      int cached_rg = -1, cached_round = -1;
      bool ok = true;
      // weight slices of group g go to buffer (g - g_beg) & 1; the load of group g + 1 is issued as
      // soon as the MMAs of group g are issued, after the MMAs of group g - 1 (same buffer) finished
      auto load_w = [&](int g, uint32_t n) -> bool {
        GroupInfo gl;
        group_info(a, g, &gl);
        const int wb = n & 1;
        if (n >= 2 && !mbar_wait(wfree + wb, ((n >> 1) - 1) & 1, abort_flag, a.err, 11)) return false;
        const uint32_t bytes = static_cast<uint32_t>(gl.nbatch * G::WSLICE);
        mbar_expect_tx(wload + wb, bytes);
        bulk_g2s(Wbuf + wb * (G::WBUF / 4), a.wt + static_cast<size_t>(gl.unit) * (G::WBUF / 4), bytes, wload + wb);
        return true;
      };
      if (g_beg < g_end) ok = load_w(g_beg, 0);
      for (int g = g_beg; g < g_end && ok; ++g) {
        GroupInfo gi;
        group_info(a, g, &gi);
        const int wb = n_loads & 1;
        ok = mbar_wait(wload + wb, (n_loads >> 1) & 1, abort_flag, a.err, 12);
        ++n_loads;
        for (int round = 0; round < gi.rounds && ok; ++round) {
          int S = 0;
#pragma unroll
          for (int q = 0; q < kConsumers; ++q) {
            const int t = tiles_of(gi.deg[q], round);
            S = t > S ? t : S;
          }
          if (gi.rg != cached_rg || round != cached_round) {
            ok = mbar_wait(rready, n_setup & 1, abort_flag, a.err, 13);
            ++n_setup;
            cached_rg = gi.rg;
            cached_round = round;
            if (!ok) break;
          }
          tc_fence_after();
          for (int b = 0; b < gi.nbatch && ok; ++b) {
            for (int s = 0; s < S; ++s) {
              const int slot = item % NSLOT;
              const uint32_t par = ((item / NSLOT) & 1) ^ 1;
              ok = mbar_wait(empty + slot, par, abort_flag, a.err, 14);
              if (!ok) break;
              tc_fence_after();
              const uint32_t d = tmem + slot * NCOL;
              const uint64_t ah = smem_desc(sptr(Atile + (s * 2 + 0) * 1024));
              const uint64_t al = smem_desc(sptr(Atile + (s * 2 + 1) * 1024));
              const float* wsl = Wbuf + wb * (G::WBUF / 4) + b * (G::WSLICE / 4);
              const uint64_t bh = smem_desc(sptr(wsl));
              const uint64_t bl = smem_desc(sptr(wsl + NCOL * 8));
              mma_tf32(d, ah, bh, idesc, 0u);
              mma_tf32(d, ah, bl, idesc, 1u);
              mma_tf32(d, al, bh, idesc, 1u);
              mma_commit(full + slot);
              ++item;
            }
          }
        }
        mma_commit(wfree + wb);   // completes once every MMA issued so far has finished
        if (ok && g + 1 < g_end) ok = load_w(g + 1, n_loads);
      }
      // drain: the last commit covers every MMA this CTA issued
      if (n_loads > 0) mbar_wait(wfree + ((n_loads - 1) & 1), ((n_loads - 1) >> 1) & 1, abort_flag, a.err, 15);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers
    const int q = warp;
    float* Yw = Ybuf + q * (kSMax * D * 32);
    float4* Xw = Xst + q * (2 * D * 32);
    float* Rw = Red + q * (32 * VS);
    uint32_t item = 0, n_setup = 0;
    int cached_rg = -1, cached_round = -1;
    int jsend[kSMax];
    bool ok = true;
    for (int g = g_beg; g < g_end && ok; ++g) {
      GroupInfo gi;
      group_info(a, g, &gi);
      const int r = gi.rg * kConsumers + q;
      const int deg = gi.deg[q];
      for (int round = 0; round < gi.rounds && ok; ++round) {
        int S = 0;
#pragma unroll
        for (int qq = 0; qq < kConsumers; ++qq) {
          const int t = tiles_of(gi.deg[qq], round);
          S = t > S ? t : S;
        }
        const int Sq = tiles_of(deg, round);
        const int e_round = gi.beg[q] + round * 32 * kSMax;
        if (gi.rg != cached_rg || round != cached_round) {
          // all four warps must have published setup n-1 before anyone publishes setup n
          if (n_setup > 0) {
            ok = mbar_wait(rready, (n_setup - 1) & 1, abort_flag, a.err, 22);
            if (!ok) break;
          }
          // per-edge geometry for this warp's receiver: Y to shared memory, R (tf32 hi/lo) to the
          // A tiles (row 32 q + lane), sender index to registers
#pragma unroll
          for (int s = 0; s < kSMax; ++s) {
            jsend[s] = -1;
            if (s < Sq) {
              const int le = round * 32 * kSMax + s * 32 + lane;
              float Y[D];
              float R[kNumBasis], dR[kNumBasis];
#pragma unroll
              for (int c = 0; c < D; ++c) Y[c] = 0.0f;
#pragma unroll
              for (int bb = 0; bb < kNumBasis; ++bb) R[bb] = 0.0f;
              if (le < deg) {
                const int e = gi.beg[q] + le;
                const float vx = a.edge_vec[3 * e], vy = a.edge_vec[3 * e + 1], vz = a.edge_vec[3 * e + 2];
                jsend[s] = a.sender[e];
                const float dd = sqrtf(vx * vx + vy * vy + vz * vz);
                const float inv_d = dd > 0.0f ? 1.0f / dd : 0.0f;
                Gn::sh(vx * inv_d, vy * inv_d, vz * inv_d, Y);
                radial_basis<false>(dd, a.inv_rc, R, dR);
              }
#pragma unroll
              for (int c = 0; c < D; ++c) Yw[(s * D + c) * 32 + lane] = Y[c];
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
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) mbar_arrive(rready);
          ++n_setup;
          cached_rg = gi.rg;
          cached_round = round;
        }
        (void)e_round;
        const int cbase = gi.unit * kUnitC;
        // gather of sender rows for (batch b, tile s) into stage st (zero-filled for padding lanes)
        auto prefetch = [&](int b, int s, int st) {
          const int jj = jsend[s];
          const float* src = a.x + static_cast<size_t>(jj < 0 ? 0 : jj) * a.dim + cbase + 4 * b;
          float4* dst = Xw + st * (D * 32) + lane;
#pragma unroll
          for (int c = 0; c < D; ++c) cp_async16(dst + c * 32, src + c * a.C, jj < 0 ? 0u : 16u);
          cp_async_commit();
        };
        int stage = 0;
        if (Sq > 0) prefetch(0, 0, 0);
        for (int b = 0; b < gi.nbatch && ok; ++b) {
          float acc[D][4];
#pragma unroll
          for (int c = 0; c < D; ++c)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[c][k] = 0.0f;
          for (int s = 0; s < S; ++s) {
            const int slot = item % NSLOT;
            const uint32_t par = (item / NSLOT) & 1;
            const bool mine = s < Sq;
            if (mine) {   // prefetch the next (batch, tile) of this receiver, then wait for this one
              int nb = b, ns = s + 1;
              if (ns >= Sq) {
                ns = 0;
                ++nb;
              }
              if (nb < gi.nbatch) {
                prefetch(nb, ns, stage ^ 1);
                cp_async_wait<1>();
              } else {
                cp_async_wait<0>();
              }
              __syncwarp();
            }
            ok = mbar_wait(full + slot, par, abort_flag, a.err, 21);
            if (!ok) break;
            tc_fence_after();
            if (mine) {
              float xv[D][4];
              const float4* xs = Xw + stage * (D * 32) + lane;
#pragma unroll
              for (int c = 0; c < D; ++c) {
                const float4 t = xs[c * 32];
                xv[c][0] = t.x; xv[c][1] = t.y; xv[c][2] = t.z; xv[c][3] = t.w;
              }
              float Y[D];
#pragma unroll
              for (int c = 0; c < D; ++c) Y[c] = Yw[(s * D + c) * 32 + lane];
              const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16) + slot * NCOL;
              float wch[32];
              auto wf = [&](auto pc, float (&wp)[4]) {
                constexpr int p = decltype(pc)::value;
                if constexpr ((p & 7) == 0) {
                  if constexpr (NCOL - 32 * (p >> 3) >= 32) tmem_ld32(tbase + 32 * (p >> 3), wch);
                  else tmem_ld16(tbase + 32 * (p >> 3), wch);
                  tmem_wait_ld();
                }
                const int o = (p & 7) * 4;
                wp[0] = wch[o]; wp[1] = wch[o + 1]; wp[2] = wch[o + 2]; wp[3] = wch[o + 3];
              };
              Gn::template fwd<4>(Y, wf, xv, acc);
              stage ^= 1;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);
            ++item;
          }
          if (!ok) break;
          // cross-lane sum of acc through shared memory, then one store (or add for later rounds)
          if (Sq > 0 || round == 0) {
#pragma unroll
            for (int c = 0; c < D; ++c)
              *reinterpret_cast<float4*>(Rw + lane * VS + 4 * c) = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
            __syncwarp();
            if (r < a.n_nodes) {
              for (int v = lane; v < V; v += 32) {
                float sum = 0.0f;
#pragma unroll 8
                for (int l2 = 0; l2 < 32; ++l2) sum += Rw[l2 * VS + v];
                const int c = v >> 2, k = v & 3;
                float* op = a.out + static_cast<size_t>(r) * a.dim + c * a.C + cbase + 4 * b + k;
                if (round == 0) *op = sum; else *op += sum;
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
  if (warp == kConsumers) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

int g_sms = 0;

template <int L>
etp_status launch(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                  const float* edge_vec, const float* x, const float* W, float* out, void* ws, cudaStream_t s) {
  (void)n_edges;
  using G = Cfg<L>;
  const int n_units = (c.channels + kUnitC - 1) / kUnitC;
  float* wt = static_cast<float*>(ws);
  int* err = reinterpret_cast<int*>(static_cast<char*>(ws) + align256(sizeof(float) * n_units * (G::WBUF / 4)));
  k_prep_weights<L><<<64, 256, 0, s>>>(W, c.channels, n_units, wt, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "weight split");
  e = cudaFuncSetAttribute(k_fwd_tc<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return cuda_status(e, "tc forward smem attribute");
  if (g_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_sms <= 0) g_sms = 148;
  }
  Args a;
  a.n_nodes = n_nodes;
  a.C = c.channels;
  a.dim = c.dim;
  a.n_units = n_units;
  a.n_groups = ((n_nodes + kConsumers - 1) / kConsumers) * n_units;
  a.inv_rc = 1.0f / c.r_cut;
  a.row_ptr = row_ptr;
  a.sender = sender;
  a.edge_vec = edge_vec;
  a.x = x;
  a.wt = wt;
  a.out = out;
  a.err = err;
  const int grid = a.n_groups < g_sms ? a.n_groups : g_sms;
  k_fwd_tc<L><<<grid, kThreads, G::SMEM, s>>>(a);
  return cuda_status(cudaGetLastError(), "tc forward launch");
}

}  // namespace

size_t forward_tc_workspace_bytes(const Ctx& c) {
  const int n_units = (c.channels + kUnitC - 1) / kUnitC;
  size_t wbuf = 0;
  switch (c.lmax) {
    case 1: wbuf = Cfg<1>::WBUF; break;
    case 2: wbuf = Cfg<2>::WBUF; break;
    default: wbuf = Cfg<3>::WBUF; break;
  }
  return align256(static_cast<size_t>(n_units) * wbuf) + 256;
}

// Reads the pipeline status word of the last tensor-core forward that used this workspace
// (synchronises the stream). Nonzero = a bounded wait gave up (the output is incomplete).
etp_status forward_tc_status(const Ctx& c, const void* ws, cudaStream_t s) {
  const int n_units = (c.channels + kUnitC - 1) / kUnitC;
  size_t wbuf = c.lmax == 1 ? Cfg<1>::WBUF : (c.lmax == 2 ? Cfg<2>::WBUF : Cfg<3>::WBUF);
  const int* err = reinterpret_cast<const int*>(static_cast<const char*>(ws) + align256(n_units * wbuf));
  int code = 0;
  cudaError_t e = cudaMemcpyAsync(&code, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e, "forward status read");
  if (code != 0) {
    set_error("tensor-core forward: pipeline wait exceeded its limit (code " + std::to_string(code) + ")");
    return ETP_ERR_CUDA;
  }
  return ETP_OK;
}

etp_status launch_forward_tc(const Ctx& c, int n_nodes, int n_edges, const int* row_ptr, const int* sender,
                             const float* edge_vec, const float* x, const float* W, float* out, void* ws,
                             cudaStream_t s) {
  switch (c.lmax) {
    case 1: return launch<1>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
    case 2: return launch<2>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
    case 3: return launch<3>(c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, ws, s);
  }
  set_error("tc forward: unsupported lmax");
  return ETP_ERR_UNSUPPORTED;
}

}  // namespace tc
}  // namespace etp

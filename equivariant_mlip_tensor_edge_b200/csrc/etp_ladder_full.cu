// The full node-local product ladder ("FlashCart", Fig. 3b dashed curves; Fig. E1 (b)): every step
// keeps the unweighted "uvu" product of each retained coupling path and compresses the paths of each
// output rank with one matrix that mixes paths and channels,
//
//   T_p[m3, u]      = sum_{m1, m2} C^{l1 l2 l3}_{m1 m2 m3} B[l1 m1 u] A[l2 m2 u]
//   B'[l3, m3, v]   = sum_{p of rank l3} sum_u W_l3[v, p' C + u] T_p[m3, u]
//   B_1 = A, B_{q+1} = step(B_q, A; W_q), out = sum_{q = 1..nu} B_q.
//
// The compression is a dense GEMM per output component (l3, m3): rows = nodes, K = P_l3 C (the
// paths of rank l3 times the channels), N = C. It runs on the tensor cores:
//   k_ladder_t:   CUDA cores, one warp per (node, 32-channel slice): the NT per-path products of the
//                 node for the lane's channel, written as the rows of the GEMM operands T_l3.
//   k_ladder_wprep: once per call, every step's W_l3 split into tf32 hi/lo and laid out as the
//                 MMA B operand tiles (canonical K-major), 32 columns of K per contiguous chunk.
//   k_ladder_mix: one CTA per (128-node tile, component). Per K-chunk of 32 columns, each of four
//                 loader warps loads its 32 node rows of T (thread = row = TMEM lane), splits them
//                 into tf32 hi/lo and writes them straight into TMEM (tcgen05.st): the MMA A operand
//                 never touches shared memory. The chunk's W tiles arrive by one cp.async.bulk.
//                 One thread issues three kind::tf32 MMAs per 8 columns (hi*hi + hi*lo + lo*hi,
//                 A from TMEM, B from shared memory) into a TMEM accumulator [128 nodes x C]; the
//                 loader warps then read it back (tcgen05.ld), store the component of B_{q+1} and
//                 add it into out.
// Every output element is written by one thread per step: the result is bitwise reproducible.
// Every mbarrier wait is bounded; a timeout records a code in the status word and the CTA drains
// the MMAs it issued before it releases TMEM.
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"
#include "etp_tc_common.h"

namespace etp {
namespace lad {
namespace {

using tc::canon;
using tc::fence_proxy_async;
using tc::idesc_tf32;
using tc::mbar_arrive;
using tc::mbar_init;
using tc::mbar_wait;
using tc::mbar_wait_drain;
using tc::mma_commit;
using tc::mma_tf32;
using tc::smem_desc;
using tc::split_tf32;
using tc::sptr;
using tc::tc_fence_after;
using tc::tc_fence_before;

constexpr int kRows = 128;                 // nodes per tile (MMA M)
constexpr int kChunk = 32;                 // K columns per pipeline stage (4 MMA K-steps of 8)
constexpr int kLoadWarps = 4;              // loaders, later the epilogue (TMEM lane quadrant = warp)
constexpr int kMmaWarp = kLoadWarps;
constexpr int kThreads = 32 * (kLoadWarps + 1);
constexpr int kStages = 3;
constexpr int kMaxC = 128;

template <int L>
struct LadderGen;
template <>
struct LadderGen<1> {
  using S = etp_gen::LadderShape<1>;
  static __device__ __forceinline__ void t(const float (&b)[4], const float (&a)[4], float (&t)[S::NT]) {
    etp_gen::ladder_t_1(b, a, t);
  }
};
template <>
struct LadderGen<2> {
  using S = etp_gen::LadderShape<2>;
  static __device__ __forceinline__ void t(const float (&b)[9], const float (&a)[9], float (&t)[S::NT]) {
    etp_gen::ladder_t_2(b, a, t);
  }
};
template <>
struct LadderGen<3> {
  using S = etp_gen::LadderShape<3>;
  static __device__ __forceinline__ void t(const float (&b)[16], const float (&a)[16], float (&t)[S::NT]) {
    etp_gen::ladder_t_3(b, a, t);
  }
};

// Shared memory of k_ladder_mix for C channels: barriers; kStages stages of the B operand of a
// K-chunk, [K-step 0..3][hi, lo][C x 8] (the layout k_ladder_wprep writes); kRaw stages of raw T
// rows, [128 rows][kRawLd floats] (each loader thread copies and reads back only its own row; the
// padding keeps the 16-byte reads of 8 consecutive rows on distinct banks).
constexpr int kRaw = 4;                    // raw T stages: kRaw - 1 chunks requested ahead
constexpr int kRawLd = kChunk + 4;
struct Smem {
  static constexpr int kBar = 1024;
  static __host__ __device__ constexpr int stage(int C) { return 4 * 2 * C * 8 * 4; }
  static __host__ __device__ constexpr int raw_stage() { return kRows * kRawLd * 4; }
  static __host__ __device__ constexpr int raw_off(int C) { return kBar + kStages * stage(C); }
  // above half an SM, so that one CTA holds the SM and its 512 TMEM columns
  static __host__ __device__ constexpr int bytes(int C) {
    return raw_off(C) + kRaw * raw_stage() > 118 * 1024 ? raw_off(C) + kRaw * raw_stage() : 118 * 1024;
  }
};

// TMEM columns of k_ladder_mix: the accumulator [0, 128), then per stage the A operand of a
// K-chunk: [K-step 0..3][hi, lo][8 columns].
constexpr uint32_t kTmemAlloc = 512;
constexpr uint32_t kAccCols = 128;
constexpr uint32_t kAStageCols = 64;

// ---------------------------------------------------------------- per-path products

// Task t: node t / n_slices, channel slice t % n_slices (32 channels). T_l3 is laid out
// [node][m3][p' C + u] after the blocks of the lower ranks (block l3 starts at N C off(l3)).
template <int L>
__global__ void __launch_bounds__(256) k_ladder_t(int n_nodes, int C, const float* __restrict__ B,
                                                  const float* __restrict__ A, float* __restrict__ T) {
  using S = typename LadderGen<L>::S;
  constexpr int D = (L + 1) * (L + 1);
  const int lane = threadIdx.x & 31;
  const int n_slices = C / 32;
  const long long n_tasks = static_cast<long long>(n_nodes) * n_slices;
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long task = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5); task < n_tasks;
       task += stride) {
    const int node = static_cast<int>(task / n_slices);
    const int u = static_cast<int>(task % n_slices) * 32 + lane;
    const size_t row = static_cast<size_t>(node) * D * C;
    float b[D], a[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      b[c] = __ldg(B + row + static_cast<size_t>(c) * C + u);
      a[c] = __ldg(A + row + static_cast<size_t>(c) * C + u);
    }
    float t[S::NT];
    LadderGen<L>::t(b, a, t);
#pragma unroll
    for (int l3 = 0; l3 <= L; ++l3) {
      const int P = S::P(l3);
      float* dst = T + static_cast<size_t>(n_nodes) * C * S::off(l3) +
                   static_cast<size_t>(node) * (2 * l3 + 1) * P * C + u;
#pragma unroll
      for (int i = 0; i < (2 * l3 + 1) * P; ++i) dst[static_cast<size_t>(i) * C] = t[S::off(l3) + i];
    }
  }
}

// ---------------------------------------------------------------- the compression GEMM

struct MixArgs {
  int n_nodes;
  int C;
  const float* T;      // the step's products (k_ladder_t layout)
  const float* Wt;     // the step's B operand tiles (k_ladder_wprep layout)
  float* b_next;       // B_{q+1} [N][D C], or null on the last step
  float* out;          // out [N][D C], += B_{q+1}
  int* err;
};

struct Bars {
  uint64_t full[kStages];    // a stage's A columns written to TMEM (kLoadWarps arrivals)
  uint64_t bfull[kStages];   // a stage's B tiles landed (transaction bytes)
  uint64_t empty[kStages];   // a stage's MMAs complete (one commit)
  uint64_t done;             // every MMA of the tile complete
  uint64_t drain;
  uint32_t tmem_holder;
  int abort_flag;
  int b_last[kStages];       // per stage: the last chunk whose B copy was issued into it
};

// W of one step as B operand tiles: rank blocks one after another; block l3 holds, per K-chunk c of
// 32 columns, [K-step s][hi, lo][C x 8] in the canonical K-major layout, so one chunk's tiles are
// 8 C 8 contiguous floats.
template <int L>
__global__ void k_ladder_wprep(int C, int steps, const float* __restrict__ W, float* __restrict__ Wt) {
  using S = typename LadderGen<L>::S;
  size_t per_step = 0;
  for (int l = 0; l <= L; ++l) per_step += static_cast<size_t>(S::P(l)) * C * C;
  const size_t total = per_step * steps;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t q = i / per_step;
    size_t r = i - q * per_step;
    int l3 = 0;
    size_t blk = 0;
    while (r >= blk + static_cast<size_t>(S::P(l3)) * C * C) {
      blk += static_cast<size_t>(S::P(l3)) * C * C;
      ++l3;
    }
    r -= blk;
    const int K = S::P(l3) * C;
    const int v = static_cast<int>(r / K), k = static_cast<int>(r % K);
    float hi, lo;
    split_tf32(W[i], &hi, &lo);
    float* dst = Wt + 2 * (q * per_step + blk) + (static_cast<size_t>(k / kChunk) * 8 + ((k % kChunk) / 8) * 2) * C * 8;
    dst[canon(v, k % 8)] = hi;
    dst[C * 8 + canon(v, k % 8)] = lo;
  }
}

// D (TMEM) += A (TMEM: 128 lanes x 8 columns of tf32) x B (shared memory descriptor)
__device__ __forceinline__ void mma_tf32_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]),
      "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]),
      "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Grid: x = 128-node tiles, y = output component (l3, m3) in (l, m) order.
template <int L>
__global__ void __launch_bounds__(kThreads, 1) k_ladder_mix(MixArgs a) {
  using S = typename LadderGen<L>::S;
  constexpr int D = (L + 1) * (L + 1);
  extern __shared__ __align__(1024) unsigned char smem[];
  Bars* bars = reinterpret_cast<Bars*>(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = a.C;
  const int comp = blockIdx.y;
  int l3 = 0;
  while ((l3 + 1) * (l3 + 1) <= comp) ++l3;
  const int m3 = comp - l3 * l3;
  const int K = S::P(l3) * C;                 // GEMM K: the paths of rank l3 times the channels
  const int n_chunks = K / kChunk;
  const int node0 = blockIdx.x * kRows;
  // T_l3 row (node, m3) has K columns
  const float* Tt = a.T + static_cast<size_t>(a.n_nodes) * C * S::off(l3) +
                    (static_cast<size_t>(node0) * (2 * l3 + 1) + m3) * K;
  const size_t t_ld = static_cast<size_t>(2 * l3 + 1) * K;
  size_t w_off = 0;
  for (int l = 0; l < l3; ++l) w_off += static_cast<size_t>(S::P(l)) * C * C;
  const float* Wl = a.Wt + 2 * w_off;        // the rank's B tiles: 64 C floats per chunk
  const uint32_t b_bytes = static_cast<uint32_t>(Smem::stage(C));
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], kLoadWarps);
      mbar_init(&bars->bfull[s], 1);
      mbar_init(&bars->empty[s], 1);
      bars->b_last[s] = -1;
    }
    mbar_init(&bars->done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sptr(&bars->tmem_holder)),
                 "r"(kTmemAlloc)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_holder;
  unsigned char* stages = smem + Smem::kBar;
  bool drained = true;

  if (warp < kLoadWarps) {
    // ---------------------------------------------------------------- loaders, then the epilogue
    const int t = threadIdx.x;                                         // tile row = TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * warp) << 16);
    const bool valid = node0 + t < a.n_nodes;
    const float* src = Tt + static_cast<size_t>(valid ? t : 0) * t_ld;
    float* raw = reinterpret_cast<float*>(smem + Smem::raw_off(C)) + t * kRawLd;
    // this thread's row of chunk k into raw stage k % kRaw (zero-filled past the last node); one
    // commit group per chunk, so chunk k's copies are complete once at most kRaw - 2 later groups
    // are pending
    auto request = [&](int k) {
      if (k < n_chunks) {
        float* dst = raw + (k % kRaw) * (kRows * kRawLd);
#pragma unroll
        for (int i = 0; i < kChunk / 4; ++i) tc::cp_async16(dst + 4 * i, src + k * kChunk + 4 * i, valid ? 16u : 0u);
      }
      tc::cp_async_commit();
    };
    for (int k = 0; k < kRaw - 1; ++k) request(k);
    bool ok = true;
    for (int c = 0; c < n_chunks && ok; ++c) {
      request(c + kRaw - 1);
      tc::cp_async_wait<kRaw - 1>();
      const int st = c % kStages;
      if (c >= kStages) ok = tc::warp_wait(&bars->empty[st], ((c / kStages) - 1) & 1, abort_flag, a.err, 61);
      if (!ok) break;
      if (warp == 0 && lane == 0) {   // the chunk's B tiles: one bulk copy (the stage's MMAs are done)
        tc::mbar_expect_tx(&bars->bfull[st], b_bytes);
        bars->b_last[st] = c;
        tc::bulk_g2s(stages + static_cast<size_t>(st) * Smem::stage(C), Wl + static_cast<size_t>(c) * 64 * C,
                     b_bytes, &bars->bfull[st]);
      }
      float4 v[kChunk / 4];
      const float4* rrow = reinterpret_cast<const float4*>(raw + (c % kRaw) * (kRows * kRawLd));
#pragma unroll
      for (int i = 0; i < kChunk / 4; ++i) v[i] = rrow[i];
      // [K-step s][hi, lo][8]: 64 TMEM columns
      float hl[64];
#pragma unroll
      for (int i = 0; i < kChunk / 4; ++i) {
        const int s = i >> 1, kk = (i & 1) * 4;
        split_tf32(v[i].x, &hl[s * 16 + kk + 0], &hl[s * 16 + 8 + kk + 0]);
        split_tf32(v[i].y, &hl[s * 16 + kk + 1], &hl[s * 16 + 8 + kk + 1]);
        split_tf32(v[i].z, &hl[s * 16 + kk + 2], &hl[s * 16 + 8 + kk + 2]);
        split_tf32(v[i].w, &hl[s * 16 + kk + 3], &hl[s * 16 + 8 + kk + 3]);
      }
      const uint32_t acol = trow + kAccCols + st * kAStageCols;
      tmem_st32(acol, *reinterpret_cast<const float(*)[32]>(&hl[0]));
      tmem_st32(acol + 32, *reinterpret_cast<const float(*)[32]>(&hl[32]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->full[st]);
    }
    tc::cp_async_wait<0>();   // no copy into this CTA's shared memory outlives the loop
    if (ok) ok = tc::warp_wait(&bars->done, 0, abort_flag, a.err, 62);
    if (ok) {
      tc_fence_after();
      const int node = node0 + t;
      for (int v0 = 0; v0 < C; v0 += 32) {
        float d[32];
        tc::tmem_ld32(trow + v0, d);
        tc::tmem_wait_ld();
        if (valid) {
          const size_t off = static_cast<size_t>(node) * D * C + static_cast<size_t>(comp) * C + v0;
          float4* o = reinterpret_cast<float4*>(a.out + off);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 s = o[i];
            s.x += d[4 * i];
            s.y += d[4 * i + 1];
            s.z += d[4 * i + 2];
            s.w += d[4 * i + 3];
            o[i] = s;
          }
          if (a.b_next) {
            float4* bn = reinterpret_cast<float4*>(a.b_next + off);
#pragma unroll
            for (int i = 0; i < 8; ++i) bn[i] = make_float4(d[4 * i], d[4 * i + 1], d[4 * i + 2], d[4 * i + 3]);
          }
        }
      }
    }
  } else if (lane == 0) {
    // ---------------------------------------------------------------- MMA thread
    const uint32_t idesc = idesc_tf32(C);
    bool ok = true;
    for (int c = 0; c < n_chunks && ok; ++c) {
      const int st = c % kStages;
      ok = mbar_wait(&bars->full[st], (c / kStages) & 1, abort_flag, a.err, 63);
      if (ok) ok = mbar_wait(&bars->bfull[st], (c / kStages) & 1, abort_flag, a.err, 65);
      if (!ok) break;
      tc_fence_after();
      const float* bst = reinterpret_cast<const float*>(stages + static_cast<size_t>(st) * Smem::stage(C));
      const uint32_t acol = tmem + kAccCols + st * kAStageCols;
#pragma unroll
      for (int s = 0; s < kChunk / 8; ++s) {
        const uint64_t dbh = smem_desc(sptr(bst + (2 * s) * C * 8));
        const uint64_t dbl = smem_desc(sptr(bst + (2 * s + 1) * C * 8));
        const uint32_t ah = acol + s * 16, al = ah + 8;
        mma_tf32_ta(tmem, ah, dbh, idesc, (c > 0 || s > 0) ? 1u : 0u);
        mma_tf32_ta(tmem, ah, dbl, idesc, 1u);
        mma_tf32_ta(tmem, al, dbh, idesc, 1u);
      }
      mma_commit(&bars->empty[st]);
    }
    if (ok) mma_commit(&bars->done);
    // drain, ignoring the abort flag: one more commit tracks every MMA issued so far
    mma_commit(&bars->drain);
    if (!mbar_wait_drain(&bars->drain, 0)) {
      tc::report_code(a.err, 64);
      bars->abort_flag = 1;
      drained = false;
    }
  }
  if (warp == kMmaWarp) drained = __shfl_sync(0xffffffffu, drained ? 1 : 0, 0) != 0;
  __syncthreads();
  // B copies still in flight (on abort no MMA waited for them) are drained before the CTA exits: a
  // stage is refilled only after its MMAs completed, which waited for its previous copy.
  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) {
      const int c = bars->b_last[st];
      if (c >= 0 && !mbar_wait_drain(&bars->bfull[st], (c / kStages) & 1)) {
        tc::report_code(a.err, 66);
        break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp && drained) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemAlloc) : "memory");
  }
}

bool supported_shape(int lmax, int C) {
  return lmax >= 1 && lmax <= 3 && C >= 32 && C <= kMaxC && C % 32 == 0;
}

template <int L>
size_t t_floats(int n_nodes, int C) {
  return static_cast<size_t>(n_nodes) * C * LadderGen<L>::S::NT;
}

size_t t_floats_rt(int lmax, int n_nodes, int C) {
  switch (lmax) {
    case 1: return t_floats<1>(n_nodes, C);
    case 2: return t_floats<2>(n_nodes, C);
    default: return t_floats<3>(n_nodes, C);
  }
}

template <int L>
size_t step_weights(int C) {
  using S = typename LadderGen<L>::S;
  size_t w = 0;
  for (int l = 0; l <= L; ++l) w += static_cast<size_t>(S::P(l)) * C * C;
  return w;
}

template <int L>
etp_status run(int C, int order, int n_nodes, const float* A, const float* W, float* out, float* bufs, float* T,
               float* Wt, int* status, cudaStream_t s) {
  constexpr int D = (L + 1) * (L + 1);
  const size_t row = static_cast<size_t>(D) * C;
  cudaError_t e = cudaMemcpyAsync(out, A, sizeof(float) * row * n_nodes, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return cuda_status(e, "full ladder: out = A");
  if (order <= 1 || n_nodes == 0) return ETP_OK;
  e = cudaFuncSetAttribute(k_ladder_mix<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem::bytes(C));
  if (e != cudaSuccess) return cuda_status(e, "full ladder smem attribute");
  const float* b_cur = A;
  const size_t wstep = step_weights<L>(C);
  const long long tasks = static_cast<long long>(n_nodes) * (C / 32);
  long long tblocks = (tasks + 7) / 8;
  if (tblocks > 148LL * 16) tblocks = 148LL * 16;
  for (int q = 1; q < order; ++q) {
    float* b_next = q + 1 < order ? bufs + static_cast<size_t>(q & 1) * row * n_nodes : nullptr;
    k_ladder_t<L><<<static_cast<int>(tblocks), 256, 0, s>>>(n_nodes, C, b_cur, A, T);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "full ladder products");
    k_ladder_wprep<L><<<static_cast<int>((wstep + 255) / 256 < 4096 ? (wstep + 255) / 256 : 4096), 256, 0, s>>>(
        C, 1, W + static_cast<size_t>(q - 1) * wstep, Wt);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "full ladder weight tiles");
    MixArgs m;
    m.n_nodes = n_nodes;
    m.C = C;
    m.T = T;
    m.Wt = Wt;
    m.b_next = b_next;
    m.out = out;
    m.err = status;
    dim3 grid((n_nodes + kRows - 1) / kRows, D);
    k_ladder_mix<L><<<grid, kThreads, Smem::bytes(C), s>>>(m);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "full ladder mixing");
    b_cur = b_next;
  }
  return ETP_OK;
}

}  // namespace

size_t step_weight_floats(int lmax, int channels);

// [status][B ping-pong: 2 x N x dim][T][one step of B operand tiles: 2 x step floats]
size_t workspace_bytes(int lmax, int channels, int n_nodes) {
  if (!supported_shape(lmax, channels) || n_nodes < 0) return 0;
  const size_t row = static_cast<size_t>((lmax + 1) * (lmax + 1)) * channels;
  return align256(sizeof(int)) + 2 * align256(sizeof(float) * row * n_nodes) +
         align256(sizeof(float) * t_floats_rt(lmax, n_nodes, channels)) +
         align256(sizeof(float) * 2 * step_weight_floats(lmax, channels));
}

size_t step_weight_floats(int lmax, int channels) {
  switch (lmax) {
    case 1: return step_weights<1>(channels);
    case 2: return step_weights<2>(channels);
    default: return step_weights<3>(channels);
  }
}

bool supported(int lmax, int channels) { return supported_shape(lmax, channels); }

etp_status launch(int lmax, int channels, int order, int n_nodes, const float* A, const float* W, float* out,
                  void* ws, cudaStream_t s, int** status_dev) {
  char* p = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(p);
  p += align256(sizeof(int));
  const size_t row = static_cast<size_t>((lmax + 1) * (lmax + 1)) * channels;
  float* bufs = reinterpret_cast<float*>(p);
  p += 2 * align256(sizeof(float) * row * n_nodes);
  float* T = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * t_floats_rt(lmax, n_nodes, channels));
  float* Wt = reinterpret_cast<float*>(p);
  *status_dev = status;
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e != cudaSuccess) return cuda_status(e, "full ladder status");
  switch (lmax) {
    case 1: return run<1>(channels, order, n_nodes, A, W, out, bufs, T, Wt, status, s);
    case 2: return run<2>(channels, order, n_nodes, A, W, out, bufs, T, Wt, status, s);
    default: return run<3>(channels, order, n_nodes, A, W, out, bufs, T, Wt, status, s);
  }
}

}  // namespace lad
}  // namespace etp

// Blackwell (sm_100a) building blocks shared by the tensor-core convolution kernels: mbarriers
// with bounded waits, tcgen05 MMA / TMEM access, async copies, and the canonical operand layout.
// Internal to libetp.
#pragma once

#include <cstdint>

namespace etp {
namespace tc {

constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 2 GHz: bounded waits
constexpr int kTmemCols = 512;

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

__device__ __forceinline__ void mbar_arrive_lane0(uint64_t* b, int lane) {
  if (lane == 0) mbar_arrive(b);
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

// Records a pipeline error code in the handle's status word. The word lives in pinned host memory
// mapped into the device address space, so it is written with a plain store (atomics on host
// memory are not relied on) and made visible to the host with a system-scope fence.
__device__ __forceinline__ void report_code(int* err, int code) {
  *reinterpret_cast<volatile int*>(err) = code;
  __threadfence_system();
}

// try_wait with a suspend-time hint: a thread whose phase is not complete sleeps in hardware until
// the phase completes or about `ns` nanoseconds pass, instead of spinning on issue slots that the
// working warps of its scheduler need.
__device__ __forceinline__ bool mbar_test_sleep(uint64_t* b, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(sptr(b)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Bounded wait on the phase of the given parity. Returns false (and raises the CTA abort flag and
// records the error code) when the limit is exceeded or another thread has aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* err,
                                          int code) {
  if (mbar_test(b, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_test_sleep(b, parity, 20000u)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      report_code(err, code);
      *abort_flag = 1;
      return false;
    }
  }
}

// Warp-uniform bounded wait: every lane waits (and so acquires), the warp follows lane 0's outcome,
// so a timeout can never split the warp's control flow.
__device__ __forceinline__ bool warp_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* err,
                                          int code) {
  const bool ok = mbar_wait(b, parity, abort_flag, err, code);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Drain wait: ignores the abort flag. Used before a CTA releases TMEM or shared memory that
// asynchronous copies or MMAs it issued may still write. Returns false if the bound is exceeded.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* b, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_test(b, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
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
// L1-allocating variant: sender rows shared by the receivers of a group hit in L1
__device__ __forceinline__ void cp_async16_ca(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16, %2;" ::"r"(sptr(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
// 8-byte copy (the .ca form is the one that takes sizes below 16)
__device__ __forceinline__ void cp_async8(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(sptr(dst)), "l"(src), "r"(src_bytes)
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

}  // namespace tc
}  // namespace etp

// common.cuh -- sm_100a building blocks shared by the HASTE kernels: mbarriers with
// bounded waits, cp.async staging, tcgen05 (TMEM allocation, MMA issue/commit,
// TMEM loads) and the shared-memory / instruction descriptors of the 5th-gen
// tensor cores.  Everything is inline PTX written for this library.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace haste {

// ---------------------------------------------------------------------------
// Device-side error word.  A kernel whose bounded wait runs out records
// kErrTimeout here (first writer wins) and unwinds; the host reads it with
// haste_device_status().  Lives in static device memory: no allocation.
// ---------------------------------------------------------------------------
enum : int { kErrNone = 0, kErrTimeout = 1, kErrBadShape = 2 };
// Defined here: the library is one translation unit.
__device__ int g_device_error = 0;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_error, 0, code); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Upper bound of any single wait inside a kernel: 2 s of wall time or 2^31
// polls, whichever comes first.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kWaitLimitPolls = 0x80000000u;
// Limit of the waits between the warps of a pipelined kernel (a producer waiting
// for a free stage, a consumer for a full one).  kWaitLimitNs unless the host
// shortens it (haste_set_wait_limit_ns) to exercise the abort paths.  Waits for
// a thread's own copies or MMAs in flight always use kWaitLimitNs, so that no
// CTA exits while they can still write its shared memory or TMEM.
__device__ uint64_t g_wait_limit_ns = kWaitLimitNs;
constexpr uint32_t kWaitSuspendNs = 20000;  // longest sleep of one poll

__device__ __forceinline__ uint32_t align1024(uint32_t a) { return (a + 1023u) & ~1023u; }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of the phase with the given parity (mbarrier.test_wait never
// suspends the thread, unlike try_wait): for threads that poll several barriers.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// As mbar_try_wait, but a thread whose phase is not complete yet is suspended
// (it issues nothing) until the phase completes or about hint_ns pass.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity to complete.  Waiting
// threads sleep in the barrier instead of spinning, so they leave the issue
// slots to the warps doing work.  Returns false (and records kErrTimeout) when
// the limit runs out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t polls = 0; polls < kWaitLimitPolls; ++polls) {
    if (mbar_try_wait_suspend(bar, parity, kWaitSuspendNs)) return true;
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
  record_error(kErrTimeout);
  return false;
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// ------------------------------------------------------------------- TMA
// 2D tiled load of one box at coordinates (c0 = innermost, c1) into shared
// memory; completion is signalled on the mbarrier as transaction bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 2D tiled store of one box from shared memory at coordinates (c0 = innermost,
// c1) of the tensor map, as a bulk async-group of the executing thread; parts of
// the box outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(tm), "r"(src),
               "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every bulk group of this thread has completed (its writes performed).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Hint: bring `bytes` (a multiple of 16, 16-byte aligned) of global memory into
// L2 without waiting for them; a later load of the range then finds it there.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- cp.async
// 16-byte global->shared copy through L2 only; src_bytes < 16 zero-fills the rest.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// Named barrier over a subset of warps (ids 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also ORs a predicate over its threads: every thread gets the
// same answer.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred c, p;\n\tsetp.ne.u32 c, %2, 0;\n\tbar.red.or.pred p, %1, %3, c;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(id), "r"((uint32_t)pred), "r"(nthreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Wait until at most N of this thread's committed cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Make generic-proxy shared-memory writes visible to the tensor core (async proxy).
// The mbarrier receives one arrival once every cp.async this thread issued so
// far has landed (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive_on(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 128-byte swizzle (16-byte chunk index XOR row-in-atom) of a byte offset inside
// a 1024-byte aligned region.
__device__ __forceinline__ uint32_t sw128(uint32_t off) { return off ^ (((off >> 7) & 7u) << 4); }
// 128-byte swizzle with 32-byte granularity (32-byte chunk index XOR row-in-atom,
// 4 rows of 128 B per 512-byte atom): the shared-memory layout that MN-major
// tf32 operands of tcgen05.mma require.
__device__ __forceinline__ uint32_t sw128_32b(uint32_t off) { return off ^ (((off >> 7) & 3u) << 5); }

// Swizzle of rows of rb = 32, 64 or 128 bytes inside a 1024-byte aligned region
// (16-byte chunk index XOR bits 7.. of the offset), the pattern of the TMA and
// UMMA 32B / 64B / 128B swizzle modes.
__device__ __forceinline__ uint32_t swz_rows(uint32_t off, int rb) {
  const uint32_t m = (uint32_t)(rb / 16 - 1);
  return off ^ (((off >> 7) & m) << 4);
}

// Swizzle of a 128B-row tile for element type T read as a K-major (kMN = false)
// or MN-major (kMN = true) operand.
template <typename T, bool kMN>
__device__ __forceinline__ uint32_t swz(uint32_t off) {
  if constexpr (kMN && sizeof(T) == 4) return sw128_32b(off);
  else return sw128(off);
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, one instruction; kind::f16 (bf16 inputs) or
// kind::tf32 (fp32 inputs read as tf32).  accumulate = 0 overwrites D.
template <bool kTF32>
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  if constexpr (kTF32) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}
// Weight-stationary form, cta_group::1 (tcgen05.mma.ws): M in {32, 64, 128}, N in
// {64, 128, 256}.  Where D sits in TMEM (N columns of fp32 in total):
//   M = 32: row m in lane 32q + m of every lane quarter q, which holds the
//           columns n in [qN/4, (q+1)N/4) at column offset n - qN/4;
//   M = 64: rows 0-63 in lanes 0-63 for n < N/2 and in lanes 64-127 for
//           n >= N/2, at column offset n mod N/2.
// For a small M the instruction costs far less than a 128-row one of the same N.
__device__ __forceinline__ void mma_ws(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.ws.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier when all previously issued MMAs of this thread finish.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp receives lane
// (32*(warp%4) + i), columns [col, col+16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// ------------------------------------------------------------- descriptors
// Layout codes of the shared-memory matrix descriptor (bits 61..63).
enum : uint32_t { kLayoutNone = 0, kLayoutSw128Base32 = 1, kLayoutSw128 = 2, kLayoutSw64 = 4, kLayoutSw32 = 6 };

// Descriptor layout code of rows of rb bytes (128, 64 or 32).
__host__ __device__ constexpr uint32_t layout_for_rows(int rb) {
  return rb == 128 ? kLayoutSw128 : rb == 64 ? kLayoutSw64 : kLayoutSw32;
}

// Shared-memory matrix descriptor: start address, leading-dimension byte offset
// (LBO), stride-dimension byte offset (SBO), descriptor version 1 (bit 46) and
// the swizzle layout.  For the no-swizzle layout LBO steps between 8x16B core
// matrices along K and SBO along M/N; for 128B-swizzled K-major operands SBO
// steps between 8-row groups (LBO unused); for 128B-swizzled MN-major operands
// LBO steps between 64-element (bf16) MN blocks and SBO between 8-row K groups.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)layout << 61;
  return d;
}

// Descriptor of a 128B-swizzled MN-major operand: lbo = stride between
// 128-byte MN blocks; K groups are 8 rows (1024 B) apart, or 4 rows (512 B) in
// the 32-byte-granular swizzle of tf32.
template <typename T>
__device__ __forceinline__ uint64_t mn_desc(uint32_t saddr, uint32_t lbo) {
  if constexpr (sizeof(T) == 4) return make_sdesc(saddr, lbo, 512, kLayoutSw128Base32);
  else return make_sdesc(saddr, lbo, 1024, kLayoutSw128);
}

// Instruction descriptor for dense MMAs with fp32 accumulation.
// fmt: 1 = bf16 (kind::f16), 2 = tf32 (kind::tf32).  a_mn/b_mn: operand is
// MN-major (1) or K-major (0).  M in {64,128}; N multiple of 16 up to 256.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t fmt, uint32_t a_mn, uint32_t b_mn, uint32_t M,
                                                  uint32_t N) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) |
         ((M >> 4) << 24);
}

// ------------------------------------------------------------------ math
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 32-byte global store (sm_100): 16 bf16 values packed from v[0..16); p must be
// 32-byte aligned.  One store covers a whole 32-byte sector.
__device__ __forceinline__ void st_global_bf16x16(void* p, const float* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(pack_bf16x2(v[0], v[1])),
               "r"(pack_bf16x2(v[2], v[3])), "r"(pack_bf16x2(v[4], v[5])), "r"(pack_bf16x2(v[6], v[7])),
               "r"(pack_bf16x2(v[8], v[9])), "r"(pack_bf16x2(v[10], v[11])), "r"(pack_bf16x2(v[12], v[13])),
               "r"(pack_bf16x2(v[14], v[15]))
               : "memory");
}

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  static constexpr bool kTF32 = true;
  static constexpr uint32_t kFmt = 2;
  static constexpr int kMmaK = 8;   // K per tcgen05.mma instruction
  __device__ static float to_f(float v) { return v; }
  __device__ static float from_f(float v) { return v; }
};
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr bool kTF32 = false;
  static constexpr uint32_t kFmt = 1;
  static constexpr int kMmaK = 16;
  __device__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  __device__ static __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

}  // namespace haste

// Thin inline-PTX wrappers for the sm_100a features the attention kernels use:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM alloc, MMA, commit,
// TMEM load/store) and the UMMA shared-memory / instruction descriptors.
//
// Every wait here is bounded: past a time limit it records an error code
// in the device status word and returns false, so a kernel can drain and exit
// instead of hanging the GPU.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace attn {

// Device status word of the library (the whole device side is one translation
// unit): 0 = ok; otherwise the first error code recorded.
// Code 1 = an mbarrier wait timed out (the only code the kernels record).
__device__ int g_attn_status = 0;

// Work-unit counters for dynamically scheduled kernels: each launch takes one
// slot (rotated by the host) and a generation number; sched_reset_kernel, on the
// same stream just before the launch, sets the slot to (generation << 32) | 0, and a
// claim is one 64-bit atomicAdd whose old value carries the generation it counted
// in.  A claim that finds another generation (more than kSchedSlots launches in
// flight at once, so a later launch has reset the slot) stops its launch and records
// error 3; its stray increment may cost the later launch a unit, which is why the
// error stands for both launches.  A compare-and-swap claim would keep the later
// launch intact, but it serialises under contention (up to 60% slower measured on
// workloads of many short units).
constexpr int kSchedSlots = 128;
constexpr int kSchedSelftestSlot = kSchedSlots;   // one more, used only by the scheduler self-test
__device__ unsigned long long g_sched[kSchedSlots + 1];

__global__ void sched_reset_kernel(int slot, unsigned int gen) {
  if (threadIdx.x == 0) g_sched[slot] = static_cast<unsigned long long>(gen) << 32;
}

__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Checking build (compiled with -DATTN_CHECKS): every tile coordinate, head index and
// global row the kernels compute is tested against the tensor it addresses before the
// access; a value out of range records error 2 in the status word and the access is
// skipped (stores) or kept harmless (TMA tile loads, which zero-fill outside the
// tensor).  No trap, no assert.  In the normal build the tests compile away.
#ifdef ATTN_CHECKS
constexpr bool kChecks = true;
#else
constexpr bool kChecks = false;
#endif
__device__ __forceinline__ bool in_range(long long idx, long long n) {
  if constexpr (kChecks) {
    if (idx < 0 || idx >= n) {
      record_error(&g_attn_status, 2);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}


// One lane of a converged warp (elect.sync); the others get false.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Orders later uses of registers written by an asynchronous TMEM load after the
// tcgen05.wait::ld that precedes this call (both are volatile asm, kept in order).
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
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

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool status_set() {
  return *reinterpret_cast<volatile int*>(&g_attn_status) != 0;
}

// A legitimate wait inside these kernels lasts microseconds to milliseconds;
// anything past this bound is treated as a lost arrival.
constexpr uint64_t kWaitTimeoutNs = 4000000000ull;

// Bounded wait for the mbarrier phase with the given parity to complete.  Gives
// up (returns false) after kWaitTimeoutNs, recording error 1, or as soon as any
// CTA has recorded an error.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (status_set()) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        record_error(&g_attn_status, 1);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_for(bar, parity, kWaitTimeoutNs);
}

// Bounded wait used only on error paths, to let copies already in flight land.
__device__ __forceinline__ void mbar_drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > 100000000ull) return;
}

// Ring of work-unit indices: one producer thread claims units from g_sched and
// posts them; each consumer warp takes them in the same order.  A posted -1 ends
// the sequence.
struct UnitRing {
  uint64_t full[4];     // count 1: the producer posted slot k & 3
  uint64_t empty[4];    // count = number of consumer warps
  int idx[4];
};

__device__ __forceinline__ void unit_ring_init(UnitRing& r, uint32_t consumers) {
  for (int i = 0; i < 4; ++i) {
    mbar_init(&r.full[i], 1);
    mbar_init(&r.empty[i], consumers);
  }
}

// Producer (one thread): claim the k-th unit of this CTA from counter `slot` of
// generation `gen`, post it (or -1 once u >= n, or once the slot belongs to another
// launch), return it; -2 if a wait failed.
__device__ __forceinline__ int unit_ring_claim(UnitRing& r, int k, int slot, unsigned int gen, int n) {
  const int i = k & 3;
  if (k >= 4 && !mbar_wait(&r.empty[i], ((k >> 2) - 1) & 1)) return -2;
  const unsigned long long old = atomicAdd(&g_sched[slot], 1ull);
  int u = static_cast<int>(old & 0xffffffffull);
  if (static_cast<unsigned int>(old >> 32) != gen) {
    record_error(&g_attn_status, 3);
    u = -1;
  }
  if (u >= n) u = -1;
  r.idx[i] = u;
  mbar_arrive(&r.full[i]);              // release: the index is visible before the arrival
  return u;
}


// Consumer (whole warp): the k-th unit of this CTA, -1 when none is left.
__device__ __forceinline__ int unit_ring_take(UnitRing& r, int k, int lane, bool& ok) {
  const int i = k & 3;
  ok = __all_sync(0xffffffffu, mbar_wait(&r.full[i], (k >> 2) & 1));
  if (!ok) return -1;
  const int u = *reinterpret_cast<volatile int*>(&r.idx[i]);
  __syncwarp();
  if (lane == 0) mbar_arrive(&r.empty[i]);
  return u;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 3-D tiled load: coordinates are (x = column, y = row, z = head), x in elements.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Same load with an L2 eviction-priority policy (from l2_policy_*).
__device__ __forceinline__ void tma_load_3d_hint(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y,
                                                 int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}

// L2 cache policies for loads: keep data that other CTAs will read again, let
// data read once leave first.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}



// Split shared-memory descriptors (128B swizzle): the low word holds the start
// address and the leading byte offset, the high word the stride byte offset,
// the descriptor version and the swizzle mode.  Offsets inside a tile are added
// to the low word (start address field, 16-byte units; shared addresses stay
// below 2^18, so the field never carries).
__host__ __device__ constexpr uint32_t sdesc_hi_sw128(uint32_t sbo_bytes) {
  return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}
__device__ __forceinline__ uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}

// D[tmem] (+)= A[smem] * B[smem]^T from split descriptors sharing one high word.
__device__ __forceinline__ void umma_ss_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T with B from a split descriptor.
__device__ __forceinline__ void umma_ts_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same two products with 8-bit operands (kind::f8f6f4; e4m3 here): K = 32
// elements (32 bytes) per instruction instead of 16.
__device__ __forceinline__ void umma_ss_f8_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_ts_f8_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on an mbarrier when all previously issued tcgen05 ops of this thread finish.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Warp-collective TMEM load: thread t of the warp reads lane (quadrant*32 + t),
// 32 consecutive 32-bit columns starting at the column in taddr.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
      "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}


__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}



// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulate:
//   [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format (1 = bf16),
//   [15] A major (0 = K, 1 = MN), [16] B major, [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                       bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor for kind::f8f6f4 with e4m3 A/B (format code 0) and fp32
// accumulate; the other fields as in idesc_bf16_f32.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------- math
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Three-input max (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic): two lanes of work per instruction.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// exp2 of a pair on the FMA pipe, to take load off the MUFU pipe (16 ex2 per SM
// per clock).  Range reduction x = n + f with n = round(x), |f| <= 1/2, via the
// 1.5 * 2^23 rounding constant; 2^f from a cubic fitted for minimum relative error
// on [-1/2, 1/2] (gen_exp2_poly.py: bound 7.5e-5, far below bf16 rounding); 2^n
// added to the exponent field as an integer.  Inputs below -126 are clamped, so
// the result is at least 2^-126.5 instead of underflowing (vanishing next to the
// row's other terms, which include 2^0 or more).
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716648042202f;

__device__ __forceinline__ void exp2_fma_pair(float x0, float x1, float& y0, float& y1) {
  const uint64_t x = f2pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = fadd2(x, f2pack(12582912.f, 12582912.f));            // 1.5 * 2^23 + n
  const uint64_t r = fadd2(t, f2pack(-12582912.f, -12582912.f));          // n as a float
  const uint64_t f = ffma2(r, f2pack(-1.f, -1.f), x);                     // x - n
  uint64_t q = ffma2(f, f2pack(kExp2C3, kExp2C3), f2pack(kExp2C2, kExp2C2));
  q = ffma2(q, f, f2pack(kExp2C1, kExp2C1));
  q = ffma2(q, f, f2pack(kExp2C0, kExp2C0));
  float q0, q1, t0, t1;
  f2unpack(q, q0, q1);
  f2unpack(t, t0, t1);
  // the low bits of t's pattern hold n; shifted by 23 only n's bits survive
  y0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}


// Two floats to two e4m3 bytes (round to nearest even, saturating to +-448); lo in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two packed fp32 to one bf16x2 word (round to nearest even), first value in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2_2(uint64_t v) {
  float lo, hi;
  f2unpack(v, lo, hi);
  return pack_bf16x2(lo, hi);
}

// Row-per-lane tiles to row-contiguous stores.  A thread that owns one row of a
// tile holds NC 16-byte chunks of it; a warp storing chunk k of its 32 rows per
// instruction touches 32 separate lines.  This exchanges chunks inside each group
// of NC lanes (an NC x NC transpose in log2(NC) butterfly steps of shuffles), so
// that afterwards lane NC*g + i holds chunk i of the group's rows NC*g + t in c[t]:
// storing c[t] from every lane writes 32 / NC whole row segments of NC * 16 bytes.
template <int NC>
__device__ __forceinline__ void transpose_row_chunks(uint32_t (&c)[NC][4], int lane) {
  static_assert(NC == 2 || NC == 4 || NC == 8, "NC must be 2, 4 or 8");
#pragma unroll
  for (int m = NC / 2; m >= 1; m >>= 1) {
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int lo = 0; lo < NC; ++lo) {
      if (lo & m) continue;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        // the lower lane of a pair sends its upper chunk and takes the partner's lower one
        const uint32_t r = __shfl_xor_sync(0xffffffffu, up ? c[lo][w] : c[lo | m][w], m);
        if (up)
          c[lo][w] = r;
        else
          c[lo | m][w] = r;
      }
    }
  }
}

}  // namespace attn

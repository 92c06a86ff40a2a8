// sm100.cuh - thin inline-PTX wrappers for the sm_100a features the kernels
// use: mbarriers (with bounded waits), TMA tile loads, bulk copies, and the
// 5th-generation tensor core (tcgen05: TMEM allocation, MMA, commit, TMEM
// loads/stores, fences) plus the UMMA shared-memory and instruction
// descriptors.  Written from the PTX ISA; every TMA and bulk load writes
// the shared memory of the issuing CTA only.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace vdn {

// ------------------------------------------------------------------ basics

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }
__device__ __forceinline__ uint32_t warp_id() { return threadIdx.x >> 5; }

// Warp-uniform: true in exactly one lane of the (fully active) warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Register re-split between warpgroups (all 128 threads of a warpgroup execute it).
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------------ packed fp32 math

__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// (a * b + c) on two fp32 lanes in one instruction
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA/ALU pipes (no special-function unit), for x <= 64.
// Cody-Waite style reduction x = n + f, n = round(x) by the 1.5 * 2^23
// magic-number addition, f in [-1/2, 1/2]; 2^f by a degree-3 polynomial
// fitted for minimax relative error (Lawson's algorithm; coefficients from
// csrc/exp2_poly.py, max relative error 7.5e-5 in float32); 2^n applied by
// adding n to the exponent field.  x is clamped at -126 so the result stays a
// (tiny) non-negative float; masked -inf scores give 2^-126-ish, not 0.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -126.0f);
  const float t = __fadd_rn(x, 12582912.0f);  // 1.5 * 2^23: n in the low mantissa bits
  const float n = __fadd_rn(t, -12582912.0f);
  const float f = __fadd_rn(x, -n);
  float p = fmaf(0.05517149344086647f, f, 0.24261093139648438f);
  p = fmaf(p, f, 0.6932609677314758f);
  p = fmaf(p, f, 0.9999280571937561f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f32x2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x of two values at once on the FMA pipe, packed f32x2 arithmetic: the
// same reduction and polynomial as exp2_fma (x clamped at -126; n = round(x)
// by the 1.5 * 2^23 addition, f = x - n in [-1/2, 1/2], 2^f by the fitted
// cubic, 2^n added into the exponent field).  Ten instructions per pair;
// valid for x <= 64.
__device__ __forceinline__ uint64_t exp2x2_fma(uint64_t x) {
  float x0, x1;
  f32x2_unpack(x, x0, x1);
  x = f32x2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t magic = f32x2_pack(12582912.0f, 12582912.0f);
  const uint64_t t = f32x2_add(x, magic);   // n in the low mantissa bits
  const uint64_t n = f32x2_sub(t, magic);   // round(x)
  const uint64_t f = f32x2_sub(x, n);
  uint64_t p = f32x2_fma(f32x2_pack(0.05517149344086647f, 0.05517149344086647f), f,
                         f32x2_pack(0.24261093139648438f, 0.24261093139648438f));
  p = f32x2_fma(p, f, f32x2_pack(0.6932609677314758f, 0.6932609677314758f));
  p = f32x2_fma(p, f, f32x2_pack(0.9999280571937561f, 0.9999280571937561f));
  float p0, p1, t0, t1;
  f32x2_unpack(p, p0, p1);
  f32x2_unpack(t, t0, t1);
  return f32x2_pack(__int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23)),
                    __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23)));
}

// sigmoid(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh (one special-function op)
__device__ __forceinline__ float sigmoid_tanh(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

// sigmoid of two packed fp32 values: the arithmetic of sigmoid_tanh on each,
// the multiply and the fma packed
__device__ __forceinline__ uint64_t sigmoid2_tanh(uint64_t x) {
  const uint64_t half = f32x2_pack(0.5f, 0.5f);
  float h0, h1, t0, t1;
  f32x2_unpack(f32x2_mul(x, half), h0, h1);
  asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(h0));
  asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(h1));
  return f32x2_fma(half, f32x2_pack(t0, t1), half);
}

// ------------------------------------------------------------------ abort / status

// Status shared by the warps of one CTA.  A wait that runs out sets `abort`
// (so every other waiter gives up quickly), records VDN_ERR_TIMEOUT (6) in
// the global status word and describes itself in the timeout record.
struct CtaAbort {
  int* flag;           // shared memory
  int* global_status;  // device memory, may be null
  int* record;         // device memory (kRec* words), may be null
  int kernel;          // kernel id written into the record
};

constexpr int kStatusTimeout = 6;
// Waits are bounded in global time (%globaltimer, nanoseconds), not in SM
// cycles: after a compute preemption a CTA may resume on another SM, whose
// cycle counter has no relation to the one read before.
constexpr long long kWaitNs = 1000000000ll;  // 1 s

// Timeout record (int words): the first wait that ran out since the record
// was cleared.
enum : int {
  kRecTimeouts = 0,  // waits that ran out
  kRecKernel = 1,    // kernel id of the first
  kRecBlock = 2,     // its blockIdx.x
  kRecWarp = 3,      // its warp
  kRecBarOff = 4,    // byte distance from its barrier to the CTA's abort flag
  kRecParity = 5,    // the phase parity it waited for
  kRecNs = 6,        // global nanoseconds it waited (two words, low first)
  kRecSm = 8,        // SM it ran on
  kRecWords = 16
};

__device__ __forceinline__ long long global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return (long long)t;
}

__device__ __forceinline__ int sm_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
  return (int)r;
}

// Sleep for about `ns` nanoseconds of global time (debug stalls only).
__device__ __forceinline__ void sleep_ns(long long ns) {
  const long long t0 = global_ns();
  while (global_ns() - t0 < ns) __nanosleep(1000);
}

__device__ __forceinline__ bool aborted(const CtaAbort& ab) {
  return *reinterpret_cast<volatile int*>(ab.flag) != 0;
}

__device__ __forceinline__ void raise_abort(const CtaAbort& ab) {
  *reinterpret_cast<volatile int*>(ab.flag) = 1;
  if (ab.global_status) atomicExch(ab.global_status, kStatusTimeout);
}

// Out of line: only a wait that ran out gets here.
static __device__ __noinline__ void record_timeout(const CtaAbort& ab, const void* bar, uint32_t parity, long long ns) {
  if (!ab.record) return;
  if (atomicAdd(ab.record + kRecTimeouts, 1) != 0) return;
  int* r = ab.record;
  r[kRecKernel] = ab.kernel;
  r[kRecBlock] = (int)blockIdx.x;
  r[kRecWarp] = (int)(threadIdx.x >> 5);
  r[kRecBarOff] = (int)(smem_u32(ab.flag) - smem_u32(bar));
  r[kRecParity] = (int)parity;
  r[kRecNs] = (int)(ns & 0xffffffffll);
  r[kRecNs + 1] = (int)(ns >> 32);
  r[kRecSm] = sm_id();
  __threadfence();
}

// Named barrier `id` over `nthreads` threads (whole warps) that also ORs a
// predicate: every participant leaves with the same answer.
__device__ __forceinline__ bool bar_any(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of a phase (no suspension).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Bounded: gives up
// after `limit_ns` nanoseconds of global time (kWaitNs by default) or when
// another warp of the CTA has given up, returning false.  Every thread that
// calls it must act on a false return.  The clock is read every 64 probes
// only, the first reading starting the count.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const CtaAbort& ab,
                                          long long limit_ns = kWaitNs) {
  if (mbar_test_wait(bar, parity)) return true;  // already complete: no suspension
  if (mbar_try_wait(bar, parity)) return true;
  long long g0 = 0;
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++n & 63u) == 0) {
      if (aborted(ab)) return false;
      const long long g1 = global_ns();
      if (n == 64) {
        g0 = g1;
      } else if (g1 - g0 > limit_ns) {
        record_timeout(ab, bar, parity, g1 - g0);
        raise_abort(ab);
        return false;
      }
    }
  }
}

// Bounded wait until the gpu-scope counter *counter has reached `target`
// (an acquire load, so that what the counting threads wrote before their
// release is visible after it); false, with the timeout recorded (barrier
// offset 0, parity 2: a counter wait), after limit_ns of global time or when
// the CTA gave up.
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ bool counter_wait(const unsigned* counter, unsigned target, const CtaAbort& ab,
                                             long long limit_ns = kWaitNs) {
  if (ld_acquire_u32(counter) >= target) return true;
  const long long g0 = global_ns();
  while (true) {
    __nanosleep(256);
    if (ld_acquire_u32(counter) >= target) return true;
    if (aborted(ab)) return false;
    const long long g1 = global_ns();
    if (g1 - g0 > limit_ns) {
      record_timeout(ab, ab.flag, 2u, g1 - g0);
      raise_abort(ab);
      return false;
    }
  }
}

// Short bounded wait (kWaitNs / 4) used only while draining on the abort path.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = global_ns();
  uint32_t n = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++n & 63u) == 0 && global_ns() - t0 > (kWaitNs >> 2)) return;
  }
}

// ------------------------------------------------------------------ TMA / bulk copies

// 2-D tiled TMA load, into this CTA's shared memory, of the box at element coordinates
// (x = innermost, y) into shared memory; completes `bytes` on bar.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Prefetch the same box into L2 (no shared-memory write, no barrier).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

// Bring a global 128-byte line into L2 ahead of use.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Contiguous global -> shared bulk copy (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Make generic-proxy writes to shared memory visible to the async proxy
// (TMA, tensor core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Global memory written through the generic proxy (plain stores, made visible
// by a release/acquire pair) and then read through the async proxy (a bulk
// copy): the reading thread fences between its acquire and the copy.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05: TMEM

// Allocate `ncols` (power of two >= 32) TMEM columns; the base address is
// written to *slot (shared).  Executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
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
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM address: lane in bits [16, 32), column in bits [0, 16).
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

// TMEM loads/stores of shape 32x32b: thread t of the warp reads/writes lane
// (lane base + t); .xN covers N consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld1(uint32_t taddr, uint32_t& r0) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r0) : "r"(taddr) : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ tcgen05: MMA

// UMMA shared-memory matrix descriptor (sm_100 "version 1" format):
// start address >> 4 in [0,14), leading byte offset >> 4 in [16,30), stride
// byte offset >> 4 in [32,46), version 1 at bit 46, base offset 0, layout type
// in [61,64) (0 none, 2 = 128-byte swizzle, 4 = 64-byte, 6 = 32-byte).
enum : uint32_t { kLayoutNone = 0, kLayoutSw128 = 2 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B and fp32 accumulation.
// a_mn / b_mn: operand stored MN-major (1) or K-major (0).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((uint32_t)a_mn << 15)       // A major
         | ((uint32_t)b_mn << 16)       // B major
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; one thread issues.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]; A is M x K with 16-bit elements packed
// two per 32-bit column (lane = row).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f8f6f4 with e4m3 A and B (both K-major) and
// fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                      // D format: f32
         | (0u << 7)                    // A format: e4m3
         | (0u << 10)                   // B format: e4m3
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// The same products with 8-bit operands (K = 32 per instruction).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// A from TMEM: M x K 8-bit elements packed four per 32-bit column (lane = row).
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The mbarrier tracks completion of every earlier tcgen05 async op of this thread.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ------------------------------------------------------------------ packing helpers

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&t);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

}  // namespace vdn

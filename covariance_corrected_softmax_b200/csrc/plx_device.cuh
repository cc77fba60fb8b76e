// plx_device.cuh -- device-side building blocks shared by the Parallax kernels
// (sm_100a): mbarriers with bounded waits, TMA tensor loads, tcgen05 tensor
// memory and MMA wrappers, bf16 helpers.  Inline PTX written from the PTX ISA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace plx {

// ---------------------------------------------------------------------------
// Device error word.  Kernels never spin forever: every wait is bounded by a
// wall-clock limit; on expiry the kernel records a code here and returns.
// ---------------------------------------------------------------------------
enum DeviceError : unsigned {
  kDevOk = 0,
  kDevTimeoutMbarrier = 1,   // an mbarrier wait ran out of time
  kDevBadArgument = 2,       // a kernel saw inconsistent arguments
  kDevNonFinite = 3,         // a result was not finite (inputs out of range)
};

// The device status block lives in the library (plx_abi.cu), one per device;
// kernels get the address of its first word (the error code) as a parameter.
// The wall-clock limit of every bounded wait sits in the same block, so a
// diagnostic entry point can shorten it without rebuilding the kernels.
struct DeviceStatus {
  unsigned error;                   // first DeviceError recorded (0 = none)
  unsigned reserved;
  unsigned long long wait_limit_ns; // limit of one bounded wait
};

__device__ __forceinline__ void record_error(unsigned* err, unsigned code) {
  if (err) atomicCAS(err, 0u, code);
}

// This launch's grid identifier (unique per launch in the context, graph
// replays included): tags data one launch leaves for another CTA of the same
// launch, so that what an earlier launch left behind is never mistaken for it.
__device__ __forceinline__ int launch_tag() {
  uint64_t id;
  asm volatile("mov.u64 %0, %%gridid;" : "=l"(id));
  return (int)((id ^ (id >> 31)) & 0x7fffffffu);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Default wall-clock limit of a single wait (ns).  Long enough for any
// legitimate stall (including profiler replay), short enough to give the GPU
// back.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Backstop on the number of polls of one wait, should the wall clock stop: a
// poll takes tens of nanoseconds or more, so this is tens of seconds.
constexpr uint32_t kWaitMaxPolls = 1u << 30;

// The wait limit in force on this device (the status block's, or the default
// when a kernel runs without one).
__device__ __forceinline__ uint64_t wait_limit_ns(const unsigned* err) {
  if (!err) return kWaitLimitNs;
  return reinterpret_cast<const volatile DeviceStatus*>(err)->wait_limit_ns;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
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

// Non-blocking probe: has the phase with this parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
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

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start before the previous kernel in the stream has
// finished; grid_dep_wait() blocks until that kernel has completed and its
// memory is visible.  grid_dep_launch_dependents() lets such a dependent
// kernel be scheduled before this one finishes.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Three-input max / min (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair, on the FMA pipe instead of the special-function unit.
// Range reduction after Cody and Waite: x = n + f with n = round(x) (added to a
// 1.5 * 2^23 bias, so n sits in the low mantissa bits) and f in [-1/2, 1/2];
// 2^f by a degree-4 polynomial, relative-error minimax on [-1/2, 1/2] (fit by
// exp2_poly_fit.py beside this file; max relative error 2.7e-6); 2^n added to
// the exponent field.  Inputs are clamped to >= -32 (2^-32: below fp16's
// smallest subnormal, which is all the callers keep) and must be <= 64.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -32.f);
  x.y = fmaxf(x.y, -32.f);
  const float2 bias = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23
  const float2 y = __fadd2_rn(x, bias);
  const float2 n = __fadd2_rn(y, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 r = make_float2(9.569985792e-03f, 9.569985792e-03f);
  r = __ffma2_rn(r, f, make_float2(5.591785908e-02f, 5.591785908e-02f));
  r = __ffma2_rn(r, f, make_float2(2.402474731e-01f, 2.402474731e-01f));
  r = __ffma2_rn(r, f, make_float2(6.931217909e-01f, 6.931217909e-01f));
  r = __ffma2_rn(r, f, make_float2(9.999992847e-01f, 9.999992847e-01f));
  // low bits of y hold n (two's complement); << 23 moves them to the exponent
  return make_float2(__int_as_float(__float_as_int(r.x) + (__float_as_int(y.x) << 23)),
                     __int_as_float(__float_as_int(r.y) + (__float_as_int(y.y) << 23)));
}

// 2^x with the hardware approximation (ex2.approx.ftz.f32, about 2 ulp).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Waits until the phase with the given parity has completed.  Returns false
// (and records kDevTimeoutMbarrier) if the wall-clock limit runs out (or the
// poll backstop is reached) or if *abort becomes nonzero (another role of the
// CTA gave up).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort, unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint64_t limit = 0;
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++spins & 63u) == 0) {
      if (*abort) return false;
      if (limit == 0) limit = wait_limit_ns(err);
      if (globaltimer_ns() - t0 > limit || spins >= kWaitMaxPolls) {
        record_error(err, kDevTimeoutMbarrier);
        *abort = 1;
        return false;
      }
    }
  }
  return true;
}

// A barrier among whole warps on an mbarrier initialised with their number (one
// arrival per warp), bounded like mbar_wait: false in every lane of the warp if
// the wait gave up (a warp that left its loop early never arrives, so the
// others record a timeout instead of waiting for good).  `phase` counts the
// caller's completed uses of the barrier.
__device__ __forceinline__ bool warps_sync(uint64_t* bar, uint32_t& phase, volatile int* abort,
                                           unsigned* err) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase & 1u, abort, err);
  ++phase;
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), plain tile loads into this CTA's
// shared memory, completing on an mbarrier with a transaction count.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Pull a 4-D tile into L2 ahead of its use (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* map, int c0, int c1,
                                                   int c2, int c3) {
  asm volatile(
      "cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory (TMEM) and the 5th-generation tensor-core MMA.
// TMEM addresses: bits [31:16] lane, [15:0] column (32-bit columns).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
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

// D[tmem] (+)= A[smem desc] * B[smem desc]; kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc].
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16: fp32 accumulator, A and B both bf16 or
// both fp16, A K-major, B K-major or MN-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_f16kind(int M, int N, bool b_mn_major,
                                                          bool fp16_operands) {
  return (1u << 4)                                  // D format: f32
         | ((fp16_operands ? 0u : 1u) << 7)         // A format: f16 = 0, bf16 = 1
         | ((fp16_operands ? 0u : 1u) << 10)        // B format: f16 = 0, bf16 = 1
         | ((b_mn_major ? 1u : 0u) << 16)           // B major-ness
         | ((uint32_t)(N >> 3) << 17)               // N / 8
         | ((uint32_t)(M >> 4) << 24);              // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 layout, version 1).
// lbo/sbo in bytes: K-major tiles use lbo = 16 (unused) and sbo = the stride of
// 8-row groups; MN-major tiles use lbo = the stride of 64-element column blocks
// and sbo = the stride of 8-row (K) groups.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo,
                                                    uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // version (sm100)
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// 32 lanes x 32 bits, repeated over consecutive columns: each thread of the warp
// moves its own lane's columns.
// Loads are asynchronous until tcgen05.wait::ld; the wait sits in the same asm
// statement as the load(s), so no instruction can read the registers early.
#define PLX_R8(a, i) "=r"(a[i]), "=r"(a[i + 1]), "=r"(a[i + 2]), "=r"(a[i + 3]), \
                     "=r"(a[i + 4]), "=r"(a[i + 5]), "=r"(a[i + 6]), "=r"(a[i + 7])
__device__ __forceinline__ void tmem_ld32_sync(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : PLX_R8(r, 0), PLX_R8(r, 8), PLX_R8(r, 16), PLX_R8(r, 24)
      : "r"(taddr)
      : "memory");
}
// Two 32-column loads (from two TMEM addresses) under one wait.
__device__ __forceinline__ void tmem_ld2x32_sync(uint32_t ta, uint32_t tb, uint32_t (&a)[32],
                                                 uint32_t (&b)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, "
      "%41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, "
      "%58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : PLX_R8(a, 0), PLX_R8(a, 8), PLX_R8(a, 16), PLX_R8(a, 24), PLX_R8(b, 0), PLX_R8(b, 8),
        PLX_R8(b, 16), PLX_R8(b, 24)
      : "r"(ta), "r"(tb)
      : "memory");
}
// Two 16-column loads (from two TMEM addresses) under one wait.
__device__ __forceinline__ void tmem_ld2x16_sync(uint32_t ta, uint32_t tb, uint32_t (&a)[16],
                                                 uint32_t (&b)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16, %17, %18, %19, %20, %21, %22, %23, %24, "
      "%25, %26, %27, %28, %29, %30, %31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : PLX_R8(a, 0), PLX_R8(a, 8), PLX_R8(b, 0), PLX_R8(b, 8)
      : "r"(ta), "r"(tb)
      : "memory");
}
// One 16-column load.
__device__ __forceinline__ void tmem_ld16_sync(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : PLX_R8(r, 0), PLX_R8(r, 8)
      : "r"(taddr)
      : "memory");
}
// One column from each of two TMEM addresses under one wait.
__device__ __forceinline__ void tmem_ld2x1_sync(uint32_t ta, uint32_t tb, uint32_t& a,
                                                uint32_t& b) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%2];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%1}, [%3];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a), "=r"(b)
      : "r"(ta), "r"(tb)
      : "memory");
}
#undef PLX_R8
#define PLX_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), \
                  "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      PLX_W8(0), PLX_W8(8), PLX_W8(16), PLX_W8(24)
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      PLX_W8(0), PLX_W8(8)
      : "memory");
}
#undef PLX_W8
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Named barriers for a subset of the CTA's warps.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads: every
// thread gets the same answer, so a group can leave a loop together.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.cta.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------------------
// bf16 <-> fp32
// ---------------------------------------------------------------------------
// Two bf16 packed in a 32-bit word -> (low, high) as fp32 (exact).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  float2 r;
  r.x = __uint_as_float(w << 16);
  r.y = __uint_as_float(w & 0xffff0000u);
  return r;
}

// Round two fp32 to fp16 (nearest-even) and pack (lo in the low half).
__device__ __forceinline__ uint32_t float2_to_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Element-wise maximum of two bf16 pairs (max.bf16x2).
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Two fp16 packed in a 32-bit word -> (low, high) as fp32 (exact).
__device__ __forceinline__ float2 f16x2_to_float2(uint32_t w) {
  float2 r;
  asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "r"(w));
  return r;
}

// fence.proxy.async: make this thread's generic-proxy shared-memory writes
// visible to later async-proxy (tensor core, TMA) reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The fp32 values nearest to x with 11 significant bits (fp16's precision in
// its normal range), by Veltkamp-Dekker splitting: g = (2^13 + 1) x,
// hi = g - (g - x).  Three packed fp32x2 operations on the FMA pipe.
__device__ __forceinline__ float2 round_to_11_bits(float2 x) {
  const float2 m1 = make_float2(-1.f, -1.f);
  const float2 g = __fmul2_rn(x, make_float2(8193.f, 8193.f));
  const float2 d = __ffma2_rn(x, m1, g);   // g - x
  return __ffma2_rn(d, m1, g);             // g - (g - x)
}

// Round two fp32 to bf16 (nearest-even) and pack (lo in the low half).
__device__ __forceinline__ uint32_t float2_to_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace plx

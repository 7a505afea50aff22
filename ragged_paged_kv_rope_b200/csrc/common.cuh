// common.cuh -- device helpers shared by the librpk kernels (sm_100a only).
//
// Thin wrappers over PTX for mbarriers, TMA tensor loads and the global
// timer, plus the error-word convention of rpk.h. Every wait on an mbarrier
// is bounded in time: when the bound is hit the caller gets `false`, sets
// RPK_DEVERR_TIMEOUT and returns instead of spinning forever.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rpk.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "librpk is written for sm_100a only"
#endif

namespace rpk {

// Default upper bound of a single wait inside a kernel (nanoseconds of
// %globaltimer); launches take theirs from rpk_set_wait_limit_ns. Waits for
// copies or tensor-core operations already in flight while a CTA gives up
// always use this bound.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;

__device__ __forceinline__ void raise_error(int32_t* error_word, unsigned bits) {
  if (error_word) atomicOr(reinterpret_cast<unsigned*>(error_word), bits);
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- bf16 / f32

template <typename T> struct Elt;
template <> struct Elt<float> {
  static constexpr int kVec = 4;  // elements per 16-byte vector
  __device__ __forceinline__ static float to_f32(float x) { return x; }
  __device__ __forceinline__ static float from_f32(float x) { return x; }
};
template <> struct Elt<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ __forceinline__ static float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

// 16 bytes of elements as fp32 values.
template <typename T> struct Vec16 {
  float v[Elt<T>::kVec];
};

template <typename T>
__device__ __forceinline__ void load16(const T* p, float* out) {
  uint4 raw = *reinterpret_cast<const uint4*>(p);
  const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
  for (int i = 0; i < Elt<T>::kVec; ++i) out[i] = Elt<T>::to_f32(e[i]);
}

template <typename T>
__device__ __forceinline__ void store16(T* p, const float* in) {
  uint4 raw;
  T* e = reinterpret_cast<T*>(&raw);
#pragma unroll
  for (int i = 0; i < Elt<T>::kVec; ++i) e[i] = Elt<T>::from_f32(in[i]);
  *reinterpret_cast<uint4*>(p) = raw;
}

// ------------------------------------------------------------------- e4m3

// Two fp32 values -> two e4m3 codes, lo in bits 0-7 and hi in bits 8-15:
// rounded to nearest with ties to even, magnitudes beyond 448 saturating to
// +-448 (the largest finite code), NaN kept (PTX cvt .satfinite .e4m3x2).
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two e4m3 codes (bits 0-7, 8-15) -> two f16 values (bits 0-15, 16-31); every
// e4m3 value is exactly representable in f16.
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint32_t codes) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)codes));
  return r;
}

// Four e4m3 codes (bytes 0-3) -> four f16 values: bytes 0-1 into lo, 2-3 into hi.
__device__ __forceinline__ void f16x4_from_e4m3x4(uint32_t codes, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 c0, c1;\n\t"
      "mov.b32 {c0, c1}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, c0;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, c1;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(codes));
}

// One e4m3 code -> fp32 (exact).
__device__ __forceinline__ float f32_from_e4m3(uint8_t code) {
  const uint32_t h2 = f16x2_from_e4m3x2(code);
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Two fp32 values -> f16x2 (round to nearest even), lo in bits 0-15.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Natural log-sum-exp of a row from its running state in log2 units: the
// scores' maximum m (times log2 e) and the sum l of 2^(score - m); -inf for a
// row with no key (l = 0).
__device__ __forceinline__ float lse_from_log2_state(float m, float l) {
  return l > 0.f ? (m + log2f(l)) * 0.693147180559945309f : -INFINITY;
}

// 2^x by the MUFU approximation (relative error ~2^-22; 2^-inf = +0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------- warp-level tensor cores

// Four 8x8 matrices of 16-bit elements from shared memory; lane i gives the
// address of row i % 8 of matrix i / 8, and lane t receives row t / 4,
// columns 2 (t % 4), +1 of each matrix (of its transpose with .trans).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------ ragged offsets

// Sequence b with off[b] <= t < off[b+1] (off non-decreasing, batch >= 1).
__device__ __forceinline__ int find_sequence(const int32_t* __restrict__ off, int batch, int t) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(off + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that lets the hardware suspend the thread until the phase completes
// or `hint_ns` nanoseconds pass, so waiting warps do not spend issue slots on
// polling.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar_addr, uint32_t parity,
                                                      uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Sleep hint of one try_wait inside a wait bounded by `limit_ns`.
__device__ __forceinline__ uint32_t wait_hint_ns(unsigned long long limit_ns) {
  return limit_ns < 200000ull ? (uint32_t)limit_ns : 200000u;
}

// Limits below this give up at the first test of a phase that is not
// complete: the global timer does not resolve shorter intervals.
constexpr unsigned long long kTimerResolutionNs = 1000ull;

// Wait for the phase with the given parity to complete; false once more than
// `limit_ns` have passed. The first test does not block; a limit under
// kTimerResolutionNs gives up right there when the phase is not complete, and
// each later try sleeps at most the limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long limit_ns = kWaitTimeoutNs) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait(a, parity)) return true;
  if (limit_ns < kTimerResolutionNs) return false;
  const uint32_t hint = wait_hint_ns(limit_ns);
  const unsigned long long t0 = global_timer_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait_suspend(a, parity, hint)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// --------------------------------------------------------------------- TMA

// 3-D tiled TMA load into shared memory, completing on `bar` (no multicast).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, int32_t c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy accesses (TMA writes, tcgen05.mma reads) of the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a tile that
// TMA wrote with CU_TENSOR_MAP_SWIZZLE_128B (rows of 128 bytes; the tile base
// is 1024-byte aligned, so the XOR uses the row index within its 8-row group).
__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// ------------------------------------------------- packed fp32 arithmetic

// Packed and three-input fp32 instructions of sm_100: softmax-like passes over
// tensor-memory tiles are bound by instruction issue and the exponential unit,
// so two values per instruction where the hardware allows it.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// (d0, d1) = (a0, a1) * b + c
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %4};\n\t"
      "mov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
// (s0, s1) += (a0, a1)
__device__ __forceinline__ void add2(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(s0), "=f"(s1)
      : "f"(a0), "f"(a1), "f"(s0), "f"(s1));
}

// (d0, d1) = (a0, a1) + (b0, b1)
__device__ __forceinline__ void add2_to(float& d0, float& d1, float a0, float a1, float b0,
                                        float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// (d0, d1) = (a0, a1) * (b0, b1) + (c0, c1)
__device__ __forceinline__ void fma2_v(float& d0, float& d1, float a0, float a1, float b0,
                                       float b1, float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// (d0, d1) = (a0, a1) * (b0, b1)
__device__ __forceinline__ void mul2(float& d0, float& d1, float a0, float a1, float b0,
                                     float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// ------------------------------------- bounded waits of persistent kernels

// A CTA that gives up on a wait publishes RPK_DEVERR_TIMEOUT in the error
// word; every other CTA of the launch (and of later launches, until the caller
// clears the word) sees it and stops early instead of waiting out its own
// bound, so a broken launch ends in about one bound, not one per CTA.
__device__ __forceinline__ bool timed_out_elsewhere(const int32_t* error_word) {
  return error_word &&
         (*reinterpret_cast<const volatile int32_t*>(error_word) & (int32_t)RPK_DEVERR_TIMEOUT);
}

// Bounded wait by one thread; false on timeout (after `limit_ns`; at the first
// incomplete test for a limit under kTimerResolutionNs) or abort.
// The first test does not block; then the thread sleeps in try_wait (woken
// when the phase completes, at most 0.2 ms or the limit per try), so
// waiting warps leave the issue slots to the warps that compute; between
// tries it looks at the abort flag, the timer and, once the wait has lasted
// longer than any healthy one (50 us), the global error word.
__device__ __forceinline__ bool thread_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                            const int32_t* error_word,
                                            unsigned long long limit_ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait(a, parity)) return true;
  if (limit_ns < kTimerResolutionNs) return false;
  const uint32_t hint = wait_hint_ns(limit_ns);
  const unsigned long long t0 = global_timer_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait_suspend(a, parity, hint)) return true;
    if (*abort) return false;
    const unsigned long long dt = global_timer_ns() - t0;
    if (dt > limit_ns) return false;
    if (dt > 50000ull && timed_out_elsewhere(error_word)) return false;
  }
}

// Bounded wait shared by the whole warp: every lane polls (so each lane has
// acquired the phase) and the lanes agree on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const int32_t* error_word,
                                          unsigned long long limit_ns) {
  const bool ok = thread_wait(bar, parity, abort, error_word, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait for two barriers at once: the two tests are issued back to
// back, so a warp that finds both phases complete pays one barrier round
// trip, not two.
__device__ __forceinline__ bool warp_wait2(uint64_t* bar_a, uint32_t par_a, uint64_t* bar_b,
                                           uint32_t par_b, volatile int* abort,
                                           const int32_t* error_word,
                                           unsigned long long limit_ns) {
  uint32_t ok_a, ok_b;
  asm volatile(
      "{\n\t.reg .pred pa, pb;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 pa, [%2], %3;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 pb, [%4], %5;\n\t"
      "selp.u32 %0, 1, 0, pa;\n\t"
      "selp.u32 %1, 1, 0, pb;\n\t}"
      : "=r"(ok_a), "=r"(ok_b)
      : "r"(smem_u32(bar_a)), "r"(par_a), "r"(smem_u32(bar_b)), "r"(par_b)
      : "memory");
  bool ok = (ok_a != 0 || thread_wait(bar_a, par_a, abort, error_word, limit_ns)) &&
            (ok_b != 0 || thread_wait(bar_b, par_b, abort, error_word, limit_ns));
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void do_abort(volatile int* abort, int32_t* error_word) {
  if (!*abort) {
    *abort = 1;
    raise_error(error_word, RPK_DEVERR_TIMEOUT);
  }
}

}  // namespace rpk

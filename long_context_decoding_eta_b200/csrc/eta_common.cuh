// Shared device helpers of the ETA sm_100a kernels: bf16 unpacking, mbarrier
// waits with an iteration limit, and 1-D TMA bulk copies global -> shared.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "../../include/eta.h"

#define ETA_DEV __device__ __forceinline__

namespace eta {

// Iteration limit of every mbarrier wait.  try_wait already suspends the thread
// for a hardware-defined interval per call, so 2^22 polls is far beyond any
// legitimate wait (seconds) while still ending a lost wait.
constexpr uint32_t kWaitLimit = 1u << 22;

// Programmatic dependent launch: every kernel of the library is launched with
// programmatic stream serialization allowed, waits for the grid before it in the
// stream (completion and memory flush) before touching any global memory, and
// then lets the grid after it start launching.  Only launch latency overlaps;
// the data dependencies stay exactly those of plain stream order.
ETA_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
ETA_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
#define ETA_PDL_ENTRY() \
  do {                  \
    eta::pdl_wait();    \
    eta::pdl_trigger(); \
  } while (0)

ETA_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
ETA_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
ETA_DEV float bf16_to_f(uint16_t h) { return __uint_as_float(((uint32_t)h) << 16); }

ETA_DEV void set_status(int32_t* st, int32_t bits) {
  if (st) atomicOr(st, bits);
}

// Checked build (-DETA_CHECKED): every global load or store whose index a kernel
// computes from its inputs or its schedule is guarded by ETA_IN_BOUNDS(i, n, status),
// false when i lies outside [0, n): ETA_DEVSTAT_BOUNDS is then OR-ed into the status
// word (when the call has one), the first such event of the source file is printed
// with its file and line, and the caller skips the access.  In the release build the
// guard is the constant true and generates no code.
#ifdef ETA_CHECKED
static __device__ int g_bounds_reported = 0;

static __device__ __noinline__ bool in_bounds_report(long long i, long long n, int32_t* st,
                                                     const char* file, int line) {
  set_status(st, ETA_DEVSTAT_BOUNDS);
  if (atomicExch(&g_bounds_reported, 1) == 0)
    printf("eta checked build: index %lld outside [0, %lld) at %s:%d\n", i, n, file, line);
  return false;
}

ETA_DEV bool in_bounds(long long i, long long n, int32_t* st, const char* file, int line) {
  return (i >= 0 && i < n) ? true : in_bounds_report(i, n, st, file, line);
}
#define ETA_IN_BOUNDS(i, n, st) \
  eta::in_bounds((long long)(i), (long long)(n), (st), __FILE__, __LINE__)
// The half-open index range [lo, hi) lies inside [0, n) (true when it is empty).
#define ETA_RANGE_IN_BOUNDS(lo, hi, n, st) \
  ((long long)(hi) <= (long long)(lo) ||    \
   (ETA_IN_BOUNDS(lo, n, st) && ETA_IN_BOUNDS((long long)(hi) - 1, n, st)))
constexpr bool kChecked = true;
#else
#define ETA_IN_BOUNDS(i, n, st) true
#define ETA_RANGE_IN_BOUNDS(lo, hi, n, st) true
constexpr bool kChecked = false;
#endif

ETA_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

ETA_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

ETA_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

ETA_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

ETA_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

ETA_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of `bar`.  Returns false when `limit` polls ran
// out or when *abort became non-zero (another thread of the CTA gave up).
ETA_DEV bool mbar_wait_n(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
  }
  return false;
}

ETA_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait_n(bar, parity, abort, kWaitLimit);
}

// 1-D bulk copy (TMA engine) of `bytes` from global to this CTA's shared memory,
// completing `bytes` transaction bytes on `bar`.  Both addresses 16-byte aligned,
// bytes a multiple of 16.
ETA_DEV void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// gpu-scope acquire load / release store of an int32 flag in global memory.
ETA_DEV int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

ETA_DEV void st_release_gpu(int32_t* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

ETA_DEV void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

ETA_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

ETA_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace eta

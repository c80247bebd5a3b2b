// Device helpers shared by the liblla kernels (sm_100a): shared-memory
// addresses, mbarriers with bounded waits, bulk async copies, programmatic
// dependent launch, and bf16 unpacking.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lla {

// A bounded device wait gives up after this many nanoseconds of wall time
// (read from %globaltimer), sets the sticky status word and lets the kernel
// return instead of hanging the GPU.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s
constexpr unsigned int kStatusWaitTimeout = 0x1u;
constexpr unsigned int kStatusBadPagedInput = 0x2u;
constexpr unsigned int kStatusPlanMismatch = 0x4u;
constexpr unsigned int kStatusOutOfBounds = 0x8u;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete. Returns false if
// the wait ran past `timeout_ns`; the caller then records the failure and
// returns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          unsigned long long timeout_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
}

__device__ __forceinline__ void report_status(unsigned int* status, unsigned int bits) {
  if (status) atomicOr(status, bits);
}

// The extent of a device buffer, [p, p + n) in bytes. The default span has
// no extent and admits every address.
struct Span {
  const char* p = nullptr;
  unsigned long long n = ~0ull;
};
inline Span span_of(const void* p, unsigned long long bytes) {
  return Span{static_cast<const char*>(p), bytes};
}

// Bounds-check build (compiled with LLA_BOUNDS_CHECK): the kernels test each
// computed global access against the span of the buffer it belongs to. An
// access outside its span sets the status bit kStatusOutOfBounds and is not
// made (a store is skipped, a load or copy takes zeros or nothing). The
// release build compiles every check to `true`.
#ifdef LLA_BOUNDS_CHECK
__device__ __forceinline__ bool in_span(const Span& s, const void* q, unsigned long long bytes,
                                        unsigned int* status) {
  const char* c = static_cast<const char*>(q);
  const bool ok = s.p == nullptr || (c >= s.p && bytes <= s.n && c - s.p <= (long long)(s.n - bytes));
  if (!ok) report_status(status, kStatusOutOfBounds);
  return ok;
}
#else
__device__ __forceinline__ constexpr bool in_span(const Span&, const void*, unsigned long long,
                                                  unsigned int*) {
  return true;
}
#endif

// A store of v at p that the bounds-check build makes only inside span s.
template <class T>
__device__ __forceinline__ void st_chk(T* p, T v, const Span& s, unsigned int* status) {
  if (in_span(s, p, sizeof(T), status)) *p = v;
}

// A read-only load from p, or `dflt` when the bounds-check build finds p
// outside span s.
template <class T>
__device__ __forceinline__ T ld_chk(const T* p, const Span& s, unsigned int* status, T dflt) {
  return in_span(s, p, sizeof(T), status) ? __ldg(p) : dflt;
}

// L2 policy for data read exactly once (the latent stream).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// One bulk async copy global -> shared, completion counted in bytes on the
// mbarrier. Source and destination 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue, and wait for the previous kernel's results.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// bf16 pair in one 32-bit word -> two floats (exact widening).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace lla

// Per-head decode for callers that cannot allocate device memory.
//
// lla_decode_attn needs a caller-provided workspace (the absorbed queries,
// the lse offsets and one partial record per streaming piece). Some callers
// cannot allocate it: for example a plugin running inside a serving engine
// that has already reserved the whole device for its own memory pool, or
// code that must not call cudaMalloc after start-up because an allocation
// can synchronise the device at an unpredictable point. This entry point
// runs the same kernels with the same launch plan, but its scratch is a
// fixed array compiled into the library: every GPU that loads liblla holds
// LLA_NOALLOC_SCRATCH_BYTES of it until the process exits.
//
// Under CUDA's default lazy module loading the array is placed on a device
// when this file's module loads there, which happens at the first call's
// address lookup; a caller that reserves the rest of the device up front
// should make one call before that reservation (or load modules eagerly).
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace lla {
namespace {

constexpr size_t kScratchBytes = LLA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch itself. In host code this name is only a stand-in for the
// symbol, not a device address: its address on a device comes from
// cudaGetSymbolAddress with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];

// Identifier of the calling thread's current CUDA context, or 0 when there
// is none yet or the driver cannot say. cudaDeviceReset destroys a device's
// primary context and the next runtime call creates a new one, with a new
// identifier and a new copy of the scratch, so an address looked up in one
// context is reused only within that context.
unsigned long long current_context_id() {
  static std::once_flag once;
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    cudaGetLastError();
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch on the current device. It is looked up once
// per device and context: the first call on a device (and the first after a
// cudaDeviceReset) does this set-up.
lla_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return check_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return fail(LLA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> g(g_mutex);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return check_cuda(e, "cudaGetSymbolAddress(noalloc scratch)");
    g_scratch_ptr[dev] = p;
    // the lookup made the device's context current if it was not yet
    g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
  }
  *out = g_scratch_ptr[dev];
  return LLA_OK;
}

}  // namespace
}  // namespace lla

using namespace lla;

extern "C" lla_status lla_decode_attn_noalloc(const float* q, const void* zk, const void* zv,
                                              lla_dtype zdt, int B, int H, int d_h, int N,
                                              int n_cap, int r_k, int r_v, const float* dk_t,
                                              const float* dv_t, const float* mu_k_t,
                                              const float* mu_v_t, float scale, float* out,
                                              float* lse, void* stream) {
  int esz = 0;
  lla_status st = check_decode_args(q, zk, zv, zdt, B, H, d_h, N, n_cap, r_k, r_v, dk_t, dv_t,
                                    mu_k_t, mu_v_t, out, lse, nullptr, &esz);
  if (st != LLA_OK) return st;
  DecodePlan plan;
  st = plan_decode(B, H, N, r_k, r_v, esz, &plan);
  if (st != LLA_OK) return st;
  if (plan.ws_bytes > kScratchBytes)
    return fail(LLA_ERR_WORKSPACE,
                "this shape needs %zu bytes of scratch; the built-in scratch holds %zu "
                "(use lla_decode_attn with a caller workspace)",
                plan.ws_bytes, kScratchBytes);
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != LLA_OK) return st;
  // Nothing in the scratch has to start at zero: every call writes the
  // absorbed queries, lse offsets and partial records before reading them.
  return run_decode(q, zk, zv, esz, B, H, d_h, N, (long long)n_cap, r_k, r_v, dk_t, dv_t, mu_k_t,
                    mu_v_t, scale, out, lse, scratch, kScratchBytes,
                    static_cast<cudaStream_t>(stream));
}

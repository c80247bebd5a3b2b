// C ABI entry points of liblla: argument checks, status reporting and the
// per-device state (SM count, sticky status word).
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace lla {

namespace {

constexpr int kMaxDevices = 64;

// Sticky device status word: kernels OR bits into it when a bounded wait
// runs out. One instance per device (a module-scope __device__ variable).
__device__ unsigned int g_status_word = 0u;

thread_local char g_last_error[512] = "";
thread_local cudaEvent_t g_ev_begin = nullptr;
thread_local cudaEvent_t g_ev_end = nullptr;

std::mutex g_dev_mutex;
bool g_dev_ready[kMaxDevices];
DeviceInfo g_dev_info[kMaxDevices];
unsigned int* g_status_ptr[kMaxDevices];

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return dev;
}

void init_device(int dev) {
  // caller holds g_dev_mutex
  if (dev < 0 || dev >= kMaxDevices || g_dev_ready[dev]) return;
  DeviceInfo info{148, 227 * 1024};
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
    info.sms = v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess &&
      v > 0)
    info.smem_optin = v;
  cudaGetLastError();
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) {
    cudaGetLastError();
    p = nullptr;
  }
  g_dev_info[dev] = info;
  g_status_ptr[dev] = static_cast<unsigned int*>(p);
  g_dev_ready[dev] = true;
}

}  // namespace

DeviceInfo device_info() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return DeviceInfo{148, 227 * 1024};
  std::lock_guard<std::mutex> g(g_dev_mutex);
  init_device(dev);
  return g_dev_info[dev];
}

unsigned int* status_word() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> g(g_dev_mutex);
  init_device(dev);
  return g_status_ptr[dev];
}

void timing_events(cudaEvent_t* begin, cudaEvent_t* end) {
  *begin = g_ev_begin;
  *end = g_ev_end;
}

cudaError_t record_timing(bool begin, cudaStream_t stream) {
  if (!g_ev_begin || !g_ev_end) return cudaSuccess;
  return cudaEventRecord(begin ? g_ev_begin : g_ev_end, stream);
}

lla_status fail(lla_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

lla_status check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return LLA_OK;
  return fail(LLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace lla

using namespace lla;

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

lla_status lla::check_decode_args(const float* q, const void* zk, const void* zv, lla_dtype zdt,
                             int B, int H, int d_h, int N, int n_cap, int r_k, int r_v,
                             const float* dk, const float* dv, const float* mu_k,
                             const float* mu_v, float* out, float* lse, void* ws, int* esz) {
  if (zdt != LLA_BF16 && zdt != LLA_F32) return fail(LLA_ERR_INVALID_ARG, "zdt must be LLA_BF16 or LLA_F32");
  *esz = (zdt == LLA_BF16) ? 2 : 4;
  if (!q || !zk || !zv || !dk || !dv || !out)
    return fail(LLA_ERR_INVALID_ARG, "q, zk, zv, dk_t, dv_t and out must be non-NULL");
  if (B < 1 || H < 1) return fail(LLA_ERR_INVALID_ARG, "B and H must be >= 1");
  if (d_h < 1 || d_h > 256) return fail(LLA_ERR_INVALID_ARG, "d_h must be in 1..256");
  if (N < 1) return fail(LLA_ERR_INVALID_ARG, "N must be >= 1 (empty context is undefined)");
  if (N > n_cap) return fail(LLA_ERR_INVALID_ARG, "N must be <= n_cap");
  const int rmax = (*esz == 2) ? 256 : 128;
  if (r_k < 8 || r_v < 8 || r_k % 8 || r_v % 8 || r_k > rmax || r_v > rmax)
    return fail(LLA_ERR_INVALID_ARG, "r_k and r_v must be multiples of 8 in 8..%d", rmax);
  if (!aligned(zk, 16) || !aligned(zv, 16) || !aligned(dk, 16) || !aligned(dv, 16))
    return fail(LLA_ERR_INVALID_ARG, "zk, zv, dk_t and dv_t must be 16-byte aligned");
  if (!aligned(q, 4) || !aligned(out, 4) ||
      (mu_k && !aligned(mu_k, 4)) || (mu_v && !aligned(mu_v, 4)) || (lse && !aligned(lse, 4)))
    return fail(LLA_ERR_INVALID_ARG, "fp32 arrays must be 4-byte aligned");
  if (ws && !aligned(ws, 16)) return fail(LLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  return LLA_OK;
}

namespace {

// Argument checks shared by the encode entry points. `rows` is the number
// of rows of one group that the strides lay out (N for a dense write,
// page_size inside a page of a paged store).
lla_status check_encode_args(const void* x, lla_dtype xdt, int T, int N, int G, int d_loop, int r,
                             const void* w_down_t, const float* mu, void* z,
                             long long z_row_stride, long long z_group_stride, int rows) {
  if (xdt != LLA_BF16) return fail(LLA_ERR_INVALID_ARG, "xdt must be LLA_BF16");
  if (!x || !w_down_t || !z) return fail(LLA_ERR_INVALID_ARG, "x, w_down_t and z must be non-NULL");
  if (!aligned(x, 16) || !aligned(w_down_t, 16) || !aligned(z, 16))
    return fail(LLA_ERR_INVALID_ARG, "x, w_down_t and z must be 16-byte aligned");
  if (mu && !aligned(mu, 4)) return fail(LLA_ERR_INVALID_ARG, "mu must be 4-byte aligned");
  if (T < 1 || N < 1 || G < 1) return fail(LLA_ERR_INVALID_ARG, "T, N and G must be >= 1");
  if (d_loop < 64 || d_loop % 64)
    return fail(LLA_ERR_INVALID_ARG, "d_loop must be a positive multiple of 64");
  if ((long long)T * d_loop > (1LL << 30)) return fail(LLA_ERR_INVALID_ARG, "T*d_loop too large");
  if (r < 8 || r > 256 || r % 8) return fail(LLA_ERR_INVALID_ARG, "r must be a multiple of 8 in 8..256");
  if (z_row_stride < r || z_group_stride < 0 || z_row_stride % 8 || z_group_stride % 8)
    return fail(LLA_ERR_INVALID_ARG, "z strides must be multiples of 8 with z_row_stride >= r");
  if (G > 1) {
    const bool groups_outer = z_group_stride >= (long long)(rows - 1) * z_row_stride + r;
    const bool rows_outer = z_row_stride >= (long long)(G - 1) * z_group_stride + r && z_group_stride >= r;
    if (!groups_outer && !rows_outer)
      return fail(LLA_ERR_INVALID_ARG, "z strides make output rows overlap");
  }
  return LLA_OK;
}

// Checks shared by the paged calls: the pool's geometry, the block table
// and lengths (device arrays, read only on the device) and the eviction set.
lla_status check_paged_table(int page_size, int num_pages, const int* block_table,
                             int max_blocks, const int* seq_lens, int sink, int window,
                             bool two_d) {
  if (!block_table || !seq_lens)
    return fail(LLA_ERR_INVALID_ARG, "block_table and seq_lens must be non-NULL");
  if (!aligned(block_table, 4) || !aligned(seq_lens, 4))
    return fail(LLA_ERR_INVALID_ARG, "block_table and seq_lens must be 4-byte aligned");
  if (two_d && (page_size < 64 || page_size % 64))
    return fail(LLA_ERR_UNSUPPORTED, "LLA-2D pages hold a positive multiple of 64 tokens");
  if (page_size < 1 || num_pages < 1 || max_blocks < 1)
    return fail(LLA_ERR_INVALID_ARG, "page_size, num_pages and max_blocks must be >= 1");
  if ((long long)page_size * max_blocks > 0x7fffffffLL)
    return fail(LLA_ERR_INVALID_ARG, "page_size * max_blocks must fit in 31 bits");
  if (sink < 0 || window < 0) return fail(LLA_ERR_INVALID_ARG, "sink and window must be >= 0");
  return LLA_OK;
}

// The per-head paged call in each mode (plan and decode, or decode on a plan
// already in the workspace).
lla_status paged_call(const float* q, const void* zk_pages, const void* zv_pages, lla_dtype zdt,
                      int B, int H, int d_h, int r_k, int r_v, int page_size, int num_pages,
                      const int* block_table, int max_blocks, const int* seq_lens, int sink,
                      int window, const float* dk_t, const float* dv_t, const float* mu_k_t,
                      const float* mu_v_t, float scale, float* out, float* lse, void* workspace,
                      size_t ws_bytes, void* stream, PagedMode mode) {
  g_last_error[0] = '\0';
  int esz = 0;
  // the shared checks; lengths live on the device and are checked there
  lla_status st = check_decode_args(q, zk_pages, zv_pages, zdt, B, H, d_h, 1, 1, r_k, r_v, dk_t,
                                    dv_t, mu_k_t, mu_v_t, out, lse, workspace, &esz);
  if (st != LLA_OK) return st;
  st = check_paged_table(page_size, num_pages, block_table, max_blocks, seq_lens, sink, window,
                         false);
  if (st != LLA_OK) return st;
  return run_decode_paged(q, zk_pages, zv_pages, esz, B, H, d_h, r_k, r_v, page_size, num_pages,
                          block_table, max_blocks, seq_lens, sink, window, dk_t, dv_t, mu_k_t,
                          mu_v_t, scale, out, lse, workspace, ws_bytes,
                          static_cast<cudaStream_t>(stream), mode);
}

lla_status paged2d_call(const float* q, const void* zk_pages, const void* zv_pages, lla_dtype zdt,
                        int B, int H, int d_h, int r_k, int r_v, int page_size, int num_pages,
                        const int* block_table, int max_blocks, const int* seq_lens, int sink,
                        int window, const float* dk_t, const float* dv_t, const float* mu_k_t,
                        const float* mu_v_t, float scale, float* out, float* lse,
                        void* workspace, size_t ws_bytes, void* stream, PagedMode mode) {
  g_last_error[0] = '\0';
  int esz = 0;
  lla_status st = check_decode_args(q, zk_pages, zv_pages, zdt, B, H, d_h, 1, 1, r_k, r_v, dk_t,
                                    dv_t, mu_k_t, mu_v_t, out, lse, workspace, &esz);
  if (st != LLA_OK) return st;
  if (zdt != LLA_BF16) return fail(LLA_ERR_UNSUPPORTED, "LLA-2D latents must be LLA_BF16");
  if (H > 32) return fail(LLA_ERR_UNSUPPORTED, "LLA-2D supports H <= 32");
  st = check_paged_table(page_size, num_pages, block_table, max_blocks, seq_lens, sink, window,
                         true);
  if (st != LLA_OK) return st;
  return run_decode_2d_paged(q, zk_pages, zv_pages, B, H, d_h, r_k, r_v, page_size, num_pages,
                             block_table, max_blocks, seq_lens, sink, window, dk_t, dv_t, mu_k_t,
                             mu_v_t, scale, out, lse, workspace, ws_bytes,
                             static_cast<cudaStream_t>(stream), mode);
}

// The plan-only calls: the ranks and table checks of the decode calls,
// without the query-side arrays.
lla_status paged_plan_call(lla_dtype zdt, int B, int H, int r_k, int r_v, int page_size,
                           int num_pages, const int* block_table, int max_blocks,
                           const int* seq_lens, int sink, int window, void* workspace,
                           size_t ws_bytes, void* stream, bool two_d) {
  g_last_error[0] = '\0';
  if (zdt != LLA_BF16 && zdt != LLA_F32)
    return fail(LLA_ERR_INVALID_ARG, "zdt must be LLA_BF16 or LLA_F32");
  if (B < 1 || H < 1) return fail(LLA_ERR_INVALID_ARG, "B and H must be >= 1");
  const int esz = zdt == LLA_BF16 ? 2 : 4;
  const int rmax = esz == 2 ? 256 : 128;
  if (r_k < 8 || r_v < 8 || r_k % 8 || r_v % 8 || r_k > rmax || r_v > rmax)
    return fail(LLA_ERR_INVALID_ARG, "r_k and r_v must be multiples of 8 in 8..%d", rmax);
  if (two_d && zdt != LLA_BF16) return fail(LLA_ERR_UNSUPPORTED, "LLA-2D latents must be LLA_BF16");
  if (two_d && H > 32) return fail(LLA_ERR_UNSUPPORTED, "LLA-2D supports H <= 32");
  if (workspace && !aligned(workspace, 16))
    return fail(LLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  lla_status st = check_paged_table(page_size, num_pages, block_table, max_blocks, seq_lens,
                                    sink, window, two_d);
  if (st != LLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (two_d)
    return run_decode_2d_paged(nullptr, nullptr, nullptr, B, H, 1, r_k, r_v, page_size, num_pages,
                               block_table, max_blocks, seq_lens, sink, window, nullptr, nullptr,
                               nullptr, nullptr, 0.f, nullptr, nullptr, workspace, ws_bytes, s,
                               kPlanOnly);
  return run_decode_paged(nullptr, nullptr, nullptr, esz, B, H, 1, r_k, r_v, page_size, num_pages,
                          block_table, max_blocks, seq_lens, sink, window, nullptr, nullptr,
                          nullptr, nullptr, 0.f, nullptr, nullptr, workspace, ws_bytes, s,
                          kPlanOnly);
}

}  // namespace

extern "C" {

const char* lla_status_string(lla_status s) {
  switch (s) {
    case LLA_OK: return "LLA_OK";
    case LLA_ERR_INVALID_ARG: return "LLA_ERR_INVALID_ARG";
    case LLA_ERR_UNSUPPORTED: return "LLA_ERR_UNSUPPORTED";
    case LLA_ERR_WORKSPACE: return "LLA_ERR_WORKSPACE";
    case LLA_ERR_CUDA: return "LLA_ERR_CUDA";
  }
  return "LLA_ERR_UNKNOWN";
}

const char* lla_last_error(void) { return g_last_error; }

int lla_version(void) { return 100; }

void lla_set_timing_events(void* ev_begin, void* ev_end) {
  g_ev_begin = static_cast<cudaEvent_t>(ev_begin);
  g_ev_end = static_cast<cudaEvent_t>(ev_end);
}

lla_status lla_device_status(unsigned int* status, int clear) {
  if (!status) return fail(LLA_ERR_INVALID_ARG, "status must be non-NULL");
  unsigned int* p = status_word();
  if (!p) return fail(LLA_ERR_CUDA, "no device status word on the current device");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return check_cuda(e, "cudaDeviceSynchronize");
  e = cudaMemcpy(status, p, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return check_cuda(e, "read status word");
  if (clear) {
    e = cudaMemset(p, 0, sizeof(unsigned int));
    if (e != cudaSuccess) return check_cuda(e, "clear status word");
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return check_cuda(e, "cudaDeviceSynchronize");
  }
  return LLA_OK;
}

lla_status lla_merge_attn(const float* out_parts, const float* lse_parts, int R, long long U,
                          int d, float* out, float* lse, void* stream) {
  g_last_error[0] = '\0';
  if (!out_parts || !lse_parts || !out)
    return fail(LLA_ERR_INVALID_ARG, "out_parts, lse_parts and out must be non-NULL");
  if (R < 1 || U < 1 || d < 1) return fail(LLA_ERR_INVALID_ARG, "R, U and d must be >= 1");
  if ((U + 7) / 8 > 0x7fffffffLL) return fail(LLA_ERR_INVALID_ARG, "U too large");
  if (!aligned(out_parts, 4) || !aligned(lse_parts, 4) || !aligned(out, 4) ||
      (lse && !aligned(lse, 4)))
    return fail(LLA_ERR_INVALID_ARG, "arrays must be 4-byte aligned");
  return run_merge_attn(out_parts, lse_parts, R, U, d, out, lse, static_cast<cudaStream_t>(stream));
}

lla_status lla_selftest_wait_timeout(unsigned int timeout_us, void* stream) {
  g_last_error[0] = '\0';
  if (timeout_us < 1 || timeout_us > 1000000)
    return fail(LLA_ERR_INVALID_ARG, "timeout_us must be in 1..1000000");
  return run_selftest_wait(timeout_us, static_cast<cudaStream_t>(stream));
}

size_t lla_decode_attn_workspace(int B, int H, int N, int r_k, int r_v) {
  if (B < 1 || H < 1 || N < 1 || r_k < 8 || r_v < 8 || r_k % 8 || r_v % 8) return 0;
  // The bf16 plan needs at least as much workspace as the fp32 one.
  DecodePlan p2, p4;
  size_t need = 0;
  if (plan_decode(B, H, N, r_k, r_v, 2, &p2) == LLA_OK) need = p2.ws_bytes;
  if (r_k <= 128 && r_v <= 128 && plan_decode(B, H, N, r_k, r_v, 4, &p4) == LLA_OK)
    need = need > p4.ws_bytes ? need : p4.ws_bytes;
  return need;
}

lla_status lla_decode_attn(const float* q, const void* zk, const void* zv, lla_dtype zdt, int B,
                           int H, int d_h, int N, int n_cap, int r_k, int r_v, const float* dk_t,
                           const float* dv_t, const float* mu_k_t, const float* mu_v_t,
                           float scale, float* out, float* lse, void* workspace, size_t ws_bytes,
                           void* stream) {
  g_last_error[0] = '\0';
  int esz = 0;
  lla_status st = check_decode_args(q, zk, zv, zdt, B, H, d_h, N, n_cap, r_k, r_v, dk_t, dv_t,
                                    mu_k_t, mu_v_t, out, lse, workspace, &esz);
  if (st != LLA_OK) return st;
  return run_decode(q, zk, zv, esz, B, H, d_h, N, (long long)n_cap, r_k, r_v, dk_t, dv_t,
                    mu_k_t, mu_v_t, scale, out, lse, workspace, ws_bytes,
                    static_cast<cudaStream_t>(stream));
}

lla_status lla_decode_attn_rope(const float* q, const float* q_rope, const void* zk, const void* zv,
                                lla_dtype zdt, int B, int H, int d_h, int d_r, int N, int n_cap,
                                int r_k, int r_v, const float* dk_t, const float* dv_t,
                                const float* mu_k_t, const float* mu_v_t, float scale, float* out,
                                float* lse, void* workspace, size_t ws_bytes, void* stream) {
  g_last_error[0] = '\0';
  if (!q_rope) return fail(LLA_ERR_INVALID_ARG, "q_rope must be non-NULL");
  if (!aligned(q_rope, 4)) return fail(LLA_ERR_INVALID_ARG, "q_rope must be 4-byte aligned");
  if (d_r < 8 || d_r % 8) return fail(LLA_ERR_INVALID_ARG, "d_r must be a positive multiple of 8");
  if (r_k < 8 || r_k % 8) return fail(LLA_ERR_INVALID_ARG, "r_k must be a positive multiple of 8");
  int esz = 0;
  // the key row (latent and rotary key) is checked as one rank-(r_k + d_r) row
  lla_status st = check_decode_args(q, zk, zv, zdt, B, H, d_h, N, n_cap, r_k + d_r, r_v, dk_t, dv_t,
                                    mu_k_t, mu_v_t, out, lse, workspace, &esz);
  if (st != LLA_OK) return st;
  return run_decode(q, zk, zv, esz, B, H, d_h, N, (long long)n_cap, r_k, r_v, dk_t, dv_t, mu_k_t,
                    mu_v_t, scale, out, lse, workspace, ws_bytes, static_cast<cudaStream_t>(stream),
                    q_rope, d_r);
}

size_t lla_decode_attn_paged_workspace(int B, int H, int r_k, int r_v) {
  if (B < 1 || H < 1 || r_k < 8 || r_v < 8 || r_k % 8 || r_v % 8) return 0;
  size_t need = workspace_paged(B, H, r_k, r_v, 2);
  if (r_k <= 128 && r_v <= 128) {
    const size_t n4 = workspace_paged(B, H, r_k, r_v, 4);
    need = need > n4 ? need : n4;
  }
  return need;
}

lla_status lla_decode_attn_paged(const float* q, const void* zk_pages, const void* zv_pages,
                                 lla_dtype zdt, int B, int H, int d_h, int r_k, int r_v,
                                 int page_size, int num_pages, const int* block_table,
                                 int max_blocks, const int* seq_lens, int sink, int window,
                                 const float* dk_t, const float* dv_t, const float* mu_k_t,
                                 const float* mu_v_t, float scale, float* out, float* lse,
                                 void* workspace, size_t ws_bytes, void* stream) {
  return paged_call(q, zk_pages, zv_pages, zdt, B, H, d_h, r_k, r_v, page_size, num_pages,
                    block_table, max_blocks, seq_lens, sink, window, dk_t, dv_t, mu_k_t, mu_v_t,
                    scale, out, lse, workspace, ws_bytes, stream, kPlanAndDecode);
}

lla_status lla_decode_attn_paged_plan(lla_dtype zdt, int B, int H, int r_k, int r_v,
                                      int page_size, int num_pages, const int* block_table,
                                      int max_blocks, const int* seq_lens, int sink, int window,
                                      void* workspace, size_t ws_bytes, void* stream) {
  return paged_plan_call(zdt, B, H, r_k, r_v, page_size, num_pages, block_table, max_blocks,
                         seq_lens, sink, window, workspace, ws_bytes, stream, false);
}

lla_status lla_decode_attn_paged_planned(const float* q, const void* zk_pages,
                                         const void* zv_pages, lla_dtype zdt, int B, int H,
                                         int d_h, int r_k, int r_v, int page_size, int num_pages,
                                         const int* block_table, int max_blocks,
                                         const int* seq_lens, int sink, int window,
                                         const float* dk_t, const float* dv_t,
                                         const float* mu_k_t, const float* mu_v_t, float scale,
                                         float* out, float* lse, void* workspace,
                                         size_t ws_bytes, void* stream) {
  return paged_call(q, zk_pages, zv_pages, zdt, B, H, d_h, r_k, r_v, page_size, num_pages,
                    block_table, max_blocks, seq_lens, sink, window, dk_t, dv_t, mu_k_t, mu_v_t,
                    scale, out, lse, workspace, ws_bytes, stream, kDecodePlanned);
}

size_t lla2d_decode_attn_workspace(int B, int H, int N, int r_k, int r_v) {
  // r_k is the key row width (r_k + d_r for lla2d_decode_attn_rope)
  if (B < 1 || H < 1 || H > 32 || N < 1 || r_k < 8 || r_k > 384 || r_k % 8 || r_v < 8 ||
      r_v > 256 || r_v % 8)
    return 0;
  return workspace_2d(B, H, N, r_k, r_v);
}

lla_status lla2d_decode_attn(const float* q, const void* zk, const void* zv, lla_dtype zdt, int B,
                             int H, int d_h, int N, int n_cap, int r_k, int r_v,
                             const float* dk_t, const float* dv_t, const float* mu_k_t,
                             const float* mu_v_t, float scale, float* out, float* lse,
                             void* workspace, size_t ws_bytes, void* stream) {
  g_last_error[0] = '\0';
  int esz = 0;
  lla_status st = check_decode_args(q, zk, zv, zdt, B, H, d_h, N, n_cap, r_k, r_v, dk_t, dv_t,
                                    mu_k_t, mu_v_t, out, lse, workspace, &esz);
  if (st != LLA_OK) return st;
  if (zdt != LLA_BF16) return fail(LLA_ERR_UNSUPPORTED, "LLA-2D latents must be LLA_BF16");
  if (H > 32) return fail(LLA_ERR_UNSUPPORTED, "LLA-2D supports H <= 32");
  return run_decode_2d(q, zk, zv, B, H, d_h, N, (long long)n_cap, r_k, r_v, dk_t, dv_t, mu_k_t,
                       mu_v_t, scale, out, lse, workspace, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

lla_status lla2d_decode_attn_rope(const float* q, const float* q_rope, const void* zk,
                                  const void* zv, lla_dtype zdt, int B, int H, int d_h, int d_r,
                                  int N, int n_cap, int r_k, int r_v, const float* dk_t,
                                  const float* dv_t, const float* mu_k_t, const float* mu_v_t,
                                  float scale, float* out, float* lse, void* workspace,
                                  size_t ws_bytes, void* stream) {
  g_last_error[0] = '\0';
  if (!q_rope) return fail(LLA_ERR_INVALID_ARG, "q_rope must be non-NULL");
  if (!aligned(q_rope, 4)) return fail(LLA_ERR_INVALID_ARG, "q_rope must be 4-byte aligned");
  if (d_r < 8 || d_r % 8) return fail(LLA_ERR_INVALID_ARG, "d_r must be a positive multiple of 8");
  if (r_k < 8 || r_k % 8) return fail(LLA_ERR_INVALID_ARG, "r_k must be a positive multiple of 8");
  int esz = 0;
  // shared checks on the latent part; the key-row limits follow
  lla_status st = check_decode_args(q, zk, zv, zdt, B, H, d_h, N, n_cap, 8, r_v, dk_t, dv_t, mu_k_t,
                                    mu_v_t, out, lse, workspace, &esz);
  if (st != LLA_OK) return st;
  if (zdt != LLA_BF16) return fail(LLA_ERR_UNSUPPORTED, "LLA-2D latents must be LLA_BF16");
  if (H > 32) return fail(LLA_ERR_UNSUPPORTED, "LLA-2D supports H <= 32");
  const int rq = r_k + d_r;
  if (rq > 384)
    return fail(LLA_ERR_UNSUPPORTED, "LLA-2D with a rotary branch needs r_k + d_r <= 384");
  return run_decode_2d(q, zk, zv, B, H, d_h, N, (long long)n_cap, r_k, r_v, dk_t, dv_t, mu_k_t,
                       mu_v_t, scale, out, lse, workspace, ws_bytes,
                       static_cast<cudaStream_t>(stream), q_rope, d_r);
}

size_t lla2d_decode_attn_paged_workspace(int B, int H, int r_k, int r_v) {
  if (B < 1 || H < 1 || H > 32 || r_k < 8 || r_k > 256 || r_k % 8 || r_v < 8 || r_v > 256 ||
      r_v % 8)
    return 0;
  return workspace_2d_paged(B, H, r_k, r_v);
}

lla_status lla2d_decode_attn_paged(const float* q, const void* zk_pages, const void* zv_pages,
                                   lla_dtype zdt, int B, int H, int d_h, int r_k, int r_v,
                                   int page_size, int num_pages, const int* block_table,
                                   int max_blocks, const int* seq_lens, int sink, int window,
                                   const float* dk_t, const float* dv_t, const float* mu_k_t,
                                   const float* mu_v_t, float scale, float* out, float* lse,
                                   void* workspace, size_t ws_bytes, void* stream) {
  return paged2d_call(q, zk_pages, zv_pages, zdt, B, H, d_h, r_k, r_v, page_size, num_pages,
                      block_table, max_blocks, seq_lens, sink, window, dk_t, dv_t, mu_k_t, mu_v_t,
                      scale, out, lse, workspace, ws_bytes, stream, kPlanAndDecode);
}

lla_status lla2d_decode_attn_paged_plan(int B, int H, int r_k, int r_v, int page_size,
                                        int num_pages, const int* block_table, int max_blocks,
                                        const int* seq_lens, int sink, int window,
                                        void* workspace, size_t ws_bytes, void* stream) {
  return paged_plan_call(LLA_BF16, B, H, r_k, r_v, page_size, num_pages, block_table, max_blocks,
                         seq_lens, sink, window, workspace, ws_bytes, stream, true);
}

lla_status lla2d_decode_attn_paged_planned(const float* q, const void* zk_pages,
                                           const void* zv_pages, lla_dtype zdt, int B, int H,
                                           int d_h, int r_k, int r_v, int page_size,
                                           int num_pages, const int* block_table, int max_blocks,
                                           const int* seq_lens, int sink, int window,
                                           const float* dk_t, const float* dv_t,
                                           const float* mu_k_t, const float* mu_v_t, float scale,
                                           float* out, float* lse, void* workspace,
                                           size_t ws_bytes, void* stream) {
  return paged2d_call(q, zk_pages, zv_pages, zdt, B, H, d_h, r_k, r_v, page_size, num_pages,
                      block_table, max_blocks, seq_lens, sink, window, dk_t, dv_t, mu_k_t, mu_v_t,
                      scale, out, lse, workspace, ws_bytes, stream, kDecodePlanned);
}

lla_status lla_encode(const void* x, lla_dtype xdt, int T, int N, int G, int d_loop, int r,
                      const void* w_down_t, const float* mu, void* z, long long z_row_stride,
                      long long z_group_stride, void* stream) {
  g_last_error[0] = '\0';
  lla_status st = check_encode_args(x, xdt, T, N, G, d_loop, r, w_down_t, mu, z, z_row_stride,
                                    z_group_stride, N);
  if (st != LLA_OK) return st;
  return run_encode(x, T, N, G, d_loop, r, w_down_t, mu, z, z_row_stride, z_group_stride,
                    static_cast<cudaStream_t>(stream));
}

lla_status lla_encode_bias(const void* w_down_t, const float* mu, int G, int K, int r, float* muw,
                           void* stream) {
  g_last_error[0] = '\0';
  if (!w_down_t || !mu || !muw) return fail(LLA_ERR_INVALID_ARG, "w_down_t, mu and muw must be non-NULL");
  if (!aligned(w_down_t, 16) || !aligned(mu, 16) || !aligned(muw, 4))
    return fail(LLA_ERR_INVALID_ARG, "w_down_t and mu must be 16-byte aligned, muw 4-byte");
  if (G < 1 || K < 8 || K % 8) return fail(LLA_ERR_INVALID_ARG, "G >= 1 and K a positive multiple of 8");
  if (r < 1 || r > 65535 * 8) return fail(LLA_ERR_INVALID_ARG, "r out of range");
  return run_encode_bias(w_down_t, mu, G, K, r, muw, static_cast<cudaStream_t>(stream));
}

size_t lla_encode_with_bias_workspace(int T, int N, int G, int d_loop, int r) {
  if (T < 1 || N < 1 || G < 1 || d_loop < 64 || d_loop % 64 || r < 8 || r > 256 || r % 8) return 0;
  return encode_workspace(T, N, G, d_loop, r);
}

lla_status lla_encode_with_bias(const void* x, lla_dtype xdt, int T, int N, int G, int d_loop,
                                int r, const void* w_down_t, const float* muw, void* z,
                                long long z_row_stride, long long z_group_stride, void* workspace,
                                size_t ws_bytes, void* stream) {
  g_last_error[0] = '\0';
  lla_status st = check_encode_args(x, xdt, T, N, G, d_loop, r, w_down_t, nullptr, z,
                                    z_row_stride, z_group_stride, N);
  if (st != LLA_OK) return st;
  if (muw && !aligned(muw, 16)) return fail(LLA_ERR_INVALID_ARG, "muw must be 16-byte aligned");
  if (workspace && !aligned(workspace, 16))
    return fail(LLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  return run_encode(x, T, N, G, d_loop, r, w_down_t, nullptr, z, z_row_stride, z_group_stride,
                    static_cast<cudaStream_t>(stream), muw, workspace, ws_bytes);
}

lla_status lla_encode_paged(const void* x, lla_dtype xdt, int T, int N, int G, int d_loop, int r,
                            const void* w_down_t, const float* muw, void* z_pages,
                            long long z_page_stride, long long z_group_stride,
                            long long z_row_stride, int page_size, int num_pages,
                            const int* block_table, int n_seq, int max_blocks, const int* seq_idx,
                            const int* positions, void* workspace, size_t ws_bytes,
                            void* stream) {
  g_last_error[0] = '\0';
  if (page_size < 1 || num_pages < 1 || n_seq < 1 || max_blocks < 1)
    return fail(LLA_ERR_INVALID_ARG, "page_size, num_pages, n_seq and max_blocks must be >= 1");
  if ((long long)page_size * max_blocks > 0x7fffffffLL)
    return fail(LLA_ERR_INVALID_ARG, "page_size * max_blocks must fit in 31 bits");
  // the rows of one page are laid out like a dense write of page_size tokens
  lla_status st = check_encode_args(x, xdt, T, N, G, d_loop, r, w_down_t, nullptr, z_pages,
                                    z_row_stride, z_group_stride, page_size);
  if (st != LLA_OK) return st;
  const long long page_extent =
      (long long)(G - 1) * z_group_stride + (long long)(page_size - 1) * z_row_stride + r;
  if (z_page_stride % 8 || z_page_stride < page_extent)
    return fail(LLA_ERR_INVALID_ARG,
                "z_page_stride must be a multiple of 8 covering a page (>= %lld)", page_extent);
  if (!block_table || !positions)
    return fail(LLA_ERR_INVALID_ARG, "block_table and positions must be non-NULL");
  if (!aligned(block_table, 4) || !aligned(positions, 4) || (seq_idx && !aligned(seq_idx, 4)))
    return fail(LLA_ERR_INVALID_ARG, "block_table, seq_idx and positions must be 4-byte aligned");
  if (muw && !aligned(muw, 16)) return fail(LLA_ERR_INVALID_ARG, "muw must be 16-byte aligned");
  if (workspace && !aligned(workspace, 16))
    return fail(LLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  PagedOut pd{block_table, seq_idx, positions, n_seq, max_blocks, page_size, num_pages,
              z_page_stride};
  return run_encode(x, T, N, G, d_loop, r, w_down_t, nullptr, z_pages, z_row_stride,
                    z_group_stride, static_cast<cudaStream_t>(stream), muw, workspace, ws_bytes,
                    &pd);
}

}  // extern "C"

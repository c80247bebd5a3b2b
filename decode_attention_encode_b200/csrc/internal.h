// Host-side internals of liblla shared between translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "lla.h"

namespace lla {

// SM count and shared-memory limit of a device, queried once per device.
// Without any visible device these describe a B200 (148 SMs, 227 KB), so
// workspace queries still work on a host with no GPU.
struct DeviceInfo {
  int sms;
  int smem_optin;
};
DeviceInfo device_info();

// Device address of the sticky status word on the current device (one per
// device, set up once with cudaGetSymbolAddress). NULL on failure.
unsigned int* status_word();

// Records a one-line reason for the calling thread and returns `s`.
lla_status fail(lla_status s, const char* fmt, ...);

// Timing hook events of the calling thread (lla_set_timing_events).
void timing_events(cudaEvent_t* begin, cudaEvent_t* end);
// Records the hook's begin (or end) event on `stream` if a hook is set.
cudaError_t record_timing(bool begin, cudaStream_t stream);

// Maps a CUDA error to LLA_ERR_CUDA with its message, or LLA_OK.
lla_status check_cuda(cudaError_t e, const char* what);

// Integer tuning override from the environment (planner sweeps); `dflt`
// when the variable is unset or empty.
int env_int(const char* name, int dflt);

// Host-side argument checks shared by the decode entry points; sets *esz to
// the latent element size.
lla_status check_decode_args(const float* q, const void* zk, const void* zv, lla_dtype zdt, int B,
                             int H, int d_h, int N, int n_cap, int r_k, int r_v, const float* dk,
                             const float* dv, const float* mu_k, const float* mu_v, float* out,
                             float* lse, void* ws, int* esz);

// Launch plan of the per-head absorbed decode. See decode.cu.
struct DecodePlan {
  int esz;             // bytes per latent element (2 or 4)
  int nseg_k, nseg_v;  // 16-byte segments per latent row
  int lpt;             // lanes cooperating on one token
  int sk, sv;          // segments each lane holds (registers)
  bool exact;          // every lane's segments are all in range
  int tile;            // tokens per pipeline stage
  int nstage;          // pipeline depth per warp
  int warps;           // warps per CTA of the stream kernel
  int stage_bytes;     // bytes of one stage (K then V)
  long long P;         // tokens each warp streams
  int W;               // warps that stream
  int grid;            // CTAs of the stream kernel
  int pstride;         // floats per partial record
  size_t off_qp, off_c0, off_part, ws_bytes;
  size_t smem_bytes;   // dynamic shared memory of the stream kernel
};

lla_status plan_decode(int B, int H, int N, int r_k, int r_v, int esz, DecodePlan* plan);

// q_rope [B*H][d_r] (or null): the decoupled rotary branch; the key rows of
// zk then hold r_k latent values followed by d_r rotated rotary-key values.
lla_status run_decode(const float* q, const void* zk, const void* zv, int esz, int B, int H,
                      int d_h, int N, long long n_cap, int r_k, int r_v, const float* dk,
                      const float* dv, const float* mu_k, const float* mu_v, float scale,
                      float* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream,
                      const float* q_rope = nullptr, int d_r = 0);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Piece map of a ragged (paged) plan, all device arrays written by
// k_plan_paged: per-sequence records {kept tokens n, sink part, gap, 0},
// the flattened range's prefix sums [B+1] and {total, tokens per warp}.
struct RaggedMap {
  const int4* seqinfo;
  const long long* cum;
  const long long* plan;      // {total, share, stamp}
  unsigned long long stamp;   // the stamp plan[2] must hold (else: no work)
};

// What a paged decode call runs: the plan kernel and the decode kernels
// (kPlanAndDecode), the plan alone (kPlanOnly), or the decode kernels on a
// plan an earlier kPlanOnly call left in the same workspace (kDecodePlanned).
enum PagedMode { kPlanAndDecode = 0, kPlanOnly = 1, kDecodePlanned = 2 };

// Identifies a paged plan: a 64-bit hash (FNV-1a) of everything the plan
// depends on except the contents of the lengths and the table. k_plan_paged
// stores it next to the plan; the kernels that read the plan compare it
// first and do nothing (status LLA_DEVICE_PAGED_PLAN_MISMATCH) on a
// mismatch, so a workspace that holds no plan for this call is never used.
unsigned long long paged_plan_stamp(int family, int esz, int B, int H, int r_k, int r_v,
                                    int page_size, int num_pages, const int* block_table,
                                    int max_blocks, const int* seq_lens, int sink, int window,
                                    int W, int pmin, int tile_tokens);

size_t workspace_paged(int B, int H, int r_k, int r_v, int esz);

// Log-sum-exp merge of (out, lse) over R disjoint context parts (merge.cu).
lla_status run_merge_attn(const float* outs, const float* lses, int R, long long U, int d,
                          float* out, float* lse, cudaStream_t stream);

// Launches the bounded-wait self-test (selftest.cu).
lla_status run_selftest_wait(unsigned int timeout_us, cudaStream_t stream);

// k_plan_paged: per-sequence records, prefix sums of the flattened range,
// {total, share} and each worker's start (paged.cu). tile_tokens > 0 plans
// LLA-2D: units are tiles of that many tokens, records {tiles, tokens}, and
// the workers are CTAs.
lla_status launch_plan_paged(const int* seq_lens, const int* block_table, int B, int H,
                             int page_size, int num_pages, int max_blocks, int sink, int window,
                             int W, int pmin, int tile_tokens, int4* seqinfo, long long* cum,
                             long long* plan, int4* wstart, unsigned long long stamp,
                             cudaStream_t stream);

size_t workspace_2d_paged(int B, int H, int r_k, int r_v);
lla_status run_decode_2d_paged(const float* q, const void* zk, const void* zv, int B, int H,
                               int d_h, int r_k, int r_v, int page_size, int num_pages,
                               const int* block_table, int max_blocks, const int* seq_lens,
                               int sink, int window, const float* dk, const float* dv,
                               const float* mu_k, const float* mu_v, float scale, float* out,
                               float* lse, void* ws, size_t ws_bytes, cudaStream_t stream,
                               PagedMode mode = kPlanAndDecode);
lla_status run_decode_paged(const float* q, const void* zk, const void* zv, int esz, int B, int H,
                            int d_h, int r_k, int r_v, int page_size, int num_pages,
                            const int* block_table, int max_blocks, const int* seq_lens, int sink,
                            int window, const float* dk, const float* dv, const float* mu_k,
                            const float* mu_v, float scale, float* out, float* lse, void* ws,
                            size_t ws_bytes, cudaStream_t stream,
                            PagedMode mode = kPlanAndDecode);

// Kernels shared by the per-head and LLA-2D decode paths (decode.cu).
// k_absorb writes q' (fp32, [B*H][r_k + d_r]) to qp when qp is non-null, and
// when qsw is non-null also the bf16 copy LLA-2D stages per sequence: for
// each b, an hp x (r_k + d_r) K-major 128B-swizzled operand (rows >= H
// zero), r_k + d_r a multiple of 64, at qsw + b * ((r_k + d_r) / 64) * hp *
// 128. With q_rope non-null the last d_r columns of q' are the rotary query
// [B*H][d_r] times scale * log2(e) (not absorbed). With tc the contraction
// runs on the tensor cores (split bf16 operands, fp32 accumulation; d_h of
// 64 or 128, r_k a multiple of 8, q and W^K 16-byte aligned, else the
// CUDA-core form runs); callers pass it for bf16 latents (absorb_tc).
// launch_combine's tc is chosen by small_gemm_tc.
lla_status launch_absorb(const float* q, const float* dk, const float* mu_k, int B, int H,
                         int d_h, int r_k, float scale, float* qp, float* c0, cudaStream_t stream,
                         unsigned char* qsw = nullptr, int hp = 0, const float* q_rope = nullptr,
                         int d_r = 0, bool tc = false, Span ws = Span{});
// whether per-head decode runs launch_combine / launch_absorb with tc
bool small_gemm_tc(int esz, int B, int r_k, int r_v);
bool absorb_tc(int esz, int B);
lla_status launch_combine(const float* part, int pstride, const float* c0, const float* dv,
                          const float* mu_v, int B, int H, int d_h, int r_v, long long N,
                          long long P, int shared, float* out, float* lse, cudaStream_t stream,
                          const RaggedMap* ragged = nullptr, bool tc = false, Span ws = Span{});

size_t workspace_2d(int B, int H, int N, int r_k, int r_v);
lla_status run_decode_2d(const float* q, const void* zk, const void* zv, int B, int H, int d_h,
                         int N, long long n_cap, int r_k, int r_v, const float* dk,
                         const float* dv, const float* mu_k, const float* mu_v, float scale,
                         float* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream,
                         const float* q_rope = nullptr, int d_r = 0);

// Destination of a latent write into a paged store (lla_encode_paged): token
// n of sequence seq[n] (n when seq is null) at position pos[n] goes to row
// pos % page_size of page block_table[s][pos / page_size]; page_stride is in
// elements. Device arrays: block_table [n_seq][max_blocks], seq and pos [N].
struct PagedOut {
  const int* block_table;
  const int* seq;
  const int* pos;
  int n_seq, max_blocks, page_size, num_pages;
  long long page_stride;
};

// The latent write. With `paged` the output rows go to each token's slot of
// a paged store (zrs, zgs are then the row and group strides inside a page).
lla_status run_encode(const void* x, int T, int N, int G, int d_loop, int r, const void* wt,
                      const float* mu, void* z, long long zrs, long long zgs, cudaStream_t stream,
                      const float* muw = nullptr, void* ws = nullptr, size_t ws_bytes = 0,
                      const PagedOut* paged = nullptr);

// Bytes of the split-K workspace run_encode uses for this shape (0: the
// shape has enough tiles and runs unsplit).
size_t encode_workspace(int T, int N, int G, int d_loop, int r);

// muw[g][c] = sum_k mu[g][k] W_down[g][k][c] over K = T * d_loop (fp32).
lla_status run_encode_bias(const void* wt, const float* mu, int G, int K, int r, float* muw,
                           cudaStream_t stream);

}  // namespace lla

// Merge of attention results over disjoint parts of one context (sm_100a).
//
// Source: the log-sum-exp split of softmax attention that every split-K
// decode in this library already uses inside a call (partial (m, l, u)
// records), applied here across calls. "Looped Latent Attention" §7
// measures the absorbed path at 262k-token contexts; when one sequence's
// latent store is spread over several GPUs, each GPU decodes its part and
// the parts' (out, lse) pairs merge exactly:
//   L = ln sum_r exp(lse_r),  out = sum_r exp(lse_r - L) out_r,  lse = L,
// because out_r = W^V ubar_r + mu^V with weights that sum to one. A part
// with lse_r = -inf (no token) has weight 0.
#include "common.cuh"
#include "internal.h"

namespace lla {
namespace {

// One warp per unit: lanes find the maximum lse over the parts, then each
// lane forms its columns of the weighted sum.
__global__ void __launch_bounds__(256) k_merge_attn(const float* outs, const float* lses, int R,
                                                    long long U, int d, float* out, float* lse) {
  const long long u = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (u >= U) return;
  float M = -INFINITY;
  for (int r = lane; r < R; r += 32) M = fmaxf(M, __ldg(lses + (size_t)r * U + u));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (M == -INFINITY) {  // every part empty
    for (int c = lane; c < d; c += 32) out[u * d + c] = 0.f;
    if (lse && lane == 0) lse[u] = -INFINITY;
    return;
  }
  float L = 0.f;
  for (int r = lane; r < R; r += 32) {
    const float l = __ldg(lses + (size_t)r * U + u);
    L += l == -INFINITY ? 0.f : expf(l - M);
  }
  L = warp_sum(L);
  const float inv = 1.f / L;
  for (int c = lane; c < d; c += 32) {
    float acc = 0.f;
    for (int r = 0; r < R; ++r) {
      const float l = __ldg(lses + (size_t)r * U + u);
      if (l != -INFINITY) acc = fmaf(expf(l - M), __ldg(outs + ((size_t)r * U + u) * d + c), acc);
    }
    out[u * d + c] = acc * inv;
  }
  if (lse && lane == 0) lse[u] = M + logf(L);
}

}  // namespace

lla_status run_merge_attn(const float* outs, const float* lses, int R, long long U, int d,
                          float* out, float* lse, cudaStream_t stream) {
  const long long blocks = (U + 7) / 8;
  k_merge_attn<<<(unsigned)blocks, 256, 0, stream>>>(outs, lses, R, U, d, out, lse);
  return check_cuda(cudaGetLastError(), "launch k_merge_attn");
}

}  // namespace lla

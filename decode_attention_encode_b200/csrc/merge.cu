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

// Extents of the merge's arrays (bounds-check build).
struct MergeSpans {
  Span outs, lses, out, lse;
  unsigned int* status;
};

// One warp per unit: lanes find the maximum lse over the parts, then each
// lane forms its columns of the weighted sum.
__global__ void __launch_bounds__(256) k_merge_attn(const float* outs, const float* lses, int R,
                                                    long long U, int d, float* out, float* lse,
                                                    MergeSpans sp) {
  const long long u = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (u >= U) return;
  auto lse_of = [&](int r) { return ld_chk(lses + (size_t)r * U + u, sp.lses, sp.status, -INFINITY); };
  float M = -INFINITY;
  for (int r = lane; r < R; r += 32) M = fmaxf(M, lse_of(r));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (M == -INFINITY) {  // every part empty
    for (int c = lane; c < d; c += 32) st_chk(&out[u * d + c], 0.f, sp.out, sp.status);
    if (lse && lane == 0) st_chk(&lse[u], -INFINITY, sp.lse, sp.status);
    return;
  }
  float L = 0.f;
  for (int r = lane; r < R; r += 32) {
    const float l = lse_of(r);
    L += l == -INFINITY ? 0.f : expf(l - M);
  }
  L = warp_sum(L);
  const float inv = 1.f / L;
  for (int c = lane; c < d; c += 32) {
    float acc = 0.f;
    for (int r = 0; r < R; ++r) {
      const float l = lse_of(r);
      if (l != -INFINITY)
        acc = fmaf(expf(l - M), ld_chk(outs + ((size_t)r * U + u) * d + c, sp.outs, sp.status, 0.f),
                   acc);
    }
    st_chk(&out[u * d + c], acc * inv, sp.out, sp.status);
  }
  if (lse && lane == 0) st_chk(&lse[u], M + logf(L), sp.lse, sp.status);
}

}  // namespace

lla_status run_merge_attn(const float* outs, const float* lses, int R, long long U, int d,
                          float* out, float* lse, cudaStream_t stream) {
  const long long blocks = (U + 7) / 8;
  const unsigned long long RU = (unsigned long long)R * U;
  MergeSpans sp{span_of(outs, RU * d * 4), span_of(lses, RU * 4),
                span_of(out, (unsigned long long)U * d * 4),
                lse ? span_of(lse, (unsigned long long)U * 4) : Span{}, status_word()};
  k_merge_attn<<<(unsigned)blocks, 256, 0, stream>>>(outs, lses, R, U, d, out, lse, sp);
  return check_cuda(cudaGetLastError(), "launch k_merge_attn");
}

}  // namespace lla

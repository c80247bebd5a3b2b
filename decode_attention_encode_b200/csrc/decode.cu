// Per-head absorbed LLA decode for sm_100a.
//
// Source: "Looped Latent Attention: Cross-Loop KV Compression for Looped
// Transformers" (arXiv 2607.15456), §3 Eq. 3 (loop-specific reconstruction)
// and §7 "Per-head LLA versus LLA-2D at inference" (the absorbed form: the
// K up-projection moves onto the query, the V up-projection is applied once
// to the latent-space value sum).
//
// One (layer, loop) step runs three kernels on the caller's stream:
//   k_absorb   q' = scale*log2(e) * W^K_up,t^T q for every (b, h), and
//              c0 = scale * q . mu^K_t. Tiny; D^K comes from L2.
//   k_stream   the HBM-bound part. The flattened (unit, token) range is cut
//              into equal contiguous pieces, one per warp of a one-wave grid,
//              so every warp streams the same number of latent bytes whatever
//              B, H and N are. Each warp runs its own bulk-async-copy
//              pipeline (cp.async.bulk into a ring of shared-memory stages,
//              completion on an mbarrier per stage), computes scores
//              q' . z^K_j, keeps an online softmax per token slot and
//              accumulates sum_j p_j z^V_j in latent space. Each (warp,
//              unit) piece ends with one partial (m, l, u).
//   k_combine  merges the partials of each unit, divides by the softmax
//              mass and applies W^V_up,t once: out = W^V (u / l) + mu^V.
// k_stream and k_combine are launched with programmatic dependent launch, so
// the latent copies of k_stream start while k_absorb is still running.
#include <algorithm>
#include <cstdio>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "stream.cuh"

namespace lla {
namespace {

constexpr int kAbsorbRows = 64;   // batch rows per k_absorb CTA (8 per warp)
constexpr int kCombineRows = 32;  // batch rows per k_combine CTA (4 per warp)
constexpr int kColChunk = 32;     // decoder columns (absorb) / rows (combine) per CTA

// ---------------------------------------------------------------------------
// k_absorb
// ---------------------------------------------------------------------------
struct AbsorbArgs {
  const float* q;
  const float* dk;
  const float* mu_k;
  int B, H, d_h, r_k;
  int rows;  // batch rows per CTA: 8, 16, 32 or 64
  float qscale;  // scale * log2(e): scores leave k_stream in log2 units
  float scale;
  float* qp;  // [B*H][r_k]
  float* c0;  // [B*H], natural-log units
};

// One CTA per (head, `rows` batch rows, 32 latent columns). The CTA stages
// the d_h x 32 slice of W^K_up,t once and its query rows in shared memory;
// thread (warp w, lane l) forms q'[b][c0 + l] for the rows b = w + 8k, so
// each decoder value read from shared memory feeds rows/8 FMAs. `rows` is
// chosen on the host so the grid stays near 512-1024 CTAs.
__global__ void __launch_bounds__(256) k_absorb(AbsorbArgs a) {
  extern __shared__ __align__(16) float sm_absorb[];
  float* q_s = sm_absorb;                        // [rows][d_h4]
  const int d_h4 = (a.d_h + 3) & ~3;             // rows padded to float4
  float* d_s = sm_absorb + a.rows * d_h4;        // [d_h][kColChunk]
  pdl_launch_dependents();
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * a.rows;
  const int c0 = blockIdx.z * kColChunk;
  const int nb = min(a.rows, a.B - b0);
  const int nc = min(kColChunk, a.r_k - c0);
  for (int idx = threadIdx.x; idx < nb * d_h4; idx += blockDim.x) {
    const int bb = idx / d_h4, i = idx - bb * d_h4;
    q_s[idx] = i < a.d_h ? a.q[((size_t)(b0 + bb) * a.H + h) * a.d_h + i] : 0.f;
  }
  const float* D = a.dk + (size_t)h * a.d_h * a.r_k + c0;
  const int n4 = nc / 4;  // nc is a multiple of 8
  for (int idx = threadIdx.x; idx < a.d_h * n4; idx += blockDim.x) {
    const int i = idx / n4, j = idx - i * n4;
    reinterpret_cast<float4*>(d_s + i * kColChunk)[j] =
        __ldg(reinterpret_cast<const float4*>(D + (size_t)i * a.r_k) + j);
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.z == 0) {
    // c0 = scale * q . mu_k (natural-log units), one warp per row
    for (int bb = warp; bb < nb; bb += 8) {
      float acc = 0.f;
      if (a.mu_k)
        for (int i = lane; i < a.d_h; i += 32)
          acc += q_s[bb * d_h4 + i] * a.mu_k[(size_t)h * a.d_h + i];
      acc = warp_sum(acc);
      if (lane == 0) a.c0[(size_t)(b0 + bb) * a.H + h] = a.scale * acc;
    }
  }
  constexpr int kPer = kAbsorbRows / 8;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  if (lane < nc) {
    for (int i = 0; i < a.d_h; i += 4) {
      float dv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) dv[e] = (i + e < a.d_h) ? d_s[(i + e) * kColChunk + lane] : 0.f;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int bb = warp + 8 * k;
        if (bb < nb) {
          const float4 qv = *reinterpret_cast<const float4*>(q_s + bb * d_h4 + i);
          acc[k] = fmaf(dv[0], qv.x, fmaf(dv[1], qv.y, fmaf(dv[2], qv.z, fmaf(dv[3], qv.w, acc[k]))));
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int bb = warp + 8 * k;
      if (bb < nb) a.qp[((size_t)(b0 + bb) * a.H + h) * a.r_k + c0 + lane] = acc[k] * a.qscale;
    }
  }
}

// ---------------------------------------------------------------------------
// k_combine
// ---------------------------------------------------------------------------
struct CombineArgs {
  const float* part;
  int pstride;
  const float* c0;
  const float* dv;
  const float* mu_v;
  int B, H, d_h, r_v;
  long long N, P;  // per-sequence and per-piece extents of the split
  int shared;      // 1: one split per sequence shared by all heads (LLA-2D)
  int rows;        // batch rows per CTA: 8, 16 or 32
  float* out;
  float* lse;
};

// One CTA per (head, `rows` batch rows, 32 output channels). Warp w merges
// the partial records of rows w, w+8, ... into ubar (lanes across the latent
// index); the CTA stages the 32 x r_v slice of W^V_up,t once (rows padded by
// 4 floats, so float4 reads of 8 consecutive rows hit 8 distinct bank
// groups); thread (warp w, lane l) forms out[b][h][i0 + l] for its rows.
__global__ void __launch_bounds__(256) k_combine(CombineArgs a) {
  extern __shared__ __align__(16) float sm_combine[];
  const int pitch = a.r_v + 4;
  float* ub = sm_combine;                         // [rows][r_v]
  float* d_s = sm_combine + a.rows * a.r_v;       // [kColChunk][pitch]
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * a.rows;
  const int i0 = blockIdx.z * kColChunk;
  const int nb = min(a.rows, a.B - b0);
  const int ni = min(kColChunk, a.d_h - i0);
  // W^V does not depend on the streaming kernel: stage it before waiting
  const float* D = a.dv + ((size_t)h * a.d_h + i0) * a.r_v;
  const int r4 = a.r_v / 4;
  for (int idx = threadIdx.x; idx < ni * r4; idx += blockDim.x) {
    const int i = idx / r4, j = idx - i * r4;
    reinterpret_cast<float4*>(d_s + i * pitch)[j] =
        __ldg(reinterpret_cast<const float4*>(D + (size_t)i * a.r_v) + j);
  }
  pdl_wait();  // partials come from the streaming kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int bb = warp; bb < nb; bb += 8) {
    const long long u = (long long)(b0 + bb) * a.H + h;
    // The split runs over units (b, h) for per-head LLA and over sequences
    // b for LLA-2D; piece w of split key k is partial record w + k.
    const long long key = a.shared ? (long long)(b0 + bb) : u;
    const long long wf = (key * a.N) / a.P;
    const long long wl = ((key + 1) * a.N - 1) / a.P;
    auto rec = [&](long long w) {
      return a.shared ? a.part + ((w + key) * a.H + h) * a.pstride : a.part + (w + key) * a.pstride;
    };
    const int np = (int)(wl - wf + 1);
    float M = kNegBig;
    for (int k = lane; k < np; k += 32) M = fmaxf(M, rec(wf + k)[0]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int k = lane; k < np; k += 32) {
      const float* pp = rec(wf + k);
      L += pp[1] * exp2f(pp[0] - M);
    }
    L = warp_sum(L);
    const float inv = 1.f / L;
    for (int c = lane; c < a.r_v; c += 32) {
      float acc = 0.f;
      for (int k = 0; k < np; ++k) {
        const float* pp = rec(wf + k);
        acc = fmaf(exp2f(pp[0] - M), pp[4 + c], acc);
      }
      ub[bb * a.r_v + c] = acc * inv;
    }
    if (blockIdx.z == 0 && lane == 0 && a.lse) a.lse[u] = (M + log2f(L)) * kLn2 + a.c0[u];
  }
  __syncthreads();
  if (lane < ni) {
    constexpr int kPer = kCombineRows / 8;
    float acc[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
    const float* drow = d_s + lane * pitch;
    for (int c = 0; c < a.r_v; c += 4) {
      const float4 dv = *reinterpret_cast<const float4*>(drow + c);
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int bb = warp + 8 * k;
        if (bb < nb) {
          const float4 uv = *reinterpret_cast<const float4*>(ub + bb * a.r_v + c);
          acc[k] = fmaf(dv.x, uv.x, fmaf(dv.y, uv.y, fmaf(dv.z, uv.z, fmaf(dv.w, uv.w, acc[k]))));
        }
      }
    }
    const float mu = a.mu_v ? a.mu_v[(size_t)h * a.d_h + i0 + lane] : 0.f;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int bb = warp + 8 * k;
      if (bb < nb) a.out[((size_t)(b0 + bb) * a.H + h) * a.d_h + i0 + lane] = acc[k] + mu;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
bool exact_variant(int lpt, int s) { return lpt >= 1 && lpt <= 8 && s >= 1 && s <= 4; }

int env_int(const char* name, int dflt) {
  const char* v = std::getenv(name);
  if (!v || !*v) return dflt;
  return std::atoi(v);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

lla_status launch_absorb(const float* q, const float* dk, const float* mu_k, int B, int H,
                         int d_h, int r_k, float scale, float* qp, float* c0, cudaStream_t stream) {
  const int zc = (r_k + kColChunk - 1) / kColChunk;
  int rows = 8;
  while (rows < kAbsorbRows && (long long)H * zc * ((B + rows - 1) / rows) > 1024) rows *= 2;
  AbsorbArgs a{q, dk, mu_k, B, H, d_h, r_k, rows, scale * kLog2e, scale, qp, c0};
  dim3 grid(H, (B + rows - 1) / rows, zc);
  const size_t smem = ((size_t)rows * ((d_h + 3) & ~3) + (size_t)d_h * kColChunk) * 4;
  cudaError_t e = cudaFuncSetAttribute(k_absorb, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_absorb)");
  k_absorb<<<grid, 256, smem, stream>>>(a);
  return check_cuda(cudaGetLastError(), "launch k_absorb");
}

lla_status launch_combine(const float* part, int pstride, const float* c0, const float* dv,
                          const float* mu_v, int B, int H, int d_h, int r_v, long long N,
                          long long P, int shared, float* out, float* lse, cudaStream_t stream) {
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  const int zc = (d_h + kColChunk - 1) / kColChunk;
  int rows = 8;
  while (rows < kCombineRows && (long long)H * zc * ((B + rows - 1) / rows) > 1024) rows *= 2;
  CombineArgs a{part, pstride, c0, dv, mu_v, B, H, d_h, r_v, N, P, shared, rows, out, lse};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(H, (B + rows - 1) / rows, zc);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = ((size_t)rows * r_v + (size_t)kColChunk * (r_v + 4)) * 4;
  cudaError_t e = cudaFuncSetAttribute(k_combine, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)cfg.dynamicSmemBytes);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_combine)");
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return check_cuda(cudaLaunchKernelEx(&cfg, k_combine, a), "launch k_combine");
}

lla_status plan_decode(int B, int H, int N, int r_k, int r_v, int esz, DecodePlan* p) {
  DecodePlan d{};
  d.esz = esz;
  d.nseg_k = r_k * esz / 16;
  d.nseg_v = r_v * esz / 16;
  auto v2 = [](int x) {
    int k = 0;
    while ((x & 1) == 0 && k < 3) {
      x >>= 1;
      ++k;
    }
    return k;
  };
  // Lanes per token: the largest power of two (<= 8) dividing both segment
  // counts. With it, the 8 lanes of each shared-memory phase touch 8
  // distinct 16-byte bank groups (the per-lane segment count is odd, or one
  // phase is one contiguous 128-byte row piece), so row reads are
  // conflict-free.
  int lpt = 1 << std::min(v2(d.nseg_k), v2(d.nseg_v));
  // tuning override (power of two dividing both segment counts)
  const int lpt_env = env_int("LLA_DECODE_LPT", 0);
  if (lpt_env == 1 || lpt_env == 2 || lpt_env == 4 || lpt_env == 8)
    if (d.nseg_k % lpt_env == 0 && d.nseg_v % lpt_env == 0) lpt = lpt_env;
  if (d.nseg_k == d.nseg_v && exact_variant(lpt, d.nseg_k / lpt)) {
    d.exact = true;
    d.sk = d.sv = d.nseg_k / lpt;
  } else {
    auto fits = [&](int l) { return (d.nseg_k + l - 1) / l <= 4 && (d.nseg_v + l - 1) / l <= 4; };
    while (lpt < 8 && !fits(lpt)) lpt *= 2;
    if (!fits(lpt)) return fail(LLA_ERR_UNSUPPORTED, "latent rank too large for the decode kernel");
    d.exact = false;
    d.sk = d.sv = 4;
  }
  d.lpt = lpt;
  const int ns = 32 / lpt;
  const int tok_bytes = (r_k + r_v) * esz;
  const DeviceInfo di = device_info();
  d.warps = std::max(1, std::min(8, env_int("LLA_DECODE_WARPS", 8)));
  d.nstage = std::max(2, std::min(8, env_int("LLA_DECODE_STAGES", 2)));
  const int target = std::max(1024, env_int("LLA_DECODE_STAGE_BYTES", 10240));
  const int pair = 2 * ns;
  d.tile = std::max(pair, (target / tok_bytes) / pair * pair);
  // fit the CTA's shared memory
  auto smem_of = [&](int tile, int nst) {
    return (size_t)((d.warps * nst * 8 + 127) & ~127) + (size_t)d.warps * nst * tile * tok_bytes;
  };
  while (smem_of(d.tile, d.nstage) > (size_t)di.smem_optin && d.tile > pair) d.tile -= pair;
  while (smem_of(d.tile, d.nstage) > (size_t)di.smem_optin && d.nstage > 2) --d.nstage;
  while (smem_of(d.tile, d.nstage) > (size_t)di.smem_optin && d.warps > 1) --d.warps;
  if (smem_of(d.tile, d.nstage) > (size_t)di.smem_optin)
    return fail(LLA_ERR_UNSUPPORTED, "decode stage does not fit in shared memory");
  d.stage_bytes = d.tile * tok_bytes;
  d.smem_bytes = smem_of(d.tile, d.nstage);

  const long long units = (long long)B * H;
  const long long total = units * N;
  const long long ideal = (long long)di.sms * d.warps;
  const long long pmin = 2LL * d.tile;
  d.P = std::max(pmin, (total + ideal - 1) / ideal);
  d.W = (int)((total + d.P - 1) / d.P);
  d.grid = (d.W + d.warps - 1) / d.warps;
  d.pstride = 4 + r_v;

  d.off_qp = 0;
  d.off_c0 = align256(d.off_qp + (size_t)units * r_k * sizeof(float));
  d.off_part = align256(d.off_c0 + (size_t)units * sizeof(float));
  d.ws_bytes = align256(d.off_part + (size_t)(d.W + units) * d.pstride * sizeof(float));
  *p = d;
  return LLA_OK;
}

lla_status run_decode(const float* q, const void* zk, const void* zv, int esz, int B, int H,
                      int d_h, int N, long long n_cap, int r_k, int r_v, const float* dk,
                      const float* dv, const float* mu_k, const float* mu_v, float scale,
                      float* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  DecodePlan d;
  lla_status st = plan_decode(B, H, N, r_k, r_v, esz, &d);
  if (st != LLA_OK) return st;
  if (ws == nullptr || ws_bytes < d.ws_bytes)
    return fail(LLA_ERR_WORKSPACE, "decode workspace needs %zu bytes, got %zu", d.ws_bytes,
                ws_bytes);
  char* wsb = static_cast<char*>(ws);
  float* qp = reinterpret_cast<float*>(wsb + d.off_qp);
  float* c0 = reinterpret_cast<float*>(wsb + d.off_c0);
  float* part = reinterpret_cast<float*>(wsb + d.off_part);

  StreamFn fn = pick_stream_kernel(esz, d.lpt, d.sk, d.exact);
  if (!fn) return fail(LLA_ERR_UNSUPPORTED, "no decode kernel for this latent shape");

  cudaError_t e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)d.smem_bytes);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_stream)");

  // 1. absorb
  st = launch_absorb(q, dk, mu_k, B, H, d_h, r_k, scale, qp, c0, stream);
  if (st != LLA_OK) return st;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  // 2. stream
  {
    StreamArgs a{};
    a.zk = static_cast<const char*>(zk);
    a.zv = static_cast<const char*>(zv);
    a.n_cap = n_cap;
    a.N = N;
    a.total = (long long)B * H * N;
    a.P = d.P;
    a.W = d.W;
    a.row_k = r_k * esz;
    a.row_v = r_v * esz;
    a.nseg_k = d.nseg_k;
    a.nseg_v = d.nseg_v;
    a.r_k = r_k;
    a.tile = d.tile;
    a.nstage = d.nstage;
    a.stage_bytes = d.stage_bytes;
    a.qp = qp;
    a.part = part;
    a.pstride = d.pstride;
    a.status = status_word();
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(d.grid);
    cfg.blockDim = dim3(32 * d.warps);
    cfg.dynamicSmemBytes = d.smem_bytes;
    cfg.stream = stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = record_timing(true, stream);
    if (e != cudaSuccess) return check_cuda(e, "record timing event");
    e = cudaLaunchKernelEx(&cfg, fn, a);
    if (e != cudaSuccess) return check_cuda(e, "launch k_stream");
    e = record_timing(false, stream);
    if (e != cudaSuccess) return check_cuda(e, "record timing event");
  }
  // 3. combine
  return launch_combine(part, d.pstride, c0, dv, mu_v, B, H, d_h, r_v, N, d.P, 0, out, lse, stream);
  return LLA_OK;
}

}  // namespace lla

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

namespace lla {
namespace {

constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2e = 1.44269504088896341f;
constexpr float kNegBig = -1.0e30f;
// Lazy rescaling: a slot keeps its reference maximum until a score exceeds
// it by this much (log2 units), so p_j <= 2^8 and rescales are rare.
constexpr float kRescaleSlack = 8.0f;

constexpr int kAbsorbRows = 16;   // batch rows per k_absorb CTA
constexpr int kCombineRows = 16;  // batch rows per k_combine CTA

// ---------------------------------------------------------------------------
// k_absorb
// ---------------------------------------------------------------------------
struct AbsorbArgs {
  const float* q;
  const float* dk;
  const float* mu_k;
  int B, H, d_h, r_k;
  float qscale;  // scale * log2(e): scores leave k_stream in log2 units
  float scale;
  float* qp;  // [B*H][r_k]
  float* c0;  // [B*H], natural-log units
};

__global__ void __launch_bounds__(256) k_absorb(AbsorbArgs a) {
  extern __shared__ float q_s[];  // [kAbsorbRows][d_h]
  pdl_launch_dependents();
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * kAbsorbRows;
  const int nb = min(kAbsorbRows, a.B - b0);
  for (int idx = threadIdx.x; idx < nb * a.d_h; idx += blockDim.x) {
    const int bb = idx / a.d_h, i = idx - bb * a.d_h;
    q_s[idx] = a.q[((size_t)(b0 + bb) * a.H + h) * a.d_h + i];
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int bb = warp; bb < nb; bb += nwarps) {
    float acc = 0.f;
    if (a.mu_k)
      for (int i = lane; i < a.d_h; i += 32)
        acc += q_s[bb * a.d_h + i] * a.mu_k[(size_t)h * a.d_h + i];
    acc = warp_sum(acc);
    if (lane == 0) a.c0[(size_t)(b0 + bb) * a.H + h] = a.scale * acc;
  }

  // q'[b][c] = qscale * sum_i D[i][c] q[b][i]; thread -> (column c, row group)
  const int groups = max(1, (int)blockDim.x / a.r_k);
  const int g = threadIdx.x / a.r_k;
  const int c = threadIdx.x - g * a.r_k;
  if (g >= groups) return;
  float acc[kAbsorbRows];
#pragma unroll
  for (int k = 0; k < kAbsorbRows; ++k) acc[k] = 0.f;
  const float* D = a.dk + (size_t)h * a.d_h * a.r_k + c;
  for (int i = 0; i < a.d_h; ++i) {
    const float dval = __ldg(D + (size_t)i * a.r_k);
#pragma unroll
    for (int k = 0; k < kAbsorbRows; ++k) {
      const int bb = g + k * groups;
      if (bb < nb) acc[k] = fmaf(dval, q_s[bb * a.d_h + i], acc[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < kAbsorbRows; ++k) {
    const int bb = g + k * groups;
    if (bb < nb) a.qp[((size_t)(b0 + bb) * a.H + h) * a.r_k + c] = acc[k] * a.qscale;
  }
}

// ---------------------------------------------------------------------------
// k_stream
// ---------------------------------------------------------------------------
struct StreamArgs {
  const char* zk;
  const char* zv;
  long long n_cap;
  long long N;
  long long total;  // units * N
  long long P;      // tokens per warp
  int W;            // streaming warps
  int row_k, row_v;  // bytes per latent row
  int nseg_k, nseg_v;
  int r_k;  // elements (q' row stride)
  int tile, nstage, stage_bytes;
  const float* qp;
  float* part;
  int pstride;
  unsigned int* status;
};

template <int ESZ>
__device__ __forceinline__ void unpack16(const uint4& v, float* f);
template <>
__device__ __forceinline__ void unpack16<2>(const uint4& v, float* f) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}
template <>
__device__ __forceinline__ void unpack16<4>(const uint4& v, float* f) {
  f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}

// ESZ: bytes per latent element. LPT: lanes per token. SK/SV: 16-byte
// segments per lane for K/V. EXACT: nseg == LPT*S for both axes.
template <int ESZ, int LPT, int SK, int SV, bool EXACT>
__global__ void __launch_bounds__(256, 1) k_stream(StreamArgs a) {
  constexpr int E = 16 / ESZ;   // elements per 16-byte segment
  constexpr int NS = 32 / LPT;  // token slots per warp
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ __align__(128) unsigned char smem[];

  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const long long w = (long long)blockIdx.x * nwarps + warp;
  if (w >= a.W) return;
  const int slot = lane / LPT, g = lane - slot * LPT;

  const int bar_bytes = ((nwarps * a.nstage * 8) + 127) & ~127;
  const uint32_t bar0 = smem_u32(smem) + warp * a.nstage * 8;
  unsigned char* buf = smem + bar_bytes + (size_t)warp * a.nstage * a.stage_bytes;
  const uint32_t buf0 = smem_u32(buf);
  const int v_off = a.tile * a.row_k;  // V part of a stage follows K

  if (lane == 0) {
    for (int s = 0; s < a.nstage; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();

  const long long f0 = w * a.P;
  const long long f1 = min(f0 + a.P, a.total);
  const uint64_t pol = l2_evict_first_policy();

  // Producer side (lane 0 issues): the tile sequence is the range [f0, f1)
  // cut at unit boundaries and at `tile` tokens.
  long long pf = f0;
  int issued = 0;
  auto issue = [&]() {
    const long long u = pf / a.N;
    const long long j = pf - u * a.N;
    const int len = (int)min((long long)a.tile, min(f1 - pf, a.N - j));
    const int s = issued % a.nstage;
    if (lane == 0) {
      const uint32_t kb = (uint32_t)len * a.row_k, vb = (uint32_t)len * a.row_v;
      const uint32_t bar = bar0 + 8 * s;
      const long long row = u * a.n_cap + j;
      mbar_arrive_expect_tx(bar, kb + vb);
      bulk_g2s(buf0 + s * a.stage_bytes, a.zk + row * a.row_k, kb, bar, pol);
      bulk_g2s(buf0 + s * a.stage_bytes + v_off, a.zv + row * a.row_v, vb, bar, pol);
    }
    pf += len;
    ++issued;
  };
  for (int s = 0; s < a.nstage && pf < f1; ++s) issue();

  // q' is written by k_absorb.
  pdl_wait();

  int consumed = 0;
  long long f = f0;
  while (f < f1) {
    const long long u = f / a.N;
    const long long seg_end = min(f1, (u + 1) * a.N);

    float qv[SK][E];
#pragma unroll
    for (int s = 0; s < SK; ++s) {
      const int seg = s * LPT + g;
      if (EXACT || seg < a.nseg_k) {
        const float4* src = reinterpret_cast<const float4*>(a.qp + u * a.r_k + seg * E);
#pragma unroll
        for (int e4 = 0; e4 < E / 4; ++e4) {
          const float4 t = src[e4];
          qv[s][4 * e4 + 0] = t.x; qv[s][4 * e4 + 1] = t.y;
          qv[s][4 * e4 + 2] = t.z; qv[s][4 * e4 + 3] = t.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) qv[s][e] = 0.f;
      }
    }
    float m = kNegBig, l = 0.f;
    float acc[SV][E];
#pragma unroll
    for (int s = 0; s < SV; ++s)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[s][e] = 0.f;

    while (f < seg_end) {
      const int len = (int)min((long long)a.tile, seg_end - f);
      const int st = consumed % a.nstage;
      const uint32_t par = (uint32_t)(consumed / a.nstage) & 1u;
      const bool ok = __all_sync(FULL, mbar_wait(bar0 + 8 * st, par));
      if (!ok) {
        if (lane == 0) report_status(a.status, kStatusWaitTimeout);
        for (int i = consumed; i < issued; ++i)
          (void)mbar_wait(bar0 + 8 * (i % a.nstage), (uint32_t)(i / a.nstage) & 1u,
                          kWaitTimeoutNs / 8);
        return;
      }
      const unsigned char* Ks = buf + st * a.stage_bytes;
      const unsigned char* Vs = Ks + v_off;

      for (int t0 = 0; t0 < len; t0 += 2 * NS) {
        const int ta = t0 + slot, tb = t0 + NS + slot;
        const bool va = ta < len, vb = tb < len;
        // scores of two token slots per lane
        float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
#pragma unroll
        for (int s = 0; s < SK; ++s) {
          const int seg = s * LPT + g;
          if (EXACT || seg < a.nseg_k) {
            float x[E];
            if (va) {
              unpack16<ESZ>(*reinterpret_cast<const uint4*>(Ks + ta * a.row_k + seg * 16), x);
#pragma unroll
              for (int e = 0; e < E; e += 2) {
                sa0 = fmaf(qv[s][e], x[e], sa0);
                sa1 = fmaf(qv[s][e + 1], x[e + 1], sa1);
              }
            }
            if (vb) {
              unpack16<ESZ>(*reinterpret_cast<const uint4*>(Ks + tb * a.row_k + seg * 16), x);
#pragma unroll
              for (int e = 0; e < E; e += 2) {
                sb0 = fmaf(qv[s][e], x[e], sb0);
                sb1 = fmaf(qv[s][e + 1], x[e + 1], sb1);
              }
            }
          }
        }
        float sa = sa0 + sa1, sb = sb0 + sb1;
#pragma unroll
        for (int o = LPT / 2; o > 0; o >>= 1) {
          sa += __shfl_xor_sync(FULL, sa, o);
          sb += __shfl_xor_sync(FULL, sb, o);
        }
        if (va) {
          if (sa > m + kRescaleSlack) {
            const float alpha = exp2f(m - sa);
            l *= alpha;
#pragma unroll
            for (int s = 0; s < SV; ++s)
#pragma unroll
              for (int e = 0; e < E; ++e) acc[s][e] *= alpha;
            m = sa;
          }
          const float p = exp2f(sa - m);
          l += p;
#pragma unroll
          for (int s = 0; s < SV; ++s) {
            const int seg = s * LPT + g;
            if (EXACT || seg < a.nseg_v) {
              float x[E];
              unpack16<ESZ>(*reinterpret_cast<const uint4*>(Vs + ta * a.row_v + seg * 16), x);
#pragma unroll
              for (int e = 0; e < E; ++e) acc[s][e] = fmaf(p, x[e], acc[s][e]);
            }
          }
        }
        if (vb) {
          if (sb > m + kRescaleSlack) {
            const float alpha = exp2f(m - sb);
            l *= alpha;
#pragma unroll
            for (int s = 0; s < SV; ++s)
#pragma unroll
              for (int e = 0; e < E; ++e) acc[s][e] *= alpha;
            m = sb;
          }
          const float p = exp2f(sb - m);
          l += p;
#pragma unroll
          for (int s = 0; s < SV; ++s) {
            const int seg = s * LPT + g;
            if (EXACT || seg < a.nseg_v) {
              float x[E];
              unpack16<ESZ>(*reinterpret_cast<const uint4*>(Vs + tb * a.row_v + seg * 16), x);
#pragma unroll
              for (int e = 0; e < E; ++e) acc[s][e] = fmaf(p, x[e], acc[s][e]);
            }
          }
        }
      }
      __syncwarp();
      ++consumed;
      if (pf < f1) issue();  // refill the stage just read
      f += len;
    }

    // Merge the NS token slots of this warp (log-sum-exp butterfly).
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) {
      const float mo = __shfl_xor_sync(FULL, m, o);
      const float lo = __shfl_xor_sync(FULL, l, o);
      const float M = fmaxf(m, mo);
      const float wa = exp2f(m - M), wb = exp2f(mo - M);
      l = l * wa + lo * wb;
#pragma unroll
      for (int s = 0; s < SV; ++s)
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float ao = __shfl_xor_sync(FULL, acc[s][e], o);
          acc[s][e] = acc[s][e] * wa + ao * wb;
        }
      m = M;
    }
    if (slot == 0) {
      float* pp = a.part + (size_t)(w + u) * a.pstride;
      if (g == 0) {
        pp[0] = m;
        pp[1] = l;
      }
#pragma unroll
      for (int s = 0; s < SV; ++s) {
        const int seg = s * LPT + g;
        if (EXACT || seg < a.nseg_v) {
          float4* dst = reinterpret_cast<float4*>(pp + 4 + seg * E);
#pragma unroll
          for (int e4 = 0; e4 < E / 4; ++e4)
            dst[e4] = make_float4(acc[s][4 * e4], acc[s][4 * e4 + 1], acc[s][4 * e4 + 2],
                                  acc[s][4 * e4 + 3]);
        }
      }
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
  long long N, P;
  float* out;
  float* lse;
};

__global__ void __launch_bounds__(256) k_combine(CombineArgs a) {
  extern __shared__ float ub[];  // [kCombineRows][r_v]
  pdl_wait();                    // partials come from k_stream
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * kCombineRows;
  const int nb = min(kCombineRows, a.B - b0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;

  for (int bb = warp; bb < nb; bb += nwarps) {
    const long long u = (long long)(b0 + bb) * a.H + h;
    const long long wf = (u * a.N) / a.P;
    const long long wl = ((u + 1) * a.N - 1) / a.P;
    float M = kNegBig;
    for (long long w = wf; w <= wl; ++w) M = fmaxf(M, a.part[(w + u) * a.pstride]);
    float L = 0.f;
    for (long long w = wf; w <= wl; ++w) {
      const float* pp = a.part + (w + u) * a.pstride;
      L += pp[1] * exp2f(pp[0] - M);
    }
    const float inv = 1.f / L;
    for (int c = lane; c < a.r_v; c += 32) {
      float acc = 0.f;
      for (long long w = wf; w <= wl; ++w) {
        const float* pp = a.part + (w + u) * a.pstride;
        acc = fmaf(exp2f(pp[0] - M), pp[4 + c], acc);
      }
      ub[bb * a.r_v + c] = acc * inv;
    }
    if (lane == 0 && a.lse) a.lse[u] = (M + log2f(L)) * kLn2 + a.c0[u];
  }
  __syncthreads();

  // out[b][h][i] = sum_c W^V[i][c] ubar_b[c] + mu^V[i]: one warp per row i,
  // lanes across c (coalesced reads of W^V from L2).
  for (int i = warp; i < a.d_h; i += nwarps) {
    const float* drow = a.dv + ((size_t)h * a.d_h + i) * a.r_v;
    float acc[kCombineRows];
#pragma unroll
    for (int k = 0; k < kCombineRows; ++k) acc[k] = 0.f;
    for (int c = lane; c < a.r_v; c += 32) {
      const float dval = __ldg(drow + c);
#pragma unroll
      for (int k = 0; k < kCombineRows; ++k)
        if (k < nb) acc[k] = fmaf(dval, ub[k * a.r_v + c], acc[k]);
    }
    const float mu = a.mu_v ? a.mu_v[(size_t)h * a.d_h + i] : 0.f;
#pragma unroll
    for (int k = 0; k < kCombineRows; ++k) {
      if (k < nb) {
        const float v = warp_sum(acc[k]);
        if (lane == 0) a.out[((size_t)(b0 + k) * a.H + h) * a.d_h + i] = v + mu;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
using StreamFn = void (*)(StreamArgs);

template <int ESZ>
StreamFn pick_stream(int lpt, int s, bool exact) {
  if (!exact) {
    switch (lpt) {
      case 1: return k_stream<ESZ, 1, 4, 4, false>;
      case 2: return k_stream<ESZ, 2, 4, 4, false>;
      case 4: return k_stream<ESZ, 4, 4, 4, false>;
      case 8: return k_stream<ESZ, 8, 4, 4, false>;
    }
    return nullptr;
  }
#define LLA_CASE(L, S) \
  if (lpt == L && s == S) return k_stream<ESZ, L, S, S, true>;
  LLA_CASE(1, 1) LLA_CASE(1, 3) LLA_CASE(2, 1) LLA_CASE(2, 3) LLA_CASE(4, 1)
  LLA_CASE(4, 3) LLA_CASE(8, 1) LLA_CASE(8, 2) LLA_CASE(8, 3) LLA_CASE(8, 4)
#undef LLA_CASE
  return nullptr;
}

bool exact_variant(int lpt, int s) {
  if (lpt == 8) return s >= 1 && s <= 4;
  return s == 1 || s == 3;
}

int env_int(const char* name, int dflt) {
  const char* v = std::getenv(name);
  if (!v || !*v) return dflt;
  return std::atoi(v);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

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
  d.nstage = std::max(2, std::min(8, env_int("LLA_DECODE_STAGES", 4)));
  const int target = std::max(1024, env_int("LLA_DECODE_STAGE_BYTES", 6144));
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

  StreamFn fn = (esz == 2) ? pick_stream<2>(d.lpt, d.sk, d.exact) : pick_stream<4>(d.lpt, d.sk, d.exact);
  if (!fn) return fail(LLA_ERR_UNSUPPORTED, "no decode kernel for this latent shape");

  cudaError_t e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)d.smem_bytes);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_stream)");

  // 1. absorb
  {
    AbsorbArgs a{q, dk, mu_k, B, H, d_h, r_k, scale * kLog2e, scale, qp, c0};
    dim3 grid(H, (B + kAbsorbRows - 1) / kAbsorbRows);
    const size_t sm = (size_t)kAbsorbRows * d_h * sizeof(float);
    k_absorb<<<grid, 256, sm, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return check_cuda(e, "launch k_absorb");
  }
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
    e = cudaLaunchKernelEx(&cfg, fn, a);
    if (e != cudaSuccess) return check_cuda(e, "launch k_stream");
  }
  // 3. combine
  {
    CombineArgs a{part, d.pstride, c0, dv, mu_v, B, H, d_h, r_v, (long long)N, d.P, out, lse};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(H, (B + kCombineRows - 1) / kCombineRows);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = (size_t)kCombineRows * r_v * sizeof(float);
    cfg.stream = stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_combine, a);
    if (e != cudaSuccess) return check_cuda(e, "launch k_combine");
  }
  return LLA_OK;
}

}  // namespace lla

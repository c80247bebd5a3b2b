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

constexpr int kAbsorbRows = 8;    // batch rows (one per warp) per k_absorb CTA
constexpr int kCombineRows = 8;   // batch rows (one per warp) per k_combine CTA
constexpr int kColChunk = 32;     // decoder columns (absorb) / rows (combine) per CTA

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

// One CTA per (head, 8 batch rows, 32 latent columns): the CTA stages its
// d_h x 32 slice of W^K_up,t and the 8 query rows in shared memory, and each
// thread forms one q'[b][c] as a d_h-long dot product.
__global__ void __launch_bounds__(256) k_absorb(AbsorbArgs a) {
  __shared__ float q_s[kAbsorbRows * 256];
  __shared__ __align__(16) float d_s[256 * kColChunk];
  pdl_launch_dependents();
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * kAbsorbRows;
  const int c0 = blockIdx.z * kColChunk;
  const int nb = min(kAbsorbRows, a.B - b0);
  const int nc = min(kColChunk, a.r_k - c0);
  for (int idx = threadIdx.x; idx < nb * a.d_h; idx += blockDim.x) {
    const int bb = idx / a.d_h, i = idx - bb * a.d_h;
    q_s[idx] = a.q[((size_t)(b0 + bb) * a.H + h) * a.d_h + i];
  }
  // W^K rows i, columns [c0, c0 + nc): nc is a multiple of 8, so float4 loads
  const float* D = a.dk + (size_t)h * a.d_h * a.r_k + c0;
  const int n4 = nc / 4;
  for (int idx = threadIdx.x; idx < a.d_h * n4; idx += blockDim.x) {
    const int i = idx / n4, j = idx - i * n4;
    reinterpret_cast<float4*>(d_s + i * kColChunk)[j] =
        __ldg(reinterpret_cast<const float4*>(D + (size_t)i * a.r_k) + j);
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.z == 0) {
    // c0 = scale * q . mu_k (natural-log units), one warp per row
    for (int bb = warp; bb < nb; bb += blockDim.x >> 5) {
      float acc = 0.f;
      if (a.mu_k)
        for (int i = lane; i < a.d_h; i += 32)
          acc += q_s[bb * a.d_h + i] * a.mu_k[(size_t)h * a.d_h + i];
      acc = warp_sum(acc);
      if (lane == 0) a.c0[(size_t)(b0 + bb) * a.H + h] = a.scale * acc;
    }
  }
  // thread -> (row bb = warp, column c0 + lane)
  const int bb = warp;
  if (bb < nb && lane < nc) {
    const float* qrow = q_s + bb * a.d_h;
    float s0 = 0.f, s1 = 0.f;
    int i = 0;
    for (; i + 1 < a.d_h; i += 2) {
      s0 = fmaf(d_s[i * kColChunk + lane], qrow[i], s0);
      s1 = fmaf(d_s[(i + 1) * kColChunk + lane], qrow[i + 1], s1);
    }
    if (i < a.d_h) s0 = fmaf(d_s[i * kColChunk + lane], qrow[i], s0);
    a.qp[((size_t)(b0 + bb) * a.H + h) * a.r_k + c0 + lane] = (s0 + s1) * a.qscale;
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

// Loads q' of unit u (this lane's segments) into registers.
template <int E, int LPT, int SK, bool EXACT>
__device__ __forceinline__ void load_qp(float (&qv)[SK][E], const float* qp, long long u, int r_k,
                                        int nseg_k, int g) {
#pragma unroll
  for (int s = 0; s < SK; ++s) {
    const int seg = s * LPT + g;
    if (EXACT || seg < nseg_k) {
      const float4* src = reinterpret_cast<const float4*>(qp + u * r_k + seg * E);
#pragma unroll
      for (int e4 = 0; e4 < E / 4; ++e4) {
        const float4 t = src[e4];
        qv[s][4 * e4 + 0] = t.x;
        qv[s][4 * e4 + 1] = t.y;
        qv[s][4 * e4 + 2] = t.z;
        qv[s][4 * e4 + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) qv[s][e] = 0.f;
    }
  }
}

// One token slot's online-softmax update with score sc (log2 units) and
// value row v.
template <int ESZ, int LPT, int SV, bool EXACT>
__device__ __forceinline__ void slot_update(float sc, const unsigned char* vrow, float& m, float& l,
                                            float (&acc)[SV][16 / ESZ], int nseg_v, int g) {
  constexpr int E = 16 / ESZ;
  if (sc > m + kRescaleSlack) {
    const float alpha = exp2f(m - sc);
    l *= alpha;
#pragma unroll
    for (int s = 0; s < SV; ++s)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[s][e] *= alpha;
    m = sc;
  }
  const float p = exp2f(sc - m);
  l += p;
#pragma unroll
  for (int s = 0; s < SV; ++s) {
    const int seg = s * LPT + g;
    if (EXACT || seg < nseg_v) {
      float x[E];
      unpack16<ESZ>(*reinterpret_cast<const uint4*>(vrow + seg * 16), x);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[s][e] = fmaf(p, x[e], acc[s][e]);
    }
  }
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
  // cut at unit boundaries and at `tile` tokens; (pu, pj) is the unit and
  // token of the next tile to load, ps its stage.
  long long pf = f0, pu = f0 / a.N, pj = f0 - pu * a.N;
  int ps = 0, in_flight = 0;
  auto issue = [&]() {
    const int len = (int)min((long long)a.tile, min(f1 - pf, a.N - pj));
    if (lane == 0) {
      const uint32_t kb = (uint32_t)len * a.row_k, vb = (uint32_t)len * a.row_v;
      const uint32_t bar = bar0 + 8 * ps;
      const long long row = pu * a.n_cap + pj;
      const uint32_t dst = buf0 + ps * a.stage_bytes;
      mbar_arrive_expect_tx(bar, kb + vb);
      bulk_g2s(dst, a.zk + row * a.row_k, kb, bar, pol);
      bulk_g2s(dst + v_off, a.zv + row * a.row_v, vb, bar, pol);
    }
    pf += len;
    pj += len;
    if (pj == a.N) {
      pj = 0;
      ++pu;
    }
    if (++ps == a.nstage) ps = 0;
    ++in_flight;
  };
  for (int s = 0; s < a.nstage && pf < f1; ++s) issue();

  // q' is written by k_absorb.
  pdl_wait();

  int cs = 0;          // stage being consumed
  uint32_t cpar = 0;   // its phase parity
  long long f = f0;
  long long u = f0 / a.N;
  const long long u_last = (f1 - 1) / a.N;
  float qv[SK][E], qn[SK][E];
  load_qp<E, LPT, SK, EXACT>(qv, a.qp, u, a.r_k, a.nseg_k, g);
  while (f < f1) {
    const long long seg_end = min(f1, (u + 1) * a.N);
    // the next unit's q' loads run under this unit's stream
    if (u < u_last) load_qp<E, LPT, SK, EXACT>(qn, a.qp, u + 1, a.r_k, a.nseg_k, g);
    float m = kNegBig, l = 0.f;
    float acc[SV][E];
#pragma unroll
    for (int s = 0; s < SV; ++s)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[s][e] = 0.f;

    while (f < seg_end) {
      const int len = (int)min((long long)a.tile, seg_end - f);
      const bool ok = __all_sync(FULL, mbar_wait(bar0 + 8 * cs, cpar));
      if (!ok) {
        if (lane == 0) report_status(a.status, kStatusWaitTimeout);
        int st = cs;
        uint32_t par = cpar;
        for (int i = 0; i < in_flight; ++i) {
          (void)mbar_wait(bar0 + 8 * st, par, kWaitTimeoutNs / 8);
          if (++st == a.nstage) {
            st = 0;
            par ^= 1u;
          }
        }
        return;
      }
      const unsigned char* Ks = buf + cs * a.stage_bytes;
      const unsigned char* Vs = Ks + v_off;

      for (int t0 = 0; t0 < len; t0 += 2 * NS) {
        const int ta = t0 + slot, tb = t0 + NS + slot;
        const bool va = ta < len, vb = tb < len;
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
        if (va) slot_update<ESZ, LPT, SV, EXACT>(sa, Vs + ta * a.row_v, m, l, acc, a.nseg_v, g);
        if (vb) slot_update<ESZ, LPT, SV, EXACT>(sb, Vs + tb * a.row_v, m, l, acc, a.nseg_v, g);
      }
      __syncwarp();
      --in_flight;
      if (pf < f1) issue();  // refill the stage just read
      if (++cs == a.nstage) {
        cs = 0;
        cpar ^= 1u;
      }
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
    ++u;
#pragma unroll
    for (int s = 0; s < SK; ++s)
#pragma unroll
      for (int e = 0; e < E; ++e) qv[s][e] = qn[s][e];
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
  float* out;
  float* lse;
};

// One CTA per (head, 8 batch rows, 32 output channels): warp w merges the
// partial records of row w (lanes across the latent index) into ubar, the
// CTA stages its 32 x r_v slice of W^V_up,t (rows padded by one float so
// consecutive rows fall in distinct banks), and each thread forms one
// out[b][h][i] as an r_v-long dot product.
__global__ void __launch_bounds__(256) k_combine(CombineArgs a) {
  __shared__ float ub[kCombineRows * 256];
  __shared__ float d_s[kColChunk * 257];
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * kCombineRows;
  const int i0 = blockIdx.z * kColChunk;
  const int nb = min(kCombineRows, a.B - b0);
  const int ni = min(kColChunk, a.d_h - i0);
  const int pitch = a.r_v + 1;
  // W^V does not depend on the streaming kernel: stage it before waiting
  const float* D = a.dv + ((size_t)h * a.d_h + i0) * a.r_v;
  for (int idx = threadIdx.x; idx < ni * a.r_v; idx += blockDim.x) {
    const int i = idx / a.r_v, c = idx - i * a.r_v;
    d_s[i * pitch + c] = __ldg(D + idx);
  }
  pdl_wait();  // partials come from the streaming kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bb = warp;
  if (bb < nb) {
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
  // thread -> (row bb = warp, output channel i0 + lane)
  if (bb < nb && lane < ni) {
    const float* drow = d_s + lane * pitch;
    const float* urow = ub + bb * a.r_v;
    float s0 = 0.f, s1 = 0.f;
    for (int c = 0; c < a.r_v; c += 2) {
      s0 = fmaf(drow[c], urow[c], s0);
      s1 = fmaf(drow[c + 1], urow[c + 1], s1);
    }
    const float mu = a.mu_v ? a.mu_v[(size_t)h * a.d_h + i0 + lane] : 0.f;
    a.out[((size_t)(b0 + bb) * a.H + h) * a.d_h + i0 + lane] = s0 + s1 + mu;
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
  LLA_CASE(1, 1) LLA_CASE(1, 2) LLA_CASE(1, 3) LLA_CASE(1, 4)
  LLA_CASE(2, 1) LLA_CASE(2, 2) LLA_CASE(2, 3) LLA_CASE(2, 4)
  LLA_CASE(4, 1) LLA_CASE(4, 2) LLA_CASE(4, 3) LLA_CASE(4, 4)
  LLA_CASE(8, 1) LLA_CASE(8, 2) LLA_CASE(8, 3) LLA_CASE(8, 4)
#undef LLA_CASE
  return nullptr;
}

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
  AbsorbArgs a{q, dk, mu_k, B, H, d_h, r_k, scale * kLog2e, scale, qp, c0};
  dim3 grid(H, (B + kAbsorbRows - 1) / kAbsorbRows, (r_k + kColChunk - 1) / kColChunk);
  k_absorb<<<grid, 256, 0, stream>>>(a);
  return check_cuda(cudaGetLastError(), "launch k_absorb");
}

lla_status launch_combine(const float* part, int pstride, const float* c0, const float* dv,
                          const float* mu_v, int B, int H, int d_h, int r_v, long long N,
                          long long P, int shared, float* out, float* lse, cudaStream_t stream) {
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  CombineArgs a{part, pstride, c0, dv, mu_v, B, H, d_h, r_v, N, P, shared, out, lse};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(H, (B + kCombineRows - 1) / kCombineRows, (d_h + kColChunk - 1) / kColChunk);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
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

  StreamFn fn = (esz == 2) ? pick_stream<2>(d.lpt, d.sk, d.exact) : pick_stream<4>(d.lpt, d.sk, d.exact);
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
    e = cudaLaunchKernelEx(&cfg, fn, a);
    if (e != cudaSuccess) return check_cuda(e, "launch k_stream");
  }
  // 3. combine
  return launch_combine(part, d.pstride, c0, dv, mu_v, B, H, d_h, r_v, N, d.P, 0, out, lse, stream);
  return LLA_OK;
}

}  // namespace lla

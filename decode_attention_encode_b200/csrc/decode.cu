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
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "stream.cuh"
#include "tc.cuh"

namespace lla {
namespace {

// Register block of k_absorb / k_combine threads: ROWS batch rows (1, 2, 4,
// 8) by COLS columns (1, 2, 4) per thread, the largest ROWS * COLS that
// still gives at least ~256 CTAs for `nh` heads, `ncols` output columns and
// B rows; ties go to more rows, or with prefer_cols to more columns (fewer
// column blocks, which k_combine pays for by merging the same partials in
// each). Larger blocks reuse each shared-memory read for more FMAs.
void pick_block(int nh, int ncols, int B, int* rows_out, int* cols_out, bool prefer_cols = false,
                int max_cols = 4) {
  int best_r = 1, best_c = 1, best = 0;
  for (int r : {8, 4, 2, 1})
    for (int c : {4, 2, 1}) {
      if (c > max_cols) continue;
      if (c > 1 && ncols < 32 * c) continue;  // lanes would sit idle
      const long long ctas = (long long)nh * ((ncols + 32 * c - 1) / (32 * c)) *
                             ((B + 8 * r - 1) / (8 * r));
      if (ctas < 256 && !(r == 1 && c == 1)) continue;
      if (r * c > best || (prefer_cols && r * c == best && c > best_c)) {
        best = r * c;
        best_r = r;
        best_c = c;
      }
    }
  *rows_out = best_r;
  *cols_out = best_c;
}


// Stages n float4 items into shared memory with the whole CTA (256 threads):
// each thread issues up to 8 global loads before its first shared store, so
// a staging pass costs about one memory round trip per 2048 items instead
// of one per item.
template <typename Load, typename Store>
__device__ __forceinline__ void stage_batched(int n, Load load, Store store) {
  constexpr int kBatch = 8;
  for (int base = threadIdx.x; base < n; base += 256 * kBatch) {
    float4 v[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int idx = base + k * 256;
      v[k] = idx < n ? load(idx) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int idx = base + k * 256;
      if (idx < n) store(idx, v[k]);
    }
  }
}

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
  float* qp;  // [B*H][r_k + d_r], or null
  float* c0;  // [B*H], natural-log units
  unsigned char* qsw;  // LLA-2D MMA operand copy of q' (bf16, swizzled), or null
  int hp;              // its rows (heads padded to the MMA N)
  const float* q_rope;  // [B*H][d_r] rotated rotary query, or null (d_r = 0)
  int d_r;
  Span ws_span;         // the workspace holding qp, c0 and qsw (bounds-check build)
  unsigned int* status;
};

// One CTA per (head, 32*COLS latent columns, 8*ROWS batch rows). The CTA
// stages its d_h x 32*COLS slice of W^K_up,t and its query rows in shared
// memory; thread (warp w, lane l) forms q'[b][c0 + l*COLS + j] for the ROWS
// rows b = b0 + w*ROWS + k and its COLS columns j, so one shared-memory read
// of COLS decoder values feeds ROWS*COLS FMAs and one float4 query read
// (the same address for the whole warp) feeds 4*COLS. The kernel is bound by
// shared-memory instructions, so larger ROWS*COLS blocks run faster.
template <int COLS>
__device__ __forceinline__ void lds_cols(const float* p, float (&v)[COLS]) {
  if constexpr (COLS == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else if constexpr (COLS == 2) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x; v[1] = t.y;
  } else {
    v[0] = *p;
  }
}

// Byte offset of sequence b's Q' block in the LLA-2D operand: rq columns
// rounded up to whole 64-column (128-byte) swizzle chunks of hp rows.
__device__ __forceinline__ size_t qsw_block(const AbsorbArgs& a, int rq, int b) {
  return (size_t)b * ((rq + 63) / 64) * a.hp * 128;
}

// The LLA-2D operand's columns from rq up to the next multiple of 64 are
// zero for batch rows b0 .. b0+nb-1 of head h (and of the padding heads when
// h is the last head): the tensor map fills the latent tile's matching
// columns with zeros, and those products must stay finite. Called by the
// CTA that holds the last columns.
__device__ __forceinline__ void zero_qsw_tail(const AbsorbArgs& a, int rq, int h, int b0, int nb) {
  const int npad = ((rq + 63) & ~63) - rq;
  const int nh = h == a.H - 1 ? 1 + a.hp - a.H : 1;
  for (int idx = threadIdx.x; idx < nb * npad * nh; idx += blockDim.x) {
    const int bb = idx / (npad * nh), rest = idx - bb * npad * nh;
    const int k = rest / npad, c = rq + rest - k * npad;
    const int hh = k == 0 ? h : a.H + k - 1;
    st_chk(reinterpret_cast<__nv_bfloat16*>(a.qsw + qsw_block(a, rq, b0 + bb) + sw128_off(hh, c, a.hp)),
           __float2bfloat16_rn(0.f), a.ws_span, a.status);
  }
}

template <int ROWS, int COLS>
__global__ void __launch_bounds__(256) k_absorb(AbsorbArgs a) {
  constexpr int CW = 32 * COLS;  // columns per CTA
  extern __shared__ __align__(16) float sm_absorb[];
  const int d_h4 = (a.d_h + 3) & ~3;
  float* d_s = sm_absorb;                   // [d_h4][CW]
  float* q_s = sm_absorb + d_h4 * CW;       // [8*ROWS][d_h4]
  pdl_launch_dependents();
  const int h = blockIdx.x;
  const int c0 = blockIdx.y * CW;
  const int b0 = blockIdx.z * (8 * ROWS);
  const int nb = min(8 * ROWS, a.B - b0);
  const int rq = a.r_k + a.d_r;        // q' row: latent part, then rotary part
  const int nc = min(CW, rq - c0);     // columns of this CTA, a multiple of 8
  const int n4 = max(0, min(CW, a.r_k - c0)) / 4;  // of them from W^K, in float4
  const float* D = a.dk + (size_t)h * a.d_h * a.r_k + c0;
  constexpr int F4 = CW / 4;  // float4 per staged decoder row
  stage_batched(d_h4 * F4, [&](int idx) {
    const int i = idx / F4, j = idx - i * F4;
    return (i < a.d_h && j < n4) ? __ldg(reinterpret_cast<const float4*>(D + (size_t)i * a.r_k) + j)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }, [&](int idx, float4 v) { reinterpret_cast<float4*>(d_s)[idx] = v; });
  const int q4 = d_h4 / 4;  // float4 per staged query row
  if ((a.d_h & 3) == 0 && (reinterpret_cast<uintptr_t>(a.q) & 15) == 0) {
    stage_batched(8 * ROWS * q4, [&](int idx) {
      const int bb = idx / q4, i4 = idx - bb * q4;
      return bb < nb ? __ldg(reinterpret_cast<const float4*>(
                           a.q + ((size_t)(b0 + bb) * a.H + h) * a.d_h) + i4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }, [&](int idx, float4 v) { reinterpret_cast<float4*>(q_s)[idx] = v; });
  } else {
    stage_batched(8 * ROWS * q4, [&](int idx) {
      const int bb = idx / q4, i = 4 * (idx - bb * q4);
      const float* row = a.q + ((size_t)(b0 + bb) * a.H + h) * a.d_h;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (bb < nb) {
        if (i + 0 < a.d_h) v.x = __ldg(row + i + 0);
        if (i + 1 < a.d_h) v.y = __ldg(row + i + 1);
        if (i + 2 < a.d_h) v.z = __ldg(row + i + 2);
        if (i + 3 < a.d_h) v.w = __ldg(row + i + 3);
      }
      return v;
    }, [&](int idx, float4 v) { reinterpret_cast<float4*>(q_s)[idx] = v; });
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.y == 0) {
    // c0 = scale * q . mu_k (natural-log units), one warp per row
    for (int bb = warp; bb < nb; bb += 8) {
      float acc = 0.f;
      if (a.mu_k)
        for (int i = lane; i < a.d_h; i += 32)
          acc += q_s[bb * d_h4 + i] * a.mu_k[(size_t)h * a.d_h + i];
      acc = warp_sum(acc);
      if (lane == 0) st_chk(&a.c0[(size_t)(b0 + bb) * a.H + h], a.scale * acc, a.ws_span, a.status);
    }
  }
  float acc[ROWS][COLS];
#pragma unroll
  for (int k = 0; k < ROWS; ++k)
#pragma unroll
    for (int j = 0; j < COLS; ++j) acc[k][j] = 0.f;
  const float* qrow = q_s + warp * ROWS * d_h4;
  const float* dcol = d_s + lane * COLS;
  for (int i = 0; i < d_h4; i += 4) {
    float dv[4][COLS];
#pragma unroll
    for (int e = 0; e < 4; ++e) lds_cols<COLS>(dcol + (i + e) * CW, dv[e]);
#pragma unroll
    for (int k = 0; k < ROWS; ++k) {
      const float4 qv = *reinterpret_cast<const float4*>(qrow + k * d_h4 + i);
#pragma unroll
      for (int j = 0; j < COLS; ++j)
        acc[k][j] = fmaf(dv[0][j], qv.x,
                         fmaf(dv[1][j], qv.y, fmaf(dv[2][j], qv.z, fmaf(dv[3][j], qv.w, acc[k][j]))));
    }
  }
#pragma unroll
  for (int j = 0; j < COLS; ++j) {
    const int cl = lane * COLS + j;  // column within the CTA
    if (cl >= nc) continue;
    const int c = c0 + cl;
#pragma unroll
    for (int k = 0; k < ROWS; ++k) {
      const int bb = warp * ROWS + k;
      if (bb >= nb) continue;
      const size_t unit = (size_t)(b0 + bb) * a.H + h;
      // the rotary part of the query is not absorbed: it meets the cached
      // rotated keys as it is
      const float v = (c < a.r_k ? acc[k][j] : __ldg(a.q_rope + unit * a.d_r + (c - a.r_k))) *
                      a.qscale;
      if (a.qp) st_chk(&a.qp[unit * rq + c], v, a.ws_span, a.status);
      if (a.qsw) {
        unsigned char* base = a.qsw + qsw_block(a, rq, b0 + bb);
        st_chk(reinterpret_cast<__nv_bfloat16*>(base + sw128_off(h, c, a.hp)), __float2bfloat16_rn(v),
               a.ws_span, a.status);
        // the last head's CTAs also clear the padding rows h >= H
        if (h == a.H - 1)
          for (int hz = a.H; hz < a.hp; ++hz)
            st_chk(reinterpret_cast<__nv_bfloat16*>(base + sw128_off(hz, c, a.hp)),
                   __float2bfloat16_rn(0.f), a.ws_span, a.status);
      }
    }
  }
  if (a.qsw && c0 + nc == rq) zero_qsw_tail(a, rq, h, b0, nb);
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
  RaggedMap ragged;  // seqinfo non-null: the paged plan's piece map
  unsigned int* status;
  Span ws_span, out_span, lse_span;  // extents (bounds-check build)
};

// The merge pass shared by k_combine and k_combine_tc.
//
// merge_rows: per row bb < nrows of a combine CTA (batch rows b0 .. b0+nb-1
// of head h), one thread per row: the row's first partial record and piece
// count, and the merged maximum and normaliser over its pieces, with four
// record loads in flight; it also writes lse. The split runs over units
// (b, h) for per-head LLA and over sequences b for LLA-2D; piece w of split
// key k is partial record w + k. A ragged plan places unit (b, h) at
// cum[b] + h * n_b in the range. A row with no attended token gets no piece,
// keep = 0 and lse = -inf.
__device__ __forceinline__ void merge_rows(const CombineArgs& a, int h, int b0, int nb, int nrows,
                                           int* s_np, long long* s_off, float* s_M, float* s_inv,
                                           float* s_keep) {
  if ((int)threadIdx.x >= nrows) return;
  const long long rstride = a.shared ? (long long)a.H * a.pstride : a.pstride;
  const int bb = threadIdx.x;
  // a ragged map whose plan is not this call's (its stamp differs): every
  // row is empty, and the mismatch is reported
  const bool plan_ok = !a.ragged.seqinfo || (unsigned long long)a.ragged.plan[2] == a.ragged.stamp;
  if (!plan_ok && bb == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    report_status(a.status, kStatusPlanMismatch);
  int np = 0;
  long long off = 0;
  float M = kNegBig, L = 0.f, keep = 0.f;
  if (bb < nb) {
    const long long u = (long long)(b0 + bb) * a.H + h;
    const float c0u =  // in flight with the records
        (blockIdx.y == 0 && a.lse) ? ld_chk(&a.c0[u], a.ws_span, a.status, 0.f) : 0.f;
    const long long key = a.shared ? (long long)(b0 + bb) : u;
    long long wf = 0, wl = -1;
    if (a.ragged.seqinfo) {
      const int n = plan_ok ? __ldg(&a.ragged.seqinfo[b0 + bb].x) : 0;
      if (n > 0) {
        const long long P = a.ragged.plan[1];
        // per head for per-head LLA; LLA-2D splits a sequence once for all heads
        const long long first = a.ragged.cum[b0 + bb] + (a.shared ? 0LL : (long long)h * n);
        wf = first / P;
        wl = (first + n - 1) / P;
      }
    } else {
      wf = (key * a.N) / a.P;
      wl = ((key + 1) * a.N - 1) / a.P;
    }
    np = (int)(wl - wf + 1);
    off = a.shared ? ((wf + key) * a.H + h) * a.pstride : (wf + key) * a.pstride;
    const float* rec0 = a.part + off;
    for (int p0 = 0; p0 < np; p0 += 4) {
      float2 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v[k] = p0 + k < np ? ld_chk(reinterpret_cast<const float2*>(rec0 + (p0 + k) * rstride),
                                    a.ws_span, a.status, make_float2(kNegBig, 0.f))
                           : make_float2(kNegBig, 0.f);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float Mn = fmaxf(M, v[k].x);
        L = L * exp2f(M - Mn) + v[k].y * exp2f(v[k].x - Mn);
        M = Mn;
      }
    }
    keep = np > 0 ? 1.f : 0.f;
    if (blockIdx.y == 0 && a.lse)  // no attended token: lse = -inf
      st_chk(&a.lse[u], np > 0 ? (M + log2f(L)) * kLn2 + c0u : -INFINITY, a.lse_span, a.status);
  }
  s_np[bb] = np;
  s_off[bb] = off;
  s_M[bb] = M;
  s_inv[bb] = np > 0 ? 1.f / L : 0.f;
  s_keep[bb] = keep;
}

// merge_sweep: ubar[row] = sum_p exp2(m_p - M) u_p / L over the CTA's
// (row, 4-column) items, k4 items per row of which the first r4 hold values
// (the rest are padding and come out 0), four items per thread at a time
// so their record loads are in flight together (a CTA rarely has more than
// one or two items per thread: larger blocks take k_combine_tc). Rows with
// no piece come out 0. store(bb, c4, v) places each normalised float4.
template <class Store>
__device__ __forceinline__ void merge_sweep(const CombineArgs& a, int nrows, int k4, int r4,
                                            const int* s_np, const long long* s_off,
                                            const float* s_M, const float* s_inv, Store store) {
  constexpr int kI = 4;
  const long long rstride = a.shared ? (long long)a.H * a.pstride : a.pstride;
  const int nitems = nrows * k4;
  for (int base = threadIdx.x; base < nitems; base += 256 * kI) {
    float4 acc[kI];
    const float* rb[kI];
    int npk[kI], c4k[kI];
    float Mk[kI];
    int npmax = 0;
#pragma unroll
    for (int k = 0; k < kI; ++k) {
      const int idx = base + k * 256;
      acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      npk[k] = 0;
      rb[k] = a.part;
      c4k[k] = 0;
      Mk[k] = 0.f;
      if (idx < nitems) {
        const int bb = idx / k4;
        c4k[k] = idx - bb * k4;
        npk[k] = c4k[k] < r4 ? s_np[bb] : 0;
        rb[k] = a.part + s_off[bb];
        Mk[k] = s_M[bb];
      }
      npmax = max(npmax, npk[k]);
    }
    for (int p = 0; p < npmax; ++p) {
      float mv[kI];
      float4 uv[kI];
#pragma unroll
      for (int k = 0; k < kI; ++k) {
        if (p < npk[k]) {
          mv[k] = ld_chk(rb[k] + p * rstride, a.ws_span, a.status, kNegBig);
          uv[k] = ld_chk(reinterpret_cast<const float4*>(rb[k] + p * rstride + 4) + c4k[k],
                         a.ws_span, a.status, make_float4(0.f, 0.f, 0.f, 0.f));
        }
      }
#pragma unroll
      for (int k = 0; k < kI; ++k) {
        if (p < npk[k]) {
          const float wk = exp2f(mv[k] - Mk[k]);
          acc[k].x = fmaf(wk, uv[k].x, acc[k].x);
          acc[k].y = fmaf(wk, uv[k].y, acc[k].y);
          acc[k].z = fmaf(wk, uv[k].z, acc[k].z);
          acc[k].w = fmaf(wk, uv[k].w, acc[k].w);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kI; ++k) {
      const int idx = base + k * 256;
      if (idx < nitems) {
        const int bb = idx / k4;
        const float inv = s_inv[bb];
        store(bb, c4k[k],
              make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv));
      }
    }
  }
}

// One CTA per (head, 32*COLS output channels, 8*ROWS batch rows). The CTA
// stages its 32*COLS x r_v slice of W^V_up,t (rows padded by 4 floats, so float4 reads
// of 8 consecutive rows hit distinct bank groups; staged before waiting on
// the streaming kernel), then merges the partial records of its rows into
// ubar: one thread per row forms the merged maximum and normaliser, then
// all threads sweep the (row, 4-column) items with several records in
// flight each, since this kernel is bound by memory round trips, not
// bandwidth. Thread (w, l) finally forms out[b][h][i0 + l + 32 j] for its
// ROWS rows. Three CTAs fit an SM (80 registers), so the 384 CTAs of a
// 768-sequence batch run in one wave.
template <int ROWS, int COLS>
__global__ void __launch_bounds__(256, 3) k_combine(CombineArgs a) {
  constexpr int CW = 32 * COLS;  // output channels per CTA
  extern __shared__ __align__(16) float sm_combine[];
  // per row of the CTA: pieces, offset of the first record, merged max,
  // 1 / normaliser, and 0 for a row with no attended token
  __shared__ int s_np[64];
  __shared__ long long s_off[64];
  __shared__ float s_M[64], s_inv[64], s_keep[64];
  const int pitch = a.r_v + 4;
  float* d_s = sm_combine;                        // [CW][pitch]
  float* ub = sm_combine + CW * pitch;            // [8*ROWS][r_v]
  const int h = blockIdx.x;
  const int i0 = blockIdx.y * CW;
  const int b0 = blockIdx.z * (8 * ROWS);
  const int nb = min(8 * ROWS, a.B - b0);
  const int ni = min(CW, a.d_h - i0);
  const float* D = a.dv + ((size_t)h * a.d_h + i0) * a.r_v;
  const int r4 = a.r_v / 4;
  stage_batched(ni * r4, [&](int idx) {
    const int i = idx / r4, j = idx - i * r4;
    return __ldg(reinterpret_cast<const float4*>(D + (size_t)i * a.r_v) + j);
  }, [&](int idx, float4 v) {
    const int i = idx / r4, j = idx - i * r4;
    reinterpret_cast<float4*>(d_s + i * pitch)[j] = v;
  });
  pdl_wait();  // partials come from the streaming kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrows = 8 * ROWS;
  // 1. per row: its records, merged maximum and normaliser
  merge_rows(a, h, b0, nb, nrows, s_np, s_off, s_M, s_inv, s_keep);
  __syncthreads();
  // 2. ubar rows into shared memory
  merge_sweep(a, nrows, r4, r4, s_np, s_off, s_M, s_inv, [&](int bb, int c4, float4 v) {
    reinterpret_cast<float4*>(ub + bb * a.r_v)[c4] = v;
  });
  __syncthreads();
  // thread (w, l): channels i0 + l + 32 j (j < COLS; consecutive lanes read
  // consecutive padded rows, so the float4 reads are conflict-free) for the
  // ROWS rows of warp w
  float acc[ROWS][COLS];
#pragma unroll
  for (int k = 0; k < ROWS; ++k)
#pragma unroll
    for (int j = 0; j < COLS; ++j) acc[k][j] = 0.f;
  const float4* ubase = reinterpret_cast<const float4*>(ub + warp * ROWS * a.r_v);
  for (int c4 = 0; c4 < r4; ++c4) {
    float4 dv[COLS];
#pragma unroll
    for (int j = 0; j < COLS; ++j)
      dv[j] = reinterpret_cast<const float4*>(d_s + (lane + 32 * j) * pitch)[c4];
#pragma unroll
    for (int k = 0; k < ROWS; ++k) {
      const float4 uv = ubase[k * r4 + c4];
#pragma unroll
      for (int j = 0; j < COLS; ++j)
        acc[k][j] = fmaf(dv[j].x, uv.x, fmaf(dv[j].y, uv.y, fmaf(dv[j].z, uv.z, fmaf(dv[j].w, uv.w, acc[k][j]))));
    }
  }
#pragma unroll
  for (int j = 0; j < COLS; ++j) {
    const int il = lane + 32 * j;
    if (il >= ni) continue;
    const float mu = a.mu_v ? a.mu_v[(size_t)h * a.d_h + i0 + il] : 0.f;
#pragma unroll
    for (int k = 0; k < ROWS; ++k) {
      const int bb = warp * ROWS + k;
      if (bb < nb)
        st_chk(&a.out[((size_t)(b0 + bb) * a.H + h) * a.d_h + i0 + il],
               acc[k][j] + mu * s_keep[bb], a.out_span, a.status);
    }
  }
}


// ---------------------------------------------------------------------------
// Tensor-core forms of k_absorb and k_combine (bf16 latents)
// ---------------------------------------------------------------------------
// Both kernels are small GEMMs per head (q' = q W^K, out = W^V ubar) that the
// CUDA-core forms above spend most of their time on as FFMA chains. Here the
// contraction runs on warp-level bf16 tensor-core MMAs (m16n8k16, fp32
// accumulate). Each fp32 operand x is split as hi = bf16(x), lo = bf16(x - hi)
// (x - hi is exact in fp32) and the product is hi.hi + hi.lo + lo.hi. With
// bf16's 8-bit significand |lo| <= 2^-8 |x| and |x - hi - lo| <= 2^-16 |x|,
// so the dropped lo.lo term and the two residues together stay within
// 3 * 2^-16 of each product |x y|: far under the bf16 rounding the latents
// and the LLA-2D query already carry.
// Accumulators stay in registers: no tensor memory is allocated, so these
// kernels never contend with the programmatically overlapped k_lla2d for it.
//
// Operands are staged as bf16 rows whose pitch is their width (a multiple
// of 16 elements) plus 8: the eight 16-byte rows of every ldmatrix then
// start 4*(odd) banks apart and hit 32 distinct banks.

// hi and lo bf16 parts of four consecutive fp32 values, as 8-byte stores
__device__ __forceinline__ void store_split4(__nv_bfloat16* hi, __nv_bfloat16* lo, float4 v) {
  const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 h23 = __floats2bfloat162_rn(v.z, v.w);
  const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
  const __nv_bfloat162 l01 = __floats2bfloat162_rn(v.x - f01.x, v.y - f01.y);
  const __nv_bfloat162 l23 = __floats2bfloat162_rn(v.z - f23.x, v.w - f23.y);
  uint2 uh, ul;
  uh.x = *reinterpret_cast<const uint32_t*>(&h01);
  uh.y = *reinterpret_cast<const uint32_t*>(&h23);
  ul.x = *reinterpret_cast<const uint32_t*>(&l01);
  ul.y = *reinterpret_cast<const uint32_t*>(&l23);
  *reinterpret_cast<uint2*>(hi) = uh;
  *reinterpret_cast<uint2*>(lo) = ul;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// d += a.b with both operands split: hi.hi + hi.lo + lo.hi
__device__ __forceinline__ void mma_split(float (&d)[4], const uint32_t (&ah)[4],
                                          const uint32_t (&al)[4], const uint32_t (&bh)[2],
                                          const uint32_t (&bl)[2]) {
  mma_bf16(d, al, bh);
  mma_bf16(d, ah, bl);
  mma_bf16(d, ah, bh);
}

constexpr int kTcRows = 64;  // batch rows per CTA in both kernels
constexpr int kTcCols = 64;  // q' columns per k_absorb_tc CTA
constexpr int kTcCh = 32;    // output channels per k_combine_tc CTA

size_t absorb_tc_smem(int d_h) {
  return (size_t)2 * (kTcRows * (d_h + 8) + d_h * (kTcCols + 8)) * sizeof(__nv_bfloat16);
}

size_t combine_tc_smem(int r_v) {
  const int pitch = ((r_v + 15) & ~15) + 8;
  return (size_t)2 * (kTcCh + kTcRows) * pitch * sizeof(__nv_bfloat16);
}

// Fragment loads with ldmatrix: four 8 x 8 bf16 matrices whose rows start
// at the addresses lanes 0-7, 8-15, 16-23 and 24-31 give. The plain form
// feeds an A fragment (or two B fragments of a [column][k] array), the
// transposed form two B fragments of a [k][column] array.
__device__ __forceinline__ void ldsm_x4(uint32_t (&f)[4], const __nv_bfloat16* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(f[0]), "=r"(f[1]), "=r"(f[2]), "=r"(f[3])
               : "r"(a));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&f)[4], const __nv_bfloat16* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(f[0]), "=r"(f[1]), "=r"(f[2]), "=r"(f[3])
               : "r"(a));
}

__device__ __forceinline__ void mma_split2(float (&d0)[4], float (&d1)[4], const uint32_t (&ah)[4],
                                           const uint32_t (&al)[4], const uint32_t (&bh)[4],
                                           const uint32_t (&bl)[4]) {
  const uint32_t bh0[2] = {bh[0], bh[1]}, bl0[2] = {bl[0], bl[1]};
  const uint32_t bh1[2] = {bh[2], bh[3]}, bl1[2] = {bl[2], bl[3]};
  mma_split(d0, ah, al, bh0, bl0);
  mma_split(d1, ah, al, bh1, bl1);
}

// One CTA per (head h, 64 q' columns, 64 batch rows): M = batch rows, N =
// q' columns, K = d_h = DH (64 or 128, a compile-time constant so that the
// staging index arithmetic is shifts). Warp w computes rows 16*(w%4).. and
// columns 32*(w/4).. of the tile; columns past r_k (the rotary part) take
// q_rope. Every thread issues all its loads of both operands before its
// first shared store: thread t holds float4 t % (DH/4) of query rows
// t / (DH/4) + k * 1024/DH, and float4 t % 16 of W^K_h rows t / 16 + 16 k,
// both staged as bf16 hi/lo rows with a pitch of 8 extra elements (the
// eight rows of every ldmatrix hit distinct banks). W^K_h keeps its
// [i][column] order; the transposed ldmatrix forms the B fragments. The
// LLA-2D operand leaves through a shared tile: each batch row's 64 columns
// are one 128-byte swizzled row of the operand, written as eight 16-byte
// stores.
template <int DH>
__global__ void __launch_bounds__(256, 2) k_absorb_tc(AbsorbArgs a) {
  static_assert(DH == 64 || DH == 128, "k_absorb_tc stages d_h of 64 or 128");
  constexpr int QP = DH + 8, WP = kTcCols + 8;
  constexpr int D4 = DH / 4, KB = DH / 16, QSTEP = 256 / D4;
  extern __shared__ __align__(16) unsigned char sm_abs_tc[];
  __nv_bfloat16* q_hi = reinterpret_cast<__nv_bfloat16*>(sm_abs_tc);  // [64 rows][QP]
  __nv_bfloat16* q_lo = q_hi + kTcRows * QP;
  __nv_bfloat16* w_hi = q_lo + kTcRows * QP;  // [DH][WP]: W^K_h row i, columns c0..
  __nv_bfloat16* w_lo = w_hi + DH * WP;
  pdl_launch_dependents();
  const int h = blockIdx.x;
  const int c0 = blockIdx.y * kTcCols;
  const int b0 = blockIdx.z * kTcRows;
  const int nb = min(kTcRows, a.B - b0);
  const int rq = a.r_k + a.d_r;
  const int nc = min(kTcCols, rq - c0);
  const int ncw = max(0, min(kTcCols, a.r_k - c0));  // columns from W^K, a multiple of 8
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qi4 = tid % D4, qrow0 = tid / D4;
  const int wj4 = tid & 15, wrow0 = tid >> 4;
  const float* qh = a.q + (size_t)h * DH + 4 * qi4;
  const float* D = a.dk + (size_t)h * DH * a.r_k + c0 + 4 * wj4;
  const bool wcol = 4 * wj4 < ncw;
  float4 vq[KB], vw[KB];
#pragma unroll
  for (int k = 0; k < KB; ++k) {
    const int bb = qrow0 + k * QSTEP;
    vq[k] = bb < nb ? __ldg(reinterpret_cast<const float4*>(qh + (size_t)(b0 + bb) * a.H * DH))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    vw[k] = wcol ? __ldg(reinterpret_cast<const float4*>(D + (size_t)(wrow0 + 16 * k) * a.r_k))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (blockIdx.y == 0) {
    // c0 = scale * q . mu_k (natural-log units) in fp32 from the loaded
    // query values: a row's D4 float4s sit in D4 consecutive lanes
    float mu[4] = {0.f, 0.f, 0.f, 0.f};
    if (a.mu_k)
#pragma unroll
      for (int e = 0; e < 4; ++e) mu[e] = __ldg(a.mu_k + (size_t)h * DH + 4 * qi4 + e);
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      float acc = fmaf(vq[k].x, mu[0], fmaf(vq[k].y, mu[1], fmaf(vq[k].z, mu[2], vq[k].w * mu[3])));
#pragma unroll
      for (int o = D4 / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const int bb = qrow0 + k * QSTEP;
      if (qi4 == 0 && bb < nb)
        st_chk(&a.c0[(size_t)(b0 + bb) * a.H + h], a.scale * acc, a.ws_span, a.status);
    }
  }
#pragma unroll
  for (int k = 0; k < KB; ++k) {
    const int bb = qrow0 + k * QSTEP, i = wrow0 + 16 * k;
    store_split4(q_hi + bb * QP + 4 * qi4, q_lo + bb * QP + 4 * qi4, vq[k]);
    store_split4(w_hi + i * WP + 4 * wj4, w_lo + i * WP + 4 * wj4, vw[k]);
  }
  __syncthreads();
  const int m0 = (warp & 3) * 16, n0 = (warp >> 2) * 32;
  const int lr = lane & 15, lc = (lane >> 4) * 8;
  float acc[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  if (n0 < ncw) {
#pragma unroll 4
    for (int k0 = 0; k0 < DH; k0 += 16) {
      uint32_t ah[4], al[4], bh[4], bl[4];
      ldsm_x4(ah, q_hi + (m0 + lr) * QP + k0 + lc);
      ldsm_x4(al, q_lo + (m0 + lr) * QP + k0 + lc);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        ldsm_x4_t(bh, w_hi + (k0 + lr) * WP + n0 + 16 * np + lc);
        ldsm_x4_t(bl, w_lo + (k0 + lr) * WP + n0 + 16 * np + lc);
        mma_split2(acc[2 * np], acc[2 * np + 1], ah, al, bh, bl);
      }
    }
  }
  if (a.qsw) __syncthreads();  // the output tile reuses q_hi
  __nv_bfloat16* tile = q_hi;  // [64 rows][WP] bf16 q' of this column block
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int bb = m0 + g + 8 * hr;
      const int cl = n0 + 8 * nt + 2 * t;
      const size_t unit = (size_t)(b0 + bb) * a.H + h;
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = c0 + cl + e;
        // the rotary part of the query is not absorbed: it meets the cached
        // rotated keys as it is; columns past rq are the operand's zero pad
        v[e] = (bb >= nb || cl + e >= nc) ? 0.f
               : (c < a.r_k ? acc[nt][2 * hr + e]
                            : __ldg(a.q_rope + unit * a.d_r + (c - a.r_k))) * a.qscale;
        if (a.qp && bb < nb && cl + e < nc) st_chk(&a.qp[unit * rq + c], v[e], a.ws_span, a.status);
      }
      if (a.qsw)
        *reinterpret_cast<__nv_bfloat162*>(tile + bb * WP + cl) = __floats2bfloat162_rn(v[0], v[1]);
    }
  if (!a.qsw) return;
  __syncthreads();
  // 16-byte chunk j (columns 8j..8j+7) of a batch row lands at chunk
  // j ^ (h & 7) of row h of the 128-byte swizzle row; the padding heads'
  // rows (after the last head) are zero
  const size_t cblock = (size_t)(c0 / 64) * a.hp * 128;
  for (int idx = tid; idx < kTcRows * 8; idx += 256) {
    const int bb = idx >> 3, j = idx & 7;
    if (bb >= nb) continue;
    unsigned char* rowp = a.qsw + qsw_block(a, rq, b0 + bb) + cblock;
    st_chk(reinterpret_cast<uint4*>(rowp + h * 128 + ((j ^ (h & 7)) << 4)),
           *reinterpret_cast<const uint4*>(tile + bb * WP + 8 * j), a.ws_span, a.status);
    if (h == a.H - 1)
      for (int hz = a.H; hz < a.hp; ++hz)
        st_chk(reinterpret_cast<uint4*>(rowp + hz * 128 + (j << 4)), make_uint4(0u, 0u, 0u, 0u),
               a.ws_span, a.status);
  }
}

// One CTA per (head h, 32 output channels, 64 batch rows): the merge of
// k_combine (same record map, same order of operations), with ubar written
// split into shared memory, then out = W^V ubar with M = channels, N = batch
// rows, K = r_v. Warp w computes channels 16*(w%2).. for rows 16*(w/2)...
//
// Shared-memory work is spread so that every index is a warp or lane
// number, not a quotient: warp w stages W^V rows w, w+8, .. and merges
// batch rows w, w+8, .. (a row's record offset, piece count, maximum and
// normaliser are the same for the whole warp), lane l taking the float4
// columns l, l+32, .. of each. Both tiles are [row][k] bf16 hi/lo arrays
// read with ldmatrix.
__global__ void __launch_bounds__(256, 2) k_combine_tc(CombineArgs a) {
  extern __shared__ __align__(16) unsigned char sm_cmb_tc[];
  __shared__ int s_np[kTcRows];
  __shared__ long long s_off[kTcRows];
  __shared__ float s_M[kTcRows], s_inv[kTcRows], s_keep[kTcRows], s_mu[kTcCh];
  const int kp = (a.r_v + 15) & ~15;
  const int pitch = kp + 8;
  __nv_bfloat16* d_hi = reinterpret_cast<__nv_bfloat16*>(sm_cmb_tc);  // [32 channels][pitch]
  __nv_bfloat16* d_lo = d_hi + kTcCh * pitch;
  __nv_bfloat16* u_hi = d_lo + kTcCh * pitch;                          // [64 rows][pitch]
  __nv_bfloat16* u_lo = u_hi + kTcRows * pitch;
  const int h = blockIdx.x;
  const int i0 = blockIdx.y * kTcCh;
  const int b0 = blockIdx.z * kTcRows;
  const int nb = min(kTcRows, a.B - b0);
  const int ni = min(kTcCh, a.d_h - i0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r4 = a.r_v / 4, k4 = kp / 4;
  // decoder slice, 64 float4 columns of 4 rows per warp in flight; channels
  // past d_h and columns past r_v are zero
  const float* D = a.dv + ((size_t)h * a.d_h + i0) * a.r_v;
  for (int cb = 0; cb < k4; cb += 64) {
    float4 v[4][2];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int i = warp + 8 * k, j = cb + lane + 32 * cc;
        v[k][cc] = (i < ni && j < r4)
                       ? __ldg(reinterpret_cast<const float4*>(D + (size_t)i * a.r_v) + j)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int i = warp + 8 * k, j = cb + lane + 32 * cc;
        if (j < k4) store_split4(d_hi + i * pitch + 4 * j, d_lo + i * pitch + 4 * j, v[k][cc]);
      }
  }
  if (threadIdx.x < kTcCh)
    s_mu[threadIdx.x] = (a.mu_v && (int)threadIdx.x < ni) ? __ldg(a.mu_v + (size_t)h * a.d_h + i0 + threadIdx.x) : 0.f;
  pdl_wait();  // partials come from the streaming kernel

  // 1. per row: its records, merged maximum and normaliser
  merge_rows(a, h, b0, nb, kTcRows, s_np, s_off, s_M, s_inv, s_keep);
  __syncthreads();

  // 2. ubar rows, split into shared memory: warp w takes rows w + 8k, four
  //    at a time with all their piece loads in flight; rows with no piece
  //    and the padding columns come out 0
  const long long rstride = a.shared ? (long long)a.H * a.pstride : a.pstride;
  for (int cb = 0; cb < k4; cb += 64)
    for (int k0 = 0; k0 < kTcRows / 8; k0 += 4) {
      float4 acc[4][2];
      int np[4];
      int npmax = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        np[k] = s_np[warp + 8 * (k0 + k)];
        npmax = max(npmax, np[k]);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) acc[k][cc] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      for (int p = 0; p < npmax; ++p) {
        float mv[4];
        float4 uv[4][2];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int bb = warp + 8 * (k0 + k);
          const float* rec = a.part + s_off[bb] + p * rstride;
          mv[k] = p < np[k] ? ld_chk(rec, a.ws_span, a.status, kNegBig) : kNegBig;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int j = cb + lane + 32 * cc;
            uv[k][cc] = (p < np[k] && j < r4)
                            ? ld_chk(reinterpret_cast<const float4*>(rec + 4) + j, a.ws_span,
                                     a.status, make_float4(0.f, 0.f, 0.f, 0.f))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (p < np[k]) {
            const float wk = exp2f(mv[k] - s_M[warp + 8 * (k0 + k)]);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              acc[k][cc].x = fmaf(wk, uv[k][cc].x, acc[k][cc].x);
              acc[k][cc].y = fmaf(wk, uv[k][cc].y, acc[k][cc].y);
              acc[k][cc].z = fmaf(wk, uv[k][cc].z, acc[k][cc].z);
              acc[k][cc].w = fmaf(wk, uv[k][cc].w, acc[k][cc].w);
            }
          }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int bb = warp + 8 * (k0 + k);
        const float inv = s_inv[bb];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int j = cb + lane + 32 * cc;
          if (j < k4)
            store_split4(u_hi + bb * pitch + 4 * j, u_lo + bb * pitch + 4 * j,
                         make_float4(acc[k][cc].x * inv, acc[k][cc].y * inv, acc[k][cc].z * inv,
                                     acc[k][cc].w * inv));
        }
      }
    }
  __syncthreads();

  // 3. out tile = W^V slice (32 x kp) . ubar^T (kp x 64)
  const int m0 = (warp & 1) * 16, n0 = (warp >> 1) * 16;
  float acc[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  if (m0 < ni && n0 < nb) {
    const __nv_bfloat16* pa = d_hi + (m0 + (lane & 15)) * pitch + (lane >> 4) * 8;
    const __nv_bfloat16* pb =
        u_hi + (n0 + (lane & 7) + ((lane >> 4) << 3)) * pitch + ((lane >> 3) & 1) * 8;
    const int lo_a = kTcCh * pitch, lo_b = kTcRows * pitch;
    for (int k0 = 0; k0 < kp; k0 += 16) {
      uint32_t ah[4], al[4], bh[4], bl[4];
      ldsm_x4(ah, pa + k0);
      ldsm_x4(al, pa + lo_a + k0);
      ldsm_x4(bh, pb + k0);
      ldsm_x4(bl, pb + lo_b + k0);
      mma_split2(acc[0], acc[1], ah, al, bh, bl);
    }
  }
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int il = m0 + g + (e >> 1) * 8;
      const int bb = n0 + 8 * nt + 2 * t + (e & 1);
      if (il >= ni || bb >= nb) continue;
      st_chk(&a.out[((size_t)(b0 + bb) * a.H + h) * a.d_h + i0 + il],
             acc[nt][e] + s_mu[il] * s_keep[bb], a.out_span, a.status);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

int env_int(const char* name, int dflt) {
  const char* v = std::getenv(name);
  if (!v || !*v) return dflt;
  return std::atoi(v);
}

lla_status launch_absorb(const float* q, const float* dk, const float* mu_k, int B, int H,
                         int d_h, int r_k, float scale, float* qp, float* c0, cudaStream_t stream,
                         unsigned char* qsw, int hp, const float* q_rope, int d_r, bool tc,
                         Span ws) {
  AbsorbArgs a{q, dk, mu_k, B, H, d_h, r_k, scale * kLog2e, scale, qp, c0, qsw, hp,
               q_rope, q_rope ? d_r : 0, ws, status_word()};
  const int rq = r_k + a.d_r;
  // the tensor-core form stages d_h of 64 or 128 with float4 loads of q and
  // W^K (16-byte aligned, r_k a multiple of 8)
  if (tc && (d_h == 64 || d_h == 128) && r_k % 8 == 0 &&
      ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(dk)) & 15) == 0) {
    const size_t smem = absorb_tc_smem(d_h);
    auto kern = d_h == 128 ? k_absorb_tc<128> : k_absorb_tc<64>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_absorb_tc)");
    dim3 grid(H, (rq + kTcCols - 1) / kTcCols, (B + kTcRows - 1) / kTcRows);
    kern<<<grid, 256, smem, stream>>>(a);
    return check_cuda(cudaGetLastError(), "launch k_absorb_tc");
  }
  int rows, cols;
  pick_block(H, rq, B, &rows, &cols, false, env_int("LLA_ABSORB_MAX_COLS", 2));
  dim3 grid(H, (rq + 32 * cols - 1) / (32 * cols), (B + 8 * rows - 1) / (8 * rows));
  const int d_h4 = (d_h + 3) & ~3;
  const size_t smem = ((size_t)d_h4 * 32 * cols + (size_t)8 * rows * d_h4) * sizeof(float);
  using Fn = void (*)(AbsorbArgs);
  const Fn fns[4][3] = {{k_absorb<1, 1>, k_absorb<1, 2>, k_absorb<1, 4>},
                        {k_absorb<2, 1>, k_absorb<2, 2>, k_absorb<2, 4>},
                        {k_absorb<4, 1>, k_absorb<4, 2>, k_absorb<4, 4>},
                        {k_absorb<8, 1>, k_absorb<8, 2>, k_absorb<8, 4>}};
  const Fn fn = fns[rows == 8 ? 3 : rows == 4 ? 2 : rows == 2 ? 1 : 0][cols == 4 ? 2 : cols == 2 ? 1 : 0];
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_absorb)");
  fn<<<grid, 256, smem, stream>>>(a);
  return check_cuda(cudaGetLastError(), "launch k_absorb");
}

lla_status launch_combine(const float* part, int pstride, const float* c0, const float* dv,
                          const float* mu_v, int B, int H, int d_h, int r_v, long long N,
                          long long P, int shared, float* out, float* lse, cudaStream_t stream,
                          const RaggedMap* ragged, bool tc, Span ws) {
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  CombineArgs a{part, pstride, c0, dv, mu_v, B, H, d_h, r_v, N, P, shared, out, lse,
                RaggedMap{nullptr, nullptr, nullptr, 0ull}, status_word(), ws,
                span_of(out, (unsigned long long)B * H * d_h * sizeof(float)),
                lse ? span_of(lse, (unsigned long long)B * H * sizeof(float)) : Span{}};
  if (ragged) a.ragged = *ragged;
  if (tc) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(H, (d_h + kTcCh - 1) / kTcCh, (B + kTcRows - 1) / kTcRows);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = combine_tc_smem(r_v);
    cudaError_t e = cudaFuncSetAttribute(k_combine_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)cfg.dynamicSmemBytes);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_combine_tc)");
    cfg.stream = stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return check_cuda(cudaLaunchKernelEx(&cfg, k_combine_tc, a), "launch k_combine_tc");
  }
  int rows, cols;
  // Up to four 32-channel column blocks per CTA: at large batches fewer CTAs
  // merge each row's records once for more channels (768 -> 384 CTAs at
  // B = 768); below that the CTA-count floor keeps one or two.
  pick_block(H, d_h, B, &rows, &cols, true, env_int("LLA_COMBINE_MAX_COLS", 4));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(H, (d_h + 32 * cols - 1) / (32 * cols), (B + 8 * rows - 1) / (8 * rows));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = ((size_t)32 * cols * (r_v + 4) + (size_t)8 * rows * r_v) * sizeof(float);
  using Fn = void (*)(CombineArgs);
  const Fn fns[4][3] = {{k_combine<1, 1>, k_combine<1, 2>, k_combine<1, 4>},
                        {k_combine<2, 1>, k_combine<2, 2>, k_combine<2, 4>},
                        {k_combine<4, 1>, k_combine<4, 2>, k_combine<4, 4>},
                        {k_combine<8, 1>, k_combine<8, 2>, k_combine<8, 4>}};
  const Fn fn = fns[rows == 8 ? 3 : rows == 4 ? 2 : rows == 2 ? 1 : 0][cols == 4 ? 2 : cols == 2 ? 1 : 0];
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)cfg.dynamicSmemBytes);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_combine)");
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return check_cuda(cudaLaunchKernelEx(&cfg, fn, a), "launch k_combine");
}

// Per-head decode takes the tensor-core combine for bf16 latents, large
// batches and wide ranks only, and the tensor-core absorb (its second form,
// staged by lane and warp numbers) for bf16 latents and large batches at any
// rank. Both forms are bound by memory round trips and instruction issue at
// these sizes. Measured on B200 (whole decode steps, same box): the first
// tensor-core forms lost to the CUDA-core ones at B = 64, r = 128 and at
// B = 768, r = 24; the second absorb wins at B = 768, r = 24 (70.43 ->
// 70.17 ms per step, three runs each), and the LLA-2D shape (B = 256,
// r = 256) gains on both.
bool small_gemm_tc(int esz, int B, int r_k, int r_v) {
  return esz == 2 && B >= 256 && std::max(r_k, r_v) >= 192;
}

bool absorb_tc(int esz, int B) { return esz == 2 && B >= 256; }

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
  // Rows of at most two segments (r <= 16 bf16): one lane per token. The
  // score's lane reduction would cost more than the 2-way bank conflict it
  // avoids (measured at r = 16, B = 32, N = 32768: 178 -> 164 us).
  if (d.nseg_k <= 2 && d.nseg_v <= 2) lpt = 1;
  // tuning override (power of two dividing both segment counts)
  const int lpt_env = env_int("LLA_DECODE_LPT", 0);
  if (lpt_env == 1 || lpt_env == 2 || lpt_env == 4 || lpt_env == 8)
    if (d.nseg_k % lpt_env == 0 && d.nseg_v % lpt_env == 0) lpt = lpt_env;
  // An exact kernel (every lane's segments in range) when one exists for
  // the two per-lane counts; else the fewest lanes whose masked counts fit
  // in 4, with a masked kernel sized to them, or the generic 4 / 4 one.
  if (d.nseg_k % lpt == 0 && d.nseg_v % lpt == 0 &&
      pick_stream_kernel(esz, lpt, d.nseg_k / lpt, d.nseg_v / lpt, true)) {
    d.exact = true;
    d.sk = d.nseg_k / lpt;
    d.sv = d.nseg_v / lpt;
  } else {
    auto fits = [&](int l) { return (d.nseg_k + l - 1) / l <= 4 && (d.nseg_v + l - 1) / l <= 4; };
    while (lpt < 8 && !fits(lpt)) lpt *= 2;
    if (!fits(lpt)) return fail(LLA_ERR_UNSUPPORTED, "latent rank too large for the decode kernel");
    d.exact = false;
    d.sk = (d.nseg_k + lpt - 1) / lpt;
    d.sv = (d.nseg_v + lpt - 1) / lpt;
    if (!pick_stream_kernel(esz, lpt, d.sk, d.sv, false)) d.sk = d.sv = 4;
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
  // per warp and stage: an 8-byte mbarrier and a 4-byte tile length (the
  // paged kernel's producer hands each tile's length to its consumer)
  auto smem_of = [&](int tile, int nst) {
    return (size_t)((d.warps * nst * 12 + 127) & ~127) + (size_t)d.warps * nst * tile * tok_bytes;
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
                      float* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream,
                      const float* q_rope, int d_r) {
  if (!q_rope) d_r = 0;
  const int rq = r_k + d_r;  // key row: latent, then the rotated rotary key
  DecodePlan d;
  lla_status st = plan_decode(B, H, N, rq, r_v, esz, &d);
  if (st != LLA_OK) return st;
  if (ws == nullptr || ws_bytes < d.ws_bytes)
    return fail(LLA_ERR_WORKSPACE, "decode workspace needs %zu bytes, got %zu", d.ws_bytes,
                ws_bytes);
  char* wsb = static_cast<char*>(ws);
  float* qp = reinterpret_cast<float*>(wsb + d.off_qp);
  float* c0 = reinterpret_cast<float*>(wsb + d.off_c0);
  float* part = reinterpret_cast<float*>(wsb + d.off_part);

  StreamFn fn = pick_stream_kernel(esz, d.lpt, d.sk, d.sv, d.exact);
  if (!fn) return fail(LLA_ERR_UNSUPPORTED, "no decode kernel for this latent shape");

  cudaError_t e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)d.smem_bytes);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_stream)");

  // 1. absorb
  st = launch_absorb(q, dk, mu_k, B, H, d_h, r_k, scale, qp, c0, stream, nullptr, 0, q_rope, d_r,
                     absorb_tc(esz, B), span_of(ws, ws_bytes));
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
    a.row_k = rq * esz;
    a.row_v = r_v * esz;
    a.nseg_k = d.nseg_k;
    a.nseg_v = d.nseg_v;
    a.r_k = rq;
    a.tile = d.tile;
    a.nstage = d.nstage;
    a.stage_bytes = d.stage_bytes;
    a.qp = qp;
    a.part = part;
    a.pstride = d.pstride;
    a.status = status_word();
    a.zk_span = span_of(zk, (unsigned long long)B * H * n_cap * a.row_k);
    a.zv_span = span_of(zv, (unsigned long long)B * H * n_cap * a.row_v);
    a.ws_span = span_of(ws, ws_bytes);
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
  return launch_combine(part, d.pstride, c0, dv, mu_v, B, H, d_h, r_v, N, d.P, 0, out, lse, stream,
                        nullptr, small_gemm_tc(esz, B, r_k, r_v), span_of(ws, ws_bytes));
  return LLA_OK;
}

}  // namespace lla

// Latent write (LLA encoder) on the sm_100a tensor cores.
//
// Source: "Looped Latent Attention: Cross-Loop KV Compression for Looped
// Transformers" (arXiv 2607.15456), §3 "Teacher cache" Eq. 1 (loop-major
// stacking of the T per-loop vectors) and §3 "Cross-loop codec" Eq. 2
// (c = (x - mu) W_down).
//
// Per group g this is the GEMM Z_g[N x r] = X_g[N x T*d_loop] W_g - mu_g W_g.
// X_g is never stacked in memory: the loop-major input x[T][N][G][d_loop] is
// read through a 4-D TMA tensor map, and the contraction index k = t*d_loop+i
// is walked as (t, 64-wide chunk) pairs, so each K chunk is one 128-token x
// 64-channel box of one loop.
//
// Kernel layout (persistent, one CTA per SM, warp-specialised):
//   warp 0      TMA producer: A box (128 tokens x 64 k, 128B swizzle) and
//               the matching B box (r rows of W^T x 64 k) per pipeline stage.
//   warp 1      allocates TMEM, issues tcgen05.mma (M=128, N=r padded to 16,
//               K=16 per instruction) into one of two TMEM accumulators, and
//               commits stage releases and accumulator hand-offs.
//   warps 2-5   epilogue: tcgen05.ld of the 128 x r accumulator (one TMEM
//               lane per token), subtract mu W, round to bf16 (RNE), store
//               with the caller's row and group strides, or at each token's
//               slot of a paged store (its page from the block table).
//               Double-buffered
//               accumulators let the epilogue of tile i overlap the MMAs of
//               tile i+1.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "tc.cuh"

namespace lla {
namespace {

constexpr int kTileM = 128;     // tokens per tile (TMEM lanes)
constexpr int kChunkK = 64;     // K elements per stage (128 B rows)
constexpr int kABytes = kTileM * kChunkK * 2;
constexpr int kThreads = 192;   // 6 warps
constexpr int kMaxStages = 12;  // enough bytes in flight to cover HBM latency at r = 16

// Where each token's output row goes. Dense: row n of group g starts at
// element g * zgs + n * zrs. Paged: token n belongs to sequence seq[n] (n
// when seq is null) at position pos[n], and its row is row pos % page_size
// of page block_table[s][pos / page_size], starting at element
// page * page_stride + g * zgs + (pos % page_size) * zrs.
struct OutMap {
  __nv_bfloat16* z;
  long long zrs, zgs;
  int paged;
  PagedOut pd;
  Span z_span;  // every row the map can address (bounds-check build)
};

// Element offset of token n's row (group 0), or -1 when a paged destination
// is out of range: its sequence index, position or page lies outside the
// table or the pool. Such a row is not written.
__device__ __forceinline__ long long out_row(const OutMap& o, int n) {
  if (!o.paged) return (long long)n * o.zrs;
  const int s = o.pd.seq ? __ldg(o.pd.seq + n) : n;
  const int p = __ldg(o.pd.pos + n);
  // page_size * max_blocks < 2^31 is checked on the host
  if (s < 0 || s >= o.pd.n_seq || p < 0 || p >= o.pd.max_blocks * o.pd.page_size) return -1;
  const int page = __ldg(o.pd.block_table + (size_t)s * o.pd.max_blocks + p / o.pd.page_size);
  if (page < 0 || page >= o.pd.num_pages) return -1;
  return (long long)page * o.pd.page_stride + (long long)(p % o.pd.page_size) * o.zrs;
}

struct EncodeArgs {
  // work items are (tile, K split) pairs: item = tile * ksplit + split
  int N, G, d_loop, r, r_pad, K, nk, mtiles, tiles, tiles_per_cta;
  // a tile is msub sub-tiles of 128 tokens that share each stage's W^T box
  // (one accumulator each); nacc tiles' accumulators fit in TMEM at once
  int msub, nacc;
  int ksplit, cpk;  // K splits per tile and chunks per split
  // tile order: token-major (all groups of a 128-token tile in a row, so a
  // token's G * d_loop input row is read at once) or group-major (one
  // group's tiles in a row, so the in-kernel mean term changes rarely)
  int token_major;
  float* part;      // ksplit > 1: fp32 partials [ksplit][G][N][r]
  Span ws_span;     // the workspace holding them (bounds-check build)
  int nstage, b_bytes, stage_bytes;
  uint32_t tmem_cols;
  const float* mu;
  const float* muw;  // precomputed mu W [G][r] (then mu is unused), or null
  const __nv_bfloat16* wt;
  OutMap out;
  unsigned int* status;
};

struct SmemTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t epi;  // 4-warp rendezvous of the epilogue warps
  uint32_t tmem_base;
  int abort_flag;
  float muw[256];
};

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
      *abort_flag = 1;
      report_status(status, kStatusWaitTimeout);
      return false;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    k_encode(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
             EncodeArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the 128B-swizzle atoms
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemTail* tail = reinterpret_cast<SmemTail*>(smem + (size_t)a.nstage * a.stage_bytes);
  volatile int* abort_flag = &tail->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = blockIdx.x * a.tiles_per_cta;  // work items, see EncodeArgs
  const int t_end = min(t_begin + a.tiles_per_cta, a.tiles * a.ksplit);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.nstage; ++s) {
      mbar_init(smem_u32(&tail->full[s]), 1);
      mbar_init(smem_u32(&tail->empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tail->tfull[i]), 1);
      mbar_init(smem_u32(&tail->tempty[i]), 4);
    }
    mbar_init(smem_u32(&tail->drain), 1);
    mbar_init(smem_u32(&tail->epi), 4);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tail->tmem_base), a.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tail->tmem_base;
  const int cpl = a.d_loop / kChunkK;  // chunks per loop

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_x = l2_evict_first_policy();
      const uint64_t pol_w = l2_evict_last_policy();
      int it = 0;
      bool ok = true;
      for (int item = t_begin; item < t_end && ok; ++item) {
        const int tile = item / a.ksplit, split = item - tile * a.ksplit;
        const int g = a.token_major ? tile % a.G : tile / a.mtiles;
        const int m0 = (a.token_major ? tile / a.G : tile - g * a.mtiles) * kTileM * a.msub;
        const int kc0 = split * a.cpk, kc1 = min(a.nk, kc0 + a.cpk);
        for (int kc = kc0; kc < kc1; ++kc, ++it) {
          const int s = it % a.nstage;
          const uint32_t ph = (uint32_t)(it / a.nstage) & 1u;
          if (!wait_or_abort(smem_u32(&tail->empty[s]), ph ^ 1u, abort_flag, a.status)) {
            ok = false;
            break;
          }
          const uint32_t full = smem_u32(&tail->full[s]);
          mbar_arrive_expect_tx(full, a.msub * kABytes + a.b_bytes);
          const uint32_t sa = smem_u32(smem + (size_t)s * a.stage_bytes);
          const int t = kc / cpl, i0 = (kc - t * cpl) * kChunkK;
          // rows past N (a sub-tile beyond the last token) read as zeros
          for (int sub = 0; sub < a.msub; ++sub)
            tma_load_4d(sa + sub * kABytes, &tx, i0, g, m0 + sub * kTileM, t, full, pol_x);
          tma_load_3d(sa + a.msub * kABytes, &tw, kc * kChunkK, 0, g, full, pol_w);
        }
      }
      if (!ok) {
        // let copies already issued land before the CTA can exit
        const int first = max(0, it - a.nstage);
        for (int i = first; i < it; ++i)
          (void)mbar_wait(smem_u32(&tail->full[i % a.nstage]), (uint32_t)(i / a.nstage) & 1u,
                          kWaitTimeoutNs / 8);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileM, a.r_pad, false, false);
      int it = 0;
      bool ok = true;
      for (int item = t_begin, lt = 0; item < t_end && ok; ++item, ++lt) {
        const int acc = lt % a.nacc;
        const uint32_t aph = (uint32_t)(lt / a.nacc) & 1u;
        if (!wait_or_abort(smem_u32(&tail->tempty[acc]), aph ^ 1u, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tbase + (uint32_t)(acc * a.msub * a.r_pad);
        const int split = item % a.ksplit;
        const int kc0 = split * a.cpk, kc1 = min(a.nk, kc0 + a.cpk);
        for (int kc = kc0; kc < kc1; ++kc, ++it) {
          const int s = it % a.nstage;
          const uint32_t ph = (uint32_t)(it / a.nstage) & 1u;
          if (!wait_or_abort(smem_u32(&tail->full[s]), ph, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + (size_t)s * a.stage_bytes);
          // descriptors built once per stage, advanced 32 B (2 x 16 B) per K
          // step; every sub-tile multiplies the stage's one W^T box
          const uint64_t b_base = desc_kmajor_sw128(sa + a.msub * kABytes);
          for (int sub = 0; sub < a.msub; ++sub) {
            const uint64_t a_base = desc_kmajor_sw128(sa + sub * kABytes);
#pragma unroll
            for (int kk = 0; kk < kChunkK / 16; ++kk)
              umma_bf16(d + (uint32_t)(sub * a.r_pad), a_base + (uint64_t)(kk * 2),
                        b_base + (uint64_t)(kk * 2), idesc, kc != kc0 || kk != 0);
          }
          umma_commit(smem_u32(&tail->empty[s]));
        }
        if (!ok) break;
        umma_commit(smem_u32(&tail->tfull[acc]));
      }
      // all issued MMAs complete before TMEM can be released
      umma_commit(smem_u32(&tail->drain));
      (void)mbar_wait(smem_u32(&tail->drain), 0u, kWaitTimeoutNs / 8);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    uint32_t epi_phase = 0;
    // bounded rendezvous of the 4 epilogue warps (an mbarrier, so a warp
    // that aborts cannot leave the others waiting forever)
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tail->epi));
      const bool ok = __all_sync(
          0xffffffffu, wait_or_abort(smem_u32(&tail->epi), epi_phase & 1u, abort_flag, a.status));
      ++epi_phase;
      return ok;
    };
    int cur_g = -1;
    for (int item = t_begin, lt = 0; item < t_end; ++item, ++lt) {
      const int tile = item / a.ksplit, split = item - tile * a.ksplit;
      const int g = a.token_major ? tile % a.G : tile / a.mtiles;
      const int m0 = (a.token_major ? tile / a.G : tile - g * a.mtiles) * kTileM * a.msub;
      if (g != cur_g && !a.part) {
        if (!epi_sync()) break;  // previous tile's readers of muw are done
        for (int c = ew; c < a.r; c += 4) {
          float acc = 0.f;
          if (a.muw) {
            acc = a.muw[(size_t)g * a.r + c];
          } else if (a.mu) {
            const float* mu = a.mu + (size_t)g * a.K;
            const __nv_bfloat16* w = a.wt + ((size_t)g * a.r + c) * a.K;
            for (int k = lane; k < a.K; k += 32) acc = fmaf(mu[k], __bfloat162float(w[k]), acc);
            acc = warp_sum(acc);
          }
          if (lane == 0) tail->muw[c] = acc;
        }
        if (!epi_sync()) break;
        cur_g = g;
      }
      const int acc = lt % a.nacc;
      const uint32_t aph = (uint32_t)(lt / a.nacc) & 1u;
      const bool ok = __all_sync(0xffffffffu, wait_or_abort(smem_u32(&tail->tfull[acc]), aph,
                                                            abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      for (int sub = 0; sub < a.msub; ++sub) {
        const uint32_t taddr = tbase + ((uint32_t)(quarter * 32) << 16) +
                               (uint32_t)((acc * a.msub + sub) * a.r_pad);
        const int n = m0 + sub * kTileM + row;
        long long roff = 0;
        bool write = n < a.N;
        if (write && !a.part) {
          roff = out_row(a.out, n);
          if (roff < 0) {
            write = false;
            if (g == 0) report_status(a.status, kStatusBadPagedInput);
          }
        }
        __nv_bfloat16* zrow = a.out.z + (size_t)g * a.out.zgs + roff;
        // split K: this item's fp32 partial sum; k_encode_reduce finishes it
        float* prow = a.part ? a.part + (((size_t)split * a.G + g) * a.N + n) * a.r : nullptr;
        for (int cc = 0; cc < a.r_pad; cc += 16) {
          float v[16];
          tmem_ld16(taddr + cc, v);
          if (n < a.N && prow) {
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
              const int c0 = cc + 8 * h8;
              if (c0 < a.r) {
                float4* dst = reinterpret_cast<float4*>(prow + c0);
                if (in_span(a.ws_span, dst, 32, a.status)) {
                  dst[0] = make_float4(v[8 * h8 + 0], v[8 * h8 + 1], v[8 * h8 + 2], v[8 * h8 + 3]);
                  dst[1] = make_float4(v[8 * h8 + 4], v[8 * h8 + 5], v[8 * h8 + 6], v[8 * h8 + 7]);
                }
              }
            }
          } else if (write) {
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
              const int c0 = cc + 8 * h8;
              if (c0 < a.r) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const __nv_bfloat162 p = __floats2bfloat162_rn(
                      v[8 * h8 + 2 * e] - tail->muw[c0 + 2 * e],
                      v[8 * h8 + 2 * e + 1] - tail->muw[c0 + 2 * e + 1]);
                  w[e] = *reinterpret_cast<const uint32_t*>(&p);
                }
                st_chk(reinterpret_cast<uint4*>(zrow + c0), make_uint4(w[0], w[1], w[2], w[3]),
                       a.out.z_span, a.status);
              }
            }
          }
        }
      }  // sub-tiles
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tail->tempty[acc]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, a.tmem_cols);
  }
}

using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeTiledFn get_encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// muw[g][c] = sum_k mu[g][k] W_down[g][k][c] (fp32): one warp per (g, c),
// 16-byte loads of W^T, eight in flight per lane.
__global__ void __launch_bounds__(256) k_encode_bias(const __nv_bfloat16* wt, const float* mu,
                                                     int G, int K, int r, float* muw) {
  const int g = blockIdx.x;
  const int c = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= r) return;
  const uint4* w = reinterpret_cast<const uint4*>(wt + ((size_t)g * r + c) * K);
  const float4* m = reinterpret_cast<const float4*>(mu + (size_t)g * K);
  const int n8 = K / 8;
  float acc = 0.f;
  for (int i0 = lane; i0 < n8; i0 += 32 * 8) {
    uint4 wv[8];
    float4 m0[8], m1[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = i0 + 32 * k;
      if (i < n8) {
        wv[k] = __ldg(w + i);
        m0[k] = __ldg(m + 2 * i);
        m1[k] = __ldg(m + 2 * i + 1);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (i0 + 32 * k < n8) {
        acc = fmaf(m0[k].x, bf16lo(wv[k].x), acc);
        acc = fmaf(m0[k].y, bf16hi(wv[k].x), acc);
        acc = fmaf(m0[k].z, bf16lo(wv[k].y), acc);
        acc = fmaf(m0[k].w, bf16hi(wv[k].y), acc);
        acc = fmaf(m1[k].x, bf16lo(wv[k].z), acc);
        acc = fmaf(m1[k].y, bf16hi(wv[k].z), acc);
        acc = fmaf(m1[k].z, bf16lo(wv[k].w), acc);
        acc = fmaf(m1[k].w, bf16hi(wv[k].w), acc);
      }
    }
  }
  acc = warp_sum(acc);
  if (lane == 0) muw[(size_t)g * r + c] = acc;
}

// Finishes a split-K encode: z[g][n][c..c+4) = bf16_rne(sum over splits of
// the fp32 partials - muw[g][c..c+4)), one thread per 4 outputs with eight
// partial loads in flight.
__global__ void __launch_bounds__(256) k_encode_reduce(const float* part, const float* muw,
                                                       int ksplit, int G, int N, int r,
                                                       OutMap out, unsigned int* status,
                                                       Span ws_span) {
  const int r4 = r / 4;
  const long long total = (long long)G * N * r4;
  const size_t plane4 = (size_t)G * N * r / 4;  // float4 per split
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < total; i += (long long)gridDim.x * 256) {
    const int c = (int)(i % r4) * 4;
    const long long gn = i / r4;
    const int n = (int)(gn % N), g = (int)(gn / N);
    const long long roff = out_row(out, n);
    if (roff < 0) {
      if (g == 0 && c == 0) report_status(status, kStatusBadPagedInput);
      continue;
    }
    const float4* p = reinterpret_cast<const float4*>(part) + (size_t)i;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < ksplit; k0 += 8) {
      float4 v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        v[k] = k0 + k < ksplit ? ld_chk(p + (size_t)(k0 + k) * plane4, ws_span, status,
                                        make_float4(0.f, 0.f, 0.f, 0.f))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        s.x += v[k].x;
        s.y += v[k].y;
        s.z += v[k].z;
        s.w += v[k].w;
      }
    }
    if (muw) {
      const float4 m = __ldg(reinterpret_cast<const float4*>(muw + (size_t)g * r + c));
      s.x -= m.x;
      s.y -= m.y;
      s.z -= m.z;
      s.w -= m.w;
    }
    const __nv_bfloat162 b0 = __floats2bfloat162_rn(s.x, s.y), b1 = __floats2bfloat162_rn(s.z, s.w);
    st_chk(reinterpret_cast<uint2*>(out.z + (size_t)g * out.zgs + roff + c),
           make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1)),
           out.z_span, status);
  }
}

}  // namespace

bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) {
    fail(LLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t gd[5];
  cuuint64_t gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                  gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(LLA_ERR_INVALID_ARG, "tensor map rejected by the driver (CUresult %d)", (int)r);
    return false;
  }
  return true;
}

lla_status run_encode_bias(const void* wt, const float* mu, int G, int K, int r, float* muw,
                           cudaStream_t stream) {
  k_encode_bias<<<dim3(G, (r + 7) / 8), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(wt),
                                                          mu, G, K, r, muw);
  return check_cuda(cudaGetLastError(), "launch k_encode_bias");
}

int encode_ksplit(int T, int N, int G, int d_loop) {
  const int tiles = (N + kTileM - 1) / kTileM * G;
  const int nk = T * d_loop / kChunkK;
  const int sms = device_info().sms;
  if (2 * tiles > sms) return 1;
  // at most 16 splits: beyond that the partial traffic and the final sum
  // cost more than the idle SMs they would fill
  const int S = std::min(std::min(nk / 2, sms / tiles), 16);
  if (S < 2) return 1;
  const int cpk = (nk + S - 1) / S;
  return (nk + cpk - 1) / cpk;
}

size_t encode_workspace(int T, int N, int G, int d_loop, int r) {
  const int S = encode_ksplit(T, N, G, d_loop);
  return S > 1 ? (size_t)S * G * N * r * sizeof(float) : 0;
}

lla_status run_encode(const void* x, int T, int N, int G, int d_loop, int r, const void* wt,
                      const float* mu, void* z, long long zrs, long long zgs,
                      cudaStream_t stream, const float* muw, void* ws, size_t ws_bytes,
                      const PagedOut* paged) {
  const int K = T * d_loop;
  const int r_pad = (r + 15) / 16 * 16;
  EncodeArgs a{};
  a.N = N;
  a.G = G;
  a.d_loop = d_loop;
  a.r = r;
  a.r_pad = r_pad;
  a.K = K;
  a.nk = K / kChunkK;
  a.msub = 1;
  a.mtiles = (N + kTileM - 1) / kTileM;
  a.tiles = a.mtiles * G;
  // Few tiles and a long K (a wide LLA-2D stack at decode time) leave most
  // SMs idle: with a workspace, K is split so every SM gets work, and a
  // second kernel sums the fp32 partials.
  a.ksplit = 1;
  a.cpk = a.nk;
  a.part = nullptr;
  if (ws && !mu) {
    const int S = encode_ksplit(T, N, G, d_loop);
    if (S > 1 && ws_bytes >= (size_t)S * G * N * r * sizeof(float)) {
      a.ksplit = S;
      a.cpk = (a.nk + S - 1) / S;
      a.part = static_cast<float*>(ws);
    }
  }
  a.token_major = env_int("LLA_ENCODE_TOKEN_MAJOR", 0);
  a.b_bytes = r_pad * kChunkK * 2;
  // A wide W^T (r >= 128: its box is at least the 16 KB token box) is
  // re-read from L2 for every tile. Tiles of two 128-token sub-tiles read
  // each W^T box once for both, cutting the stage bytes per MMA by a third
  // at r = 256. Unsplit writes only: split-K partials stay per 128 rows.
  if (a.ksplit == 1 && r_pad >= 128 && N > kTileM)
    a.msub = std::max(1, std::min(2, env_int("LLA_ENCODE_MSUB", 2)));
  a.mtiles = (N + kTileM * a.msub - 1) / (kTileM * a.msub);
  a.tiles = a.mtiles * G;
  a.stage_bytes = a.msub * kABytes + a.b_bytes;
  // two tiles' accumulators when they fit in the 512 TMEM columns, so the
  // epilogue of one tile overlaps the next tile's MMAs
  a.nacc = 2 * a.msub * r_pad <= 512 ? 2 : 1;
  uint32_t cols = 32;
  while (cols < (uint32_t)(a.nacc * a.msub * r_pad)) cols <<= 1;
  a.tmem_cols = cols;
  a.mu = mu;
  a.muw = muw;
  a.wt = static_cast<const __nv_bfloat16*>(wt);
  a.out.z = static_cast<__nv_bfloat16*>(z);
  a.out.zrs = zrs;
  a.out.zgs = zgs;
  a.out.paged = paged != nullptr;
  if (paged) a.out.pd = *paged;
  // the last element any row can reach, in elements from z
  const unsigned long long zlast =
      paged ? (unsigned long long)(paged->num_pages - 1) * paged->page_stride +
                  (unsigned long long)(G - 1) * zgs + (unsigned long long)(paged->page_size - 1) * zrs + r
            : (unsigned long long)(G - 1) * zgs + (unsigned long long)(N - 1) * zrs + r;
  a.out.z_span = span_of(z, zlast * 2);
  a.ws_span = span_of(ws, ws_bytes);
  a.status = status_word();

  const DeviceInfo di = device_info();
  const size_t fixed = sizeof(SmemTail) + 1024;
  // CTAs per SM: several independent producer / MMA / epilogue pipelines
  // per SM stream faster than one (measured at r = 16: 104 us with one,
  // 91 us with three). Take the most, up to 3, that leave each CTA 4
  // stages, fit the SM's 512 TMEM columns and still have a tile each.
  const int items_all = a.tiles * a.ksplit;
  int per_sm = 1;
  for (int p = 3; p >= 2; --p) {
    const size_t per_cta = (size_t)di.smem_optin / p - 1024;
    if ((size_t)p * cols <= 512 && per_cta > fixed && (per_cta - fixed) / a.stage_bytes >= 4 &&
        items_all >= p * di.sms) {
      per_sm = p;
      break;
    }
  }
  per_sm = std::max(1, std::min(3, env_int("LLA_ENCODE_CTAS_PER_SM", per_sm)));
  const size_t smem_cta = (size_t)di.smem_optin / per_sm - (per_sm > 1 ? 1024 : 0);
  int nst = (int)std::min<size_t>(std::max(2, std::min(kMaxStages, env_int("LLA_ENCODE_STAGES", kMaxStages))),
                                  (smem_cta - fixed) / a.stage_bytes);
  if (nst < 2) return fail(LLA_ERR_UNSUPPORTED, "encode stage does not fit in shared memory");
  a.nstage = nst;
  const size_t smem = (size_t)nst * a.stage_bytes + fixed;
  const int items = a.tiles * a.ksplit;
  const int grid0 = std::min(items, di.sms * per_sm);
  a.tiles_per_cta = (items + grid0 - 1) / grid0;
  const int grid = (items + a.tiles_per_cta - 1) / a.tiles_per_cta;

  CUtensorMap tx, tw;
  {
    const uint64_t dims[4] = {(uint64_t)d_loop, (uint64_t)G, (uint64_t)N, (uint64_t)T};
    const uint64_t strides[3] = {(uint64_t)d_loop * 2, (uint64_t)G * d_loop * 2,
                                 (uint64_t)N * G * d_loop * 2};
    const uint32_t box[4] = {(uint32_t)kChunkK, 1, (uint32_t)kTileM, 1};
    if (!make_tmap_bf16(&tx, x, 4, dims, strides, box)) return LLA_ERR_INVALID_ARG;
  }
  {
    const uint64_t dims[3] = {(uint64_t)K, (uint64_t)r, (uint64_t)G};
    const uint64_t strides[2] = {(uint64_t)K * 2, (uint64_t)r * K * 2};
    const uint32_t box[3] = {(uint32_t)kChunkK, (uint32_t)r_pad, 1};
    if (!make_tmap_bf16(&tw, wt, 3, dims, strides, box)) return LLA_ERR_INVALID_ARG;
  }
  cudaError_t e = cudaFuncSetAttribute(k_encode, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_encode)");
  e = record_timing(true, stream);
  if (e != cudaSuccess) return check_cuda(e, "record timing event");
  k_encode<<<grid, kThreads, smem, stream>>>(tx, tw, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return check_cuda(e, "launch k_encode");
  if (a.part) {
    const long long outs = (long long)G * N * (r / 4);
    const int rgrid = (int)std::min<long long>((outs + 255) / 256, 4LL * di.sms);
    k_encode_reduce<<<rgrid, 256, 0, stream>>>(a.part, muw, a.ksplit, G, N, r, a.out, a.status,
                                               a.ws_span);
    e = cudaGetLastError();
    if (e != cudaSuccess) return check_cuda(e, "launch k_encode_reduce");
  }
  e = record_timing(false, stream);
  if (e != cudaSuccess) return check_cuda(e, "record timing event");
  return LLA_OK;
}

}  // namespace lla

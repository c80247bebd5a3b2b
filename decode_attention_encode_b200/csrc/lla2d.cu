// LLA-2D absorbed decode on the sm_100a tensor cores.
//
// Source: "Looped Latent Attention: Cross-Loop KV Compression for Looped
// Transformers" (arXiv 2607.15456), §3 "The LLA-2D variant" (one latent per
// token and layer, decoded into every head) and §7 "Per-head LLA versus
// LLA-2D at inference" (absorbed attention reads latents directly).
//
// Every head of a sequence reads the same latents, so the H absorbed queries
// against the shared latent store form real contractions (ranks that are
// not whole 64-column boxes or 128-row tiles are zero-padded by the tensor
// maps' out-of-range fill, which reads nothing from memory):
//   S  [128 tokens x H] = Z^K_tile [128 x r_k] . Q'^T [r_k x H]
//   U  [r_v x H]       += Z^V_tile^T [r_v x 128] . P [128 x H]
// Both run as tcgen05.mma kind::f16 (bf16 operands, fp32 accumulators in
// TMEM). The softmax over tokens sits between them on CUDA cores: one thread
// per token row reads its H scores from TMEM, keeps a per-head reference
// maximum that is raised only when a score passes it by 2^8 (a CTA vote, then
// a tile max and an in-TMEM rescale of U), and writes bf16 weights P into
// shared memory in the layout the second MMA reads.
//
// Work split: the (sequence, 128-token tile) space is cut into equal runs of
// whole tiles, one run per CTA of a one-wave grid. Each (CTA, sequence) piece
// ends in one partial record per head (m, l, U); k_combine merges them and
// applies W^V_up,t. k_absorb (shared with the per-head path) forms q'.
//
// CTA roles (8 warps):
//   warp 0     K producer: 128 x 128-column Z^K groups (two 64-column
//              128B-swizzled boxes, 32 KB) into the K ring; stages Q' (bf16,
//              swizzled K-major) for each new sequence.
//   warp 1     TMEM owner and score MMA issuer (up to one tile ahead of the
//              softmax, two S buffers).
//   warps 2-5  softmax and epilogue (one thread per TMEM lane).
//   warp 6     V producer: Z^V groups into the V ring.
//   warp 7     value MMA issuer.
// The MMAs here are small (N = H), so their issue cost, not the tensor pipe,
// sets their time: one thread issues one about every 60 cycles, two threads
// together one about every 40. Two issuers also decouple the rings: a V slot
// is released as soon as its tile's value MMA retires, whatever the K
// stream is doing, and a K slot as soon as its score MMA retires.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "tc.cuh"

namespace lla {
namespace {

constexpr int kRows = 128;
constexpr int kBoxBytes = kRows * 64 * 2;  // 16 KB: 128 rows x 64 bf16
constexpr int kStageBytes = 2 * kBoxBytes;
constexpr int kSubBytesV = kBoxBytes / 2;  // one 64-row half of a 64-column block
constexpr int kThreads = 256;
constexpr int kMaxStages = 4;  // per ring
constexpr float kNegBig = -1.0e30f;
constexpr float kSlack = 8.0f;
// Each contraction is split over independent TMEM accumulators whose MMAs
// are issued interleaved: with N = 16 a single accumulator serialises the
// small MMAs on its own read-modify-write. The partial sums are added when
// read back.
constexpr int kSAcc = 4;  // score accumulators per S buffer
constexpr int kUAcc = 2;  // value accumulators per r_v half

struct D2Args {
  int B, H, N, tps, tiles, tpc;
  int r_k, r_v, nkg, nvg, nks, nvs;  // groups per tile; stages per ring
  int off_q, off_p, off_tail, qbuf_bytes, pbuf_bytes;
  uint32_t tmem_cols;
  const unsigned char* qsw;  // per sequence: Q' as bf16 in the MMA operand layout
  // paged store (seqinfo non-null): written by k_plan_paged
  const int4* seqinfo;      // [B] {kept tiles, tokens, sink tiles, first window tile}
  const long long* plan;    // {total tiles, tiles per CTA, stamp}
  unsigned long long stamp; // plan[2] must equal it, else no tile is taken
  const int4* cstart;       // [grid] first (sequence, 0, tile) of each CTA
  const int* block_table;   // [B][max_blocks]
  int max_blocks, page_size;
  int sink, window;         // eviction set (window 0: every token)
  float* part;
  int pstride;
  unsigned int* status;
  Span ws_span;             // the workspace (bounds-check build)
};

struct Tail2 {
  uint64_t kfull[kMaxStages], kempty[kMaxStages];
  uint64_t vfull[kMaxStages], vempty[kMaxStages];
  uint64_t s_full[2], s_empty[2], p_full[2], u_done[2], q_full[2], q_empty[2];
  uint64_t epi;    // 4-warp rendezvous of the softmax warps
  uint64_t drain[2];  // score issuer, value issuer
  uint32_t tmem_base;
  int abort_flag;
  int vote[2][4];
  float red[2][4][32];
  float lsum[4][32];
};

__device__ __forceinline__ bool wait_ab(uint32_t bar, uint32_t parity, volatile int* abort_flag,
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// The (sequence b, kept tile j) a role is at, with sequence b's kept tile
// count nt, token count n, sink tiles st and first window tile fw (kept tile
// j is tile j below st, tile fw + j - st from there), and its kept positions
// [0, sk) and [ws, n). Every role walks its CTA's tiles in order with its
// own cursor: uniformly sized sequences (tps tiles of N tokens each) or the
// ragged, possibly evicted sequences of a paged plan.
struct TileCur {
  int b, j, nt, n, st, fw, sk, ws;
};

__device__ __forceinline__ void tcur_load(TileCur& c, const D2Args& a) {
  if (a.seqinfo) {
    const int4 v = ld_chk(a.seqinfo + c.b, a.ws_span, a.status, make_int4(0, 0, 0, 0));
    c.nt = v.x;
    c.n = v.y;
    c.st = v.z;
    c.fw = v.w;
  } else {
    c.nt = c.st = c.fw = a.tps;
    c.n = a.N;
  }
  if (a.window > 0 && c.n > a.sink + a.window) {
    c.sk = a.sink;
    c.ws = c.n - a.window;
  } else {
    c.sk = c.ws = c.n;
  }
}

// first token position of the cursor's tile
__device__ __forceinline__ int tcur_pos(const TileCur& c) {
  return (c.j < c.st ? c.j : c.fw + c.j - c.st) * kRows;
}

// whether the token at `pos` of the cursor's sequence is attended
__device__ __forceinline__ bool tcur_kept(const TileCur& c, int pos) {
  return pos < c.n && (pos < c.sk || pos >= c.ws);
}

__device__ __forceinline__ TileCur tcur_start(const D2Args& a) {
  TileCur c;
  if (a.seqinfo) {
    // a CTA with no tiles (or a workspace that holds no plan for this call)
    // still builds a cursor: its sequence index is kept inside [0, B)
    const int4 s = ld_chk(a.cstart + blockIdx.x, a.ws_span, a.status, make_int4(0, 0, 0, 0));
    c.b = min(max(s.x, 0), a.B - 1);
    c.j = s.z;
  } else {
    const int t = blockIdx.x * a.tpc;
    c.b = t / a.tps;
    c.j = t - c.b * a.tps;
  }
  tcur_load(c, a);
  return c;
}

__device__ __forceinline__ void tcur_next(TileCur& c, const D2Args& a) {
  if (++c.j == c.nt) {
    c.j = 0;
    do {
      ++c.b;
    } while (a.seqinfo && c.b < a.B && __ldg(&a.seqinfo[c.b].x) == 0);
    if (c.b < a.B) tcur_load(c, a);
  }
}

template <int HP, int NSUB, bool VPAIR = false>
__global__ void __launch_bounds__(kThreads, 1)
    k_lla2d(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
            D2Args a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Tail2* tl = reinterpret_cast<Tail2*>(smem + a.off_tail);
  volatile int* abort_flag = &tl->abort_flag;
  const uint32_t s_kring = smem_u32(smem);
  const uint32_t s_vring = s_kring + (uint32_t)a.nks * kStageBytes;
  const uint32_t s_q0 = smem_u32(smem + a.off_q);
  const uint32_t s_p0 = smem_u32(smem + a.off_p);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a paged plan sizes the split on the device (k_plan_paged finished before
  // k_absorb started, so this is safe before griddepcontrol.wait)
  const bool plan_ok = !a.seqinfo || (unsigned long long)a.plan[2] == a.stamp;
  const long long tiles = a.seqinfo ? (plan_ok ? a.plan[0] : 0LL) : (long long)a.tiles;
  const long long tpc = a.seqinfo ? a.plan[1] : (long long)a.tpc;
  const long long t_begin = blockIdx.x * tpc;
  const int ntile = (int)max(0LL, min(t_begin + tpc, tiles) - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.nks; ++s) {
      mbar_init(smem_u32(&tl->kfull[s]), 1);
      mbar_init(smem_u32(&tl->kempty[s]), 1);
    }
    for (int s = 0; s < a.nvs; ++s) {
      mbar_init(smem_u32(&tl->vfull[s]), 1);
      mbar_init(smem_u32(&tl->vempty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tl->s_full[i]), 1);
      mbar_init(smem_u32(&tl->s_empty[i]), 4);
      mbar_init(smem_u32(&tl->p_full[i]), 4);
      mbar_init(smem_u32(&tl->u_done[i]), 1);
      mbar_init(smem_u32(&tl->q_full[i]), 1);
      mbar_init(smem_u32(&tl->q_empty[i]), 1);
    }
    mbar_init(smem_u32(&tl->epi), 4);
    mbar_init(smem_u32(&tl->drain[0]), 1);
    mbar_init(smem_u32(&tl->drain[1]), 1);
    tl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tl->tmem_base), a.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tl->tmem_base;

  // 64-column boxes of K group kg; the last one may run past r_k, where the
  // tensor map fills zeros (and Q' holds zeros)
  auto kboxes = [&](int kg) { return min(2, (a.r_k - kg * 128 + 63) / 64); };

  if (warp == 0 || warp == 6) {
    // ------------------------------ producers ------------------------------
    // warp 0 streams Z^K groups (and stages Q'), warp 6 streams Z^V groups.
    const bool is_k = warp == 0;
    const uint64_t pol = l2_evict_first_policy();
    const int ng = is_k ? a.nkg : a.nvg;
    const int nring = is_k ? a.nks : a.nvs;
    const uint32_t ring = is_k ? s_kring : s_vring;
    uint64_t* fullb = is_k ? tl->kfull : tl->vfull;
    uint64_t* emptyb = is_k ? tl->kempty : tl->vempty;
    const CUtensorMap* map = is_k ? &tk : &tv;
    const int total = ntile * ng;
    // Cursor at the tile of the next group to load, and that tile's TMA
    // rows and third coordinates: (row, sequence) in the dense store, (row
    // in page, page) in a paged pool. Pages of a multiple of 128 tokens hold
    // whole tiles; pages of an odd multiple of 64 give each 64-row half of a
    // tile its own page, and a half that holds no kept token is zero-filled
    // in shared memory instead of read (its page may be unallocated or
    // evicted). The block-table entries of the next tile are loaded one tile
    // ahead.
    TileCur pc = tcur_start(a);
    constexpr int kSubRows = kRows / NSUB, kSubBytes = kBoxBytes / NSUB;
    int pc_lt = 0;
    int c_row[NSUB], c_z[NSUB], n_z[NSUB];
#pragma unroll
    for (int sb = 0; sb < NSUB; ++sb) c_row[sb] = c_z[sb] = n_z[sb] = 0;
    // page of rows [pos, pos + kSubRows) of the cursor's tile; whole-tile
    // boxes always hold a kept token, halves may not (-1: not read)
    auto lookup = [&](const TileCur& c, int sb) -> int {
      const int p0 = tcur_pos(c) + sb * kSubRows;
      const int* row = a.block_table + (size_t)c.b * a.max_blocks;
      if (NSUB == 1) return __ldg(row + p0 / a.page_size);
      const bool kept = p0 < c.sk || (p0 < c.n && p0 + kSubRows > c.ws);
      return kept ? __ldg(row + p0 / a.page_size) : -1;
    };
    auto place = [&]() {
      if (a.seqinfo) {
        const int pos = tcur_pos(pc);
#pragma unroll
        for (int sb = 0; sb < NSUB; ++sb) {
          c_row[sb] = (pos + sb * kSubRows) % a.page_size;
          c_z[sb] = n_z[sb];
        }
        TileCur nx = pc;
        tcur_next(nx, a);
        if (pc_lt + 1 < ntile) {
#pragma unroll
          for (int sb = 0; sb < NSUB; ++sb) n_z[sb] = lookup(nx, sb);
        }
      } else {
        c_row[0] = tcur_pos(pc);
        c_z[0] = pc.b;
      }
    };
    if (a.seqinfo && ntile > 0) {
#pragma unroll
      for (int sb = 0; sb < NSUB; ++sb) n_z[sb] = lookup(pc, sb);
    }
    if (ntile > 0) place();
    auto tile_of = [&](int lt) {
      while (pc_lt < lt) {
        tcur_next(pc, a);
        ++pc_lt;
        place();
      }
    };
    auto issue = [&](int it) -> bool {
      const int s = it % nring;
      const uint32_t ph = (uint32_t)(it / nring) & 1u;
      const bool ok = __all_sync(0xffffffffu,
                                 wait_ab(smem_u32(&emptyb[s]), ph ^ 1u, abort_flag, a.status));
      if (!ok) return false;
      const int lt = it / ng, grp = it - lt * ng;
      tile_of(lt);
      const uint32_t dst = ring + (uint32_t)s * kStageBytes;
      const int nb = is_k ? kboxes(grp) : 2;
      // VPAIR (V ring, 64-token halves): one load brings both 64-column
      // blocks of a half, laid out [half][block][64 rows]; otherwise a
      // stage is [block][half][64 rows]
      const bool pair = VPAIR && !is_k;
      int loaded = NSUB;
      if (NSUB > 1) {
        // a half with no kept token: zeros (generic stores, made visible to
        // the tensor cores before the stage is announced full)
        bool zeroed = false;
#pragma unroll
        for (int sb = 0; sb < NSUB; ++sb) {
          if (c_z[sb] >= 0) continue;
          --loaded;
          zeroed = true;
          for (int x = 0; x < nb; ++x) {
            const int off = pair ? sb * kBoxBytes + x * kSubBytes : x * kBoxBytes + sb * kSubBytes;
            uint4* z = reinterpret_cast<uint4*>(smem + (dst - s_kring) + off);
            for (int k = lane; k < kSubBytes / 16; k += 32) z[k] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        if (zeroed) fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        const uint32_t full = smem_u32(&fullb[s]);
        mbar_arrive_expect_tx(full, (uint32_t)(nb * loaded * kSubBytes));
        if (pair) {
#pragma unroll
          for (int sb = 0; sb < NSUB; ++sb)
            if (c_z[sb] >= 0)
              tma_load_4d(dst + sb * kBoxBytes, map, 0, c_row[sb], grp * 2, c_z[sb], full, pol);
        } else {
          for (int x = 0; x < nb; ++x) {
#pragma unroll
            for (int sb = 0; sb < NSUB; ++sb)
              if (NSUB == 1 || c_z[sb] >= 0)
                tma_load_3d(dst + x * kBoxBytes + sb * kSubBytes, map, grp * 128 + x * 64,
                            c_row[sb], c_z[sb], full, pol);
          }
        }
      }
      return true;
    };
    // Q' of sequence b arrives by one bulk copy: k_absorb already wrote it
    // as bf16 in the swizzled K-major layout the score MMA reads.
    int q_issued = -1;  // last sequence segment whose Q' copy was issued
    auto stage_q = [&](int seg, int b) -> bool {
      const int qb = seg & 1;
      const bool ok = __all_sync(
          0xffffffffu,
          wait_ab(smem_u32(&tl->q_empty[qb]), (uint32_t)((seg >> 1) & 1) ^ 1u, abort_flag, a.status));
      if (!ok) return false;
      if (lane == 0) {
        const uint32_t qfull = smem_u32(&tl->q_full[qb]);
        const unsigned char* qsrc = a.qsw + (size_t)b * a.qbuf_bytes;
        if (in_span(a.ws_span, qsrc, (unsigned long long)a.qbuf_bytes, a.status)) {
          mbar_arrive_expect_tx(qfull, (uint32_t)a.qbuf_bytes);
          bulk_g2s(s_q0 + (uint32_t)(qb * a.qbuf_bytes), qsrc, (uint32_t)a.qbuf_bytes, qfull,
                   l2_evict_first_policy());
        } else {
          mbar_arrive(qfull);  // nothing copied
        }
      }
      q_issued = seg;
      return true;
    };

    bool ok = true;
    int it = 0;
    if (!is_k || ntile > 0) {
      // One loop for both rings, so the load code is laid down once. The
      // K ring's loads of its first sequence (up to a ring's worth) do not
      // depend on k_absorb; before anything else it waits for that grid
      // and stages the sequence's Q', and each later sequence's Q' when
      // its first tile comes up. The V ring never waits.
      const int b0 = pc.b;
      bool waited = !is_k;
      int seg = 0, cur_b = b0;
      for (; ok && it < total; ++it) {
        const int lt = it / ng;
        tile_of(lt);
        if (!waited && (pc.b != b0 || it >= nring)) {
          pdl_wait();
          waited = true;
          ok = stage_q(0, b0);
          if (!ok) break;
        }
        if (is_k && waited && it - lt * ng == 0 && pc.b != cur_b) {
          cur_b = pc.b;
          ok = stage_q(++seg, cur_b);
          if (!ok) break;
        }
        ok = issue(it);
      }
      if (ok && !waited) {  // every tile fitted in the first ring's worth
        pdl_wait();
        ok = stage_q(0, b0);
      }
    } else {
      pdl_wait();
    }
    if (!ok && lane == 0) {
      const int first = max(0, it - nring);
      for (int i = first; i < it; ++i)
        (void)mbar_wait(smem_u32(&fullb[i % nring]), (uint32_t)(i / nring) & 1u,
                        kWaitTimeoutNs / 8);
      if (is_k && q_issued >= 0)  // the last Q' copy may still be landing
        (void)mbar_wait(smem_u32(&tl->q_full[q_issued & 1]), (uint32_t)((q_issued >> 1) & 1),
                        kWaitTimeoutNs / 8);
    }
  } else if (warp == 1) {
    // --------------------------- score MMA issuer ---------------------------
    // S[tokens x heads] = Z^K tile . Q'^T, one tile ahead of the softmax at
    // most (two S buffers). Independent of the value issuer, so a late value
    // group never holds up the next tile's scores.
    if (lane == 0 && ntile > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kRows, HP, false, false);
      bool ok = true;
      auto mma_scores = [&](int lt, int seg) -> bool {
        const int sb = lt & 1;
        if (!wait_ab(smem_u32(&tl->s_empty[sb]), (uint32_t)((lt >> 1) & 1) ^ 1u, abort_flag,
                     a.status))
          return false;
        tc_fence_after();
        const uint32_t d0 = tbase + (uint32_t)(sb * kSAcc * HP);
        const uint32_t qaddr = s_q0 + (uint32_t)((seg & 1) * a.qbuf_bytes);
        for (int kg = 0; kg < a.nkg; ++kg) {
          const int it = lt * a.nkg + kg;
          const int s = it % a.nks;
          if (!wait_ab(smem_u32(&tl->kfull[s]), (uint32_t)(it / a.nks) & 1u, abort_flag,
                       a.status))
            return false;
          tc_fence_after();
          // Descriptors are built once per stage and advanced by constant
          // start-address offsets (in 16-byte units): 32 B per K step inside
          // a 128B-swizzled row, one box (16 KB) per 64 columns.
          const uint64_t a_base = desc_kmajor_sw128(s_kring + (uint32_t)s * kStageBytes);
          const uint64_t b_base = desc_kmajor_sw128(qaddr + (uint32_t)(kg * 2 * HP * 128));
          const bool first = kg == 0;
          if (kboxes(kg) == 2) {
#pragma unroll
            for (int st = 0; st < 8; ++st) {
              const int x = st >> 2, kk = st & 3;
              const uint64_t a_d = a_base + (uint64_t)(x * (kBoxBytes >> 4) + kk * 2);
              const uint64_t b_d = b_base + (uint64_t)(x * (HP * 128 >> 4) + kk * 2);
              umma_bf16(d0 + (uint32_t)((st % kSAcc) * HP), a_d, b_d, idesc_s,
                        !(first && st < kSAcc));
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(d0 + (uint32_t)((kk % kSAcc) * HP), a_base + (uint64_t)(kk * 2),
                        b_base + (uint64_t)(kk * 2), idesc_s, !(first && kk < kSAcc));
          }
          umma_commit(smem_u32(&tl->kempty[s]));
        }
        umma_commit(smem_u32(&tl->s_full[sb]));
        return true;
      };

      int seg = 0;
      TileCur cur = tcur_start(a);
      ok = wait_ab(smem_u32(&tl->q_full[0]), 0u, abort_flag, a.status);
      for (int lt = 0; ok && lt < ntile; ++lt, tcur_next(cur, a)) {
        if (lt > 0 && cur.j == 0) {
          umma_commit(smem_u32(&tl->q_empty[seg & 1]));  // after the last score MMA of seg
          ++seg;
          ok = wait_ab(smem_u32(&tl->q_full[seg & 1]), (uint32_t)((seg >> 1) & 1), abort_flag,
                       a.status);
          if (!ok) break;
        }
        ok = mma_scores(lt, seg);
      }
      umma_commit(smem_u32(&tl->drain[0]));
      (void)mbar_wait(smem_u32(&tl->drain[0]), 0u, kWaitTimeoutNs / 8);
    }
  } else if (warp == 7) {
    // --------------------------- value MMA issuer ---------------------------
    // U[r_v x heads] += Z^V tile^T . P, per 128-column group of r_v, as soon
    // as the softmax has written P for the tile.
    if (lane == 0 && ntile > 0) {
      const uint32_t idesc_u = idesc_bf16_f32(kRows, HP, true, false);
      bool ok = true;
      TileCur cur = tcur_start(a);
      for (int lt = 0; ok && lt < ntile; ++lt, tcur_next(cur, a)) {
        const bool first_of_seg = (lt == 0) || cur.j == 0;
        const int pb = lt & 1;
        ok = wait_ab(smem_u32(&tl->p_full[pb]), (uint32_t)((lt >> 1) & 1), abort_flag, a.status);
        if (!ok) break;
        tc_fence_after();
        for (int vg = 0; vg < a.nvg && ok; ++vg) {
          const int it = lt * a.nvg + vg;
          const int s = it % a.nvs;
          ok = wait_ab(smem_u32(&tl->vfull[s]), (uint32_t)(it / a.nvs) & 1u, abort_flag,
                       a.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tbase + (uint32_t)(2 * kSAcc * HP + vg * kUAcc * HP);
          // A (MN-major latents): 16 token rows (2 KB) per K step;
          // B (K-major P): 32 B per K step inside a 64-token chunk.
          // With VPAIR the two 64-column blocks of a half sit 8 KB apart and
          // the second half's rows start 16 KB in.
          const uint64_t a_base = desc_mnmajor_sw128(s_vring + (uint32_t)s * kStageBytes,
                                                     VPAIR ? kSubBytesV : kBoxBytes);
          const uint64_t b_base = desc_kmajor_sw128(s_p0 + (uint32_t)(pb * a.pbuf_bytes));
#pragma unroll
          for (int ks = 0; ks < kRows / 16; ++ks)
            umma_bf16(d + (uint32_t)((ks % kUAcc) * HP),
                      a_base + (uint64_t)((VPAIR ? (ks >> 2) * kBoxBytes + (ks & 3) * 2048
                                                 : ks * 2048) >> 4),
                      b_base + (uint64_t)((ks >> 2) * (HP * 128 >> 4) + (ks & 3) * 2), idesc_u,
                      !(first_of_seg && ks < kUAcc));
          umma_commit(smem_u32(&tl->vempty[s]));
        }
        if (!ok) break;
        umma_commit(smem_u32(&tl->u_done[pb]));
      }
      umma_commit(smem_u32(&tl->drain[1]));
      (void)mbar_wait(smem_u32(&tl->drain[1]), 0u, kWaitTimeoutNs / 8);
    }
  } else {
    // --------------------------- softmax / epilogue ---------------------------
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tbase + ((uint32_t)(quarter * 32) << 16);
    uint32_t epi_phase = 0;
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tl->epi));
      const bool ok = __all_sync(
          0xffffffffu, wait_ab(smem_u32(&tl->epi), epi_phase & 1u, abort_flag, a.status));
      ++epi_phase;
      return ok;
    };
    float m[HP], l[HP];
    TileCur cur = tcur_start(a);
    for (int lt = 0; lt < ntile; ++lt, tcur_next(cur, a)) {
      const int b = cur.b;
      const int row0 = tcur_pos(cur);
      const bool first_of_seg = (lt == 0) || cur.j == 0;
      const bool last_of_seg = (lt == ntile - 1) || cur.j == cur.nt - 1;
      if (first_of_seg) {
#pragma unroll
        for (int h = 0; h < HP; ++h) {
          m[h] = kNegBig;
          l[h] = 0.f;
        }
      }
      const int sb = lt & 1;
      bool ok = __all_sync(0xffffffffu, wait_ab(smem_u32(&tl->s_full[sb]), (uint32_t)((lt >> 1) & 1),
                                                abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      float s[HP];
#pragma unroll
      for (int h0 = 0; h0 < HP; h0 += 16) {
        tmem_ld16(lane_base + (uint32_t)(sb * kSAcc * HP + h0), s + h0);
#pragma unroll
        for (int j = 1; j < kSAcc; ++j) {
          float t[16];
          tmem_ld16(lane_base + (uint32_t)(sb * kSAcc * HP + j * HP + h0), t);
#pragma unroll
          for (int e = 0; e < 16; ++e) s[h0 + e] += t[e];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tl->s_empty[sb]));

      const bool valid = tcur_kept(cur, row0 + row);
      bool need = false;
#pragma unroll
      for (int h = 0; h < HP; ++h) need |= valid && h < a.H && s[h] > m[h] + kSlack;
      const int vb = lt & 1;
      const int any_need = __any_sync(0xffffffffu, need);
      if (lane == 0) tl->vote[vb][ew] = any_need ? 1 : 0;
      if (!epi_sync()) break;
      const bool need_any = tl->vote[vb][0] | tl->vote[vb][1] | tl->vote[vb][2] | tl->vote[vb][3];
      if (need_any) {
#pragma unroll
        for (int h = 0; h < HP; ++h) {
          float v = valid ? s[h] : kNegBig;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) tl->red[vb][ew][h] = v;
        }
        if (!epi_sync()) break;
        float alpha[HP];
#pragma unroll
        for (int h = 0; h < HP; ++h) {
          const float mx = fmaxf(fmaxf(tl->red[vb][0][h], tl->red[vb][1][h]),
                                 fmaxf(tl->red[vb][2][h], tl->red[vb][3][h]));
          const float mn = fmaxf(m[h], mx);
          alpha[h] = exp2f(m[h] - mn);
          m[h] = mn;
          l[h] *= alpha[h];
        }
        if (!first_of_seg) {
          // U holds the value MMAs up to tile lt-1: wait for the last one
          const int pb = (lt - 1) & 1;
          ok = __all_sync(0xffffffffu,
                          wait_ab(smem_u32(&tl->u_done[pb]), (uint32_t)(((lt - 1) >> 1) & 1),
                                  abort_flag, a.status));
          if (!ok) break;
          tc_fence_after();
          for (int j = 0; j < a.nvg * kUAcc; ++j) {
#pragma unroll
            for (int h0 = 0; h0 < HP; h0 += 16) {
              float u[16];
              const uint32_t ta = lane_base + (uint32_t)(2 * kSAcc * HP + j * HP + h0);
              tmem_ld16(ta, u);
#pragma unroll
              for (int e = 0; e < 16; ++e) u[e] *= alpha[h0 + e];
              tmem_st16(ta, u);
            }
          }
        }
      }
      float p[HP];
#pragma unroll
      for (int h = 0; h < HP; ++h) {
        p[h] = (valid && h < a.H) ? exp2f(s[h] - m[h]) : 0.f;
        l[h] += p[h];
      }
      // P buffer lt&1 was read by the value MMA of tile lt-2
      if (lt >= 2) {
        ok = __all_sync(0xffffffffu,
                        wait_ab(smem_u32(&tl->u_done[lt & 1]), (uint32_t)(((lt - 2) >> 1) & 1),
                                abort_flag, a.status));
        if (!ok) break;
      }
      unsigned char* pbuf = smem + a.off_p + (lt & 1) * a.pbuf_bytes;
#pragma unroll
      for (int h = 0; h < HP; ++h)
        *reinterpret_cast<__nv_bfloat16*>(pbuf + sw128_off(h, row, HP)) = __float2bfloat16_rn(p[h]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tl->p_full[lt & 1]));

      if (last_of_seg) {
        ok = __all_sync(0xffffffffu, wait_ab(smem_u32(&tl->u_done[lt & 1]), (uint32_t)((lt >> 1) & 1),
                                             abort_flag, a.status));
        if (!ok) break;
        tc_fence_after();
        const long long slot = (long long)blockIdx.x + b;
        float* rec = a.part + slot * a.H * a.pstride;
        for (int vg = 0; vg < a.nvg; ++vg) {
#pragma unroll
          for (int h0 = 0; h0 < HP; h0 += 16) {
            float u[16];
            tmem_ld16(lane_base + (uint32_t)(2 * kSAcc * HP + vg * kUAcc * HP + h0), u);
#pragma unroll
            for (int j = 1; j < kUAcc; ++j) {
              float t[16];
              tmem_ld16(lane_base + (uint32_t)(2 * kSAcc * HP + (vg * kUAcc + j) * HP + h0), t);
#pragma unroll
              for (int e = 0; e < 16; ++e) u[e] += t[e];
            }
            // rows past r_v (zero-filled latent columns) are not stored
            if (vg * 128 + row < a.r_v) {
#pragma unroll
              for (int e = 0; e < 16; ++e)
                if (h0 + e < a.H)
                  st_chk(&rec[(size_t)(h0 + e) * a.pstride + 4 + vg * 128 + row], u[e], a.ws_span,
                         a.status);
            }
          }
        }
#pragma unroll
        for (int h = 0; h < HP; ++h) {
          const float v = warp_sum(l[h]);
          if (lane == 0) tl->lsum[ew][h] = v;
        }
        if (!epi_sync()) break;
        if (ew == 0 && lane < a.H) {
          float mm = 0.f;
#pragma unroll
          for (int h = 0; h < HP; ++h)
            if (h == lane) mm = m[h];
          st_chk(&rec[(size_t)lane * a.pstride + 0], mm, a.ws_span, a.status);
          st_chk(&rec[(size_t)lane * a.pstride + 1],
                 tl->lsum[0][lane] + tl->lsum[1][lane] + tl->lsum[2][lane] + tl->lsum[3][lane],
                 a.ws_span, a.status);
        }
        tc_fence_before();
        if (!epi_sync()) break;  // lsum is reused by the next sequence
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, a.tmem_cols);
  }
}

struct D2Plan {
  int hp, tps, tiles, tpc, grid, nkg, nvg, nks, nvs;
  int off_q, off_p, off_tail, qbuf_bytes, pbuf_bytes;
  size_t smem;
  uint32_t tmem_cols;
  int pstride;
  size_t off_qsw, off_c0, off_part, ws_bytes;
};

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

lla_status plan_2d(int B, int H, int N, int r_k, int r_v, D2Plan* p) {
  D2Plan d{};
  d.hp = H <= 16 ? 16 : 32;
  d.tps = (N + kRows - 1) / kRows;
  d.tiles = B * d.tps;
  const DeviceInfo di = device_info();
  const int grid0 = std::max(1, std::min(d.tiles, di.sms));
  d.tpc = (d.tiles + grid0 - 1) / grid0;
  d.grid = (d.tiles + d.tpc - 1) / d.tpc;
  // ranks that are not whole 64-column boxes (K) or 128-row MMA tiles (V)
  // are padded up: the tensor maps fill the missing columns with zeros
  d.nkg = (r_k + 127) / 128;
  d.nvg = (r_v + 127) / 128;
  d.qbuf_bytes = ((r_k + 63) / 64) * d.hp * 128;
  d.pbuf_bytes = 2 * d.hp * 128;
  const size_t fixed = 2 * (size_t)d.qbuf_bytes + 2 * (size_t)d.pbuf_bytes + sizeof(Tail2) + 1024;
  // Split the stages between the rings: each ring needs at least one
  // tile's groups (its slots are reused only by later tiles) and gets at
  // most kMaxStages. A split that uses every stage and gives each ring a
  // whole number of tiles is taken when there is one (the most even such
  // split, then the deeper V ring): at r_k = r_v = 256 (two groups per
  // tile and ring, six stages) 2 K + 4 V and 4 K + 2 V stages both ran the
  // decode in 312 us against 330 us for 3 + 3. Otherwise V gets half and K
  // the odd one out.
  const int nst = (int)std::min<size_t>(2 * kMaxStages,
                                        ((size_t)di.smem_optin - fixed) / kStageBytes);
  d.nvs = std::min(kMaxStages, std::max(d.nvg, nst / 2));
  int best = -1;
  for (int v = d.nvg; v <= kMaxStages && v < nst; ++v) {
    const int k = nst - v;
    if (k > kMaxStages || k < d.nkg || v % d.nvg || k % d.nkg) continue;
    if (best < 0 || std::abs(k - v) < std::abs((nst - best) - best) ||
        (std::abs(k - v) == std::abs((nst - best) - best) && v > best))
      best = v;
  }
  if (best > 0) d.nvs = best;
  d.nks = std::min(kMaxStages, nst - d.nvs);
  if (d.nks < d.nkg || d.nvs < d.nvg)
    return fail(LLA_ERR_UNSUPPORTED, "LLA-2D stage rings do not fit in shared memory");
  d.off_q = (d.nks + d.nvs) * kStageBytes;
  d.off_p = d.off_q + 2 * d.qbuf_bytes;
  d.off_tail = d.off_p + 2 * d.pbuf_bytes;
  d.smem = (size_t)d.off_tail + sizeof(Tail2) + 1024;
  const int cols = (2 * kSAcc + d.nvg * kUAcc) * d.hp;
  uint32_t c = 32;
  while (c < (uint32_t)cols) c <<= 1;
  d.tmem_cols = c;
  d.pstride = 4 + r_v;
  const size_t units = (size_t)B * H;
  d.off_qsw = 0;
  d.off_c0 = al256((size_t)B * d.qbuf_bytes);
  d.off_part = al256(d.off_c0 + units * sizeof(float));
  d.ws_bytes = al256(d.off_part + ((size_t)d.grid + B) * H * d.pstride * sizeof(float));
  *p = d;
  return LLA_OK;
}

}  // namespace

size_t workspace_2d(int B, int H, int N, int r_k, int r_v) {
  D2Plan d;
  if (plan_2d(B, H, N, r_k, r_v, &d) != LLA_OK) return 0;
  return d.ws_bytes;
}

namespace {

// Paged-store arrays of one LLA-2D call (device), or none.
struct Paged2D {
  const int4* seqinfo;
  long long* cum;
  long long* plan;
  const int4* cstart;
  const int* block_table;
  int max_blocks, page_size, sink, window;
  unsigned long long stamp;
  bool vpair;  // 64-token pages: the V map loads both blocks of a half at once
};

// Absorb, the tensor-core kernel and the merge, shared by the dense and the
// paged entry points.
// r_k is the width of a key row, the latent part plus d_r rotary values
// when q_rope is given.
lla_status launch_2d(const float* q, const CUtensorMap& tk, const CUtensorMap& tv, int B, int H,
                     int d_h, int N, int r_k, int r_v, const float* dk, const float* dv,
                     const float* mu_k, const float* mu_v, float scale, float* out, float* lse,
                     const D2Plan& d, char* wsb, Span ws, const Paged2D* pg, cudaStream_t stream,
                     const float* q_rope = nullptr, int d_r = 0) {
  unsigned char* qsw = reinterpret_cast<unsigned char*>(wsb + d.off_qsw);
  float* c0 = reinterpret_cast<float*>(wsb + d.off_c0);
  float* part = reinterpret_cast<float*>(wsb + d.off_part);
  lla_status st = launch_absorb(q, dk, mu_k, B, H, d_h, r_k - d_r, scale, nullptr, c0, stream, qsw,
                                d.hp, q_rope, d_r, true, ws);
  if (st != LLA_OK) return st;

  D2Args a{};
  a.B = B;
  a.H = H;
  a.N = N;
  a.tps = d.tps;
  a.tiles = d.tiles;
  a.tpc = d.tpc;
  a.r_k = r_k;
  a.r_v = r_v;
  a.nkg = d.nkg;
  a.nvg = d.nvg;
  a.nks = d.nks;
  a.nvs = d.nvs;
  a.off_q = d.off_q;
  a.off_p = d.off_p;
  a.off_tail = d.off_tail;
  a.qbuf_bytes = d.qbuf_bytes;
  a.pbuf_bytes = d.pbuf_bytes;
  a.tmem_cols = d.tmem_cols;
  a.qsw = qsw;
  a.part = part;
  a.pstride = d.pstride;
  a.status = status_word();
  a.ws_span = ws;
  if (pg) {
    a.seqinfo = pg->seqinfo;
    a.plan = pg->plan;
    a.stamp = pg->stamp;
    a.cstart = pg->cstart;
    a.block_table = pg->block_table;
    a.max_blocks = pg->max_blocks;
    a.page_size = pg->page_size;
    a.sink = pg->sink;
    a.window = pg->window;
  }

  // pages of an odd multiple of 64 tokens: each tile half from its own page
  const bool split = pg && pg->page_size % kRows;
  const bool vpair = split && pg->vpair;
  auto kern = d.hp == 16
                  ? (vpair ? k_lla2d<16, 2, true> : split ? k_lla2d<16, 2> : k_lla2d<16, 1>)
                  : (vpair ? k_lla2d<32, 2, true> : split ? k_lla2d<32, 2> : k_lla2d<32, 1>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)d.smem);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_lla2d)");
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(d.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = d.smem;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  e = record_timing(true, stream);
  if (e != cudaSuccess) return check_cuda(e, "record timing event");
  e = cudaLaunchKernelEx(&cfg, kern, tk, tv, a);
  if (e != cudaSuccess) return check_cuda(e, "launch k_lla2d");
  e = record_timing(false, stream);
  if (e != cudaSuccess) return check_cuda(e, "record timing event");

  if (pg) {  // sequence b's pieces: the CTAs of its tiles, cum[b] .. cum[b] + tiles - 1
    RaggedMap rm{pg->seqinfo, pg->cum, pg->plan, pg->stamp};
    return launch_combine(part, d.pstride, c0, dv, mu_v, B, H, d_h, r_v, 0, 0, 1, out, lse, stream,
                          &rm, true, ws);
  }
  return launch_combine(part, d.pstride, c0, dv, mu_v, B, H, d_h, r_v,
                        (long long)d.tps * kRows, (long long)d.tpc * kRows, 1, out, lse, stream,
                        nullptr, true, ws);
}

// The paged plan: the dense plan's kernel shape with a one-wave grid (the
// tile count is known only on the device), plus the planner's arrays.
struct D2PagedPlan {
  D2Plan d;
  size_t off_seqinfo, off_cum, off_plan, off_cstart, ws_bytes;
};

lla_status plan_2d_paged(int B, int H, int r_k, int r_v, D2PagedPlan* pp) {
  D2PagedPlan p{};
  lla_status st = plan_2d(B, H, kRows, r_k, r_v, &p.d);
  if (st != LLA_OK) return st;
  p.d.grid = device_info().sms;
  p.d.tpc = 0;
  p.d.off_part = al256(p.d.off_c0 + (size_t)B * H * sizeof(float));
  p.off_seqinfo =
      al256(p.d.off_part + ((size_t)p.d.grid + B) * H * p.d.pstride * sizeof(float));
  p.off_cum = al256(p.off_seqinfo + (size_t)B * sizeof(int4));
  p.off_plan = al256(p.off_cum + (size_t)(B + 1) * sizeof(long long));
  p.off_cstart = al256(p.off_plan + 3 * sizeof(long long));
  p.ws_bytes = al256(p.off_cstart + (size_t)p.d.grid * sizeof(int4));
  *pp = p;
  return LLA_OK;
}

}  // namespace

lla_status run_decode_2d(const float* q, const void* zk, const void* zv, int B, int H, int d_h,
                         int N, long long n_cap, int r_k, int r_v, const float* dk,
                         const float* dv, const float* mu_k, const float* mu_v, float scale,
                         float* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream,
                         const float* q_rope, int d_r) {
  if (!q_rope) d_r = 0;
  r_k += d_r;  // the key row: latent, then the rotary key
  D2Plan d;
  lla_status st = plan_2d(B, H, N, r_k, r_v, &d);
  if (st != LLA_OK) return st;
  if (ws == nullptr || ws_bytes < d.ws_bytes)
    return fail(LLA_ERR_WORKSPACE, "LLA-2D workspace needs %zu bytes, got %zu", d.ws_bytes, ws_bytes);
  CUtensorMap tk, tv;
  {
    const uint64_t dims[3] = {(uint64_t)r_k, (uint64_t)N, (uint64_t)B};
    const uint64_t strides[2] = {(uint64_t)r_k * 2, (uint64_t)n_cap * r_k * 2};
    const uint32_t box[3] = {64, (uint32_t)kRows, 1};
    if (!make_tmap_bf16(&tk, zk, 3, dims, strides, box)) return LLA_ERR_INVALID_ARG;
  }
  {
    const uint64_t dims[3] = {(uint64_t)r_v, (uint64_t)N, (uint64_t)B};
    const uint64_t strides[2] = {(uint64_t)r_v * 2, (uint64_t)n_cap * r_v * 2};
    const uint32_t box[3] = {64, (uint32_t)kRows, 1};
    if (!make_tmap_bf16(&tv, zv, 3, dims, strides, box)) return LLA_ERR_INVALID_ARG;
  }
  return launch_2d(q, tk, tv, B, H, d_h, N, r_k, r_v, dk, dv, mu_k, mu_v, scale, out, lse, d,
                   static_cast<char*>(ws), span_of(ws, ws_bytes), nullptr, stream, q_rope, d_r);
}

size_t workspace_2d_paged(int B, int H, int r_k, int r_v) {
  D2PagedPlan p;
  if (plan_2d_paged(B, H, r_k, r_v, &p) != LLA_OK) return 0;
  return p.ws_bytes;
}

lla_status run_decode_2d_paged(const float* q, const void* zk, const void* zv, int B, int H,
                               int d_h, int r_k, int r_v, int page_size, int num_pages,
                               const int* block_table, int max_blocks, const int* seq_lens,
                               int sink, int window, const float* dk, const float* dv,
                               const float* mu_k, const float* mu_v, float scale, float* out,
                               float* lse, void* ws, size_t ws_bytes, cudaStream_t stream,
                               PagedMode mode) {
  D2PagedPlan pp;
  lla_status st = plan_2d_paged(B, H, r_k, r_v, &pp);
  if (st != LLA_OK) return st;
  if (ws == nullptr || ws_bytes < pp.ws_bytes)
    return fail(LLA_ERR_WORKSPACE, "paged LLA-2D workspace needs %zu bytes, got %zu", pp.ws_bytes,
                ws_bytes);
  char* wsb = static_cast<char*>(ws);
  Paged2D pg{};
  pg.seqinfo = reinterpret_cast<const int4*>(wsb + pp.off_seqinfo);
  pg.cum = reinterpret_cast<long long*>(wsb + pp.off_cum);
  pg.plan = reinterpret_cast<long long*>(wsb + pp.off_plan);
  pg.cstart = reinterpret_cast<const int4*>(wsb + pp.off_cstart);
  pg.block_table = block_table;
  pg.max_blocks = max_blocks;
  pg.page_size = page_size;
  pg.sink = sink;
  pg.window = window;
  pg.stamp = paged_plan_stamp(2, 2, B, 1, r_k, r_v, page_size, num_pages, block_table, max_blocks,
                              seq_lens, sink, window, pp.d.grid, 1, kRows);
  // 1. plan: tiles of kRows tokens, one worker per CTA (skipped when an
  //    earlier plan-only call already left it in this workspace)
  if (mode != kDecodePlanned) {
    st = launch_plan_paged(seq_lens, block_table, B, 1, page_size, num_pages, max_blocks, sink,
                           window, pp.d.grid, 1, kRows, const_cast<int4*>(pg.seqinfo), pg.cum,
                           pg.plan, const_cast<int4*>(pg.cstart), pg.stamp, stream);
    if (st != LLA_OK || mode == kPlanOnly) return st;
  }
  // The pool read page by page: rows of a page, pages outermost; boxes of
  // 64 rows when pages hold an odd multiple of 64 tokens.
  const uint32_t box_rows = page_size % kRows ? kRows / 2 : kRows;
  CUtensorMap tk, tv;
  {
    const uint64_t dims[3] = {(uint64_t)r_k, (uint64_t)page_size, (uint64_t)num_pages};
    const uint64_t strides[2] = {(uint64_t)r_k * 2, (uint64_t)page_size * r_k * 2};
    const uint32_t box[3] = {64, box_rows, 1};
    if (!make_tmap_bf16(&tk, zk, 3, dims, strides, box)) return LLA_ERR_INVALID_ARG;
  }
  // 64-token pages with r_v a multiple of 64: the V pool viewed as
  // [pages][64-column blocks][rows][64 columns], so one box of two blocks x
  // 64 rows loads a whole half of a value group
  pg.vpair = page_size % kRows != 0 && r_v % 64 == 0;
  if (pg.vpair) {
    const uint64_t dims[4] = {64, (uint64_t)page_size, (uint64_t)(r_v / 64), (uint64_t)num_pages};
    const uint64_t strides[3] = {(uint64_t)r_v * 2, 128, (uint64_t)page_size * r_v * 2};
    const uint32_t box[4] = {64, box_rows, 2, 1};
    if (!make_tmap_bf16(&tv, zv, 4, dims, strides, box)) return LLA_ERR_INVALID_ARG;
  } else {
    const uint64_t dims[3] = {(uint64_t)r_v, (uint64_t)page_size, (uint64_t)num_pages};
    const uint64_t strides[2] = {(uint64_t)r_v * 2, (uint64_t)page_size * r_v * 2};
    const uint32_t box[3] = {64, box_rows, 1};
    if (!make_tmap_bf16(&tv, zv, 3, dims, strides, box)) return LLA_ERR_INVALID_ARG;
  }
  return launch_2d(q, tk, tv, B, H, d_h, 0, r_k, r_v, dk, dv, mu_k, mu_v, scale, out, lse, pp.d,
                   wsb, span_of(ws, ws_bytes), &pg, stream);
}

}  // namespace lla

// Per-head absorbed LLA decode, streaming kernel (sm_100a).
//
// Source: "Looped Latent Attention: Cross-Loop KV Compression for Looped
// Transformers" (arXiv 2607.15456), §7 "Per-head LLA versus LLA-2D at
// inference": scores read latents directly through the absorbed query, and
// the value side is summed in latent space.
//
// The flattened (unit, token) range of one (layer, loop) step is cut into
// equal contiguous pieces, one per warp of a one-wave grid. Each warp runs
// its own bulk-async-copy pipeline (cp.async.bulk into a ring of shared-
// memory stages, completion counted on one mbarrier per stage), computes
// scores q' . z^K_j, keeps an online softmax per token slot and accumulates
// sum_j p_j z^V_j in latent space. Each (warp, unit) piece ends in one
// partial record (m, l, u) that k_combine merges.
#include "common.cuh"
#include "stream.cuh"

namespace lla {
namespace {



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
                                        int nseg_k, int g, const StreamArgs& a) {
#pragma unroll
  for (int s = 0; s < SK; ++s) {
    const int seg = s * LPT + g;
    if ((EXACT || seg < nseg_k) && in_span(a.ws_span, qp + u * r_k + seg * E, E * 4, a.status)) {
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

// Scores and online-softmax updates for the `len` tokens of one stage: token
// slot `slot` takes tokens slot, slot + NS, ... two at a time.
template <int ESZ, int LPT, int SK, int SV, bool EXACT>
__device__ __forceinline__ void stream_tile(const unsigned char* Ks, const unsigned char* Vs,
                                            int len, const float (&qv)[SK][16 / ESZ], float& m,
                                            float& l, float (&acc)[SV][16 / ESZ],
                                            const StreamArgs& a, int slot, int g) {
  constexpr int E = 16 / ESZ;
  constexpr int NS = 32 / LPT;
  constexpr unsigned FULL = 0xffffffffu;
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
}

// Merges the NS token slots of a warp (log-sum-exp butterfly) and writes the
// piece's partial record (m, l, u) at pp.
template <int ESZ, int LPT, int SV, bool EXACT>
__device__ __forceinline__ void stream_merge_write(float m, float l, float (&acc)[SV][16 / ESZ],
                                                   float* pp, const StreamArgs& a, int slot,
                                                   int g) {
  constexpr int E = 16 / ESZ;
  constexpr unsigned FULL = 0xffffffffu;
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
  // the whole record [m, l, pad, pad, u[nseg_v * E]] must lie in the workspace
  if (slot == 0 && in_span(a.ws_span, pp, (4 + (size_t)a.nseg_v * E) * 4, a.status)) {
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

// ESZ: bytes per latent element. LPT: lanes per token. SK/SV: 16-byte
// segments per lane for K/V. EXACT: nseg == LPT*S for both axes.
template <int ESZ, int LPT, int SK, int SV, bool EXACT>
__global__ void __launch_bounds__(256, 1) k_stream(StreamArgs a) {
  constexpr int E = 16 / ESZ;  // elements per 16-byte segment
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ __align__(128) unsigned char smem[];

  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const long long w = (long long)blockIdx.x * nwarps + warp;
  if (w >= a.W) return;
  const int slot = lane / LPT, g = lane - slot * LPT;

  const int bar_bytes = ((nwarps * a.nstage * 12) + 127) & ~127;
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
      const char* ksrc = a.zk + row * a.row_k;
      const char* vsrc = a.zv + row * a.row_v;
      if (in_span(a.zk_span, ksrc, kb, a.status) && in_span(a.zv_span, vsrc, vb, a.status)) {
        mbar_arrive_expect_tx(bar, kb + vb);
        bulk_g2s(dst, ksrc, kb, bar, pol);
        bulk_g2s(dst + v_off, vsrc, vb, bar, pol);
      } else {
        mbar_arrive(bar);  // nothing copied: the stage completes as it is
      }
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
  load_qp<E, LPT, SK, EXACT>(qv, a.qp, u, a.r_k, a.nseg_k, g, a);
  while (f < f1) {
    const long long seg_end = min(f1, (u + 1) * a.N);
    // the next unit's q' loads run under this unit's stream
    if (u < u_last) load_qp<E, LPT, SK, EXACT>(qn, a.qp, u + 1, a.r_k, a.nseg_k, g, a);
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

      stream_tile<ESZ, LPT, SK, SV, EXACT>(Ks, Vs, len, qv, m, l, acc, a, slot, g);
      __syncwarp();
      --in_flight;
      if (pf < f1) issue();  // refill the stage just read
      if (++cs == a.nstage) {
        cs = 0;
        cpar ^= 1u;
      }
      f += len;
    }

    stream_merge_write<ESZ, LPT, SV, EXACT>(m, l, acc, a.part + (size_t)(w + u) * a.pstride, a,
                                            slot, g);
    ++u;
#pragma unroll
    for (int s = 0; s < SK; ++s)
#pragma unroll
      for (int e = 0; e < E; ++e) qv[s][e] = qn[s][e];
  }
}


// ---------------------------------------------------------------------------
// paged / ragged store
// ---------------------------------------------------------------------------

// Position in the flattened range of a paged plan: sequence b, head h, kept
// index i, sequence b's record (kept tokens n, sink part s, gap), and the
// page position of kept index i: block blk, row pp (tracked incrementally,
// so a tile costs no division).
struct PCursor {
  int b, h, i;
  int n, s, gap;
  int blk, pp;
};

__device__ __forceinline__ void pc_load_seq(PCursor& c, const StreamArgs& a) {
  const int4 v = in_span(a.ws_span, a.seqinfo + c.b, sizeof(int4), a.status)
                     ? __ldg(a.seqinfo + c.b)
                     : make_int4(0, 0, 0, 0);
  c.n = v.x;
  c.s = v.y;
  c.gap = v.z;
}

// Page position of kept index c.i (a division; only at range starts and
// where the kept set jumps over evicted tokens).
__device__ __forceinline__ void pc_place(PCursor& c, int page_size) {
  const int pos = c.i < c.s ? c.i : c.i + c.gap;
  c.blk = pos / page_size;
  c.pp = pos - c.blk * page_size;
}

// Tokens of the next tile: at most `tile`, and ending no later than the
// warp's range, the unit, the sink part and the page.
__device__ __forceinline__ int pc_len(const PCursor& c, long long f, long long f1, int tile,
                                      int page_size) {
  int lim = (int)min((long long)tile, f1 - f);
  lim = min(lim, (c.i < c.s ? c.s : c.n) - c.i);
  return min(lim, page_size - c.pp);
}

// Moves the cursor `len` tokens on; len never crosses a unit end, and at one
// the cursor moves to the next head, or the next non-empty sequence.
__device__ __forceinline__ void pc_advance(PCursor& c, int len, const StreamArgs& a) {
  c.i += len;
  c.pp += len;
  if (c.pp == a.page_size) {
    c.pp = 0;
    ++c.blk;
  }
  if (c.i == c.n) {
    c.i = 0;
    if (++c.h == a.H) {
      c.h = 0;
      do {
        ++c.b;
      } while (c.b < a.B && __ldg(&a.seqinfo[c.b].x) == 0);
      if (c.b < a.B) pc_load_seq(c, a);
    }
    // kept index 0 is position 0, or the window start when the sink is empty
    c.blk = 0;
    c.pp = 0;
    if (c.s == 0 && c.gap != 0) pc_place(c, a.page_size);
  } else if (c.i == c.s && c.gap != 0) {
    pc_place(c, a.page_size);  // jump to the window part
  }
}

// Moves a cursor at any token of a unit to the start of the next unit
// (next head, or next non-empty sequence). Page fields are not kept.
__device__ __forceinline__ void pc_next_unit(PCursor& c, const StreamArgs& a) {
  c.i = 0;
  if (++c.h == a.H) {
    c.h = 0;
    do {
      ++c.b;
    } while (c.b < a.B && __ldg(&a.seqinfo[c.b].x) == 0);
    if (c.b < a.B) pc_load_seq(c, a);
  }
}

// The streaming kernel over a paged store [pages][H][page_size][r] with
// per-sequence lengths and the optional sink + window eviction set. The
// flattened range, each warp's share P and each warp's starting cursor come
// from k_plan_paged, which finished before k_absorb started, so they are
// read before griddepcontrol.wait. Tiles are cut at page ends and at the
// end of the sink part, so each is one contiguous run of rows.
template <int ESZ, int LPT, int SK, int SV, bool EXACT>
__global__ void __launch_bounds__(256, 1) k_stream_paged(StreamArgs a) {
  constexpr int E = 16 / ESZ;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ __align__(128) unsigned char smem[];

  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const long long w = (long long)blockIdx.x * nwarps + warp;
  if (w >= a.W) return;
  // a workspace that does not hold this call's plan: no work (the merge
  // reports it and writes empty results)
  if ((unsigned long long)a.plan[2] != a.stamp) return;
  const long long total = a.plan[0], P = a.plan[1];
  const long long f0 = w * P;
  if (f0 >= total) return;
  const long long f1 = min(f0 + P, total);
  const int slot = lane / LPT, g = lane - slot * LPT;

  const int bar_bytes = ((nwarps * a.nstage * 12) + 127) & ~127;
  const uint32_t bar0 = smem_u32(smem) + warp * a.nstage * 8;
  unsigned char* buf = smem + bar_bytes + (size_t)warp * a.nstage * a.stage_bytes;
  const uint32_t buf0 = smem_u32(buf);
  const int v_off = a.tile * a.row_k;
  // tile length of each stage, written by the producer before its copies
  volatile int* slen = reinterpret_cast<volatile int*>(smem + nwarps * a.nstage * 8) +
                       warp * a.nstage;

  if (lane == 0) {
    for (int s = 0; s < a.nstage; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_evict_first_policy();

  const int4 st0 = in_span(a.ws_span, a.wstart + w, sizeof(int4), a.status)
                       ? a.wstart[w]
                       : make_int4(0, 0, 0, 0);
  PCursor pc{st0.x, st0.y, st0.z, 0, 0, 0, 0, 0};
  pc_load_seq(pc, a);
  pc_place(pc, a.page_size);
  PCursor cc = pc;

  // Producer (lane 0 issues). Block-table entries are cached, and the next
  // entry of the same sequence is loaded ahead so a page change seldom
  // waits on a global load. Entries past a sequence's used blocks are read
  // only as that look-ahead and never used.
  int cb = -1, cblk = -1, cpage = 0, nblk = -1, npage = 0;
  auto page_of = [&](int b, int blk) -> int {
    if (b != cb || blk != cblk) {
      cpage = (b == cb && blk == nblk)
                  ? npage
                  : __ldg(a.block_table + (size_t)b * a.max_blocks + blk);
      cb = b;
      cblk = blk;
      nblk = blk + 1 < a.max_blocks ? blk + 1 : -1;
      if (nblk >= 0) npage = __ldg(a.block_table + (size_t)b * a.max_blocks + nblk);
      // The plan checked every page it uses, but a table changed after the
      // plan was made is read here: an index outside the pool is reported
      // and replaced by page 0, so no copy leaves the pool.
      if (cpage < 0 || cpage >= a.num_pages) {
        report_status(a.status, kStatusBadPagedInput);
        cpage = 0;
      }
    }
    return cpage;
  };
  long long pf = f0;
  int ps = 0, in_flight = 0;
  auto issue = [&]() {
    const int len = pc_len(pc, pf, f1, a.tile, a.page_size);
    if (lane == 0) {
      const int page = page_of(pc.b, pc.blk);
      const long long row = ((long long)page * a.H + pc.h) * a.page_size + pc.pp;
      const uint32_t kb = (uint32_t)len * a.row_k, vb = (uint32_t)len * a.row_v;
      const uint32_t bar = bar0 + 8 * ps;
      const uint32_t dst = buf0 + ps * a.stage_bytes;
      slen[ps] = len;  // ordered before the consumer's wait by the arrive
      const char* ksrc = a.zk + row * a.row_k;
      const char* vsrc = a.zv + row * a.row_v;
      if (in_span(a.zk_span, ksrc, kb, a.status) && in_span(a.zv_span, vsrc, vb, a.status)) {
        mbar_arrive_expect_tx(bar, kb + vb);
        bulk_g2s(dst, ksrc, kb, bar, pol);
        bulk_g2s(dst + v_off, vsrc, vb, bar, pol);
      } else {
        mbar_arrive(bar);  // nothing copied: the stage completes as it is
      }
    }
    pf += len;
    pc_advance(pc, len, a);
    if (++ps == a.nstage) ps = 0;
    ++in_flight;
  };
  for (int s = 0; s < a.nstage && pf < f1; ++s) issue();

  // q' is written by k_absorb.
  pdl_wait();

  int cs = 0;
  uint32_t cpar = 0;
  long long f = f0;
  long long u = (long long)cc.b * a.H + cc.h;
  float qv[SK][E], qn[SK][E];
  load_qp<E, LPT, SK, EXACT>(qv, a.qp, u, a.r_k, a.nseg_k, g, a);
  while (f < f1) {
    const long long seg_end = min(f1, f + (cc.n - cc.i));
    long long un = -1;
    PCursor nx = cc;
    if (seg_end < f1) {  // the next unit's q' loads run under this unit's stream
      pc_next_unit(nx, a);
      un = (long long)nx.b * a.H + nx.h;
      load_qp<E, LPT, SK, EXACT>(qn, a.qp, un, a.r_k, a.nseg_k, g, a);
    }
    float m = kNegBig, l = 0.f;
    float acc[SV][E];
#pragma unroll
    for (int s = 0; s < SV; ++s)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[s][e] = 0.f;

    while (f < seg_end) {
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
      const int len = slen[cs];
      const unsigned char* Ks = buf + cs * a.stage_bytes;
      stream_tile<ESZ, LPT, SK, SV, EXACT>(Ks, Ks + v_off, len, qv, m, l, acc, a, slot, g);
      __syncwarp();
      --in_flight;
      if (pf < f1) issue();
      if (++cs == a.nstage) {
        cs = 0;
        cpar ^= 1u;
      }
      f += len;
    }
    cc = nx;

    stream_merge_write<ESZ, LPT, SV, EXACT>(m, l, acc, a.part + (size_t)(w + u) * a.pstride, a,
                                            slot, g);
    u = un;
#pragma unroll
    for (int s = 0; s < SK; ++s)
#pragma unroll
      for (int e = 0; e < E; ++e) qv[s][e] = qn[s][e];
  }
}

template <int ESZ, bool PAGED>
StreamFn pick_stream(int lpt, int sk, int sv, bool exact) {
#define LLA_KERNEL(L, SK_, SV_, EX) \
  (PAGED ? k_stream_paged<ESZ, L, SK_, SV_, EX> : k_stream<ESZ, L, SK_, SV_, EX>)
#define LLA_CASE(L, SK_, SV_, EX) \
  if (lpt == L && sk == SK_ && sv == SV_ && exact == EX) return LLA_KERNEL(L, SK_, SV_, EX);
  // every lanes-per-token count: equal K/V segment counts, exact; and the
  // generic masked kernel
  LLA_CASE(1, 1, 1, true) LLA_CASE(1, 2, 2, true) LLA_CASE(1, 3, 3, true) LLA_CASE(1, 4, 4, true)
  LLA_CASE(2, 1, 1, true) LLA_CASE(2, 2, 2, true) LLA_CASE(2, 3, 3, true) LLA_CASE(2, 4, 4, true)
  LLA_CASE(4, 1, 1, true) LLA_CASE(4, 2, 2, true) LLA_CASE(4, 3, 3, true) LLA_CASE(4, 4, 4, true)
  LLA_CASE(8, 1, 1, true) LLA_CASE(8, 2, 2, true) LLA_CASE(8, 3, 3, true) LLA_CASE(8, 4, 4, true)
  LLA_CASE(1, 4, 4, false) LLA_CASE(2, 4, 4, false) LLA_CASE(4, 4, 4, false)
  LLA_CASE(8, 4, 4, false)
  if constexpr (ESZ == 2) {
    // bf16 rows of different K and V widths (asymmetric ranks, a rotary
    // branch on the key side) at 8 lanes per token: exact when both widths
    // are multiples of 128 bytes, else masked with per-axis segment counts
    LLA_CASE(8, 1, 2, true) LLA_CASE(8, 1, 3, true) LLA_CASE(8, 1, 4, true)
    LLA_CASE(8, 2, 1, true) LLA_CASE(8, 2, 3, true) LLA_CASE(8, 2, 4, true)
    LLA_CASE(8, 3, 1, true) LLA_CASE(8, 3, 2, true) LLA_CASE(8, 3, 4, true)
    LLA_CASE(8, 4, 1, true) LLA_CASE(8, 4, 2, true) LLA_CASE(8, 4, 3, true)
    LLA_CASE(8, 1, 1, false) LLA_CASE(8, 1, 2, false) LLA_CASE(8, 1, 3, false)
    LLA_CASE(8, 1, 4, false) LLA_CASE(8, 2, 1, false) LLA_CASE(8, 2, 2, false)
    LLA_CASE(8, 2, 3, false) LLA_CASE(8, 2, 4, false) LLA_CASE(8, 3, 1, false)
    LLA_CASE(8, 3, 2, false) LLA_CASE(8, 3, 3, false) LLA_CASE(8, 3, 4, false)
    LLA_CASE(8, 4, 1, false) LLA_CASE(8, 4, 2, false) LLA_CASE(8, 4, 3, false)
    // rows of 160 bf16 (20 segments; r_v = 160 of the 96 / 160 split at 4x,
    // r = 80 at 2 lanes) exactly, five segments per lane
    LLA_CASE(4, 3, 5, true) LLA_CASE(4, 5, 3, true) LLA_CASE(4, 5, 5, true)
    LLA_CASE(2, 5, 5, true)
  }
#undef LLA_CASE
#undef LLA_KERNEL
  return nullptr;
}

}  // namespace

StreamFn pick_stream_kernel(int esz, int lpt, int sk, int sv, bool exact, bool paged) {
  if (paged)
    return esz == 2 ? pick_stream<2, true>(lpt, sk, sv, exact)
                    : pick_stream<4, true>(lpt, sk, sv, exact);
  return esz == 2 ? pick_stream<2, false>(lpt, sk, sv, exact)
                  : pick_stream<4, false>(lpt, sk, sv, exact);
}

}  // namespace lla

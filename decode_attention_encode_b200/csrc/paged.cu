// Per-head absorbed LLA decode over a paged latent store with per-sequence
// lengths (sm_100a).
//
// Source: "Looped Latent Attention: Cross-Loop KV Compression for Looped
// Transformers" (arXiv 2607.15456), §7 "Per-head LLA versus LLA-2D at
// inference" (the absorbed form) and §7 "Memory" / App. C Table 9 (LLA
// stacks with attention-sink + window eviction: the sequence keeps its first
// `sink` tokens and its last `window`). The pages measure capacity with a
// latent store; keeping it in fixed-size pages shared by sequences of
// different lengths is how a serving engine holds such a store.
//
// One call runs four kernels on the caller's stream:
//   k_plan_paged  one CTA: reads the lengths, checks every used block-table
//                 entry, forms each sequence's kept-token record, the
//                 flattened range's prefix sums, each streaming warp's share
//                 and its starting (sequence, head, token). Nothing goes back
//                 to the host.
//   k_absorb      as in the dense path.
//   k_stream_paged  the dense streaming kernel's pipeline over the page pool.
//   k_combine     as in the dense path, with the ragged piece map.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "stream.cuh"

namespace lla {
namespace {

constexpr int kPlanThreads = 1024;

struct PlanArgs {
  const int* seq_lens;
  const int* block_table;
  int B, H, page_size, num_pages, max_blocks, sink, window;
  int W;     // streaming warps (LLA-2D: CTAs)
  int pmin;  // smallest share per warp
  int tile_tokens;  // LLA-2D: the range counts tiles of this many tokens
  int4* seqinfo;
  long long* cum;
  long long* plan;
  int4* wstart;
  unsigned long long stamp;
  unsigned int* status;
  Span bt_span;  // the block table (bounds-check build)
};

// Every page index the kept positions [lo, hi) of sequence b touch lies in
// the pool. The warp's lanes check the pages together, so a long sequence in
// small pages (hundreds of table entries) costs a few round trips.
__device__ bool pages_ok(const PlanArgs& p, int b, int lo, int hi, int lane) {
  if (lo >= hi) return true;
  const int* row = p.block_table + (size_t)b * p.max_blocks;
  bool bad = false;
  for (int blk = lo / p.page_size + lane; blk <= (hi - 1) / p.page_size; blk += 32) {
    const int pg = ld_chk(row + blk, p.bt_span, p.status, -1);
    bad |= pg < 0 || pg >= p.num_pages;
  }
  return !__any_sync(0xffffffffu, bad);
}

__global__ void __launch_bounds__(kPlanThreads) k_plan_paged(PlanArgs p) {
  __shared__ long long scan[kPlanThreads];
  __shared__ long long s_total, s_P;
  const int t = threadIdx.x, lane = t & 31;
  const long long cap = (long long)p.max_blocks * p.page_size;

  // 1. per-sequence records, one warp per sequence; a sequence with a bad
  //    length or page is empty
  bool bad = false;
  for (int b = t >> 5; b < p.B; b += kPlanThreads / 32) {
    const int N = p.seq_lens[b];
    // per-head: {kept tokens n, sink part s, gap}; LLA-2D: {kept tiles n,
    // tokens, sink tiles, first window tile}
    int4 rec = make_int4(0, 0, 0, 0);
    bool ok = N >= 0 && N <= cap;
    if (ok && p.tile_tokens > 0) {
      // The kept positions are [0, sk) and [ws, N); a tile is kept when it
      // holds one, so the kept tiles are the sink tiles [0, st) and the
      // window tiles [fw, ceil(N / T)).
      const int T = p.tile_tokens;
      int sk = N, ws = N;
      if (p.window > 0 && N > p.sink + p.window) {
        sk = p.sink;
        ws = N - p.window;
      }
      const int st = (sk + T - 1) / T;
      const int fw = max(ws / T, st);
      rec = make_int4(st + max(0, (N + T - 1) / T - fw), N, st, fw);
      ok = pages_ok(p, b, 0, sk, lane) && pages_ok(p, b, ws, N, lane);
    } else if (ok) {
      int n = N, s = N, gap = 0;
      if (p.window > 0 && N > p.sink + p.window) {
        n = p.sink + p.window;
        s = p.sink;
        gap = N - n;
      }
      rec = make_int4(n, s, gap, 0);
      ok = pages_ok(p, b, 0, s, lane) && pages_ok(p, b, s + gap, N, lane);
    }
    if (!ok) {
      bad = true;
      rec = make_int4(0, 0, 0, 0);
    }
    if (lane == 0) p.seqinfo[b] = rec;
  }
  if (bad && lane == 0) report_status(p.status, kStatusBadPagedInput);
  __syncthreads();

  const int chunk = (p.B + kPlanThreads - 1) / kPlanThreads;
  const int b0 = min(p.B, t * chunk), b1 = min(p.B, b0 + chunk);
  long long sum = 0;
  for (int b = b0; b < b1; ++b) sum += (long long)p.seqinfo[b].x * p.H;

  // 2. prefix sums of the flattened (sequence, head, token) range
  scan[t] = sum;
  __syncthreads();
  for (int off = 1; off < kPlanThreads; off <<= 1) {
    const long long v = t >= off ? scan[t - off] : 0;
    __syncthreads();
    scan[t] += v;
    __syncthreads();
  }
  long long run = scan[t] - sum;
  for (int b = b0; b < b1; ++b) {
    p.cum[b] = run;
    run += (long long)p.seqinfo[b].x * p.H;
  }
  if (t == kPlanThreads - 1) {
    const long long total = scan[t];
    const long long P = max((long long)p.pmin, (total + p.W - 1) / p.W);
    p.cum[p.B] = total;
    p.plan[0] = total;
    p.plan[1] = P;
    p.plan[2] = (long long)p.stamp;  // this plan's identity, checked by its readers
    s_total = total;
    s_P = P;
  }
  __syncthreads();

  // 3. each warp's first (sequence, head, kept index)
  const long long total = s_total, P = s_P;
  for (int w = t; w < p.W; w += kPlanThreads) {
    const long long f0 = (long long)w * P;
    int4 c = make_int4(0, 0, 0, 0);
    if (f0 < total) {
      int lo = 0, hi = p.B - 1;  // the last b with cum[b] <= f0 (never empty)
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.cum[mid] <= f0) lo = mid;
        else hi = mid - 1;
      }
      const long long off = f0 - p.cum[lo];
      const int n = p.seqinfo[lo].x;
      const int h = (int)(off / n);
      c = make_int4(lo, h, (int)(off - (long long)h * n), 0);
    }
    p.wstart[w] = c;
  }
}

struct PagedPlan {
  DecodePlan d;
  size_t off_seqinfo, off_cum, off_plan, off_wstart, ws_bytes;
};

lla_status plan_paged(int B, int H, int r_k, int r_v, int esz, PagedPlan* pp) {
  PagedPlan p{};
  // kernel shape (lanes per token, tile, stages) does not depend on N
  lla_status st = plan_decode(B, H, 1, r_k, r_v, esz, &p.d);
  if (st != LLA_OK) return st;
  const DeviceInfo di = device_info();
  p.d.grid = di.sms;
  p.d.W = di.sms * p.d.warps;
  p.d.P = 0;  // set on the device
  const long long units = (long long)B * H;
  p.d.off_qp = 0;
  p.d.off_c0 = align_up((size_t)units * r_k * sizeof(float), 256);
  p.d.off_part = align_up(p.d.off_c0 + (size_t)units * sizeof(float), 256);
  p.off_seqinfo =
      align_up(p.d.off_part + (size_t)(p.d.W + units) * p.d.pstride * sizeof(float), 256);
  p.off_cum = align_up(p.off_seqinfo + (size_t)B * sizeof(int4), 256);
  p.off_plan = align_up(p.off_cum + (size_t)(B + 1) * sizeof(long long), 256);
  p.off_wstart = align_up(p.off_plan + 3 * sizeof(long long), 256);
  p.ws_bytes = align_up(p.off_wstart + (size_t)p.d.W * sizeof(int4), 256);
  p.d.ws_bytes = p.ws_bytes;
  *pp = p;
  return LLA_OK;
}

}  // namespace

unsigned long long paged_plan_stamp(int family, int esz, int B, int H, int r_k, int r_v,
                                    int page_size, int num_pages, const int* block_table,
                                    int max_blocks, const int* seq_lens, int sink, int window,
                                    int W, int pmin, int tile_tokens) {
  const unsigned long long v[] = {(unsigned long long)family, (unsigned long long)esz,
                                  (unsigned long long)B, (unsigned long long)H,
                                  (unsigned long long)r_k, (unsigned long long)r_v,
                                  (unsigned long long)page_size, (unsigned long long)num_pages,
                                  (unsigned long long)(uintptr_t)block_table,
                                  (unsigned long long)max_blocks,
                                  (unsigned long long)(uintptr_t)seq_lens,
                                  (unsigned long long)sink, (unsigned long long)window,
                                  (unsigned long long)W, (unsigned long long)pmin,
                                  (unsigned long long)tile_tokens};
  unsigned long long h = 1469598103934665603ull;  // FNV-1a, byte by byte
  for (unsigned long long x : v)
    for (int i = 0; i < 8; ++i) {
      h ^= (x >> (8 * i)) & 0xffu;
      h *= 1099511628211ull;
    }
  return h ? h : 1ull;
}

lla_status launch_plan_paged(const int* seq_lens, const int* block_table, int B, int H,
                             int page_size, int num_pages, int max_blocks, int sink, int window,
                             int W, int pmin, int tile_tokens, int4* seqinfo, long long* cum,
                             long long* plan, int4* wstart, unsigned long long stamp,
                             cudaStream_t stream) {
  PlanArgs p{};
  p.seq_lens = seq_lens;
  p.block_table = block_table;
  p.B = B;
  p.H = H;
  p.page_size = page_size;
  p.num_pages = num_pages;
  p.max_blocks = max_blocks;
  p.sink = sink;
  p.window = window;
  p.W = W;
  p.pmin = pmin;
  p.tile_tokens = tile_tokens;
  p.seqinfo = seqinfo;
  p.cum = cum;
  p.plan = plan;
  p.wstart = wstart;
  p.stamp = stamp;
  p.status = status_word();
  p.bt_span = span_of(block_table, (unsigned long long)B * max_blocks * sizeof(int));
  k_plan_paged<<<1, kPlanThreads, 0, stream>>>(p);
  return check_cuda(cudaGetLastError(), "launch k_plan_paged");
}

size_t workspace_paged(int B, int H, int r_k, int r_v, int esz) {
  PagedPlan p;
  if (plan_paged(B, H, r_k, r_v, esz, &p) != LLA_OK) return 0;
  return p.ws_bytes;
}

lla_status run_decode_paged(const float* q, const void* zk, const void* zv, int esz, int B, int H,
                            int d_h, int r_k, int r_v, int page_size, int num_pages,
                            const int* block_table, int max_blocks, const int* seq_lens, int sink,
                            int window, const float* dk, const float* dv, const float* mu_k,
                            const float* mu_v, float scale, float* out, float* lse, void* ws,
                            size_t ws_bytes, cudaStream_t stream, PagedMode mode) {
  PagedPlan pp;
  lla_status st = plan_paged(B, H, r_k, r_v, esz, &pp);
  if (st != LLA_OK) return st;
  const DecodePlan& d = pp.d;
  if (ws == nullptr || ws_bytes < pp.ws_bytes)
    return fail(LLA_ERR_WORKSPACE, "paged decode workspace needs %zu bytes, got %zu", pp.ws_bytes,
                ws_bytes);
  char* wsb = static_cast<char*>(ws);
  float* qp = reinterpret_cast<float*>(wsb + d.off_qp);
  float* c0 = reinterpret_cast<float*>(wsb + d.off_c0);
  float* part = reinterpret_cast<float*>(wsb + d.off_part);
  int4* seqinfo = reinterpret_cast<int4*>(wsb + pp.off_seqinfo);
  long long* cum = reinterpret_cast<long long*>(wsb + pp.off_cum);
  long long* plan = reinterpret_cast<long long*>(wsb + pp.off_plan);
  int4* wstart = reinterpret_cast<int4*>(wsb + pp.off_wstart);

  StreamFn fn = pick_stream_kernel(esz, d.lpt, d.sk, d.sv, d.exact, true);
  if (!fn) return fail(LLA_ERR_UNSUPPORTED, "no decode kernel for this latent shape");
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)d.smem_bytes);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(k_stream_paged)");
  const unsigned long long stamp =
      paged_plan_stamp(1, esz, B, H, r_k, r_v, page_size, num_pages, block_table, max_blocks,
                       seq_lens, sink, window, d.W, 2 * d.tile, 0);

  // 1. plan (a plain launch: it completes before k_absorb starts, so the
  //    streaming kernel may read its results before griddepcontrol.wait; a
  //    planned call relies on the plan call having been ordered before it)
  if (mode != kDecodePlanned) {
    st = launch_plan_paged(seq_lens, block_table, B, H, page_size, num_pages, max_blocks, sink,
                           window, d.W, 2 * d.tile, 0, seqinfo, cum, plan, wstart, stamp, stream);
    if (st != LLA_OK || mode == kPlanOnly) return st;
  }
  // 2. absorb (plain launch)
  st = launch_absorb(q, dk, mu_k, B, H, d_h, r_k, scale, qp, c0, stream, nullptr, 0, nullptr, 0,
                     absorb_tc(esz, B), span_of(ws, ws_bytes));
  if (st != LLA_OK) return st;
  // 3. stream
  {
    StreamArgs a{};
    a.zk = static_cast<const char*>(zk);
    a.zv = static_cast<const char*>(zv);
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
    a.zk_span = span_of(zk, (unsigned long long)num_pages * H * page_size * a.row_k);
    a.zv_span = span_of(zv, (unsigned long long)num_pages * H * page_size * a.row_v);
    a.ws_span = span_of(ws, ws_bytes);
    a.seqinfo = seqinfo;
    a.cum = cum;
    a.plan = plan;
    a.stamp = stamp;
    a.wstart = wstart;
    a.block_table = block_table;
    a.max_blocks = max_blocks;
    a.page_size = page_size;
    a.num_pages = num_pages;
    a.H = H;
    a.B = B;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
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
    if (e != cudaSuccess) return check_cuda(e, "launch k_stream_paged");
    e = record_timing(false, stream);
    if (e != cudaSuccess) return check_cuda(e, "record timing event");
  }
  // 4. combine over the ragged piece map
  RaggedMap rm{seqinfo, cum, plan, stamp};
  return launch_combine(part, d.pstride, c0, dv, mu_v, B, H, d_h, r_v, 0, 0, 0, out, lse, stream,
                        &rm, small_gemm_tc(esz, B, r_k, r_v), span_of(ws, ws_bytes));
}

}  // namespace lla

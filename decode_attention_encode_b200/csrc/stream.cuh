// Shared declarations of the per-head streaming kernel (stream.cu) and its
// host-side launcher (decode.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lla {

// Softmax bookkeeping shared by the streaming and merge kernels: scores are
// in log2 units (the absorbed query carries scale * log2(e)).
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2e = 1.44269504088896341f;
constexpr float kNegBig = -1.0e30f;
// Lazy rescaling: a slot keeps its reference maximum until a score exceeds
// it by this much (log2 units), so p_j <= 2^8 and rescales are rare.
constexpr float kRescaleSlack = 8.0f;


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
  // Paged / ragged store (paged kernels only; written by k_plan_paged):
  const int4* seqinfo;     // [B] {kept tokens n, sink part s, position gap, 0}
  const long long* cum;    // [B+1] start of sequence b in the flattened range
  const long long* plan;   // {total tokens, tokens per warp, stamp}
  unsigned long long stamp;  // plan[2] must equal it, else the kernel does nothing
  const int4* wstart;      // [W] first (b, h, i) of each warp's range
  const int* block_table;  // [B][max_blocks]
  int max_blocks, page_size, H, B;
  int num_pages;           // page indices are checked against it as they are read
  // extents for the bounds-check build: the latent stores and the workspace
  Span zk_span, zv_span, ws_span;
};

// Per-sequence record of the paged plan: sequence b attends n tokens; kept
// index i < s is position i, index i >= s is position i + gap (the sink +
// window eviction set; s = n and gap = 0 when nothing is evicted).
struct SeqInfo {
  int n, s, gap, pad;
};

using StreamFn = void (*)(StreamArgs);

// The k_stream instantiation for a latent element size (2 or 4 bytes),
// lanes per token and K / V segments per lane; exact means every lane's
// segments are in range; paged selects the paged / ragged store. nullptr if
// there is none.
StreamFn pick_stream_kernel(int esz, int lpt, int sk, int sv, bool exact, bool paged = false);

}  // namespace lla

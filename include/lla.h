/*
 * lla.h - C ABI of liblla, the B200 (sm_100a) decode hot path of Looped
 * Latent Attention (LLA).
 *
 * Source of the operations: "Looped Latent Attention: Cross-Loop KV
 * Compression for Looped Transformers" (O'Neill & Reid, arXiv 2607.15456).
 * A looped, weight-tied decoder runs T loops over D layers. For each
 * (token, layer, head, axis) LLA keeps one latent c in R^r instead of the T
 * per-loop vectors (§3 Eq. 2) and rebuilds loop t on read as
 * xhat_t = W_up,t c + mu_t (§3 Eq. 3, written here in column form). The
 * decode calls below never rebuild K or V: they use the absorbed form of §7
 * ("Per-head LLA versus LLA-2D at inference"), moving W^K_up,t onto the
 * query and applying W^V_up,t once to the latent-space value sum.
 *
 * Conventions shared by every call
 *  - All array arguments are DEVICE pointers owned by the caller. The library
 *    allocates nothing and keeps no per-call state.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream). The library never synchronises.
 *  - The decode, merge and encode calls may be captured into a CUDA graph
 *    on a capturing stream once the library has run on that device (its
 *    first call there allocates the device status word); a replay runs the
 *    same kernels on the same pointers.
 *  - Within a decode call the streaming and merge kernels are launched
 *    programmatically (they may start before the kernel ahead of them ends
 *    and wait for it before reading its results); every call's first
 *    kernel is ordered after all earlier work on the stream.
 *  - Arrays are dense, row-major, in the layouts stated per call.
 *  - A call returns LLA_OK once its kernels are queued; an argument problem
 *    found on the host returns an error before anything is launched; a launch
 *    failure returns LLA_ERR_CUDA. lla_last_error() gives a one-line reason
 *    for the last failure on the calling thread.
 *  - Device-side waits inside the kernels are bounded in time. A wait that
 *    runs out sets a sticky device status word instead of hanging; read it
 *    with lla_device_status() (which synchronises the device).
 *  - Latent element types: LLA_BF16 or LLA_F32 where stated. Decoders,
 *    queries, means and outputs are fp32.
 */
#ifndef LLA_H
#define LLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LLA_API __attribute__((visibility("default")))
#else
#define LLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LLA_OK = 0,
    LLA_ERR_INVALID_ARG = 1, /* bad size, null or misaligned pointer */
    LLA_ERR_UNSUPPORTED = 2, /* valid but outside the supported shapes */
    LLA_ERR_WORKSPACE = 3,   /* workspace missing or too small */
    LLA_ERR_CUDA = 4         /* a CUDA runtime call or launch failed */
} lla_status;

typedef enum { LLA_F32 = 0, LLA_BF16 = 1 } lla_dtype;

/* Device status bits reported by lla_device_status(). */
#define LLA_DEVICE_WAIT_TIMEOUT 0x1u     /* a bounded device wait ran out */
#define LLA_DEVICE_BAD_PAGED_INPUT 0x2u  /* a paged decode found a length or
                                            page index out of range (that
                                            sequence was treated as empty),
                                            or lla_encode_paged a token's
                                            sequence, position or page (that
                                            token was not written) */
#define LLA_DEVICE_PAGED_PLAN_MISMATCH 0x4u /* a *_paged_planned call found no
                                            plan for itself in its workspace
                                            (nothing was decoded: out = 0,
                                            lse = -inf) */
#define LLA_DEVICE_OUT_OF_BOUNDS 0x8u    /* bounds-check build only (compiled
                                            with LLA_BOUNDS_CHECK): a kernel
                                            computed a global address outside
                                            the buffer it belongs to, and did
                                            not make that access */

/* Human-readable name of a status code. Never NULL. */
LLA_API const char *lla_status_string(lla_status s);

/* One-line reason for the most recent non-OK return on this thread, or "". */
LLA_API const char *lla_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
LLA_API int lla_version(void);

/*
 * Reads (and, if `clear` is nonzero, clears) the sticky device status word
 * of the current device: 0 when no kernel has reported a problem, else a set
 * of LLA_DEVICE_* bits. Synchronises the device. Returns LLA_ERR_CUDA if the
 * runtime fails.
 */
LLA_API lla_status lla_device_status(unsigned int *status, int clear);

/*
 * Merge of attention results over disjoint parts of one context, for a
 * context split across GPUs (each GPU decodes its part of a long sequence's
 * latent store with any decode call above, the (out, lse) pairs are
 * gathered, and this call combines them):
 *   L = ln sum_r exp(lse_parts[r][u]),
 *   out[u] = sum_r exp(lse_parts[r][u] - L) out_parts[r][u],  lse[u] = L.
 * This is exact: each part's out is a convex combination of reconstructed
 * values, and the weights renormalise the parts' softmax masses (§7's
 * absorbed decode is a softmax over the union of the parts). A part with
 * lse = -inf (no token) has weight 0; if all are, out = 0 and lse = -inf.
 *   out_parts [R][U][d] fp32, lse_parts [R][U] fp32 (device); out [U][d];
 *   lse [U] or NULL. R, U, d >= 1.
 * -------------------------------------------------------------------------- */
LLA_API lla_status lla_merge_attn(const float *out_parts, const float *lse_parts,
                                  int R, long long U, int d, float *out,
                                  float *lse, void *stream);

/*
 * Self-test of the failure path of the bounded device waits. The paper has
 * no counterpart; this exists so that tests can exercise the path without a
 * fault. A one-thread kernel waits on a barrier that nothing arrives at,
 * with the same bounded wait the decode and encode kernels use, gives up
 * after timeout_us (1..1000000) microseconds and sets
 * LLA_DEVICE_WAIT_TIMEOUT in the device status word. Read and clear it with
 * lla_device_status.
 */
LLA_API lla_status lla_selftest_wait_timeout(unsigned int timeout_us, void *stream);

/*
 * Timing hook for benchmarks and profilers. When both arguments are non-NULL
 * (cudaEvent_t handles passed as void*), every later lla_decode_attn,
 * lla_decode_attn_noalloc, lla2d_decode_attn or lla_encode call made on the
 * calling thread records ev_begin on its stream just before its main kernel
 * (the latent stream, the LLA-2D tensor-core kernel, or the encoder) and
 * ev_end just after it. The recordings separate that kernel from its
 * neighbours, so launch overlap between them is lost while a hook is set.
 * Pass NULL, NULL to clear.
 */
LLA_API void lla_set_timing_events(void *ev_begin, void *ev_end);

/* --------------------------------------------------------------------------
 * Per-head absorbed decode, one (layer d, loop t) step.
 *
 * Defines (§3 Eq. 3 and the §7 absorption identities), for each batch row b
 * and head h, over the first N cached tokens j:
 *   khat_j = dk_t[h] zk[b][h][j] + mu_k_t[h]
 *   vhat_j = dv_t[h] zv[b][h][j] + mu_v_t[h]
 *   s_j    = scale * q[b][h] . khat_j
 *   out[b][h] = sum_j softmax(s)_j vhat_j,    lse[b][h] = ln sum_j exp(s_j)
 * computed as q' = scale dk_t[h]^T q, s_j = q' . zk_j + scale q . mu_k,
 * ubar = sum_j p_j zv_j, out = dv_t[h] ubar + mu_v_t[h].
 * Arithmetic is fp32. For bf16 latents with B >= 256 and a rank of 192 or
 * more, the two small products q' and dv_t ubar run on the tensor cores
 * with each fp32 operand split into two bf16 parts (hi + lo) and fp32
 * accumulation; their error stays within 3 * 2^-16 of each product term.
 *
 * Arguments
 *   q        [B][H][d_h] fp32: this loop's query of each sequence and head.
 *   zk, zv   [B][H][n_cap][r_k] and [B][H][n_cap][r_v], element type zdt
 *            (LLA_BF16 or LLA_F32): the per-head latent store of layer d.
 *            Rows [N, n_cap) are never read. 16-byte aligned.
 *   B, H     batch and heads, >= 1.
 *   d_h      head width, 1..256.
 *   N        cached tokens attended, 1 <= N <= n_cap.
 *   r_k, r_v latent ranks, multiples of 8, at most 256 (bf16) or 128 (fp32).
 *   dk_t     [H][d_h][r_k] fp32: W^K_up,t of layer d, loop t, per head.
 *            16-byte aligned.
 *   dv_t     [H][d_h][r_v] fp32: W^V_up,t. 16-byte aligned.
 *   mu_k_t, mu_v_t  [H][d_h] fp32 loop-t slices of the codec means, or NULL
 *            for zero.
 *   scale    softmax scale (usually 1/sqrt(d_h)).
 *   out      [B][H][d_h] fp32 output.
 *   lse      [B][H] fp32 natural-log normaliser, or NULL.
 *   workspace, ws_bytes  device scratch of at least
 *            lla_decode_attn_workspace(B, H, N, r_k, r_v) bytes, 16-byte
 *            aligned; its contents need no initialisation and are
 *            overwritten. Calls that share a workspace must be ordered
 *            (same stream, or synchronised).
 * The workspace size depends on the current device's SM count: query it on
 * the device that will run the call.
 * -------------------------------------------------------------------------- */
LLA_API size_t lla_decode_attn_workspace(int B, int H, int N, int r_k, int r_v);

LLA_API lla_status lla_decode_attn(const float *q, const void *zk, const void *zv,
                           lla_dtype zdt, int B, int H, int d_h, int N,
                           int n_cap, int r_k, int r_v, const float *dk_t,
                           const float *dv_t, const float *mu_k_t,
                           const float *mu_v_t, float scale, float *out,
                           float *lse, void *workspace, size_t ws_bytes,
                           void *stream);

/* --------------------------------------------------------------------------
 * Per-head absorbed decode with a decoupled rotary branch, one (layer d,
 * loop t) step.
 *
 * §7 ("Per-head LLA versus LLA-2D at inference") notes that RoPE blocks
 * exact absorption of the positional part and splits attention, MLA-style,
 * into a NoPE latent content path and a small explicit rotary branch that a
 * looped model shares across the loops of a token. Scores become
 *   s_j = scale * ( q[b][h] . khat_j + q_rope[b][h] . krope_j ),
 * with khat_j = dk_t[h] z_j + mu_k_t[h] as in lla_decode_attn; out and lse
 * are defined from s_j as there. The rotary keys are stored already rotated
 * at their own positions (they do not change between loops), and q_rope is
 * this loop's rotary query, already rotated at the current position.
 *
 * Arguments as lla_decode_attn, plus:
 *   q_rope  [B][H][d_r] fp32, 4-byte aligned.
 *   d_r     rotary width, a positive multiple of 8.
 *   zk      [B][H][n_cap][r_k + d_r]: each key row holds the r_k latent
 *           values followed by the d_r rotated rotary-key values, so one
 *           row read serves both paths. r_k + d_r obeys the rank limits of
 *           lla_decode_attn (at most 256 for bf16, 128 for fp32).
 *   workspace  at least lla_decode_attn_workspace(B, H, N, r_k + d_r, r_v)
 *           bytes.
 * -------------------------------------------------------------------------- */
LLA_API lla_status lla_decode_attn_rope(const float *q, const float *q_rope,
                                        const void *zk, const void *zv,
                                        lla_dtype zdt, int B, int H, int d_h,
                                        int d_r, int N, int n_cap, int r_k,
                                        int r_v, const float *dk_t,
                                        const float *dv_t, const float *mu_k_t,
                                        const float *mu_v_t, float scale,
                                        float *out, float *lse, void *workspace,
                                        size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * Per-head absorbed decode without a caller workspace. The paper has no
 * counterpart: this is a deployment convenience of this library.
 *
 * Some callers cannot allocate device memory: for example a plugin running
 * inside a serving engine that has already reserved the whole device for its
 * own pool, or code that must not call cudaMalloc after start-up because an
 * allocation can synchronise the device at an unpredictable point. This call
 * computes exactly what lla_decode_attn computes, with the same kernels and
 * launch plan, and takes the same arguments minus the workspace. Its scratch
 * is a fixed array of LLA_NOALLOC_SCRATCH_BYTES compiled into the library,
 * which every GPU that loads liblla holds until the process exits.
 *  - It allocates nothing and calls no allocating routine.
 *  - Shapes whose workspace (lla_decode_attn_workspace) exceeds the scratch
 *    return LLA_ERR_WORKSPACE before anything is launched.
 *  - The first call on each device looks up the scratch's device address
 *    (cudaGetSymbolAddress with that device current); make that first call
 *    before any stream capture. The lookup is repeated once after a
 *    cudaDeviceReset (a new context holds a new copy of the scratch).
 *  - Under CUDA's default lazy module loading the scratch is placed on a
 *    device when that first lookup loads it. A caller that reserves the
 *    rest of the device for its own pool should make one call at start-up,
 *    before that reservation, or set CUDA_MODULE_LOADING=EAGER.
 *  - All calls on a device share the one scratch array, and it keeps the
 *    last call's contents (nothing in it needs to start at zero). Calls
 *    whose kernels overlap on the GPU (different streams without ordering)
 *    race on it and give wrong results: order them.
 * -------------------------------------------------------------------------- */
#define LLA_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20) /* 4 MiB per device */

LLA_API lla_status lla_decode_attn_noalloc(const float *q, const void *zk,
                                           const void *zv, lla_dtype zdt, int B,
                                           int H, int d_h, int N, int n_cap,
                                           int r_k, int r_v, const float *dk_t,
                                           const float *dv_t,
                                           const float *mu_k_t,
                                           const float *mu_v_t, float scale,
                                           float *out, float *lse, void *stream);

/* --------------------------------------------------------------------------
 * Per-head absorbed decode over a paged latent store with per-sequence
 * lengths and optional attention-sink + window eviction, one (layer d,
 * loop t) step.
 *
 * Same definition as lla_decode_attn, except that sequence b attends its own
 * set of cached tokens. The pages measure capacity with a latent store whose
 * size bounds the batch (§7 "Memory", Table 7), and stack LLA with
 * StreamingLLM-style eviction (§7, App. C Table 9: 4 sink tokens plus a
 * 256-token window). Keeping the store in fixed-size pages shared by
 * sequences of different lengths is this library's layout, not the
 * paper's. The set is
 *   window == 0:                         tokens [0, N_b),
 *   window > 0 and N_b <= sink + window: tokens [0, N_b),
 *   otherwise:                           [0, sink) and [N_b - window, N_b),
 * with N_b = seq_lens[b]. A sequence with an empty set gets out = 0 and
 * lse = -inf (no attention mass; the neutral element of a log-sum-exp
 * merge). The pages leave that case undefined; this is the library's reading.
 *
 * Arguments beyond (or replacing) lla_decode_attn's:
 *   zk_pages  [num_pages][H][page_size][r_k], zv_pages
 *             [num_pages][H][page_size][r_v], element type zdt: the page
 *             pool. Token j of sequence b, head h, is row j % page_size of
 *             head h in page block_table[b][j / page_size]. 16-byte aligned.
 *   page_size tokens per page, >= 1; num_pages >= 1.
 *   block_table  [B][max_blocks] int32 device array of page indices;
 *             max_blocks >= 1 and page_size * max_blocks < 2^31. Entries of
 *             blocks holding no attended token are not read (except as a
 *             look-ahead whose value is never used) and may hold anything.
 *   seq_lens  [B] int32 device array, 0 <= N_b <= max_blocks * page_size.
 *   sink, window  eviction set as above, both >= 0.
 *   workspace, ws_bytes  at least lla_decode_attn_paged_workspace(B, H, r_k,
 *             r_v) bytes, 16-byte aligned, no initialisation needed.
 * Lengths and page indices are read only on the device: nothing is copied
 * back to the host. Before any latent is read, a device kernel checks each
 * length and every page index among the blocks of the attended set; a
 * failure sets LLA_DEVICE_BAD_PAGED_INPUT in the device status word and
 * that sequence is treated as empty. Host-side errors are as for
 * lla_decode_attn.
 * -------------------------------------------------------------------------- */
LLA_API size_t lla_decode_attn_paged_workspace(int B, int H, int r_k, int r_v);

LLA_API lla_status lla_decode_attn_paged(const float *q, const void *zk_pages,
                                         const void *zv_pages, lla_dtype zdt, int B,
                                         int H, int d_h, int r_k, int r_v,
                                         int page_size, int num_pages,
                                         const int *block_table, int max_blocks,
                                         const int *seq_lens, int sink, int window,
                                         const float *dk_t, const float *dv_t,
                                         const float *mu_k_t, const float *mu_v_t,
                                         float scale, float *out, float *lse,
                                         void *workspace, size_t ws_bytes,
                                         void *stream);

/* --------------------------------------------------------------------------
 * A paged decode step planned once. Every paged decode call first runs a
 * small plan kernel: it checks the lengths and the block-table entries in
 * use and splits the ragged token range over the streaming warps. A
 * looped model makes T x L calls per decode step over the same lengths and
 * table, so the plan can be made once per step:
 *   lla_decode_attn_paged_plan  runs only that kernel, writing the plan into
 *     the workspace (arguments as lla_decode_attn_paged; the query-side
 *     arrays are not needed);
 *   lla_decode_attn_paged_planned  is lla_decode_attn_paged without the
 *     plan kernel: it reuses the plan in its workspace.
 * The planned call must use the same workspace, zdt, B, H, r_k, r_v,
 * page_size, num_pages, block_table and seq_lens pointers, max_blocks, sink
 * and window as the plan call, be ordered after it (same stream, or
 * synchronised), and come before the lengths or the table change. The plan
 * carries a stamp of those arguments: a planned call whose workspace holds
 * no matching plan decodes nothing (out = 0, lse = -inf) and sets
 * LLA_DEVICE_PAGED_PLAN_MISMATCH. If the table's contents change after the
 * plan, a page index outside the pool is still caught as it is read (page 0
 * is read instead, and LLA_DEVICE_BAD_PAGED_INPUT is set), so no copy leaves
 * the pool; the result is then undefined. Calls that share the workspace
 * between the plan and its planned calls must not overwrite it (the plan
 * region is written only by plan calls and unplanned paged calls).
 * -------------------------------------------------------------------------- */
LLA_API lla_status lla_decode_attn_paged_plan(lla_dtype zdt, int B, int H, int r_k, int r_v,
                                              int page_size, int num_pages,
                                              const int *block_table, int max_blocks,
                                              const int *seq_lens, int sink, int window,
                                              void *workspace, size_t ws_bytes, void *stream);

LLA_API lla_status lla_decode_attn_paged_planned(const float *q, const void *zk_pages,
                                                 const void *zv_pages, lla_dtype zdt, int B,
                                                 int H, int d_h, int r_k, int r_v,
                                                 int page_size, int num_pages,
                                                 const int *block_table, int max_blocks,
                                                 const int *seq_lens, int sink, int window,
                                                 const float *dk_t, const float *dv_t,
                                                 const float *mu_k_t, const float *mu_v_t,
                                                 float scale, float *out, float *lse,
                                                 void *workspace, size_t ws_bytes,
                                                 void *stream);

/* --------------------------------------------------------------------------
 * LLA-2D absorbed decode, one (layer d, loop t) step (§3 "The LLA-2D
 * variant": one latent per token and layer, decoded into every head).
 *
 * Same definition as lla_decode_attn, except that every head reads the same
 * latents: zk [B][n_cap][r_k], zv [B][n_cap][r_v] (bf16 only). dk_t
 * [H][d_h][r_k] and dv_t [H][d_h][r_v] are the per-(head, loop) decoders.
 * The score and value contractions run on the tensor cores with bf16
 * operands (the absorbed query and the softmax weights are rounded to bf16)
 * and fp32 accumulation. The absorbed query and dv_t ubar are formed on the
 * tensor cores from split (hi + lo) bf16 operands with fp32 accumulation,
 * within 3 * 2^-16 of each product term.
 * Limits: H <= 32 (padded to 16 or 32 inside), r_k and r_v multiples of 8,
 * at most 256, d_h 1..256, 1 <= N <= n_cap. Inside, r_k is padded to whole
 * 64-column boxes and r_v to whole 128-row tiles with zeros that the tensor
 * maps supply without reading memory (the padding costs tensor-core work,
 * not HBM traffic). Outside the limits the call returns LLA_ERR_UNSUPPORTED
 * and the workspace query returns 0.
 * -------------------------------------------------------------------------- */
LLA_API size_t lla2d_decode_attn_workspace(int B, int H, int N, int r_k, int r_v);

LLA_API lla_status lla2d_decode_attn(const float *q, const void *zk, const void *zv,
                             lla_dtype zdt, int B, int H, int d_h, int N,
                             int n_cap, int r_k, int r_v, const float *dk_t,
                             const float *dv_t, const float *mu_k_t,
                             const float *mu_v_t, float scale, float *out,
                             float *lse, void *workspace, size_t ws_bytes,
                             void *stream);

/* --------------------------------------------------------------------------
 * LLA-2D absorbed decode with a decoupled rotary branch, one (layer d,
 * loop t) step: lla_decode_attn_rope's definition on the LLA-2D store.
 * Each token's key row [latent r_k | rotated rotary key d_r] is shared by
 * every head, as MLA shares its rotary key (the pages' MLA-style split of
 * §7 "Per-head LLA versus LLA-2D at inference" applied to §3 "The LLA-2D
 * variant"); q_rope [B][H][d_r] fp32 is each head's rotated rotary query.
 *   zk  [B][n_cap][r_k + d_r] bf16; zv [B][n_cap][r_v] bf16.
 *   r_k + d_r at most 384; r_k and d_r positive multiples of 8;
 *   r_v a multiple of 8, at most 256; H <= 32.
 *   workspace  lla2d_decode_attn_workspace(B, H, N, r_k + d_r, r_v) bytes
 *   (that query takes the key-row width, up to 384).
 * The rotary query is rounded to bf16 with the absorbed query for the
 * tensor cores.
 * -------------------------------------------------------------------------- */
LLA_API lla_status lla2d_decode_attn_rope(const float *q, const float *q_rope,
                                          const void *zk, const void *zv,
                                          lla_dtype zdt, int B, int H, int d_h,
                                          int d_r, int N, int n_cap, int r_k,
                                          int r_v, const float *dk_t,
                                          const float *dv_t, const float *mu_k_t,
                                          const float *mu_v_t, float scale,
                                          float *out, float *lse, void *workspace,
                                          size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * LLA-2D absorbed decode over a paged latent store with per-sequence
 * lengths, one (layer d, loop t) step: lla2d_decode_attn's definition with
 * sequence b attending its first seq_lens[b] tokens (the paged-store
 * reading of lla_decode_attn_paged, for the one-latent-per-token store).
 *   zk_pages [num_pages][page_size][r_k], zv_pages [num_pages][page_size][r_v]
 *             bf16: token j of sequence b is row j % page_size of page
 *             block_table[b][j / page_size]. 16-byte aligned.
 *   page_size a positive multiple of 64; num_pages, max_blocks >= 1. With
 *             a multiple of 128 a 128-token tile lies in one page; otherwise
 *             each 64-token half of a tile is read from its own page.
 *   block_table [B][max_blocks], seq_lens [B]: int32 device arrays, checked
 *             on the device as for lla_decode_attn_paged (a bad length or
 *             page index sets LLA_DEVICE_BAD_PAGED_INPUT and that sequence
 *             is treated as empty: out = 0, lse = -inf).
 *   sink, window  the eviction set of lla_decode_attn_paged (window 0: every
 *             token). The tensor cores take the 128-token tiles that hold a
 *             kept token and weight the others' rows by zero; only the pages
 *             of kept tokens are read or checked (with 64-token pages a tile
 *             half that holds no kept token is zero-filled, not read).
 *   workspace lla2d_decode_attn_paged_workspace(B, H, r_k, r_v) bytes.
 * Rows of a page that holds a kept token but are themselves past the
 * length or evicted may be read (the tensor cores take whole 64- or
 * 128-token boxes) and are weighted by zero: they must hold finite values,
 * as a zero-initialised pool does. Other limits as
 * lla2d_decode_attn.
 * -------------------------------------------------------------------------- */
LLA_API size_t lla2d_decode_attn_paged_workspace(int B, int H, int r_k, int r_v);

LLA_API lla_status lla2d_decode_attn_paged(const float *q, const void *zk_pages,
                                           const void *zv_pages, lla_dtype zdt,
                                           int B, int H, int d_h, int r_k, int r_v,
                                           int page_size, int num_pages,
                                           const int *block_table, int max_blocks,
                                           const int *seq_lens, int sink, int window,
                                           const float *dk_t, const float *dv_t,
                                           const float *mu_k_t, const float *mu_v_t,
                                           float scale, float *out, float *lse,
                                           void *workspace, size_t ws_bytes,
                                           void *stream);

/* The LLA-2D paged step planned once: the same pair as
 * lla_decode_attn_paged_plan / lla_decode_attn_paged_planned (and the same
 * rules), for lla2d_decode_attn_paged. The plan call takes no element type
 * (LLA-2D latents are bf16). */
LLA_API lla_status lla2d_decode_attn_paged_plan(int B, int H, int r_k, int r_v, int page_size,
                                                int num_pages, const int *block_table,
                                                int max_blocks, const int *seq_lens, int sink,
                                                int window, void *workspace, size_t ws_bytes,
                                                void *stream);

LLA_API lla_status lla2d_decode_attn_paged_planned(const float *q, const void *zk_pages,
                                                   const void *zv_pages, lla_dtype zdt, int B,
                                                   int H, int d_h, int r_k, int r_v,
                                                   int page_size, int num_pages,
                                                   const int *block_table, int max_blocks,
                                                   const int *seq_lens, int sink, int window,
                                                   const float *dk_t, const float *dv_t,
                                                   const float *mu_k_t, const float *mu_v_t,
                                                   float scale, float *out, float *lse,
                                                   void *workspace, size_t ws_bytes,
                                                   void *stream);

/* --------------------------------------------------------------------------
 * Latent write (§3 Eq. 2 over the loop-major stack of Eq. 1):
 *   z[g][n][c] = bf16_rne( sum_k (xs[k] - mu[g][k]) * W_down[g][k][c] ),
 *   xs[t*d_loop + i] = x[t][n][g][i].
 *
 * Arguments
 *   x        [T][N][G][d_loop] bf16 (xdt must be LLA_BF16): the per-loop K
 *            (or V) vectors of N finished tokens, as each loop emits them.
 *            16-byte aligned.
 *   T, N, G  loops (>= 1), tokens (>= 1), groups (heads for per-head LLA,
 *            1 for LLA-2D with d_loop = H*d_h).
 *   d_loop   per-loop width, a multiple of 64.
 *   r        latent rank, a multiple of 8, at most 256.
 *   w_down_t [G][r][T*d_loop] bf16: the encoder W_down of each group stored
 *            transposed (row c holds column c of W_down), so both operands of
 *            the tensor-core multiply are contiguous along the stacked index.
 *            16-byte aligned.
 *   mu       [G][T*d_loop] fp32 calibration mean, or NULL for zero.
 *   z        bf16 output; row n of group g starts at element
 *            g*z_group_stride + n*z_row_stride. Strides are in elements,
 *            multiples of 8, and rows must not overlap. This lets one call
 *            write each sequence's newest token straight into its slot of a
 *            [B][H][n_cap][r] store. 16-byte aligned.
 * The multiply runs on the tensor cores (bf16 operands, fp32 accumulation);
 * the mean term mu W_down is formed in fp32 and subtracted before rounding.
 * -------------------------------------------------------------------------- */
LLA_API lla_status lla_encode(const void *x, lla_dtype xdt, int T, int N, int G,
                              int d_loop, int r, const void *w_down_t,
                              const float *mu, void *z, long long z_row_stride,
                              long long z_group_stride, void *stream);

/* --------------------------------------------------------------------------
 * The mean term of the latent write, computed once per codec.
 *
 * §3 Eq. 2 subtracts the codec mean before the down-projection; since
 * (x - mu) W_down = x W_down - mu W_down and mu, W_down are fixed codec
 * parameters, b = mu W_down is a constant of the codec:
 *   muw[g][c] = sum_k mu[g][k] * W_down[g][k][c]     (fp32 accumulation)
 * lla_encode forms it inside every call, which is cheap at the per-head
 * shapes but not for a wide LLA-2D stack (K = T H d_head). Computing it once
 * here and calling lla_encode_with_bias avoids that.
 *   w_down_t  [G][r][K] bf16 (W_down transposed, as for lla_encode),
 *             16-byte aligned; K = T * d_loop, a positive multiple of 8.
 *   mu        [G][K] fp32, 16-byte aligned.
 *   muw       [G][r] fp32 output.
 * -------------------------------------------------------------------------- */
LLA_API lla_status lla_encode_bias(const void *w_down_t, const float *mu, int G,
                                   int K, int r, float *muw, void *stream);

/* lla_encode with the mean term given as muw = mu W_down (from
 * lla_encode_bias, 16-byte aligned), or NULL for a zero mean:
 *   z[g][n][c] = bf16_rne( sum_k xs[k] * W_down[g][k][c] - muw[g][c] ).
 * Arguments and limits otherwise as lla_encode, plus an optional workspace:
 * when the shape has too few 128-token tiles to occupy the GPU (a wide
 * LLA-2D stack written for one decode step's tokens), a workspace of
 * lla_encode_with_bias_workspace(...) bytes (16-byte aligned, no
 * initialisation) lets the call split the contraction over K and add the
 * fp32 partials in a second kernel. With workspace NULL, or a query result
 * of 0, the call runs unsplit. The result is the same up to fp32 summation
 * order. */
LLA_API size_t lla_encode_with_bias_workspace(int T, int N, int G, int d_loop, int r);

LLA_API lla_status lla_encode_with_bias(const void *x, lla_dtype xdt, int T, int N,
                                        int G, int d_loop, int r,
                                        const void *w_down_t, const float *muw,
                                        void *z, long long z_row_stride,
                                        long long z_group_stride, void *workspace,
                                        size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * Latent write into a paged store: lla_encode_with_bias's latents (§3 Eq. 2
 * over the loop-major stack of Eq. 1) written at each token's slot of the
 * page pool that lla_decode_attn_paged and lla2d_decode_attn_paged read.
 * A serving loop calls it once per (layer, axis) and decode step to append
 * every sequence's newest token; a chunked prefill passes many tokens of
 * one sequence. The pages measure capacity with a latent store whose size
 * bounds the batch (§7 "Memory", Table 7); the paged layout is this
 * library's, as for the paged decode calls.
 *
 * Token n belongs to sequence s = seq_idx[n] (s = n when seq_idx is NULL)
 * at position p = positions[n]. Its row c = bf16_rne(xs_n W_down - muw) of
 * group g is written to the r elements starting at
 *   z_pages + page * z_page_stride + g * z_group_stride
 *           + (p % page_size) * z_row_stride,
 *   page = block_table[s][p / page_size].
 * For a per-head pool [num_pages][H][page_size][r] (G = H) the strides are
 * (H * page_size * r, page_size * r, r); for an LLA-2D pool
 * [num_pages][page_size][r] (G = 1) they are (page_size * r, 0, r). A key
 * row [latent r_k | rotary key d_r] takes z_row_stride = r_k + d_r and
 * keeps its rotary part. Nothing else in the pool is written.
 *
 * Arguments beyond lla_encode_with_bias's (x, xdt, T, N, G, d_loop, r,
 * w_down_t, muw, workspace, ws_bytes, stream: same meaning and limits; the
 * workspace query is lla_encode_with_bias_workspace):
 *   z_pages       bf16 page pool, 16-byte aligned.
 *   z_page_stride, z_group_stride, z_row_stride  in elements, multiples of
 *                 8, z_row_stride >= r. Rows of one page must not overlap
 *                 (groups outer or rows outer), and z_page_stride must cover
 *                 a whole page: >= (G-1) z_group_stride + (page_size-1)
 *                 z_row_stride + r.
 *   page_size     tokens per page, >= 1; num_pages >= 1.
 *   block_table   [n_seq][max_blocks] int32 device array; n_seq,
 *                 max_blocks >= 1 and page_size * max_blocks < 2^31.
 *   seq_idx       [N] int32 device array, or NULL.
 *   positions     [N] int32 device array.
 * Sequence indices, positions and page indices are read only on the device.
 * A token whose sequence index lies outside [0, n_seq), whose position
 * lies outside [0, max_blocks * page_size), or whose page lies outside
 * [0, num_pages), is not written, and LLA_DEVICE_BAD_PAGED_INPUT is set in
 * the device status word. Two tokens of one call must not name the same
 * slot (their writes would race). Host-side errors as for lla_encode.
 * -------------------------------------------------------------------------- */
LLA_API lla_status lla_encode_paged(const void *x, lla_dtype xdt, int T, int N, int G,
                                    int d_loop, int r, const void *w_down_t,
                                    const float *muw, void *z_pages,
                                    long long z_page_stride, long long z_group_stride,
                                    long long z_row_stride, int page_size, int num_pages,
                                    const int *block_table, int n_seq, int max_blocks,
                                    const int *seq_idx, const int *positions,
                                    void *workspace, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LLA_H */

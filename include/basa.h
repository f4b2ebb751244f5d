/*
 * basa.h — C ABI of the BASA forward hot path on NVIDIA B200 (sm_100a).
 *
 * BASA = "Backend-Agnostic Sparse Attention for Fast High-Resolution Visual
 * Generation" (arXiv 2610.08772). One layer of BASA replaces visual
 * self-attention by attention over shifted non-overlapping windows whose key
 * set is extended with pooled global K/V, optional routed windows and text
 * tokens. Three calls make one layer:
 *
 *   basa_pool_kv          pooled global K/V            (BASA §3.2, §A.1)
 *   basa_route_windows    top-k routed windows          (BASA §3.3, §A.2)
 *   basa_window_attn_fwd  shifted-window attention      (BASA §3.1, §A.1)
 *
 * and further entry points serve the same layer:
 *
 *   basa_pool_route           the first two from one read of q, k, v
 *   basa_route_windows_noalloc  routing without a caller workspace
 *   basa_window_attn_fwd_lse  one branch of the decomposed form, with log-sum-exp
 *   basa_merge_branches       branches merged into the joint softmax  (BASA §A.1)
 *   basa_text_attn_fwd        the text queries' output rows (dense over all keys)
 *   basa_window_attn_bwd      gradients w.r.t. q, k, v                 (BASA §3.4)
 *
 * Conventions common to every entry point
 * ---------------------------------------
 * Pointers. Every tensor pointer is a DEVICE pointer owned by the caller; the
 *   library never allocates, frees, copies to the host or synchronises. Tensor
 *   pointers must be 16-byte aligned (route_idx / route_score: 4-byte).
 * Layouts (row-major, innermost last; N = T*H*W visual tokens in raster order
 *   t, y, x; Np = (T/pt)*(H/ph)*(W/pw) pooled tokens in raster order of the
 *   pooled grid; nWin = (T/wt)*(H/wh)*(W/ww)):
 *     q, out        [B, heads, N, head_dim]
 *     k, v          [B, heads, N + n_text, head_dim]   visual rows, then text rows
 *     kp, vp        [B, heads, Np, head_dim]
 *     route_idx     int32 [B, heads, nWin, routed_k]
 *     route_score   float [B, heads, nWin, routed_k]
 *   Element type: bfloat16 (BASA_BF16) or float32 (BASA_F32) for q, k, v, kp,
 *   vp and out alike.
 * Cyclic shift. The shifted grid is Xr[t,y,x] = X[(t+st)%T, (y+sy)%H, (x+sx)%W];
 *   windows are the non-overlapping wt x wh x ww blocks of Xr, numbered in
 *   raster order of the window grid. Outputs are written at the ORIGINAL (not
 *   shifted) positions.
 * Streams. All work is enqueued on `stream` (0 = legacy default stream); each
 *   call returns as soon as its kernels are launched. Calls on one stream are
 *   ordered by the stream.
 * Errors. Arguments are checked on the host before anything is launched; an
 *   invalid call returns an error code and launches nothing. A launch failure
 *   returns BASA_ERR_CUDA. No entry point aborts, traps or prints.
 * Threads. Entry points are reentrant. Library state: the lazily resolved
 *   driver entry point used to encode TMA tensor maps, a mutex-guarded cache of
 *   window tiling plans, per-device SM counts and kernel attributes set once,
 *   and the scratch array of basa_route_windows_noalloc.
 */
#ifndef BASA_H
#define BASA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *basa_stream_t; /* identical to cudaStream_t */

typedef enum {
  BASA_OK = 0,
  BASA_ERR_INVALID_ARG = 1,    /* null pointer, bad enum, negative count, misaligned pointer */
  BASA_ERR_SHAPE = 2,          /* window or pool patch does not divide the grid, shift out of range */
  BASA_ERR_UNSUPPORTED = 3,    /* valid but not built: e.g. bfloat16 attention with head_dim 64 */
  BASA_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed */
  BASA_ERR_DEVICE_TIMEOUT = 5, /* a bounded wait inside a kernel expired (reported via dev_err) */
  BASA_ERR_BAD_INDEX = 6       /* a kernel met an out-of-range route id (reported via dev_err) */
} basa_status;

typedef enum { BASA_BF16 = 0, BASA_F32 = 1 } basa_dtype;

/* Device error word bits written (atomicOr) into *dev_err by the kernels. */
#define BASA_DEVERR_TIMEOUT_PRODUCER 0x1
#define BASA_DEVERR_TIMEOUT_MMA 0x2
#define BASA_DEVERR_TIMEOUT_SOFTMAX 0x4
/* A route id outside [0, nWin): the attention kernels (forward and backward) read
 * the routed window's tokens from the query's own window instead, so nothing is
 * accessed out of bounds, and set this bit; the results are then not valid. */
#define BASA_DEVERR_BAD_ROUTE 0x8

/* Test hook for basa_params.flags: the attention kernel's loader skips the TMA
 * load of the first key tile (the bfloat16 backward: each pass skips its first
 * ring load, a key tile in the dq pass and a query tile in the dK/dV passes), so
 * every wait on it runs into its time limit and the kernel returns with
 * BASA_DEVERR_TIMEOUT_* set. Never set in normal use. */
#define BASA_FLAG_TEST_SKIP_FIRST_KEY_LOAD 0x1u

typedef struct {
  int B, heads, head_dim;  /* head_dim in {64, 128}                                    */
  int T, H, W;             /* token grid; T = 1 for images                             */
  int wt, wh, ww;          /* window extents; each divides T, H, W                     */
  int st, sy, sx;          /* per-layer cyclic shift; 0 <= s < grid extent             */
  int pt, ph, pw;          /* pool patch; all 0 = no pooled keys; else each divides    */
  int n_text;              /* text rows appended after the N visual rows of k and v   */
  int routed_k;            /* 0 = no routing; else 1 <= routed_k <= min(16, nWin - 1)  */
  basa_dtype dtype;
  int32_t *dev_err;        /* nullable DEVICE word; kernels OR BASA_DEVERR_* bits into it
                              when a bounded wait expires. Read it after the stream has
                              synchronised; map it with basa_device_error_status().    */
  uint32_t flags;          /* 0, or BASA_FLAG_TEST_* hooks                              */
  uint32_t wait_timeout_us;/* limit of each bounded wait inside the attention kernel;
                              0 = default (2,000,000 us)                               */
  int route_radius;        /* routing candidates: 0 = every other window; r >= 1 = the
                              windows whose window-grid index differs from the query
                              window's by at most r along each axis (no wrap-around).
                              routed_k must not exceed the fewest candidates any window
                              has: prod over axes of (min(r, nW_axis - 1) + 1), minus 1 */
} basa_params;

/*
 * basa_pool_kv — pooled global K/V (BASA §3.2 "K/V-pooled global memory";
 * §A.1: pooling is a regular spatial reduction of the UNSHIFTED grid).
 *
 *   kp[b,h,P,:] = mean of k[b,h,n,:] over the tokens n of patch P
 *   vp[b,h,P,:] = mean of v[b,h,n,:] over the same tokens
 * where patch P is the P-th pt x ph x pw block of the unshifted token grid in
 * raster order. Text rows are not pooled. Sums are accumulated in float32 and
 * the mean is rounded once to the element type (round to nearest even).
 * Requires pt, ph, pw > 0. Reads k, v; writes kp, vp (no aliasing allowed).
 */
basa_status basa_pool_kv(const void *k, const void *v, void *kp, void *vp,
                         const basa_params *p, basa_stream_t stream);

/*
 * basa_route_workspace_bytes — size of the caller-allocated device workspace
 * basa_route_windows needs (the float32 window means of Q and K:
 * 2 * B * heads * nWin * head_dim * 4 bytes). Returns 0 for invalid params.
 */
size_t basa_route_workspace_bytes(const basa_params *p);

/*
 * basa_route_windows — content-adaptive true-window routing (BASA §3.3; §A.2:
 * routed windows are added as uncompressed K/V to each query window).
 *
 *   Qm[w] = mean of q over the tokens of shifted window w     (float32)
 *   Km[u] = mean of k over the tokens of shifted window u     (float32)
 *   score[w,u] = Qm[w] . Km[u]  for candidates u of w: every u != w, or with
 *                route_radius = r >= 1 only those u != w whose window-grid
 *                coordinates (jt, jy, jx) differ from w's by at most r on every
 *                axis, counted without wrap-around (BASA §A.2: one routed window
 *                per query window, candidate-window radius one, in the video
 *                configuration)
 *   route_idx[b,h,w,:] = the routed_k candidates u with the largest scores,
 *                        ties to the lower id, by descending score
 *   route_score[b,h,w,:] = their scores (optional: pass NULL to skip)
 * Requires routed_k >= 1. `workspace` is a device buffer of at least
 * basa_route_workspace_bytes(p) bytes, 16-byte aligned; its contents on entry
 * are ignored and on return are the window means [2][B][heads][nWin][head_dim].
 */
basa_status basa_route_windows(const void *q, const void *k, int32_t *route_idx,
                               float *route_score, void *workspace,
                               const basa_params *p, basa_stream_t stream);

/*
 * basa_pool_route — basa_pool_kv followed by basa_route_windows, fused into one
 * read of q, k and v (BASA §3.2 pooled global K/V, §3.3 routing; the pages run
 * them as separate reductions, this pass shares the reads).
 *
 * Same results as the two calls: kp, vp as basa_pool_kv (float32 sums, one
 * rounding), route_idx / route_score as basa_route_windows (the window means are
 * summed in another fixed order, so float32 scores can differ in the last bits).
 * Requires a pool patch and routed_k >= 1. `workspace` is a device buffer of at
 * least basa_pool_route_workspace_bytes(p) bytes, 16-byte aligned; its contents
 * on entry are ignored; on return it starts with the window means
 * [2][B][heads][nWin][head_dim] (float32), followed by per-box partial sums.
 * Returns BASA_ERR_UNSUPPORTED when the shape does not fit the fused kernel
 * (then basa_pool_route_workspace_bytes returns 0); the two separate calls
 * accept every shape this one rejects for that reason.
 */
size_t basa_pool_route_workspace_bytes(const basa_params *p);
basa_status basa_pool_route(const void *q, const void *k, const void *v,
                            void *kp, void *vp, int32_t *route_idx,
                            float *route_score, void *workspace,
                            const basa_params *p, basa_stream_t stream);

/* Key groups of the branch form (basa_window_attn_fwd_lse). */
#define BASA_KEYS_WINDOWS 1u /* the query's own window and its routed windows */
#define BASA_KEYS_POOLED 2u  /* the pooled tokens kp, vp */
#define BASA_KEYS_TEXT 4u    /* the n_text text rows of k, v */
#define BASA_KEYS_ALL 7u
#define BASA_MAX_BRANCHES 4

/*
 * basa_window_attn_fwd — shifted-window attention forward (BASA §3.1 shifted
 * windows; §A.1: the local and global/text branches equal ONE softmax over the
 * concatenated K/V, which is what is computed here in a single pass).
 *
 * For every query token i of shifted window w:
 *   keys(i) = tokens of w | tokens of route_idx[b,h,w,0..routed_k-1]
 *             | the Np pooled tokens (kp, vp) | the n_text text rows of k, v
 *   out[i]  = sum_j softmax_j( q_i . k_j / sqrt(head_dim) ) v_j
 * written at token i's original grid position. Softmax statistics and
 * accumulators are float32; with BASA_BF16 the products run on the tensor
 * cores in bfloat16 and the output is rounded once to bfloat16.
 * kp, vp must be NULL iff the pool patch is all zero; route_idx must be NULL
 * iff routed_k == 0. Route ids must lie in [0, nWin); the kernel checks them and
 * reports one outside (BASA_DEVERR_BAD_ROUTE in *dev_err, see there).
 * bfloat16 requires head_dim == 128; float32 supports 64 and 128.
 */
basa_status basa_window_attn_fwd(const void *q, const void *k, const void *v,
                                 const void *kp, const void *vp,
                                 const int32_t *route_idx, void *out,
                                 const basa_params *p, basa_stream_t stream);

/*
 * basa_window_attn_fwd_lse — one branch of the decomposed form (BASA §A.1: the
 * local-window and text/global-memory branches can be evaluated separately and
 * remain equivalent to one softmax over the concatenated K/V).
 *
 * As basa_window_attn_fwd, with the key list restricted to the groups in `keys`
 * (an OR of BASA_KEYS_*; a group the layer does not have, pooled keys without a
 * pool patch or text keys with n_text == 0, adds no keys, and a selection that
 * leaves no key at all is BASA_ERR_INVALID_ARG),
 * and, when `lse` is not NULL, the log-sum-exp of each query's scaled scores:
 *   lse[b,h,i] = log sum_j exp(q_i . k_j / sqrt(head_dim))   (natural log)
 * over the selected keys, float32 [B, heads, N] at original token positions
 * (device, 4-byte aligned). keys = BASA_KEYS_ALL with lse = NULL is exactly
 * basa_window_attn_fwd. Pointer rules for kp, vp, route_idx are those of
 * basa_window_attn_fwd (pass them whenever the layer has them).
 */
basa_status basa_window_attn_fwd_lse(const void *q, const void *k, const void *v,
                                     const void *kp, const void *vp,
                                     const int32_t *route_idx, void *out, float *lse,
                                     uint32_t keys, const basa_params *p,
                                     basa_stream_t stream);

/*
 * basa_text_attn_fwd — output rows of the text queries. The pages sparsify the
 * image queries only; a text query keeps dense joint attention over every key
 * (the N visual rows and the n_text text rows of k, v; BASA §A.1's text branch
 * seen from the text side):
 *   out_text[b,h,i] = sum_j softmax_j(q_text[b,h,i] . k[b,h,j] / sqrt(head_dim)) v[b,h,j]
 * q_text, out_text: [B, heads, n_text, head_dim] (device, 16-byte aligned);
 * k, v as for basa_window_attn_fwd. Requires n_text >= 1. `workspace` (device,
 * 16-byte aligned, contents ignored) holds basa_text_attn_workspace_bytes(p)
 * bytes of per-split partial results (0 bytes: pass NULL): with bfloat16 the key
 * range is split over CTAs and the splits are merged by their log-sum-exp.
 */
size_t basa_text_attn_workspace_bytes(const basa_params *p);
basa_status basa_text_attn_fwd(const void *q_text, const void *k, const void *v,
                               void *out_text, void *workspace, const basa_params *p,
                               basa_stream_t stream);

/*
 * basa_window_attn_bwd — gradients of basa_window_attn_fwd with respect to q, k
 * and v, for the training step of the dense-teacher adaptation (BASA §3.4).
 *
 * Inputs: the forward's arguments, its output `out` and the log-sum-exp `lse`
 * of basa_window_attn_fwd_lse with BASA_KEYS_ALL, and the output gradient
 * `dout` [B, heads, N, head_dim]. With P = softmax(q K^T / sqrt(d)) over each
 * query's keys and D_i = dout_i . out_i:
 *   dS = P (dout V^T - D),  dq = dS K / sqrt(d),  dK = dS^T q / sqrt(d),  dV = P^T dout,
 * the key rows of dK, dV added back to the tokens they came from: own and routed
 * window tokens, text rows, and pooled keys spread evenly over their patch's
 * tokens (kp, vp are means). Routing is a selection and passes no gradient.
 * Outputs (overwritten): dq [B, heads, N, d], dk, dv [B, heads, N + n_text, d],
 * element type p->dtype. head_dim 128 only (BASA_ERR_UNSUPPORTED otherwise).
 * `workspace` is a device buffer of basa_window_attn_bwd_workspace_bytes(p) bytes
 * (contents on entry ignored):
 *  - BASA_BF16: tensor cores (tcgen05), 256-byte aligned workspace holding a
 *    16-byte record {lse log2(e), dout . out} per query token, per-chunk partial
 *    gradients of the pooled and text keys and the pooled keys' gradients. Every
 *    sum has a fixed order and nothing is accumulated atomically: the results are
 *    identical run to run. P and dS are rounded to bfloat16 before the tensor-core
 *    products, each output once at the end. With routing, nWin <= 4096.
 *    BASA_ERR_UNSUPPORTED when the window tiling exceeds the kernel's limits.
 *  - BASA_F32: CUDA cores, 16-byte aligned workspace for the pooled keys'
 *    gradients (NULL when that is 0); dk, dv are accumulated with atomic adds, so
 *    their last bits can differ between runs; dq cannot.
 */
size_t basa_window_attn_bwd_workspace_bytes(const basa_params *p);
basa_status basa_window_attn_bwd(const void *q, const void *k, const void *v,
                                 const void *kp, const void *vp, const int32_t *route_idx,
                                 const void *out, const float *lse, const void *dout,
                                 void *dq, void *dk, void *dv, void *workspace,
                                 const basa_params *p, basa_stream_t stream);

/*
 * basa_merge_branches — joint softmax from n branch results (BASA §A.1).
 *
 *   L[r]   = log sum_b exp(lses[b][r])
 *   out[r] = sum_b exp(lses[b][r] - L[r]) * outs[b][r]      (float32 arithmetic)
 * for every query row r of [B, heads, N]; `lse` (nullable) receives L. `outs`
 * and `lses` are HOST arrays of n (1 <= n <= BASA_MAX_BRANCHES) DEVICE pointers:
 * outs[b] like `out` of basa_window_attn_fwd (element type p->dtype, 16-byte
 * aligned), lses[b] float32 [B, heads, N]. `out` may alias outs[0] (each
 * element is read before it is written by the same thread).
 */
basa_status basa_merge_branches(int n, const void *const *outs, const float *const *lses,
                                void *out, float *lse, const basa_params *p,
                                basa_stream_t stream);

/*
 * basa_route_windows_noalloc — basa_route_windows without a caller workspace.
 * The paper has no counterpart: this is a library convenience.
 *
 * For callers that cannot allocate device memory at the point of the call: a
 * plain C host with no allocator object to carve a workspace from, a plugin in a
 * framework whose caching allocator owns the device memory (a private
 * cudaMalloc can fail or fragment its pool), or a latency-critical path where
 * cudaMalloc's implicit device synchronisation is not allowed. Same operation,
 * arguments and results as basa_route_windows, minus `workspace`; the window
 * means go to a fixed scratch array of BASA_NOALLOC_SCRATCH_BYTES (4 MiB) that
 * lives in the library's device image: every GPU that loads the library holds
 * it until the process exits.
 *
 * Limits and caveats:
 *  - basa_route_workspace_bytes(p) must be <= BASA_NOALLOC_SCRATCH_BYTES, else
 *    BASA_ERR_UNSUPPORTED is returned and nothing is launched (e.g. Wan-shaped
 *    12 heads x 140 windows x 128 needs 1.7 MiB).
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents (nothing in it needs to start at zero). Calls whose kernels
 *    overlap on the GPU (different streams, no ordering between them) race on
 *    it; order them on one stream or with events.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define BASA_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
basa_status basa_route_windows_noalloc(const void *q, const void *k, int32_t *route_idx,
                                       float *route_score, const basa_params *p,
                                       basa_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
const char *basa_status_string(basa_status s);

/* Map a device error word (read back from basa_params.dev_err) to a status:
 * 0 -> BASA_OK, BASA_DEVERR_BAD_ROUTE -> BASA_ERR_BAD_INDEX, else (a
 * BASA_DEVERR_TIMEOUT_* bit) -> BASA_ERR_DEVICE_TIMEOUT. */
basa_status basa_device_error_status(int32_t dev_err_word);

#ifdef __cplusplus
}
#endif

#endif /* BASA_H */

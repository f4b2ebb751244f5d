// Internal declarations shared by the host layer and the kernels of libbasa.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/basa.h"

namespace basa {

// ---------------------------------------------------------------------------
// Window tiling plan of the tensor-core attention kernel.
//
// A window of the shifted grid is, in the original grid, an axis-aligned block
// that wraps around the grid edge in every axis whose shift is not a multiple
// of the window extent. Along such an axis it splits into two contiguous parts
// (lengths a and w - a, a = w - (s mod w)); all windows share the same split,
// so a window is one of at most 8 "types" (wrap in t / y / x or not).
//
// For each type the host cuts the window into "pieces": boxes of at most 128
// tokens that lie inside one part per axis, so each piece is ONE TMA box load
// (the cyclic shift costs no copy, only coordinate arithmetic). Pieces are
// packed into 128-row tiles at 8-row (1024-byte) aligned offsets, which keeps
// every TMA destination aligned to the 128-byte swizzle atom. The same tiles
// serve as query tiles (M = 128 rows of the MMA) and as key/value tiles.
// ---------------------------------------------------------------------------
constexpr int kTileRows = 128;
constexpr int kMaxShapes = 8;
constexpr int kMaxPieces = 1024;
constexpr int kMaxTiles = 512;
constexpr int kMaxRouted = 16;

struct PlanShape {
  int16_t ct, cy, cx, rows;  // box extents in t, y, x and their product
};

struct PlanPiece {
  int16_t lt, ly, lx;  // offset of the piece inside the window (window-local coordinates)
  uint8_t shape;       // index into WindowPlan::shape
  uint8_t dest;        // first row of the piece inside its tile (multiple of 8)
};

struct PlanTile {
  uint16_t first_piece, n_pieces;
  uint16_t valid_rows, pad;
  uint32_t mask[4];  // bit r set = row r of the tile holds a token
};

struct PlanType {
  uint16_t first_tile, n_tiles;
};

struct WindowPlan {
  int n_shapes, n_tiles, n_pieces, max_pairs;
  int zero_fill;  // some tile leaves rows that no TMA load writes
  PlanShape shape[kMaxShapes];
  PlanType type[8];
  PlanTile tile[kMaxTiles];
  PlanPiece piece[kMaxPieces];
};

// Builds the plan. Returns BASA_ERR_UNSUPPORTED when a limit above is exceeded.
basa_status build_window_plan(const basa_params &p, WindowPlan *plan);

// Geometry helpers shared by host and device code.
struct Geo {
  int T, H, W, wt, wh, ww, st, sy, sx;
  int nWt, nWy, nWx, nWin, N;
};

__host__ __device__ inline Geo make_geo(const basa_params &p) {
  Geo g;
  g.T = p.T; g.H = p.H; g.W = p.W;
  g.wt = p.wt; g.wh = p.wh; g.ww = p.ww;
  g.st = p.st; g.sy = p.sy; g.sx = p.sx;
  g.nWt = p.T / p.wt; g.nWy = p.H / p.wh; g.nWx = p.W / p.ww;
  g.nWin = g.nWt * g.nWy * g.nWx;
  g.N = p.T * p.H * p.W;
  return g;
}

// Origin (original-grid coordinates) of shifted window `w` and its type bits
// (1 = wraps in t, 2 = wraps in y, 4 = wraps in x).
__host__ __device__ inline void window_origin(const Geo &g, int w, int *ot, int *oy, int *ox, int *type) {
  int jx = w % g.nWx;
  int jy = (w / g.nWx) % g.nWy;
  int jt = w / (g.nWx * g.nWy);
  *ot = (jt * g.wt + g.st) % g.T;
  *oy = (jy * g.wh + g.sy) % g.H;
  *ox = (jx * g.ww + g.sx) % g.W;
  *type = (*ot + g.wt > g.T ? 1 : 0) | (*oy + g.wh > g.H ? 2 : 0) | (*ox + g.ww > g.W ? 4 : 0);
}

// Driver entry point that encodes TMA tensor maps (nullptr if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// ---------------------------------------------------------------------------
// Fused pooling + window-mean pass (one read of Q, K and V).
//
// The grid is cut into boxes of e = m * pool-patch tokens per axis (whole pool
// patches, so pooled K/V are complete inside one box). Every box writes its
// pooled K/V and, for each window it meets, the partial sums of Q and K over
// box ∩ window into a slot of its own; a second kernel adds each window's slots
// in a fixed order. Window u meets boxes b0(u), b0(u)+1, ... (mod boxes per axis)
// along each axis, b0 = floor(origin / e), and its slot along that axis is the
// box's position in that run.
struct FusedPlan {
  int e[3];       // box extents (t, y, x)
  int nb[3];      // boxes per axis
  int K[3];       // slots per window per axis
  int max_cells;  // upper bound on the cells (patch ∩ window pieces) of a box
  size_t means_bytes;  // window means of Q and K: 2 * B*heads * nWin * head_dim floats
  size_t part_bytes;   // partial slots: 2 * B*heads * nWin * K[0]*K[1]*K[2] * head_dim floats
};
// BASA_OK, or BASA_ERR_UNSUPPORTED when no box fits the kernel's limits.
basa_status plan_fused(const basa_params &p, FusedPlan *fp);

// ---------------------------------------------------------------------------
// Kernel launchers (each returns BASA_OK or BASA_ERR_CUDA).
// ---------------------------------------------------------------------------
basa_status launch_pool_kv(const void *k, const void *v, void *kp, void *vp, const basa_params &p, cudaStream_t s);
basa_status launch_route(const void *q, const void *k, int32_t *route_idx, float *route_score, void *workspace,
                         const basa_params &p, cudaStream_t s);
// Routing with the library's fixed device scratch array instead of a workspace.
basa_status launch_route_noalloc(const void *q, const void *k, int32_t *route_idx, float *route_score,
                                 const basa_params &p, cudaStream_t s);
// Top-k over window means qm, km ([B*heads][nWin][head_dim] float each).
basa_status launch_topk(const float *qm, const float *km, int32_t *route_idx, float *route_score, const basa_params &p,
                        cudaStream_t s);
// Fused pooling + window means + top-k; `workspace` holds means_bytes + part_bytes.
basa_status launch_pool_route_fused(const void *q, const void *k, const void *v, void *kp, void *vp, int32_t *route_idx,
                                    float *route_score, void *workspace, const basa_params &p, cudaStream_t s);
// `lse` (nullable) receives each query's log-sum-exp; `keys` selects key groups
// (BASA_KEYS_* bits).
basa_status launch_attn_f32(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                            const int32_t *route_idx, void *out, float *lse, uint32_t keys, const basa_params &p,
                            cudaStream_t s);
basa_status launch_attn_bf16(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                             const int32_t *route_idx, void *out, float *lse, uint32_t keys, const basa_params &p,
                             cudaStream_t s);
// out = sum_b exp(lse_b - L) out_b, L = log sum_b exp(lse_b), over n branches.
basa_status launch_merge(int n, const void *const *outs, const float *const *lses, void *out, float *lse,
                         const basa_params &p, cudaStream_t s);
// The same over `rows` rows of head_dim elements, n <= kMaxMerge.
constexpr int kMaxMerge = 8;
basa_status launch_merge_rows(int n, const void *const *outs, const float *const *lses, void *out, float *lse,
                              long long rows, int head_dim, basa_dtype dtype, cudaStream_t s);
// Text-query rows (dense attention of the n_text text queries over all k/v rows).
int device_sm_count();
size_t text_attn_workspace(const basa_params &p, int sms);  // bf16 path; 0 = none needed
basa_status launch_attn_text_bf16(const void *q_text, const void *k, const void *v, void *out_text, void *workspace,
                                  const basa_params &p, int sms, cudaStream_t s);
// Backward of the attention (float32, head_dim 128): dq, dk, dv from out, lse, dout.
size_t attn_bwd_workspace(const basa_params &p);
basa_status launch_attn_bwd_f32(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                                const int32_t *route_idx, const void *out, const float *lse, const void *dout,
                                void *dq, void *dk, void *dv, void *workspace, const basa_params &p, cudaStream_t s);
// Backward of the attention, bfloat16 (tensor cores), head_dim 128; deterministic.
size_t attn_bwd_bf16_workspace(const basa_params &p);
basa_status launch_attn_bwd_bf16(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                                 const int32_t *route_idx, const void *out, const float *lse, const void *dout,
                                 void *dq, void *dk, void *dv, void *workspace, const basa_params &p, cudaStream_t s);
basa_status launch_attn_text_f32(const void *q_text, const void *k, const void *v, void *out_text,
                                 const basa_params &p, cudaStream_t s);

}  // namespace basa

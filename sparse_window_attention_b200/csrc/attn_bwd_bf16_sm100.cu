// Backward of the shifted-window attention, bfloat16, head_dim 128, for sm_100a.
//
// Gradients of out = softmax(q K^T / sqrt(d)) V over each query's key list
// [own window | routed windows | pooled | text] (BASA §3.1-§3.3, §A.1), for the
// training step of the dense-teacher adaptation (BASA §3.4). With the forward's
// log-sum-exp L and D_i = dout_i . out_i:
//   P = exp(q K^T / sqrt(d) - L),  dS = P (dout V^T - D),
//   dq = dS K / sqrt(d),  dK = dS^T q / sqrt(d),  dV = P^T dout,
// and the key rows of dK, dV go back to the tokens they came from (pooled keys
// spread evenly over their patch: kp, vp are means).
//
// Every sum has a fixed order and nothing is accumulated with atomics, so the
// results are identical run to run. Launches, in order:
//   records      per query token {-L log2(e), -D} (16-byte records, TMA-loadable with
//                the same boxes as the query tiles; negated for the packed FMA/add)
//   dq pass      one CTA per (b*head, window, query tile): the key stream of the
//                forward; q and dout copied once into TMEM, so S = q K^T and
//                dP = dout V^T read their A operand from TMEM; dS by the compute
//                warps (written over dP), dq += dS K accumulated in TMEM.
//   dK/dV long   (pooled and text key tiles, which every query of the head sees)
//                one CTA per (b*head, key tile, chunk of the head's query tiles):
//                S^T = K q^T, dP^T = V dout^T, dV += P^T dout, dK += dS^T q in TMEM;
//                fp32 partial sums per chunk.
//   reduce       chunks summed in order: pooled-key gradients (float32, for the
//                spread) and the text rows of dk, dv.
//   dK/dV window one CTA per (b*head, window u, key tile of u): the query tiles of
//                u and of every window that routed to u (ascending window id), same
//                MMAs; the epilogue adds the pooled-key gradient of each token's
//                patch / |patch| and stores dk, dv at the tokens' positions.
//
// Warp roles (320 threads): warp 0 TMA loads, warp 1 issues tcgen05 MMAs (one
// thread), warps 2-9 compute P and dS: two warpgroups, each owning 64 of the 128
// columns of a row (the backward has no row reductions, so the columns split
// freely), a thread per (row, column half). Every wait is bounded (globaltimer):
// on expiry a bit goes to dev_err and the kernel drains and returns.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "attn_sm100_common.cuh"
#include "basa_internal.h"
#include "sm100_ptx.cuh"

namespace basa {
namespace {

using namespace sm100;

enum Mode { kDq = 0, kDkvWindow = 1, kDkvLong = 2 };

constexpr int kThreads = 320;
constexpr int kMaxSlots = 5;
constexpr uint32_t kSmemRow = 0;                            // the two row tiles
constexpr uint32_t kSmemRing = 2 * kTileBytes;              // then a ring of 32 KB tiles
constexpr uint32_t kRecBytes = kTileRows * 16;              // 128 records of 16 bytes
constexpr uint32_t kCtrlBytes = 1024;
constexpr int kMaxList = 4096;                              // windows whose query tiles one key tile sees
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kColRecBytes = 8 * 128 * 4;             // per compute warp: 64 x {-L log2 e}, 64 x {-D}

// Shared memory of each pass. dq: row tiles q, dout; five ring slots (three key
// tiles, two value tiles); each thread reads its own row's record from global
// memory. dK/dV: row tiles k, v; four slots (query and dout tiles in turn); two
// record buffers for the streamed query tiles, and per compute warp its 64
// columns' records as two arrays; the window pass adds the list of windows that
// see its key tile.
template <int MODE>
struct Smem {
  static constexpr int slots = MODE == kDq ? 5 : 4;
  static constexpr uint32_t rec = kSmemRing + slots * kTileBytes;
  static constexpr uint32_t col_rec = rec + (MODE == kDq ? 0u : 2 * kRecBytes);
  static constexpr uint32_t ctrl = col_rec + (MODE == kDq ? 0u : kColRecBytes);
  static constexpr uint32_t list = ctrl + kCtrlBytes;
  static constexpr uint32_t bytes = list + (MODE == kDkvWindow ? kMaxList * 2 : 0) + 1024;  // + alignment slack
  static_assert(bytes <= 227u * 1024u, "shared memory of a pass above the 227 KB a CTA may hold");
};

struct alignas(64) BwdParams {
  CUtensorMap map_q[kMaxShapes], map_k[kMaxShapes], map_v[kMaxShapes], map_do[kMaxShapes];
  CUtensorMap map_rec[kMaxShapes];                 // per-token records {-L log2 e, -D, 0, 0}
  CUtensorMap map_dq[kMaxShapes], map_dk[kMaxShapes], map_dv[kMaxShapes];
  CUtensorMap map_kp, map_vp, map_kt, map_vt;      // pooled and text rows, 128-row boxes
  WindowPlan plan;
  const int32_t *route;
  int32_t *dev_err;
  const float4 *rec;  // the records, [bh][N] (dq pass: each thread reads its row's)
  const float *dkvp;  // final pooled-key gradients: dkp [bh][Np][128], then dvp
  float *part;        // long key tiles: [bh][tile][chunk][dK | dV][128][128] partial sums
  Geo g;
  int bh_count, routed_k, n_pool, n_text, n_pool_tiles, n_text_tiles, n_long_tiles;
  int pt, ph, pw;
  float inv_patch;
  float scale_log2;  // log2(e) / sqrt(d)
  float scale;       // 1 / sqrt(d)
  uint32_t flags;    // basa_params.flags (test hook: skip the first ring load)
  int all_full;      // every tile of the streams is full: no column masks
  int max_tiles;     // most tiles of a window type
  int n_chunks, chunk_tiles, q_tiles;  // long mode: query tiles of a head, split in chunks
  unsigned long long timeout_ns;
};
static_assert(sizeof(BwdParams) <= 32764, "window plan too large for the kernel parameter space");

struct Ctrl {
  uint64_t full[kMaxSlots], empty[kMaxSlots];
  // dq pass: a_ready, s_full[0], s_free, dp_full[0], ds_full[0]; dK/dV passes: s_full[0],
  // dp_full[0], and per compute group p_full[g], ds_full[g]
  uint64_t row_full, s_full[2], dp_full[2], s_free, a_ready, p_full[2], ds_full[2], acc_full, drain;
  uint32_t tmem_base;
  int abort;
  int n_cols;   // column tiles streamed by this CTA
  int n_list;   // dK/dV window mode: windows in the list
  int wtype[1 + kMaxRouted];
  int org[1 + kMaxRouted][3];
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");

// ------------------------------------------------------------- dq pass: the key stream
// Segments 0..routed_k are windows (own, then routed), then pooled, then text.
struct KeyIter {
  int seg, t;
};
__device__ __forceinline__ int seg_tiles(const BwdParams &P, const Ctrl &c, int seg) {
  if (seg <= P.routed_k) return P.plan.type[c.wtype[seg]].n_tiles;
  return seg == P.routed_k + 1 ? P.n_pool_tiles : P.n_text_tiles;
}
__device__ __forceinline__ void key_first(const BwdParams &P, const Ctrl &c, KeyIter &it) {
  it.seg = 0;
  it.t = 0;
  while (it.seg <= P.routed_k + 2 && seg_tiles(P, c, it.seg) == 0) ++it.seg;
}
__device__ __forceinline__ void key_next(const BwdParams &P, const Ctrl &c, KeyIter &it) {
  ++it.t;
  while (it.seg <= P.routed_k + 2 && it.t >= seg_tiles(P, c, it.seg)) {
    ++it.seg;
    it.t = 0;
  }
}
__device__ __forceinline__ uint32_t load_key(const BwdParams &P, const Ctrl &c, const KeyIter &it, bool is_v, int bh,
                                             uint8_t *dst, uint64_t *bar) {
  if (it.seg <= P.routed_k) {
    const PlanTile &tile = P.plan.tile[P.plan.type[c.wtype[it.seg]].first_tile + it.t];
    load_window_tile(P.plan, P.g, is_v ? P.map_v : P.map_k, tile, c.org[it.seg], bh, dst, bar);
    return uint32_t(tile.valid_rows) * 256u;
  }
  const bool pooled = it.seg == P.routed_k + 1;
  const CUtensorMap *map = pooled ? (is_v ? &P.map_vp : &P.map_kp) : (is_v ? &P.map_vt : &P.map_kt);
  const int row = pooled ? it.t * kTileRows : P.g.N + it.t * kTileRows;
  ptx::tma_load_3d(dst, map, bar, 0, row, bh);
  ptx::tma_load_3d(dst + kHalfBytes, map, bar, 64, row, bh);
  return kTileBytes;
}
__device__ __forceinline__ void key_mask(const BwdParams &P, const Ctrl &c, const KeyIter &it, uint32_t *m) {
  if (it.seg <= P.routed_k) {
    const PlanTile &tile = P.plan.tile[P.plan.type[c.wtype[it.seg]].first_tile + it.t];
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = tile.mask[i];
    return;
  }
  const bool pooled = it.seg == P.routed_k + 1;
  prefix_mask(min(kTileRows, (pooled ? P.n_pool : P.n_text) - it.t * kTileRows), m);
}

// ------------------------------------------------------------- dK/dV passes: the query stream
// Window list entry li (window mode: the smem list; long mode: window li itself) and
// tile t of it.
struct QIter {
  int li, t, ntiles, type, org[3];
};
__device__ __forceinline__ void q_load(const BwdParams &P, const int16_t *list, int mode, QIter &it) {
  const int w = mode == kDkvLong ? it.li : int(list[it.li]);
  window_origin(P.g, w, &it.org[0], &it.org[1], &it.org[2], &it.type);
  it.ntiles = P.plan.type[it.type].n_tiles;
}
// Positions the iterator at global query tile `skip` of the window sequence.
__device__ __forceinline__ void q_first(const BwdParams &P, const int16_t *list, int mode, int skip, QIter &it) {
  it.li = 0;
  it.t = 0;
  q_load(P, list, mode, it);
  while (skip >= it.ntiles) {
    skip -= it.ntiles;
    ++it.li;
    q_load(P, list, mode, it);
  }
  it.t = skip;
}
__device__ __forceinline__ void q_next(const BwdParams &P, const int16_t *list, int mode, int n_windows, QIter &it) {
  if (++it.t < it.ntiles) return;
  it.t = 0;
  if (++it.li < n_windows) q_load(P, list, mode, it);
}
__device__ __forceinline__ const PlanTile &q_tile(const BwdParams &P, const QIter &it) {
  return P.plan.tile[P.plan.type[it.type].first_tile + it.t];
}

// dq pass ring: key tile j in slot j % 3 (read by S(j) and, much later, dq(j)),
// value tile j in slot 3 + j % 2 (read by dP(j) only), so the next key tiles load
// while earlier ones still wait for their dq product, and value tile j + 1 loads
// while dP(j) is computed and read.
__device__ __forceinline__ int dq_slot(int j, bool is_v) { return is_v ? 3 + (j & 1) : j % 3; }
__device__ __forceinline__ uint32_t dq_phase(int j, bool is_v) { return is_v ? ((j >> 1) & 1) : ((j / 3) & 1); }

// Sets the columns whose mask bit is clear to 0 (m0: columns 0-31, m1: 32-63).
__device__ __forceinline__ void zero_masked(float (&x)[64], uint32_t m0, uint32_t m1) {
#pragma unroll
  for (int i = 0; i < 64; ++i)
    if (!(((i < 32 ? m0 : m1) >> (i & 31)) & 1u)) x[i] = 0.f;
}

// Packs 64 fp32 values (pairs 2i, 2i+1) into 32 bf16x2 words.
__device__ __forceinline__ void pack64(const float (&x)[64], uint32_t (&w)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) w[i] = ptx::pack_bf16x2(x[2 * i], x[2 * i + 1]);
}

// 64 consecutive TMEM columns of this thread's lane, as floats.
__device__ __forceinline__ void tmem_ld64f(uint32_t taddr, float (&x)[64]) {
  uint32_t r[64];
  ptx::tmem_ld64(taddr, r);
  ptx::tmem_ld_wait(r);
#pragma unroll
  for (int i = 0; i < 64; ++i) x[i] = __uint_as_float(r[i]);
}

// Writes 64 bf16 values (columns [64 half, 64 half + 64) of row `row`) into a
// swizzled 128-row staging tile.
__device__ __forceinline__ void stage_row_half(uint8_t *tile, int row, int half, const float (&x)[64]) {
  const uint32_t base = ptx::smem_u32(tile) + uint32_t(half) * kHalfBytes + uint32_t(row) * 128u;
  const uint32_t swz = row & 7;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    ptx::st_shared_v4(base + ((uint32_t(c) ^ swz) << 4), ptx::pack_bf16x2(x[8 * c], x[8 * c + 1]),
                      ptx::pack_bf16x2(x[8 * c + 2], x[8 * c + 3]), ptx::pack_bf16x2(x[8 * c + 4], x[8 * c + 5]),
                      ptx::pack_bf16x2(x[8 * c + 6], x[8 * c + 7]));
}

// Reads 64 bf16 values (columns [64 half, 64 half + 64) of row `row`) from a swizzled
// 128-row tile as 32 bf16x2 words, the layout of an MMA A operand in TMEM.
__device__ __forceinline__ void load_row_half(const uint8_t *tile, int row, int half, uint32_t (&w)[32]) {
  const uint8_t *base = tile + uint32_t(half) * kHalfBytes + uint32_t(row) * 128u;
  const uint32_t swz = row & 7;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 v = *reinterpret_cast<const uint4 *>(base + ((uint32_t(c) ^ swz) << 4));
    w[4 * c] = v.x;
    w[4 * c + 1] = v.y;
    w[4 * c + 2] = v.z;
    w[4 * c + 3] = v.w;
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_bf16_kernel(const __grid_constant__ BwdParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using L = Smem<MODE>;
  constexpr int kSlots = L::slots;
  Ctrl &c = *reinterpret_cast<Ctrl *>(smem + L::ctrl);
  int16_t *list = reinterpret_cast<int16_t *>(smem + L::list);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ----------------------------------------------------------- unit of this CTA
  int bh, w = 0, tile_idx = 0, kt = 0, chunk = 0, ot = 0, oy = 0, ox = 0, wtype = 0;
  if (MODE == kDkvLong) {
    chunk = blockIdx.x % P.n_chunks;
    kt = (blockIdx.x / P.n_chunks) % P.n_long_tiles;
    bh = blockIdx.x / (P.n_chunks * P.n_long_tiles);
  } else {
    tile_idx = blockIdx.x % P.max_tiles;
    w = (blockIdx.x / P.max_tiles) % P.g.nWin;
    bh = blockIdx.x / (P.max_tiles * P.g.nWin);
    window_origin(P.g, w, &ot, &oy, &ox, &wtype);
    if (tile_idx >= P.plan.type[wtype].n_tiles) return;  // whole CTA: this window type has fewer tiles
  }
  const int row_org[3] = {ot, oy, ox};
  const PlanTile &row_tile = P.plan.tile[P.plan.type[wtype].first_tile + tile_idx];  // window modes

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      ptx::mbar_init(&c.full[i], 1);
      ptx::mbar_init(&c.empty[i], 1);
    }
    ptx::mbar_init(&c.row_full, 1);
    const uint32_t per_group = MODE == kDq ? 256 : 128;  // compute threads that arrive
    for (int g = 0; g < 2; ++g) {
      ptx::mbar_init(&c.s_full[g], 1);
      ptx::mbar_init(&c.dp_full[g], 1);
      ptx::mbar_init(&c.p_full[g], 128);
      ptx::mbar_init(&c.ds_full[g], per_group);
    }
    ptx::mbar_init(&c.s_free, 256);
    ptx::mbar_init(&c.a_ready, 256);
    ptx::mbar_init(&c.acc_full, 1);
    ptx::mbar_init(&c.drain, 1);
    c.abort = 0;
    if (MODE == kDq) {
      c.wtype[0] = wtype;
      c.org[0][0] = ot; c.org[0][1] = oy; c.org[0][2] = ox;
      for (int r = 0; r < P.routed_k; ++r) {
        int u = P.route[((long long)bh * P.g.nWin + w) * P.routed_k + r];
        if (u < 0 || u >= P.g.nWin) {  // reported, and replaced by the own window: accesses stay in bounds
          if (P.dev_err) atomicOr(P.dev_err, BASA_DEVERR_BAD_ROUTE);
          u = w;
        }
        int a, b, d, t;
        window_origin(P.g, u, &a, &b, &d, &t);
        c.wtype[1 + r] = t;
        c.org[1 + r][0] = a; c.org[1 + r][1] = b; c.org[1 + r][2] = d;
      }
      int n = 0;
      for (int s = 0; s <= P.routed_k + 2; ++s) n += seg_tiles(P, c, s);
      c.n_cols = n;
    } else if (MODE == kDkvLong) {
      c.n_cols = max(0, min(P.chunk_tiles, P.q_tiles - chunk * P.chunk_tiles));
    }
    ptx::fence_mbar_init();
  }
  if (MODE == kDkvWindow && warp == 0) {
    // The query windows that see key tile (w, tile_idx): w itself, then every window
    // that routed to w, in ascending id (ordered ballot compaction: a fixed order).
    int n = 1;
    if (lane == 0) list[0] = int16_t(w);
    for (int w0 = 0; P.routed_k > 0 && w0 < P.g.nWin; w0 += 32) {
      const int x = w0 + lane;
      bool hit = false;
      if (x < P.g.nWin && x != w) {
        const int32_t *r = P.route + ((long long)bh * P.g.nWin + x) * P.routed_k;
        for (int i = 0; i < P.routed_k; ++i) hit |= r[i] == w;
      }
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, hit);
      if (hit) list[n + __popc(m & ((1u << lane) - 1u))] = int16_t(x);
      n += __popc(m);
    }
    __syncwarp();
    int cols = 0;
    for (int i = lane; i < n; i += 32) {
      int a, b, d, t;
      window_origin(P.g, list[i], &a, &b, &d, &t);
      cols += P.plan.type[t].n_tiles;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cols += __shfl_xor_sync(0xFFFFFFFFu, cols, o);
    if (lane == 0) {
      c.n_list = n;
      c.n_cols = cols;
    }
  }
  {
    // Rows of a tile that no TMA box writes must hold finite values (their P and dS
    // are 0, and the MMAs multiply them by 0): tiles when the plan has such rows,
    // and always the record buffers.
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const uint32_t first = P.plan.zero_fill ? kSmemRow : L::rec;
    uint4 *z = reinterpret_cast<uint4 *>(smem + first);
    for (uint32_t i = threadIdx.x; i < (L::ctrl - first) / 16; i += kThreads) z[i] = zero;
    ptx::fence_proxy_async_smem();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&c.tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const int n_cols = c.n_cols;
  const int n_windows = MODE == kDkvLong ? P.g.nWin : c.n_list;
  uint8_t *row0 = smem + kSmemRow, *row1 = smem + kSmemRow + kTileBytes;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA loader
    if (lane == 0) {
      Waiter wt{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_PRODUCER, true};
      Waiter drain{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_PRODUCER, false};
      // row tiles: dq pass q, dout; dK/dV passes k, v
      if (MODE == kDq) {
        ptx::mbar_arrive_expect_tx(&c.row_full, uint32_t(row_tile.valid_rows) * 512u);
        load_window_tile(P.plan, P.g, P.map_q, row_tile, row_org, bh, row0, &c.row_full);
        load_window_tile(P.plan, P.g, P.map_do, row_tile, row_org, bh, row1, &c.row_full);
      } else if (MODE == kDkvWindow) {
        ptx::mbar_arrive_expect_tx(&c.row_full, uint32_t(row_tile.valid_rows) * 512u);
        load_window_tile(P.plan, P.g, P.map_k, row_tile, row_org, bh, row0, &c.row_full);
        load_window_tile(P.plan, P.g, P.map_v, row_tile, row_org, bh, row1, &c.row_full);
      } else {
        const bool pooled = kt < P.n_pool_tiles;
        const CUtensorMap *mk = pooled ? &P.map_kp : &P.map_kt, *mv = pooled ? &P.map_vp : &P.map_vt;
        const int row = pooled ? kt * kTileRows : P.g.N + (kt - P.n_pool_tiles) * kTileRows;
        ptx::mbar_arrive_expect_tx(&c.row_full, 2 * kTileBytes);
        ptx::tma_load_3d(row0, mk, &c.row_full, 0, row, bh);
        ptx::tma_load_3d(row0 + kHalfBytes, mk, &c.row_full, 64, row, bh);
        ptx::tma_load_3d(row1, mv, &c.row_full, 0, row, bh);
        ptx::tma_load_3d(row1 + kHalfBytes, mv, &c.row_full, 64, row, bh);
      }
      int last = -1, last_k = -1, last_v = -1;
      bool skipped0 = false;  // test hook: the first ring item was never loaded
      if (MODE == kDq) {
        KeyIter it;
        key_first(P, c, it);
        for (int j = 0; j < n_cols; ++j) {
          bool ok = true;
          for (int kv = 0; kv < 2; ++kv) {
            const int slot = dq_slot(j, kv == 1);
            if (!wt.wait(&c.empty[slot], dq_phase(j, kv == 1) ^ 1)) { ok = false; break; }
            if (j == 0 && kv == 0 && (P.flags & BASA_FLAG_TEST_SKIP_FIRST_KEY_LOAD)) {
              skipped0 = true;
              last_k = 0;
              continue;
            }
            const uint32_t bytes = it.seg <= P.routed_k
                                       ? uint32_t(P.plan.tile[P.plan.type[c.wtype[it.seg]].first_tile + it.t].valid_rows) * 256u
                                       : kTileBytes;
            ptx::mbar_arrive_expect_tx(&c.full[slot], bytes);
            load_key(P, c, it, kv == 1, bh, smem + kSmemRing + slot * kTileBytes, &c.full[slot]);
            (kv ? last_v : last_k) = j;
          }
          if (!ok) break;
          key_next(P, c, it);
        }
      } else if (n_cols > 0) {
        QIter it;
        q_first(P, list, MODE, MODE == kDkvLong ? chunk * P.chunk_tiles : 0, it);
        for (int j = 0; j < n_cols; ++j) {
          bool ok = true;
          const PlanTile &tile = q_tile(P, it);
          for (int kv = 0; kv < 2; ++kv) {
            const int item = 2 * j + kv, slot = item % kSlots;
            if (!wt.wait(&c.empty[slot], ((item / kSlots) & 1) ^ 1)) { ok = false; break; }
            if (item == 0 && (P.flags & BASA_FLAG_TEST_SKIP_FIRST_KEY_LOAD)) {
              skipped0 = true;
              last = 0;
              continue;
            }
            uint8_t *dst = smem + kSmemRing + slot * kTileBytes;
            if (kv == 0) {  // q tile and its records (record buffer j & 1, freed with the q slot)
              ptx::mbar_arrive_expect_tx(&c.full[slot], uint32_t(tile.valid_rows) * (256u + 16u));
              load_window_tile(P.plan, P.g, P.map_q, tile, it.org, bh, dst, &c.full[slot]);
              load_window_records(P.plan, P.g, P.map_rec, tile, it.org, bh, smem + L::rec + (j & 1) * kRecBytes,
                                  &c.full[slot]);
            } else {
              ptx::mbar_arrive_expect_tx(&c.full[slot], uint32_t(tile.valid_rows) * 256u);
              load_window_tile(P.plan, P.g, P.map_do, tile, it.org, bh, dst, &c.full[slot]);
            }
            last = item;
          }
          if (!ok) break;
          q_next(P, list, MODE, n_windows, it);
        }
      }
      // Drain: wait for the copies still in flight (immediate when all were consumed).
      // A slot's earlier copies completed before the slot was granted again.
      drain.wait(&c.row_full, 0);
      if (MODE == kDq) {
        for (int j = max(0, last_k - 2); j <= last_k; ++j)
          if (j > 0 || !skipped0) drain.wait(&c.full[dq_slot(j, false)], dq_phase(j, false));
        for (int j = max(0, last_v - 1); j <= last_v; ++j) drain.wait(&c.full[dq_slot(j, true)], dq_phase(j, true));
      }
      for (int item = max(0, last - (kSlots - 1)); item <= last; ++item)
        if (item > 0 || !skipped0) drain.wait(&c.full[item % kSlots], (item / kSlots) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      Waiter wt{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_MMA, true};
      Waiter drain{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_MMA, false};
      const uint32_t r0 = kDescLoK | (ptx::smem_u32(row0) >> 4), r1 = kDescLoK | (ptx::smem_u32(row1) >> 4);
      const uint32_t ringK = kDescLoK | (ptx::smem_u32(smem + kSmemRing) >> 4);
      const uint32_t ringMn = kDescLoMn | (ptx::smem_u32(smem + kSmemRing) >> 4);
      auto slot_of = [](int item) { return uint32_t(item % kSlots) * kTileDesc; };
      bool ok = n_cols == 0 || wt.wait(&c.row_full, 0);
      if (MODE == kDq && ok && n_cols > 0) {
        // TMEM: S at 0; dP at 128, with dS written over its first halves; dq at 256; the
        // q and dout row tiles at 384 and 448 (bf16), copied there once by the compute
        // warps, so S and dP read their A operand from TMEM and only the key or value
        // tile from shared memory. Order per key tile j: S(j+1) once every thread holds
        // S(j) in registers (it runs while P(j) is computed), then dq(j) += dS(j) K_j,
        // then dP(j+1) over dS(j).
        const uint32_t tS = tmem, tDP = tmem + 128, tDQ = tmem + 256, tQ = tmem + 384, tDO = tmem + 448;
        auto kdesc = [&](int j) { return ringK + uint32_t(dq_slot(j, false)) * kTileDesc; };
        auto wait_k = [&](int j) { return wt.wait(&c.full[dq_slot(j, false)], dq_phase(j, false)); };
        auto wait_v = [&](int j) { return wt.wait(&c.full[dq_slot(j, true)], dq_phase(j, true)); };
        auto vdesc = [&](int j) { return ringK + uint32_t(dq_slot(j, true)) * kTileDesc; };
        ok = wt.wait(&c.a_ready, 0) && wait_k(0);
        if (ok) {
          ptx::tc_fence_after();
          issue_ts_kmajor(tS, tQ, kdesc(0));  // S(0) = q K0^T
          ptx::mma_commit(&c.s_full[0]);
          ok = wait_v(0);
        }
        if (ok) {
          ptx::tc_fence_after();
          issue_ts_kmajor(tDP, tDO, vdesc(0));  // dP(0) = dout V0^T
          ptx::mma_commit(&c.dp_full[0]);
          ptx::mma_commit(&c.empty[dq_slot(0, true)]);
        }
        for (int j = 0; ok && j < n_cols; ++j) {
          const bool more = j + 1 < n_cols;
          if (more) {
            if (!wt.wait(&c.s_free, j & 1) || !wait_k(j + 1)) break;
            ptx::tc_fence_after();
            issue_ts_kmajor(tS, tQ, kdesc(j + 1));  // S(j+1)
            ptx::mma_commit(&c.s_full[0]);
          }
          if (!wt.wait(&c.ds_full[0], j & 1)) break;
          ptx::tc_fence_after();
          issue_ts_split(tDQ, tDP, ringMn + uint32_t(dq_slot(j, false)) * kTileDesc, j > 0);  // dq += dS(j) K_j
          ptx::mma_commit(&c.empty[dq_slot(j, false)]);
          if (more) {
            if (!wait_v(j + 1)) break;
            ptx::tc_fence_after();
            issue_ts_kmajor(tDP, tDO, vdesc(j + 1));  // dP(j+1), after dq(j) has read dS(j)
            ptx::mma_commit(&c.dp_full[0]);
            ptx::mma_commit(&c.empty[dq_slot(j + 1, true)]);
          }
        }
      } else if (MODE != kDq && ok && n_cols > 0) {
        // TMEM: S^T at 0, dP^T at 128, dV at 256, dK at 384. Compute group g owns query
        // columns [64 g, 64 g + 64) of S^T and dP^T; the dV and dK products are issued
        // per group (the K-steps over its queries) as soon as that group's P^T or dS^T
        // is in TMEM. S^T and dP^T stay whole N = 128 products (an N = 64 half reads
        // the same A operand from shared memory for half the work).
        const uint32_t tS = tmem, tDP = tmem + 128, tDV = tmem + 256, tDK = tmem + 384;
        ok = wt.wait(&c.full[0], 0);
        if (ok) {
          ptx::tc_fence_after();
          issue_ss(tS, r0, ringK + slot_of(0));  // S^T(0) = K q0^T
          ptx::mma_commit(&c.s_full[0]);
          ok = wt.wait(&c.full[1], 0);
        }
        if (ok) {
          ptx::tc_fence_after();
          issue_ss(tDP, r1, ringK + slot_of(1));  // dP^T(0) = V dout0^T
          ptx::mma_commit(&c.dp_full[0]);
        }
        for (int j = 0; ok && j < n_cols; ++j) {
          const int qi = 2 * j, di = 2 * j + 1, qn = qi + 2, dn = di + 2;
          const bool more = j + 1 < n_cols;
          for (int g = 0; ok && g < 2; ++g) {
            ok = wt.wait(&c.p_full[g], j & 1);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_ts_group(tDV, tS, ringMn + slot_of(di), g, j > 0 || g > 0);  // dV += P^T(j) dout_j
          }
          if (!ok) break;
          ptx::mma_commit(&c.empty[di % kSlots]);
          if (more) {
            if (!wt.wait(&c.full[qn % kSlots], (qn / kSlots) & 1)) break;
            ptx::tc_fence_after();
            issue_ss(tS, r0, ringK + slot_of(qn));  // S^T(j+1): P^T(j) has been read by dV
            ptx::mma_commit(&c.s_full[0]);
          }
          for (int g = 0; ok && g < 2; ++g) {
            ok = wt.wait(&c.ds_full[g], j & 1);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_ts_group(tDK, tDP, ringMn + slot_of(qi), g, j > 0 || g > 0);  // dK += dS^T(j) q_j
          }
          if (!ok) break;
          ptx::mma_commit(&c.empty[qi % kSlots]);
          if (more) {
            if (!wt.wait(&c.full[dn % kSlots], (dn / kSlots) & 1)) break;
            ptx::tc_fence_after();
            issue_ss(tDP, r1, ringK + slot_of(dn));  // dP^T(j+1)
            ptx::mma_commit(&c.dp_full[0]);
          }
        }
      }
      ptx::mma_commit(&c.acc_full);
      // Every MMA this thread issued must finish before TMEM is freed.
      ptx::mma_commit(&c.drain);
      drain.wait(&c.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- P and dS
    const int g = (warp - 2) / 4;  // column half
    const int sub = warp % 4;      // TMEM lane quarter this warp may access
    const int row = sub * 32 + lane;
    const uint32_t lane_off = uint32_t(sub * 32) << 16;
    const uint32_t col = uint32_t(64 * g);
    Waiter wt{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_SOFTMAX, true};
    const float sl2 = P.scale_log2;
    bool ok = true;
    if (MODE == kDq) {
      const uint32_t tS = tmem + lane_off + col, tDP = tmem + lane_off + 128 + col;
      uint64_t nl2 = 0, nd2 = 0;  // this row's -L log2 e and -D, paired for packed arithmetic
      int t, y, x;                // (a padding row keeps 0, 0: its dS is 0 as its dout row is 0)
      if (n_cols > 0 && tile_row_token(P.plan, P.g, row_tile, row_org, row, &t, &y, &x)) {
        const float4 rec = P.rec[(long long)bh * P.g.N + ((long long)t * P.g.H + y) * P.g.W + x];
        nl2 = ptx::f2_pack(rec.x, rec.x);
        nd2 = ptx::f2_pack(rec.y, rec.y);
      }
      if (n_cols > 0) {
        // This row's q and dout (this group's 64 of the head dims) into TMEM, where the
        // MMAs read them as the A operand of S and dP.
        ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.row_full, 0));
        if (ok) {
          uint32_t w[32];
          load_row_half(row0, row, g, w);
          ptx::tmem_st32(tmem + lane_off + 384 + 32 * g, w);
          load_row_half(row1, row, g, w);
          ptx::tmem_st32(tmem + lane_off + 448 + 32 * g, w);
          ptx::tmem_st_wait();
          ptx::tc_fence_before();
          ptx::mbar_arrive(&c.a_ready);
        }
      }
      const uint64_t sl2x2 = ptx::f2_pack(sl2, sl2);
      KeyIter it;
      key_first(P, c, it);
      for (int j = 0; ok && j < n_cols; ++j) {
        ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.s_full[0], j & 1));
        if (!ok) break;
        ptx::tc_fence_after();
        float s[64], dp[64];
        tmem_ld64f(tS, s);
        ptx::tc_fence_before();
        ptx::mbar_arrive(&c.s_free);  // S(j) is in registers: the MMA may overwrite it
        uint32_t m[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
        if (!P.all_full) key_mask(P, c, it, m);
        const uint32_t m0 = m[2 * g], m1 = m[2 * g + 1];
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          float x0, x1;
          ptx::f2_unpack(ptx::ffma2(ptx::f2_pack(s[i], s[i + 1]), sl2x2, nl2), x0, x1);
          s[i] = ptx::ex2(x0);
          s[i + 1] = ptx::ex2(x1);
        }
        ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.dp_full[0], j & 1));
        if (!ok) break;
        ptx::tc_fence_after();
        tmem_ld64f(tDP, dp);
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          float d0, d1;
          ptx::f2_unpack(ptx::fmul2(ptx::f2_pack(s[i], s[i + 1]), ptx::fadd2(ptx::f2_pack(dp[i], dp[i + 1]), nd2)), d0,
                         d1);
          s[i] = d0;
          s[i + 1] = d1;
        }
        if ((m0 & m1) != 0xFFFFFFFFu) zero_masked(s, m0, m1);  // warp-uniform: a partial key tile
        uint32_t pk[32];
        pack64(s, pk);
        ptx::tmem_st32(tDP, pk);  // dS (bf16) over the first half of this thread's dP columns
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&c.ds_full[0]);
        key_next(P, c, it);
      }
      if (ok) ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.acc_full, 0));
      if (ok) {
        ptx::tc_fence_after();
        float x[64];
        tmem_ld64f(tmem + lane_off + 256 + col, x);
#pragma unroll
        for (int i = 0; i < 64; ++i) x[i] *= P.scale;
        stage_row_half(row0, row, g, x);  // the q tile is no longer read
        ptx::fence_proxy_async_smem();
      }
      ptx::named_barrier(1, 256);
      if (threadIdx.x == 64 && ok && !*reinterpret_cast<volatile int *>(&c.abort)) {
        store_window_tile(P.plan, P.g, P.map_dq, row_tile, row_org, bh, row0);
        ptx::tma_store_commit();
        ptx::tma_store_wait_read_all();
      }
    } else {
      const uint32_t tS = tmem + lane_off + col, tDP = tmem + lane_off + 128 + col;
      float *wrec = reinterpret_cast<float *>(smem + L::col_rec) + (warp - 2) * 128;  // [-L log2 e x 64 | -D x 64]
      const float4 *nl4 = reinterpret_cast<const float4 *>(wrec), *nd4 = reinterpret_cast<const float4 *>(wrec + 64);
      QIter it;
      if (n_cols > 0) q_first(P, list, MODE, MODE == kDkvLong ? chunk * P.chunk_tiles : 0, it);
      for (int j = 0; ok && j < n_cols; ++j) {
        ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.s_full[0], j & 1));
        if (!ok) break;
        ptx::tc_fence_after();
        float p[64];
        tmem_ld64f(tS, p);
        {
          // This warp's 64 query records {-L log2 e, -D, 0, 0}, one load per lane
          // for two columns, rewritten as two arrays that the loops below read four
          // values at a time.
          const float4 *r = reinterpret_cast<const float4 *>(smem + L::rec + (j & 1) * kRecBytes) + col;
          const float4 a = r[lane], b = r[32 + lane];
          __syncwarp();  // every lane has read the previous tile's arrays
          wrec[lane] = a.x;
          wrec[32 + lane] = b.x;
          wrec[64 + lane] = a.y;
          wrec[96 + lane] = b.y;
          __syncwarp();
        }
        uint32_t m0 = 0xFFFFFFFFu, m1 = 0xFFFFFFFFu;
        if (!P.all_full) {
          const PlanTile &qt = q_tile(P, it);
          m0 = qt.mask[2 * g];
          m1 = qt.mask[2 * g + 1];
        }
        const uint64_t sl2x2 = ptx::f2_pack(sl2, sl2);
#pragma unroll
        for (int i = 0; i < 64; i += 4) {
          const float4 nl = nl4[i / 4];
          float x0, x1, x2, x3;
          ptx::f2_unpack(ptx::ffma2(ptx::f2_pack(p[i], p[i + 1]), sl2x2, ptx::f2_pack(nl.x, nl.y)), x0, x1);
          ptx::f2_unpack(ptx::ffma2(ptx::f2_pack(p[i + 2], p[i + 3]), sl2x2, ptx::f2_pack(nl.z, nl.w)), x2, x3);
          p[i] = ptx::ex2(x0);
          p[i + 1] = ptx::ex2(x1);
          p[i + 2] = ptx::ex2(x2);
          p[i + 3] = ptx::ex2(x3);
        }
        const bool partial = (m0 & m1) != 0xFFFFFFFFu;  // warp-uniform: a partial query tile
        if (partial) zero_masked(p, m0, m1);
        uint32_t pk[32];
        pack64(p, pk);
        ptx::tmem_st32(tS, pk);  // P^T (bf16) over the first half of this thread's S^T columns
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&c.p_full[g]);
        ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.dp_full[0], j & 1));
        if (!ok) break;
        ptx::tc_fence_after();
        float dp[64];
        tmem_ld64f(tDP, dp);
#pragma unroll
        for (int i = 0; i < 64; i += 4) {
          const float4 nd = nd4[i / 4];
          float d0, d1, d2, d3;
          ptx::f2_unpack(ptx::fmul2(ptx::f2_pack(p[i], p[i + 1]),
                                    ptx::fadd2(ptx::f2_pack(dp[i], dp[i + 1]), ptx::f2_pack(nd.x, nd.y))),
                         d0, d1);
          ptx::f2_unpack(ptx::fmul2(ptx::f2_pack(p[i + 2], p[i + 3]),
                                    ptx::fadd2(ptx::f2_pack(dp[i + 2], dp[i + 3]), ptx::f2_pack(nd.z, nd.w))),
                         d2, d3);
          dp[i] = d0;
          dp[i + 1] = d1;
          dp[i + 2] = d2;
          dp[i + 3] = d3;
        }
        if (partial) zero_masked(dp, m0, m1);  // dS = 0 there whatever dP holds
        pack64(dp, pk);
        ptx::tmem_st32(tDP, pk);  // dS^T (bf16) over the first half of this thread's dP^T columns
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&c.ds_full[g]);
        q_next(P, list, MODE, n_windows, it);
      }
      if (ok) ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.acc_full, 0));
      if (ok) {
        ptx::tc_fence_after();
        float dv[64], dk[64];
        if (n_cols > 0) {
          tmem_ld64f(tmem + lane_off + 256 + col, dv);
          tmem_ld64f(tmem + lane_off + 384 + col, dk);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) dv[i] = dk[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 64; ++i) dk[i] *= P.scale;
        if (MODE == kDkvLong) {
          // partial sums of this chunk, float32 [dK | dV][row][128]
          float *dst = P.part + ((((long long)bh * P.n_long_tiles + kt) * P.n_chunks + chunk) * 2) * (kTileRows * 128);
          float4 *pk4 = reinterpret_cast<float4 *>(dst + row * 128 + col);
          float4 *pv4 = reinterpret_cast<float4 *>(dst + kTileRows * 128 + row * 128 + col);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            pk4[i] = make_float4(dk[4 * i], dk[4 * i + 1], dk[4 * i + 2], dk[4 * i + 3]);
            pv4[i] = make_float4(dv[4 * i], dv[4 * i + 1], dv[4 * i + 2], dv[4 * i + 3]);
          }
        } else {
          int t, y, x;
          if (P.n_pool > 0 && tile_row_token(P.plan, P.g, row_tile, row_org, row, &t, &y, &x)) {
            // the pooled keys' gradient of this token's patch, spread evenly
            const int pidx = ((t / P.pt) * (P.g.H / P.ph) + y / P.ph) * (P.g.W / P.pw) + x / P.pw;
            const float4 *gk = reinterpret_cast<const float4 *>(P.dkvp + ((long long)bh * P.n_pool + pidx) * 128 + col);
            const float4 *gv = reinterpret_cast<const float4 *>(
                P.dkvp + ((long long)(P.bh_count + bh) * P.n_pool + pidx) * 128 + col);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float4 a = gk[i], b = gv[i];
              dk[4 * i] += a.x * P.inv_patch; dk[4 * i + 1] += a.y * P.inv_patch;
              dk[4 * i + 2] += a.z * P.inv_patch; dk[4 * i + 3] += a.w * P.inv_patch;
              dv[4 * i] += b.x * P.inv_patch; dv[4 * i + 1] += b.y * P.inv_patch;
              dv[4 * i + 2] += b.z * P.inv_patch; dv[4 * i + 3] += b.w * P.inv_patch;
            }
          }
          stage_row_half(row0, row, g, dk);  // the k and v tiles are no longer read
          stage_row_half(row1, row, g, dv);
          ptx::fence_proxy_async_smem();
        }
      }
      ptx::named_barrier(1, 256);
      if (MODE == kDkvWindow && threadIdx.x == 64 && ok && !*reinterpret_cast<volatile int *>(&c.abort)) {
        store_window_tile(P.plan, P.g, P.map_dk, row_tile, row_org, bh, row0);
        store_window_tile(P.plan, P.g, P.map_dv, row_tile, row_org, bh, row1);
        ptx::tma_store_commit();
        ptx::tma_store_wait_read_all();
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Per query token: {-L log2(e), -(dout . out), 0, 0}, two tokens per warp (16 lanes x
// 8 bf16 each), float32 sums in a fixed order.
__global__ void __launch_bounds__(256) bwd_records_kernel(const __nv_bfloat16 *out, const __nv_bfloat16 *dout,
                                                          const float *lse, float4 *rec, long long rows) {
  const long long r = (long long)blockIdx.x * 16 + threadIdx.x / 16;
  const int part = threadIdx.x % 16;
  float acc = 0.f;
  if (r < rows) {
    const uint4 a = reinterpret_cast<const uint4 *>(out + r * 128)[part];
    const uint4 b = reinterpret_cast<const uint4 *>(dout + r * 128)[part];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(aw[i] << 16), __uint_as_float(bw[i] << 16), acc);
      acc = fmaf(__uint_as_float(aw[i] & 0xFFFF0000u), __uint_as_float(bw[i] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (r < rows && part == 0) rec[r] = make_float4(-lse[r] * 1.4426950408889634f, -acc, 0.f, 0.f);
}

// Sums the chunks of the long key tiles in order: pooled rows -> dkvp (float32),
// text rows -> dk, dv (bf16, rows N.. of each b*head).
__global__ void __launch_bounds__(256) bwd_reduce_kernel(const float *part, float *dkvp, __nv_bfloat16 *dk,
                                                         __nv_bfloat16 *dv, int bh_count, int n_long, int n_chunks,
                                                         int n_pool, int n_pool_tiles, int n_text, long long N) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // (bh, tile, row, 4-column group)
  const long long total = (long long)bh_count * n_long * kTileRows * 32;
  if (idx >= total) return;
  const int c4 = int(idx % 32);
  const int row = int((idx / 32) % kTileRows);
  const int tile = int((idx / (32 * kTileRows)) % n_long);
  const int bh = int(idx / (32LL * kTileRows * n_long));
  const bool pooled = tile < n_pool_tiles;
  const int r = (pooled ? tile : tile - n_pool_tiles) * kTileRows + row;
  if (r >= (pooled ? n_pool : n_text)) return;
  float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
  const float *base = part + (((long long)bh * n_long + tile) * n_chunks) * 2 * (kTileRows * 128);
  for (int ch = 0; ch < n_chunks; ++ch) {
    const float *p = base + (long long)ch * 2 * (kTileRows * 128) + row * 128 + c4 * 4;
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + kTileRows * 128);
    sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
    sv.x += b.x; sv.y += b.y; sv.z += b.z; sv.w += b.w;
  }
  if (pooled) {
    *reinterpret_cast<float4 *>(dkvp + ((long long)bh * n_pool + r) * 128 + c4 * 4) = sk;
    *reinterpret_cast<float4 *>(dkvp + ((long long)bh_count * n_pool + (long long)bh * n_pool + r) * 128 + c4 * 4) = sv;
  } else {
    const long long o = ((long long)bh * (N + n_text) + N + r) * 128 + c4 * 4;
    reinterpret_cast<uint2 *>(dk + o)[0] = make_uint2(ptx::pack_bf16x2(sk.x, sk.y), ptx::pack_bf16x2(sk.z, sk.w));
    reinterpret_cast<uint2 *>(dv + o)[0] = make_uint2(ptx::pack_bf16x2(sv.x, sv.y), ptx::pack_bf16x2(sv.z, sv.w));
  }
}

// ----------------------------------------------------------------- host side
struct BwdLayout {
  size_t rec, part, dkvp, total;
  int n_long, n_chunks, chunk_tiles, q_tiles;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Query tiles per head: the sum over windows of their type's tile count.
int head_query_tiles(const basa_params &p, const WindowPlan &plan) {
  const Geo g = make_geo(p);
  int n = 0;
  for (int w = 0; w < g.nWin; ++w) {
    int a, b, d, t;
    window_origin(g, w, &a, &b, &d, &t);
    n += plan.type[t].n_tiles;
  }
  return n;
}

// Chunking of the pooled / text key tiles' query range: the chunk count n (at
// least 4 query tiles per chunk) that minimises the estimated time of the launch,
// waves x (tiles per chunk + a CTA's fixed start and end cost in tiles), for a
// 148-SM part. It depends on the shape only, so the workspace size and the order of
// the chunk sums (hence the bits of the results) are the same on every device.
constexpr long long kLongSms = 148;
constexpr double kLongCtaCostTiles = 3.5;
BwdLayout bwd_layout(const basa_params &p, const WindowPlan &plan) {
  BwdLayout L{};
  const long long bh = (long long)p.B * p.heads;
  const long long N = (long long)p.T * p.H * p.W;
  const int n_pool = p.pt > 0 ? (p.T / p.pt) * (p.H / p.ph) * (p.W / p.pw) : 0;
  L.n_long = (n_pool + kTileRows - 1) / kTileRows + (p.n_text + kTileRows - 1) / kTileRows;
  L.q_tiles = head_query_tiles(p, plan);
  L.n_chunks = 1;
  L.chunk_tiles = L.q_tiles;
  if (L.n_long > 0 && L.q_tiles > 0) {
    const long long units = bh * L.n_long;
    double best = -1.0;
    for (int n = 1; n <= std::max(1, L.q_tiles / 4); ++n) {
      const int tiles = (L.q_tiles + n - 1) / n;
      const int chunks = (L.q_tiles + tiles - 1) / tiles;
      const double cost = double((units * chunks + kLongSms - 1) / kLongSms) * (tiles + kLongCtaCostTiles);
      if (best < 0.0 || cost < best) {
        best = cost;
        L.chunk_tiles = tiles;
        L.n_chunks = chunks;
      }
    }
  }
  L.rec = align256(size_t(bh) * N * 16);
  L.part = align256(size_t(bh) * L.n_long * L.n_chunks * 2 * kTileRows * 128 * sizeof(float));
  L.dkvp = align256(size_t(bh) * n_pool * 128 * sizeof(float) * 2);
  L.total = L.rec + L.part + L.dkvp;
  return L;
}

template <int MODE>
basa_status run_bwd(const BwdParams &P, long long blocks, cudaStream_t s) {
  if (blocks <= 0) return BASA_OK;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(attn_bwd_bf16_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem<MODE>::bytes) !=
      cudaSuccess)
    return BASA_ERR_CUDA;
  attn_bwd_bf16_kernel<MODE><<<unsigned(blocks), kThreads, Smem<MODE>::bytes, s>>>(P);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

}  // namespace

size_t attn_bwd_bf16_workspace(const basa_params &p) {
  static thread_local WindowPlan plan;  // large: kept off the stack
  if (build_window_plan(p, &plan) != BASA_OK) return 0;
  return bwd_layout(p, plan).total;
}

basa_status launch_attn_bwd_bf16(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                                 const int32_t *route_idx, const void *out, const float *lse, const void *dout,
                                 void *dq, void *dk, void *dv, void *workspace, const basa_params &p, cudaStream_t s) {
  if (!tensor_map_encoder()) return BASA_ERR_CUDA;
  static thread_local BwdParams P;  // large: kept off the stack
  std::memset(&P, 0, sizeof(P));
  basa_status st = build_window_plan(p, &P.plan);
  if (st != BASA_OK) return st;
  const BwdLayout L = bwd_layout(p, P.plan);
  P.g = make_geo(p);
  if (p.routed_k > 0 && P.g.nWin > kMaxList) return BASA_ERR_UNSUPPORTED;
  const long long N = P.g.N, kv_rows = N + p.n_text, bh = (long long)p.B * p.heads;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float4 *rec = reinterpret_cast<float4 *>(ws);
  P.part = reinterpret_cast<float *>(ws + L.rec);
  float *dkvp = reinterpret_cast<float *>(ws + L.rec + L.part);
  P.dkvp = dkvp;
  P.rec = rec;
  for (int i = 0; i < P.plan.n_shapes; ++i) {
    const PlanShape &sh = P.plan.shape[i];
    if (!encode_grid_map(&P.map_q[i], q, p, N, sh) || !encode_grid_map(&P.map_k[i], k, p, kv_rows, sh) ||
        !encode_grid_map(&P.map_v[i], v, p, kv_rows, sh) || !encode_grid_map(&P.map_do[i], dout, p, N, sh) ||
        !encode_record_map(&P.map_rec[i], rec, p, sh) || !encode_grid_map(&P.map_dq[i], dq, p, N, sh) ||
        !encode_grid_map(&P.map_dk[i], dk, p, kv_rows, sh) || !encode_grid_map(&P.map_dv[i], dv, p, kv_rows, sh))
      return BASA_ERR_CUDA;
  }
  P.n_pool = p.pt > 0 ? (p.T / p.pt) * (p.H / p.ph) * (p.W / p.pw) : 0;
  P.n_text = p.n_text;
  if (P.n_pool > 0 && (!encode_rows_map(&P.map_kp, kp, p, P.n_pool) || !encode_rows_map(&P.map_vp, vp, p, P.n_pool)))
    return BASA_ERR_CUDA;
  if (p.n_text > 0 && (!encode_rows_map(&P.map_kt, k, p, kv_rows) || !encode_rows_map(&P.map_vt, v, p, kv_rows)))
    return BASA_ERR_CUDA;
  P.n_pool_tiles = (P.n_pool + kTileRows - 1) / kTileRows;
  P.n_text_tiles = (p.n_text + kTileRows - 1) / kTileRows;
  P.n_long_tiles = L.n_long;
  P.route = route_idx;
  P.bh_count = int(bh);
  P.dev_err = p.dev_err;
  P.routed_k = p.routed_k;
  P.pt = std::max(p.pt, 1);
  P.ph = std::max(p.ph, 1);
  P.pw = std::max(p.pw, 1);
  P.inv_patch = p.pt > 0 ? 1.0f / float(p.pt * p.ph * p.pw) : 0.f;
  P.scale_log2 = float(1.4426950408889634 / std::sqrt(double(p.head_dim)));
  P.scale = float(1.0 / std::sqrt(double(p.head_dim)));
  P.all_full = (P.n_pool % kTileRows == 0) && (p.n_text % kTileRows == 0);
  P.max_tiles = 0;
  for (int i = 0; i < P.plan.n_tiles; ++i) P.all_full &= P.plan.tile[i].valid_rows == kTileRows;
  for (int t = 0; t < 8; ++t) P.max_tiles = std::max<int>(P.max_tiles, P.plan.type[t].n_tiles);
  P.n_chunks = L.n_chunks;
  P.chunk_tiles = L.chunk_tiles;
  P.q_tiles = L.q_tiles;
  P.timeout_ns = (p.wait_timeout_us ? (unsigned long long)p.wait_timeout_us : 2000000ull) * 1000ull;
  P.flags = p.flags;

  const long long rows = bh * N;
  bwd_records_kernel<<<unsigned((rows + 15) / 16), 256, 0, s>>>(
      static_cast<const __nv_bfloat16 *>(out), static_cast<const __nv_bfloat16 *>(dout), lse, rec, rows);
  if (cudaGetLastError() != cudaSuccess) return BASA_ERR_CUDA;
  const long long window_blocks = bh * P.g.nWin * P.max_tiles;
  if ((st = run_bwd<kDq>(P, window_blocks, s)) != BASA_OK) return st;
  if (L.n_long > 0) {
    if ((st = run_bwd<kDkvLong>(P, bh * L.n_long * L.n_chunks, s)) != BASA_OK) return st;
    const long long threads = bh * L.n_long * kTileRows * 32;
    bwd_reduce_kernel<<<unsigned((threads + 255) / 256), 256, 0, s>>>(
        P.part, dkvp, static_cast<__nv_bfloat16 *>(dk), static_cast<__nv_bfloat16 *>(dv), int(bh), L.n_long,
        L.n_chunks, P.n_pool, P.n_pool_tiles, p.n_text, N);
    if (cudaGetLastError() != cudaSuccess) return BASA_ERR_CUDA;
  }
  return run_bwd<kDkvWindow>(P, window_blocks, s);
}

}  // namespace basa

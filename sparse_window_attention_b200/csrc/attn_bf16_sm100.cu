// Shifted-window attention forward, bfloat16, head_dim 128, for sm_100a.
//
// Operator (BASA §3.1-§3.3, §A.1): for each query of shifted window w,
//   out = softmax(q K^T / sqrt(d)) V  over K/V = [w | routed windows | pooled | text]
// written back at the query's original grid position.
//
// One CTA = (b*head, window, pair of 128-row query tiles). Warp roles:
//   warp 0      TMA loader: query tiles once, then a K, V, K, V ... stream of
//               128-row key tiles through a 5-slot shared-memory ring. Window
//               tiles are assembled from TMA box loads whose coordinates already
//               include the cyclic shift (mod the grid), so no rolled copy exists.
//   warp 1      tcgen05 issuer (one thread): S_g = Q_g K^T and O_g += P_g V with
//               fp32 accumulators in TMEM (S0, S1, O0, O1: 4 x 128 columns).
//   warps 2-3   idle (they keep the three warpgroups aligned to the SM sub-partitions)
//   warps 4-11  two softmax warpgroups, one per query tile; a thread owns one
//               query row: reads its S row from TMEM, runs the online softmax in
//               fp32 (base-2 exponent, scale folded in), writes P (bf16) back to
//               TMEM over its S row (A operand of P V), rescales its O row in TMEM when the running max grows,
//               and at the end normalises O and stores it with TMA boxes at the
//               same (unshifted) coordinates the queries were loaded from.
// Every wait is bounded (globaltimer); on expiry the kernel records a bit in
// dev_err, drains its own in-flight copies and MMAs, frees TMEM and returns.
//
// The same kernel also serves the branch form (BASA §A.1): a key-group mask drops
// the window, pooled or text segments from the key stream, and an optional
// epilogue writes each query row's log-sum-exp; and the text-query rows, where the
// queries are 128-row boxes of the text rows and the key stream is every k/v row,
// split over CTA groups whose partial results are merged by log-sum-exp.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "attn_sm100_common.cuh"
#include "basa_internal.h"
#include "sm100_ptx.cuh"

namespace basa {
namespace {

using sm100::kHalfBytes;
using sm100::kTileBytes;
using sm100::kTileDesc;
using sm100::Waiter;
using sm100::wrap;

// 12 warps = three warpgroups: warp 0 loads, warp 1 issues MMAs (warps 2-3 idle),
// warps 4-7 and 8-11 run the softmax of query tile 0 and 1. Each SM sub-partition
// then holds one warp of each group (with 10 warps, two sub-partitions held two
// softmax warps and the register limit forced spills).
constexpr int kThreads = 384;
constexpr int kStages = 5;
constexpr uint32_t kSmemQ = 0;                         // 2 query tiles (reused for the output)
constexpr uint32_t kSmemRing = 2 * kTileBytes;         // K/V ring
constexpr uint32_t kSmemCtrl = kSmemRing + kStages * kTileBytes;
constexpr uint32_t kCtrlBytes = 1024;
constexpr int kMaskTable = 64;                         // key tiles whose column masks are tabled in smem
constexpr uint32_t kSmemMask = kSmemCtrl + kCtrlBytes;
constexpr uint32_t kSmemBytes = kSmemMask + kMaskTable * 16 + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxTextSplits = 8;  // key-range splits of the text-query rows

struct alignas(64) AttnParams {
  CUtensorMap map_q[kMaxShapes];
  CUtensorMap map_k[kMaxShapes];
  CUtensorMap map_v[kMaxShapes];
  CUtensorMap map_o[kMaxShapes];
  CUtensorMap map_kp, map_vp, map_kt, map_vt;
  CUtensorMap map_kp8, map_vp8;  // pooled rows in 8-row boxes (the pooled tail, see below)
  CUtensorMap map_qd, map_od;  // text-query mode: query rows and output rows (d, row, b*head)
  WindowPlan plan;
  const int32_t *route;
  int32_t *dev_err;
  Geo g;
  int routed_k, n_pool, n_text, n_pool_tiles, n_text_tiles;
  // Pooled tail: when the pooled keys past the last full 128-row tile (pool_tail rows,
  // at most 16) fit in free 8-row blocks of the own window's key tile tail_tile[type],
  // they are loaded there (8-row boxes at rows tail_dest[type][b]) instead of taking a
  // key tile of their own; tail_mask[type] marks their rows.
  int pool_tail, tail_blocks;
  int8_t tail_tile[8];
  uint8_t tail_dest[8][2];
  uint32_t tail_mask[8][4];
  float scale_log2;
  int use_windows;  // own and routed windows are keys (else pooled and/or text only)
  // Text-query mode: the queries are the n_text text rows and attend densely to
  // every k/v row, which are streamed as the "text" segment starting at row 0.
  // The key tiles are split into n_splits ranges, one per CTA group.
  int dense, dense_rows, dense_q_tiles, dense_pairs, n_splits, split_tiles, bh_count;
  int text_row0;  // first k/v row of the text segment: N (window mode) or 0
  float *lse;       // nullable: log-sum-exp of each query row's scaled scores [B*heads][N]
  int all_full;  // every key tile of the launch is full: no column masks
  uint32_t flags;
  unsigned long long timeout_ns;
};

// __grid_constant__ kernel parameters are limited to 32764 bytes.
static_assert(sizeof(AttnParams) <= 32764, "window plan too large for the kernel parameter space");

struct Ctrl {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full, s_full[2], p_full[2], o_full[2], drain;
  uint32_t tmem_base;
  int abort;
  int tile0, ntile;  // text-query mode: this CTA's range of key tiles
  int wtype[1 + kMaxRouted];
  int org[1 + kMaxRouted][3];
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");

// Position in the key-tile stream: segments 0..routed_k are windows (own, then
// routed), then the pooled tokens, then the text tokens.
struct KeyIter {
  int seg, t;
};

__device__ __forceinline__ int seg_tiles(const AttnParams &P, const Ctrl &c, int seg) {
  if (seg <= P.routed_k) return P.use_windows ? P.plan.type[c.wtype[seg]].n_tiles : 0;
  if (seg == P.routed_k + 1) return P.n_pool_tiles;
  return P.dense ? c.ntile : P.n_text_tiles;
}
__device__ __forceinline__ void advance(const AttnParams &P, const Ctrl &c, KeyIter &it) {
  ++it.t;
  while (it.seg <= P.routed_k + 2 && it.t >= seg_tiles(P, c, it.seg)) {
    ++it.seg;
    it.t = 0;
  }
}

// First key tile of the stream (segments without tiles are skipped).
__device__ __forceinline__ KeyIter first_key(const AttnParams &P, const Ctrl &c) {
  KeyIter it{0, 0};
  while (it.seg <= P.routed_k + 2 && seg_tiles(P, c, it.seg) == 0) ++it.seg;
  return it;
}

// The own window's key tile that also carries the pooled tail.
__device__ __forceinline__ bool has_pool_tail(const AttnParams &P, const Ctrl &c, const KeyIter &it) {
  return P.pool_tail > 0 && it.seg == 0 && it.t == P.tail_tile[c.wtype[0]];
}

// Bytes the TMA loads of one key (or value) tile deliver.
__device__ __forceinline__ uint32_t key_tile_bytes(const AttnParams &P, const Ctrl &c, const KeyIter &it) {
  if (it.seg > P.routed_k) return kTileBytes;  // whole 128-row boxes (rows past the end read as zero)
  uint32_t b = uint32_t(P.plan.tile[P.plan.type[c.wtype[it.seg]].first_tile + it.t].valid_rows) * 256u;
  if (has_pool_tail(P, c, it)) b += uint32_t(P.tail_blocks) * 8u * 256u;
  return b;
}

__device__ __forceinline__ uint32_t load_key_tile(const AttnParams &P, const Ctrl &c, const KeyIter &it, bool is_v,
                                                  int bh, uint8_t *dst, uint64_t *bar) {
  if (it.seg <= P.routed_k) {
    const PlanTile &tile = P.plan.tile[P.plan.type[c.wtype[it.seg]].first_tile + it.t];
    uint32_t b = sm100::load_window_tile(P.plan, P.g, is_v ? P.map_v : P.map_k, tile, c.org[it.seg], bh, dst, bar);
    if (has_pool_tail(P, c, it)) {
      const CUtensorMap *map = is_v ? &P.map_vp8 : &P.map_kp8;
      for (int i = 0; i < P.tail_blocks; ++i) {
        uint8_t *d = dst + uint32_t(P.tail_dest[c.wtype[0]][i]) * 128u;
        const int row = P.n_pool_tiles * kTileRows + 8 * i;  // rows past n_pool read as zero
        ptx::tma_load_3d(d, map, bar, 0, row, bh);
        ptx::tma_load_3d(d + kHalfBytes, map, bar, 64, row, bh);
        b += 8u * 256u;
      }
    }
    return b;
  }
  const bool pooled = it.seg == P.routed_k + 1;
  const CUtensorMap *map = pooled ? (is_v ? &P.map_vp : &P.map_kp) : (is_v ? &P.map_vt : &P.map_kt);
  const int row = pooled ? it.t * kTileRows : P.text_row0 + (c.tile0 + it.t) * kTileRows;
  ptx::tma_load_3d(dst, map, bar, 0, row, bh);
  ptx::tma_load_3d(dst + kHalfBytes, map, bar, 64, row, bh);
  return kTileBytes;
}

// Column mask of a key tile; returns true when all 128 rows hold keys.
__device__ __forceinline__ bool key_tile_mask(const AttnParams &P, const Ctrl &c, const KeyIter &it, uint32_t *m) {
  if (it.seg <= P.routed_k) {
    const PlanTile &tile = P.plan.tile[P.plan.type[c.wtype[it.seg]].first_tile + it.t];
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = tile.mask[i];
    if (has_pool_tail(P, c, it)) {
#pragma unroll
      for (int i = 0; i < 4; ++i) m[i] |= P.tail_mask[c.wtype[0]][i];
      return false;
    }
    return tile.valid_rows == kTileRows;
  }
  const bool pooled = it.seg == P.routed_k + 1;
  const int total = pooled ? P.n_pool : (P.dense ? P.dense_rows : P.n_text);
  const int valid = min(kTileRows, total - (pooled ? it.t : c.tile0 + it.t) * kTileRows);
  sm100::prefix_mask(valid, m);
  return valid == kTileRows;
}

// The running row max is only raised when a tile's max exceeds it by more than
// 2^8 (log2 units); otherwise the old max is kept and P values up to 256 are
// produced, which float32 sums and bfloat16 P hold exactly as well. This skips
// most rescales of the O accumulator in TMEM.
constexpr float kRescaleLog2 = 8.0f;
// P = 2^x (x = s * scale_log2 - m) for the 128 scores of a row (MUFU ex2), written
// in place as the 64 bfloat16 pairs the P V MMA reads (s[i] = pair (2i, 2i+1), low
// half = even key); each pair is packed as soon as it is computed, so the live
// register set shrinks along the row. Returns the float32 row sum.
__device__ __forceinline__ float exp2_row_packed(uint32_t (&s)[128], float scale_log2, float m) {
  using namespace ptx;
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2), negm2 = f2_pack(-m, -m);
  uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
  for (int pr = 0; pr < 64; ++pr) {
    const uint64_t x = ffma2(f2_pack(__uint_as_float(s[2 * pr]), __uint_as_float(s[2 * pr + 1])), sc2, negm2);
    float x0, x1;
    f2_unpack(x, x0, x1);
    const float r0 = ex2(x0), r1 = ex2(x1);
    const uint64_t pp = f2_pack(r0, r1);
    if (pr & 1) acc1 = fadd2(acc1, pp);
    else acc0 = fadd2(acc0, pp);
    s[pr] = pack_bf16x2(r0, r1);  // s[pr] was read at pair pr / 2
  }
  float a, b, c, d;
  f2_unpack(acc0, a, b);
  f2_unpack(acc1, c, d);
  return (a + b) + (c + d);
}

// Row max of the N entries of s (raw scores).
template <int N>
__device__ __forceinline__ float row_max(const uint32_t (&s)[N]) {
  float a = __uint_as_float(s[0]), b = __uint_as_float(s[1]), c = __uint_as_float(s[2]), d = __uint_as_float(s[3]);
#pragma unroll
  for (int i = 4; i < N; i += 8) {
    a = ptx::fmax3(a, __uint_as_float(s[i]), __uint_as_float(s[i + 1]));
    b = ptx::fmax3(b, __uint_as_float(s[i + 2]), __uint_as_float(s[i + 3]));
    c = ptx::fmax3(c, __uint_as_float(s[i + 4]), __uint_as_float(s[i + 5]));
    d = ptx::fmax3(d, __uint_as_float(s[i + 6]), __uint_as_float(s[i + 7]));
  }
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// Sets every column whose mask bit is clear to -inf.
template <int N>
__device__ __forceinline__ void apply_mask(uint32_t (&s)[N], const uint32_t *mask) {
#pragma unroll
  for (int wd = 0; wd < N / 32; ++wd) {
    const uint32_t mw = mask[wd];
    if (mw != 0xFFFFFFFFu) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!((mw >> i) & 1u)) s[32 * wd + i] = __float_as_uint(-INFINITY);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) attn_bf16_kernel(const __grid_constant__ AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl &c = *reinterpret_cast<Ctrl *>(smem + kSmemCtrl);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  int pair, w = 0, bh, split = 0, ot = 0, oy = 0, ox = 0, wtype = 0, n_q_tiles;
  PlanType ty{0, 0};
  if (P.dense) {
    pair = blockIdx.x % P.dense_pairs;
    split = (blockIdx.x / P.dense_pairs) % P.n_splits;
    bh = blockIdx.x / (P.dense_pairs * P.n_splits);
    n_q_tiles = P.dense_q_tiles;
  } else {
    const int pairs = P.plan.max_pairs;
    pair = blockIdx.x % pairs;
    w = (blockIdx.x / pairs) % P.g.nWin;
    bh = blockIdx.x / (pairs * P.g.nWin);
    window_origin(P.g, w, &ot, &oy, &ox, &wtype);
    ty = P.plan.type[wtype];
    n_q_tiles = ty.n_tiles;
  }
  const int q_tile0 = 2 * pair;
  if (q_tile0 >= n_q_tiles) return;  // whole CTA: this window type has fewer query tiles
  const bool has_q1 = q_tile0 + 1 < n_q_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&c.full[i], 1);
      ptx::mbar_init(&c.empty[i], 1);
    }
    ptx::mbar_init(&c.q_full, 1);
    for (int g = 0; g < 2; ++g) {
      ptx::mbar_init(&c.s_full[g], 1);
      ptx::mbar_init(&c.p_full[g], 128);
      ptx::mbar_init(&c.o_full[g], 1);
    }
    ptx::mbar_init(&c.drain, 1);
    c.abort = 0;
    c.tile0 = P.dense ? split * P.split_tiles : 0;
    c.ntile = P.dense ? min(P.split_tiles, (P.dense_rows + kTileRows - 1) / kTileRows - c.tile0) : 0;
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
    ptx::fence_mbar_init();
  }
  if (P.plan.zero_fill) {
    // Rows of a tile that no TMA box writes must hold finite values (P is 0 there).
    uint4 *z = reinterpret_cast<uint4 *>(smem);
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (uint32_t i = threadIdx.x; i < 2 * kTileBytes / 16; i += kThreads) z[i] = zero;
    uint4 *zr = reinterpret_cast<uint4 *>(smem + kSmemRing);
    for (uint32_t i = threadIdx.x; i < kStages * kTileBytes / 16; i += kThreads) zr[i] = zero;
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

  int n_kt = 0;
  for (int s = 0; s <= P.routed_k + 2; ++s) n_kt += seg_tiles(P, c, s);

  if (warp == 0) {
    // ------------------------------------------------------------- TMA loader
    if (lane == 0) {
      Waiter wt{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_PRODUCER, true};
      Waiter drain{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_PRODUCER, false};
      if (P.dense) {
        // whole 128-row boxes (rows past the end read as zero and still count)
        ptx::mbar_arrive_expect_tx(&c.q_full, (has_q1 ? 2u : 1u) * kTileBytes);
        for (int g = 0; g < (has_q1 ? 2 : 1); ++g) {
          uint8_t *dst = smem + kSmemQ + g * kTileBytes;
          ptx::tma_load_3d(dst, &P.map_qd, &c.q_full, 0, (q_tile0 + g) * kTileRows, bh);
          ptx::tma_load_3d(dst + kHalfBytes, &P.map_qd, &c.q_full, 64, (q_tile0 + g) * kTileRows, bh);
        }
      } else {
        // a tile's TMA boxes deliver 256 bytes per valid row (two 128-byte halves)
        uint32_t qbytes = uint32_t(P.plan.tile[ty.first_tile + q_tile0].valid_rows) * 256u;
        if (has_q1) qbytes += uint32_t(P.plan.tile[ty.first_tile + q_tile0 + 1].valid_rows) * 256u;
        ptx::mbar_arrive_expect_tx(&c.q_full, qbytes);
        for (int g = 0; g < (has_q1 ? 2 : 1); ++g)
          sm100::load_window_tile(P.plan, P.g, P.map_q, P.plan.tile[ty.first_tile + q_tile0 + g], c.org[0], bh,
                                  smem + kSmemQ + g * kTileBytes, &c.q_full);
      }
      KeyIter it = first_key(P, c);
      int last = -1;
      bool skipped0 = false;
      for (int j = 0; j < n_kt; ++j) {
        bool ok = true;
        for (int kv = 0; kv < 2; ++kv) {
          const int item = 2 * j + kv;
          const int slot = item % kStages;
          if (!wt.wait(&c.empty[slot], ((item / kStages) & 1) ^ 1)) { ok = false; break; }
          if (item == 0 && (P.flags & BASA_FLAG_TEST_SKIP_FIRST_KEY_LOAD)) { skipped0 = true; last = item; continue; }
          uint8_t *dst = smem + kSmemRing + slot * kTileBytes;
          // Arm the barrier with the byte count before issuing the copies.
          const uint32_t bytes = key_tile_bytes(P, c, it);
          ptx::mbar_arrive_expect_tx(&c.full[slot], bytes);
          load_key_tile(P, c, it, kv == 1, bh, dst, &c.full[slot]);
          last = item;
        }
        if (!ok) break;
        advance(P, c, it);
      }
      // Drain: wait for the copies still in flight (immediate when all were consumed).
      drain.wait(&c.q_full, 0);
      for (int item = max(0, last - (kStages - 1)); item <= last; ++item) {
        if (item == 0 && skipped0) continue;
        drain.wait(&c.full[item % kStages], (item / kStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      Waiter wt{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_MMA, true};
      Waiter drain{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_MMA, false};
      // low descriptor halves of the query tiles and the ring slots
      const uint32_t sQ = sm100::kDescLoK | (ptx::smem_u32(smem + kSmemQ) >> 4);
      const uint32_t sRk = sm100::kDescLoK | (ptx::smem_u32(smem + kSmemRing) >> 4);
      const uint32_t sRv = sm100::kDescLoMn | (ptx::smem_u32(smem + kSmemRing) >> 4);
      const uint32_t tS0 = tmem, tS1 = tmem + 128, tO0 = tmem + 256, tO1 = tmem + 384;
      if (wt.wait(&c.q_full, 0) && wt.wait(&c.full[0], 0)) {
        ptx::tc_fence_after();
        sm100::issue_ss(tS0, sQ, sRk);
        ptx::mma_commit(&c.s_full[0]);
        if (has_q1) {
          sm100::issue_ss(tS1, sQ + kTileDesc, sRk);
          ptx::mma_commit(&c.s_full[1]);
        }
        ptx::mma_commit(&c.empty[0]);
        for (int j = 0; j < n_kt; ++j) {
          const int vi = 2 * j + 1, ki = 2 * j + 2;
          const uint32_t vaddr = sRv + (vi % kStages) * kTileDesc, kaddr = sRk + (ki % kStages) * kTileDesc;
          const bool more = j + 1 < n_kt;
          if (!wt.wait(&c.full[vi % kStages], (vi / kStages) & 1)) break;
          if (!wt.wait(&c.p_full[0], j & 1)) break;
          ptx::tc_fence_after();
          sm100::issue_ts(tO0, tS0, vaddr, j > 0);
          if (more) {
            if (!wt.wait(&c.full[ki % kStages], (ki / kStages) & 1)) break;
            ptx::tc_fence_after();
            sm100::issue_ss(tS0, sQ, kaddr);
            ptx::mma_commit(&c.s_full[0]);
          } else {
            ptx::mma_commit(&c.o_full[0]);
          }
          if (has_q1) {
            if (!wt.wait(&c.p_full[1], j & 1)) break;
            ptx::tc_fence_after();
            sm100::issue_ts(tO1, tS1, vaddr, j > 0);
          }
          ptx::mma_commit(&c.empty[vi % kStages]);
          if (more) {
            if (has_q1) {
              sm100::issue_ss(tS1, sQ + kTileDesc, kaddr);
              ptx::mma_commit(&c.s_full[1]);
            }
            ptx::mma_commit(&c.empty[ki % kStages]);
          } else if (has_q1) {
            ptx::mma_commit(&c.o_full[1]);
          }
        }
      }
      // Every MMA this thread issued must finish before TMEM is freed.
      ptx::mma_commit(&c.drain);
      drain.wait(&c.drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    // Two warpgroups, one per query tile; a thread owns one query row.
    const int g = (warp - 4) / 4;
    const int sub = warp % 4;  // TMEM lane quarter this warp may access
    const int row = sub * 32 + lane;
    const uint32_t lane_off = uint32_t(sub * 32) << 16;
    const uint32_t tS = tmem + lane_off + g * 128, tO = tmem + lane_off + 256 + g * 128;
    const bool active = g == 0 || has_q1;
    Waiter wt{&c.abort, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_SOFTMAX, true};
    uint8_t *q_tile = smem + kSmemQ + g * kTileBytes;
    const uint32_t swz = row & 7;
    const float sl2 = P.scale_log2;
    {
      // Column masks of this CTA's key tiles in stream order (all ones = full tile),
      // one tile per softmax thread; this runs while the first loads are in flight.
      const int j = threadIdx.x - 128;
      if (j < kMaskTable && j < n_kt) {
        KeyIter t{0, j};
        while (t.seg <= P.routed_k + 2 && t.t >= seg_tiles(P, c, t.seg)) {
          t.t -= seg_tiles(P, c, t.seg);
          ++t.seg;
        }
        uint32_t mk[4];
        key_tile_mask(P, c, t, mk);
        reinterpret_cast<uint4 *>(smem + kSmemMask)[j] = make_uint4(mk[0], mk[1], mk[2], mk[3]);
      }
      ptx::named_barrier(3, 256);  // the 256 softmax threads
    }
    float m = -INFINITY, l = 0.f;
    bool ok = active;
    KeyIter it = first_key(P, c);
    for (int j = 0; ok && j < n_kt; ++j) {
      ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.s_full[g], j & 1));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t s[128];
      ptx::tmem_ld128(tS, s);
      ptx::tmem_ld_wait(s);
      if (P.all_full) {
      } else if (j < kMaskTable) {
        const uint4 mt = reinterpret_cast<const uint4 *>(smem + kSmemMask)[j];
        if ((mt.x & mt.y & mt.z & mt.w) != 0xFFFFFFFFu) {
          const uint32_t mask[4] = {mt.x, mt.y, mt.z, mt.w};
          apply_mask(s, mask);
        }
      } else {
        uint32_t mask[4];
        if (!key_tile_mask(P, c, it, mask)) apply_mask(s, mask);
      }
      const float m_tile = row_max(s) * sl2;
      const bool need = m_tile > m + kRescaleLog2;  // always true on the first tile (m = -inf)
      const float m_new = need ? m_tile : m;
      const float alpha = need ? ptx::ex2(m - m_new) : 1.0f;
      const float sum = exp2_row_packed(s, sl2, m_new);
      l = l * alpha + sum;
      m = m_new;
      // P row -> TMEM over the first 64 columns of S; the MMA that overwrites S
      // next is issued after the P V that reads it.
      ptx::tmem_st64(tS, s);
      if (j > 0 && __any_sync(0xFFFFFFFFu, need)) {
        const uint64_t a2 = ptx::f2_pack(alpha, alpha);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          ptx::tmem_ld32(tO + cc * 32, r);
          ptx::tmem_ld_wait(r);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float lo, hi;
            ptx::f2_unpack(ptx::fmul2(ptx::f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), a2), lo, hi);
            r[i] = __float_as_uint(lo);
            r[i + 1] = __float_as_uint(hi);
          }
          ptx::tmem_st32(tO + cc * 32, r);
        }
      }
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&c.p_full[g]);
      if (j + 1 >= kMaskTable) {
        if (j + 1 == kMaskTable)  // past the table: walk the stream from its start once
          for (int t = 0; t < kMaskTable; ++t) advance(P, c, it);
        else
          advance(P, c, it);
      }
    }
    if (ok) ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.o_full[g], 0));
    if (ok) {
      ptx::tc_fence_after();
      const float inv = 1.0f / l;
      const uint64_t inv2 = ptx::f2_pack(inv, inv);
      const uint32_t o_row = ptx::smem_u32(q_tile) + row * 128;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        ptx::tmem_ld32(tO + cc * 32, r);
        ptx::tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float lo, hi;
          ptx::f2_unpack(ptx::fmul2(ptx::f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), inv2), lo, hi);
          r[i] = __float_as_uint(lo);
          r[i + 1] = __float_as_uint(hi);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c16 = cc * 4 + i;
          const uint32_t addr = o_row + (c16 >> 3) * kHalfBytes + (((c16 & 7) ^ swz) << 4);
          const int b = 8 * i;
          ptx::st_shared_v4(addr, ptx::pack_bf16x2(__uint_as_float(r[b]), __uint_as_float(r[b + 1])),
                            ptx::pack_bf16x2(__uint_as_float(r[b + 2]), __uint_as_float(r[b + 3])),
                            ptx::pack_bf16x2(__uint_as_float(r[b + 4]), __uint_as_float(r[b + 5])),
                            ptx::pack_bf16x2(__uint_as_float(r[b + 6]), __uint_as_float(r[b + 7])));
        }
      }
      ptx::fence_proxy_async_smem();
    }
    if (ok && P.lse != nullptr && P.dense) {
      const int qrow = (q_tile0 + g) * kTileRows + row;
      if (active && qrow < P.n_text)
        P.lse[((long long)split * P.bh_count + bh) * P.n_text + qrow] = (m + log2f(l)) * 0.6931471805599453f;
    } else if (ok && P.lse != nullptr) {
      // log-sum-exp of this row: m and l are in base 2 of the scaled scores
      int t, y, x;
      const int org[3] = {ot, oy, ox};
      if (sm100::tile_row_token(P.plan, P.g, P.plan.tile[ty.first_tile + q_tile0 + g], org, row, &t, &y, &x))
        P.lse[(long long)bh * P.g.N + ((long long)t * P.g.H + y) * P.g.W + x] = (m + log2f(l)) * 0.6931471805599453f;
    }
    ptx::named_barrier(1 + g, 128);
    if (P.dense && active && row == 0 && !*reinterpret_cast<volatile int *>(&c.abort)) {
      // rows past n_text fall outside the output map and are not written
      const int orow = (q_tile0 + g) * kTileRows, ob = split * P.bh_count + bh;
      ptx::tma_store_3d(&P.map_od, q_tile, 0, orow, ob);
      ptx::tma_store_3d(&P.map_od, q_tile + kHalfBytes, 64, orow, ob);
      ptx::tma_store_commit();
      ptx::tma_store_wait_read_all();
    } else if (active && row == 0 && !*reinterpret_cast<volatile int *>(&c.abort)) {
      const int org[3] = {ot, oy, ox};
      sm100::store_window_tile(P.plan, P.g, P.map_o, P.plan.tile[ty.first_tile + q_tile0 + g], org, bh, q_tile);
      ptx::tma_store_commit();
      ptx::tma_store_wait_read_all();
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------- host side

// Pooled tail: the pooled keys past the last full tile (1..16 rows) go into free
// 8-row blocks of one key tile of the own window when every window type has such
// blocks; the pooled segment then has one tile fewer. Returns whether it is on.
bool plan_pool_tail(AttnParams &P) {
  const int tail = P.n_pool % kTileRows;
  if (tail == 0 || tail > 16) return false;
  const int blocks = (tail + 7) / 8;
  int8_t tile_of[8];
  uint8_t dest[8][2];
  uint32_t mask[8][4];
  for (int ty = 0; ty < 8; ++ty) {
    tile_of[ty] = -1;
    const PlanType &pt = P.plan.type[ty];
    // a type no window has keeps tile -1 (never matched)
    for (int t = pt.n_tiles - 1; t >= 0 && tile_of[ty] < 0; --t) {
      const PlanTile &tile = P.plan.tile[pt.first_tile + t];
      int found = 0;
      for (int b = 0; b < kTileRows / 8 && found < blocks; ++b) {
        bool free_block = true;
        for (int r = 8 * b; r < 8 * b + 8; ++r) free_block &= !((tile.mask[r >> 5] >> (r & 31)) & 1u);
        if (free_block) dest[ty][found++] = uint8_t(8 * b);
      }
      if (found == blocks) tile_of[ty] = int8_t(t);
    }
    if (pt.n_tiles > 0 && tile_of[ty] < 0) return false;
    for (int i = 0; i < 4; ++i) mask[ty][i] = 0;
    if (tile_of[ty] >= 0)
      for (int b = 0; b < blocks; ++b)
        for (int r = 0; r < 8 && 8 * b + r < tail; ++r) {
          const int row = dest[ty][b] + r;
          mask[ty][row >> 5] |= 1u << (row & 31);
        }
  }
  P.pool_tail = tail;
  P.tail_blocks = blocks;
  P.n_pool_tiles = P.n_pool / kTileRows;
  std::memcpy(P.tail_tile, tile_of, sizeof(tile_of));
  std::memcpy(P.tail_dest, dest, sizeof(dest));
  std::memcpy(P.tail_mask, mask, sizeof(mask));
  return true;
}

basa_status run_attn(const AttnParams &P, long long blocks, cudaStream_t s) {
  if (cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return BASA_ERR_CUDA;
  attn_bf16_kernel<<<unsigned(blocks), kThreads, kSmemBytes, s>>>(P);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}


// Number of key-range splits for the text-query rows: enough CTAs to cover the SMs
// once (one CTA per SM fits), at least 4 key tiles per split.
int text_splits(const basa_params &p, int sms) {
  const long long base = (long long)p.B * p.heads * (((p.n_text + kTileRows - 1) / kTileRows + 1) / 2);
  const long long rows = (long long)p.T * p.H * p.W + p.n_text;
  const int tiles = int((rows + kTileRows - 1) / kTileRows);
  if (base >= sms) return 1;
  return std::max(1, std::min<int>(int(sms / base), std::min(kMaxTextSplits, tiles / 4)));
}

}  // namespace

// 5-D map (d, x, y, t, b*head) over the visual rows of a [B, heads, rows, 128] tensor.
bool encode_grid_map(CUtensorMap *m, const void *base, const basa_params &p, long long rows_per_bh,
                     const PlanShape &s) {
  const cuuint64_t e = 2;
  cuuint64_t dims[5] = {cuuint64_t(p.head_dim), cuuint64_t(p.W), cuuint64_t(p.H), cuuint64_t(p.T),
                        cuuint64_t(p.B) * cuuint64_t(p.heads)};
  cuuint64_t strides[4] = {p.head_dim * e, cuuint64_t(p.W) * p.head_dim * e, cuuint64_t(p.H) * p.W * p.head_dim * e,
                           cuuint64_t(rows_per_bh) * p.head_dim * e};
  cuuint32_t box[5] = {64, cuuint32_t(s.cx), cuuint32_t(s.cy), cuuint32_t(s.ct), 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map (d, row, b*head) with box_rows-row boxes; rows past the end read as zero.
bool encode_rows_map(CUtensorMap *m, const void *base, const basa_params &p, long long rows_per_bh, int box_rows) {
  const cuuint64_t e = 2;
  cuuint64_t dims[3] = {cuuint64_t(p.head_dim), cuuint64_t(rows_per_bh), cuuint64_t(p.B) * cuuint64_t(p.heads)};
  cuuint64_t strides[2] = {p.head_dim * e, cuuint64_t(rows_per_bh) * p.head_dim * e};
  cuuint32_t box[3] = {64, cuuint32_t(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 5-D map (4, x, y, t, b*head) over [B*heads, N, 4] float32 records, no swizzle.
bool encode_record_map(CUtensorMap *m, const void *base, const basa_params &p, const PlanShape &s) {
  const cuuint64_t e = 4;
  const cuuint64_t N = cuuint64_t(p.T) * p.H * p.W;
  cuuint64_t dims[5] = {4, cuuint64_t(p.W), cuuint64_t(p.H), cuuint64_t(p.T), cuuint64_t(p.B) * cuuint64_t(p.heads)};
  cuuint64_t strides[4] = {4 * e, cuuint64_t(p.W) * 4 * e, cuuint64_t(p.H) * p.W * 4 * e, N * 4 * e};
  cuuint32_t box[5] = {4, cuuint32_t(s.cx), cuuint32_t(s.cy), cuuint32_t(s.ct), 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, const_cast<void *>(base), dims, strides, box, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int device_sm_count() {
  static int n[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return 148;
  if (!n[dev] && cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n[dev] = 0;
  return n[dev];
}

basa_status launch_attn_bf16(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                             const int32_t *route_idx, void *out, float *lse, uint32_t keys, const basa_params &p,
                             cudaStream_t s) {
  if (!tensor_map_encoder()) return BASA_ERR_CUDA;
  AttnParams P;
  std::memset(&P, 0, sizeof(P));
  basa_status st = build_window_plan(p, &P.plan);
  if (st != BASA_OK) return st;
  P.g = make_geo(p);
  const long long N = P.g.N;
  const long long kv_rows = N + p.n_text;
  for (int i = 0; i < P.plan.n_shapes; ++i) {
    if (!encode_grid_map(&P.map_q[i], q, p, N, P.plan.shape[i]) ||
        !encode_grid_map(&P.map_k[i], k, p, kv_rows, P.plan.shape[i]) ||
        !encode_grid_map(&P.map_v[i], v, p, kv_rows, P.plan.shape[i]) ||
        !encode_grid_map(&P.map_o[i], out, p, N, P.plan.shape[i]))
      return BASA_ERR_CUDA;
  }
  P.n_pool = p.pt > 0 ? (p.T / p.pt) * (p.H / p.ph) * (p.W / p.pw) : 0;
  P.n_text = p.n_text;
  if (P.n_pool > 0) {
    if (!encode_rows_map(&P.map_kp, kp, p, P.n_pool) || !encode_rows_map(&P.map_vp, vp, p, P.n_pool))
      return BASA_ERR_CUDA;
  }
  if (p.n_text > 0) {
    if (!encode_rows_map(&P.map_kt, k, p, kv_rows) || !encode_rows_map(&P.map_vt, v, p, kv_rows)) return BASA_ERR_CUDA;
  }
  P.n_pool_tiles = (keys & BASA_KEYS_POOLED) ? (P.n_pool + kTileRows - 1) / kTileRows : 0;
  if ((keys & BASA_KEYS_POOLED) && (keys & BASA_KEYS_WINDOWS) && plan_pool_tail(P)) {
    if (!encode_rows_map(&P.map_kp8, kp, p, P.n_pool, 8) || !encode_rows_map(&P.map_vp8, vp, p, P.n_pool, 8))
      return BASA_ERR_CUDA;
  }
  P.n_text_tiles = (keys & BASA_KEYS_TEXT) ? (p.n_text + kTileRows - 1) / kTileRows : 0;
  P.use_windows = (keys & BASA_KEYS_WINDOWS) ? 1 : 0;
  P.lse = lse;
  P.text_row0 = int(N);
  P.route = route_idx;
  P.dev_err = p.dev_err;
  P.routed_k = p.routed_k;
  P.scale_log2 = float(1.4426950408889634 / std::sqrt(double(p.head_dim)));
  P.flags = p.flags;
  P.all_full = (P.n_pool % kTileRows == 0) && (p.n_text % kTileRows == 0);
  for (int i = 0; i < P.plan.n_tiles; ++i) P.all_full &= P.plan.tile[i].valid_rows == kTileRows;
  P.timeout_ns = (p.wait_timeout_us ? (unsigned long long)p.wait_timeout_us : 2000000ull) * 1000ull;
  const long long blocks = (long long)p.B * p.heads * P.g.nWin * P.plan.max_pairs;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  return run_attn(P, blocks, s);
}

size_t text_attn_workspace(const basa_params &p, int sms) {
  const int splits = text_splits(p, sms);
  if (splits <= 1) return 0;
  const size_t rows = size_t(splits) * p.B * p.heads * p.n_text;
  return rows * p.head_dim * 2 + rows * sizeof(float);  // partial outputs (bf16), then their log-sum-exp
}

basa_status launch_attn_text_bf16(const void *q_text, const void *k, const void *v, void *out_text, void *workspace,
                                  const basa_params &p, int sms, cudaStream_t s) {
  if (!tensor_map_encoder()) return BASA_ERR_CUDA;
  AttnParams P;
  std::memset(&P, 0, sizeof(P));
  P.g = make_geo(p);
  const long long N = P.g.N;
  const long long kv_rows = N + p.n_text;
  const int bh = p.B * p.heads;
  const int splits = text_splits(p, sms);
  uint8_t *part = static_cast<uint8_t *>(workspace);
  float *part_lse = reinterpret_cast<float *>(part + size_t(splits) * bh * p.n_text * p.head_dim * 2);
  if (!encode_rows_map(&P.map_kt, k, p, kv_rows) || !encode_rows_map(&P.map_vt, v, p, kv_rows) ||
      !encode_rows_map(&P.map_qd, q_text, p, p.n_text))
    return BASA_ERR_CUDA;
  // outputs: straight to out_text, or per-split partials [split][b*head][n_text][d]
  basa_params po = p;
  po.B = 1;
  po.heads = splits * bh;
  if (!encode_rows_map(&P.map_od, splits > 1 ? static_cast<const void *>(part) : out_text, splits > 1 ? po : p,
                       p.n_text))
    return BASA_ERR_CUDA;
  P.dense = 1;
  P.dense_rows = int(kv_rows);
  P.dense_q_tiles = (p.n_text + kTileRows - 1) / kTileRows;
  P.dense_pairs = (P.dense_q_tiles + 1) / 2;
  const int key_tiles = int((kv_rows + kTileRows - 1) / kTileRows);
  P.n_splits = splits;
  P.split_tiles = (key_tiles + splits - 1) / splits;
  P.n_splits = (key_tiles + P.split_tiles - 1) / P.split_tiles;  // no empty split
  P.bh_count = bh;
  P.n_text = p.n_text;
  P.routed_k = 0;
  P.use_windows = 0;
  P.text_row0 = 0;
  P.lse = P.n_splits > 1 ? part_lse : nullptr;
  P.dev_err = p.dev_err;
  P.scale_log2 = float(1.4426950408889634 / std::sqrt(double(p.head_dim)));
  P.flags = p.flags;
  P.all_full = kv_rows % kTileRows == 0;
  P.timeout_ns = (p.wait_timeout_us ? (unsigned long long)p.wait_timeout_us : 2000000ull) * 1000ull;
  const long long blocks = (long long)bh * P.dense_pairs * P.n_splits;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  basa_status st = run_attn(P, blocks, s);
  if (st != BASA_OK || P.n_splits == 1) return st;
  const void *outs[kMaxTextSplits];
  const float *lses[kMaxTextSplits];
  for (int i = 0; i < P.n_splits; ++i) {
    outs[i] = part + size_t(i) * bh * p.n_text * p.head_dim * 2;
    lses[i] = part_lse + size_t(i) * bh * p.n_text;
  }
  return launch_merge_rows(P.n_splits, outs, lses, out_text, nullptr, (long long)bh * p.n_text, p.head_dim, p.dtype, s);
}

}  // namespace basa

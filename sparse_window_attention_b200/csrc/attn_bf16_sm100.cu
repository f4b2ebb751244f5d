// Shifted-window attention forward, bfloat16, head_dim 128, for sm_100a.
//
// Operator (BASA §3.1-§3.3, §A.1): for each query of shifted window w,
//   out = softmax(q K^T / sqrt(d)) V  over K/V = [w | routed windows | pooled | text]
// written back at the query's original grid position.
//
// One CTA = (b*head, window, pair of 128-row query tiles). Warp roles:
//   warp 0      TMA loader: query tiles once, then a K, V, K, V ... stream of
//               128-row key tiles through a 3-slot shared-memory ring. Window
//               tiles are assembled from TMA box loads whose coordinates already
//               include the cyclic shift (mod the grid), so no rolled copy exists.
//   warp 1      tcgen05 issuer (one thread): S_g = Q_g K^T and O_g += P_g V with
//               fp32 accumulators in TMEM (S0, S1, O0, O1: 4 x 128 columns).
//   warps 2-9   two softmax warpgroups, one per query tile; a thread owns one
//               query row: reads its S row from TMEM, runs the online softmax in
//               fp32 (base-2 exponent, scale folded in), writes P (bf16) to shared
//               memory, rescales its O row in TMEM when the running max grows,
//               and at the end normalises O and stores it with TMA boxes at the
//               same (unshifted) coordinates the queries were loaded from.
// Every wait is bounded (globaltimer); on expiry the kernel records a bit in
// dev_err, drains its own in-flight copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "basa_internal.h"
#include "sm100_ptx.cuh"

namespace basa {
namespace {

constexpr int kThreads = 320;
constexpr uint32_t kHalfBytes = 16384;                 // 128 rows x 128 B (64 bf16) , 128B-swizzled
constexpr uint32_t kTileBytes = 2 * kHalfBytes;        // 128 rows x head_dim 128
constexpr int kStages = 3;
constexpr uint32_t kSmemQ = 0;                         // 2 query tiles (reused for the output)
constexpr uint32_t kSmemP = 2 * kTileBytes;            // 2 P tiles
constexpr uint32_t kSmemRing = 4 * kTileBytes;         // K/V ring
constexpr uint32_t kSmemCtrl = kSmemRing + kStages * kTileBytes;
constexpr uint32_t kCtrlBytes = 1024;
constexpr uint32_t kSmemBytes = kSmemCtrl + kCtrlBytes + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;

// tcgen05 instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9, 10-12 = 1), N >> 3 at bits 17-22, M >> 4 at bits 24-28; bit 16 marks
// B as MN-major (V is stored key-major with head_dim contiguous).
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescQK | (1u << 16);

// Shared-memory matrix descriptor, 128-byte swizzle, sm100 layout (version 1 at bit 46).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

struct alignas(64) AttnParams {
  CUtensorMap map_q[kMaxShapes];
  CUtensorMap map_k[kMaxShapes];
  CUtensorMap map_v[kMaxShapes];
  CUtensorMap map_o[kMaxShapes];
  CUtensorMap map_kp, map_vp, map_kt, map_vt;
  WindowPlan plan;
  const int32_t *route;
  int32_t *dev_err;
  Geo g;
  int routed_k, n_pool, n_text, n_pool_tiles, n_text_tiles;
  float scale_log2;
  uint32_t flags;
  unsigned long long timeout_ns;
};

struct Ctrl {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full, s_full[2], p_full[2], o_full[2], drain;
  uint32_t tmem_base;
  int abort;
  int wtype[1 + kMaxRouted];
  int org[1 + kMaxRouted][3];
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");

// Bounded mbarrier wait. Gives up when the shared abort flag is set or after
// timeout_ns; the first waiter that times out sets the flag and its dev_err bit.
struct Waiter {
  Ctrl *c;
  int32_t *dev_err;
  unsigned long long limit;
  int bit;
  bool honor_abort;
  __device__ bool wait(uint64_t *bar, uint32_t parity) const {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      if (ptx::mbar_try_wait(bar, parity)) return true;
      if ((it & 15u) == 0) {
        if (honor_abort && *reinterpret_cast<volatile int *>(&c->abort)) return false;
        if (ptx::globaltimer_ns() - t0 > limit) {
          *reinterpret_cast<volatile int *>(&c->abort) = 1;
          if (dev_err) atomicOr(dev_err, bit);
          return false;
        }
      }
    }
  }
};

// Position in the key-tile stream: segments 0..routed_k are windows (own, then
// routed), then the pooled tokens, then the text tokens.
struct KeyIter {
  int seg, t;
};

__device__ __forceinline__ int seg_tiles(const AttnParams &P, const Ctrl &c, int seg) {
  if (seg <= P.routed_k) return P.plan.type[c.wtype[seg]].n_tiles;
  if (seg == P.routed_k + 1) return P.n_pool_tiles;
  return P.n_text_tiles;
}
__device__ __forceinline__ void advance(const AttnParams &P, const Ctrl &c, KeyIter &it) {
  ++it.t;
  while (it.seg <= P.routed_k + 2 && it.t >= seg_tiles(P, c, it.seg)) {
    ++it.seg;
    it.t = 0;
  }
}

__device__ __forceinline__ int wrap(int x, int g) { return x >= g ? x - g : x; }

// Issue the TMA loads of one 128-row tile of a window (query, key or value tile).
// Returns the bytes the loads will deliver.
__device__ __forceinline__ uint32_t load_window_tile(const AttnParams &P, const CUtensorMap *maps, const PlanTile &tile,
                                                     const int *org, int bh, uint8_t *dst, uint64_t *bar) {
  uint32_t bytes = 0;
  for (int i = 0; i < tile.n_pieces; ++i) {
    const PlanPiece pc = P.plan.piece[tile.first_piece + i];
    const int x = wrap(org[2] + pc.lx, P.g.W), y = wrap(org[1] + pc.ly, P.g.H), t = wrap(org[0] + pc.lt, P.g.T);
    uint8_t *d = dst + uint32_t(pc.dest) * 128u;
    ptx::tma_load_5d(d, &maps[pc.shape], bar, 0, x, y, t, bh);
    ptx::tma_load_5d(d + kHalfBytes, &maps[pc.shape], bar, 64, x, y, t, bh);
    bytes += uint32_t(P.plan.shape[pc.shape].rows) * 256u;
  }
  return bytes;
}

__device__ __forceinline__ uint32_t load_key_tile(const AttnParams &P, const Ctrl &c, const KeyIter &it, bool is_v,
                                                  int bh, uint8_t *dst, uint64_t *bar) {
  if (it.seg <= P.routed_k) {
    const PlanTile &tile = P.plan.tile[P.plan.type[c.wtype[it.seg]].first_tile + it.t];
    return load_window_tile(P, is_v ? P.map_v : P.map_k, tile, c.org[it.seg], bh, dst, bar);
  }
  const bool pooled = it.seg == P.routed_k + 1;
  const CUtensorMap *map = pooled ? (is_v ? &P.map_vp : &P.map_kp) : (is_v ? &P.map_vt : &P.map_kt);
  const int row = (pooled ? 0 : P.g.N) + it.t * kTileRows;
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
    return tile.valid_rows == kTileRows;
  }
  const int total = (it.seg == P.routed_k + 1) ? P.n_pool : P.n_text;
  const int valid = min(kTileRows, total - it.t * kTileRows);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int v = valid - 32 * i;
    m[i] = v >= 32 ? 0xFFFFFFFFu : (v <= 0 ? 0u : ((1u << v) - 1u));
  }
  return valid == kTileRows;
}

__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
    ptx::mma_bf16_ss(d_tmem, smem_desc(q_addr + off, 16, 1024), smem_desc(k_addr + off, 16, 1024), kIdescQK, kk > 0);
  }
}
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_addr, uint32_t v_addr, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
    ptx::mma_bf16_ss(d_tmem, smem_desc(p_addr + off, 16, 1024), smem_desc(v_addr + kk * 2048, kHalfBytes, 1024),
                     kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(kThreads, 1) attn_bf16_kernel(const __grid_constant__ AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl &c = *reinterpret_cast<Ctrl *>(smem + kSmemCtrl);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const int pairs = P.plan.max_pairs;
  const int pair = blockIdx.x % pairs;
  const int w = (blockIdx.x / pairs) % P.g.nWin;
  const int bh = blockIdx.x / (pairs * P.g.nWin);
  int ot, oy, ox, wtype;
  window_origin(P.g, w, &ot, &oy, &ox, &wtype);
  const PlanType ty = P.plan.type[wtype];
  const int q_tile0 = 2 * pair;
  if (q_tile0 >= ty.n_tiles) return;  // whole CTA: this window type has fewer query tiles
  const bool has_q1 = q_tile0 + 1 < ty.n_tiles;

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
    c.wtype[0] = wtype;
    c.org[0][0] = ot; c.org[0][1] = oy; c.org[0][2] = ox;
    for (int r = 0; r < P.routed_k; ++r) {
      const int u = P.route[((long long)bh * P.g.nWin + w) * P.routed_k + r];
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

  int n_kt = P.n_pool_tiles + P.n_text_tiles;
  for (int s = 0; s <= P.routed_k; ++s) n_kt += P.plan.type[c.wtype[s]].n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA loader
    if (lane == 0) {
      Waiter wt{&c, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_PRODUCER, true};
      Waiter drain{&c, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_PRODUCER, false};
      uint32_t qbytes = 0;
      for (int g = 0; g < (has_q1 ? 2 : 1); ++g) {
        const PlanTile &tile = P.plan.tile[ty.first_tile + q_tile0 + g];
        for (int i = 0; i < tile.n_pieces; ++i)
          qbytes += uint32_t(P.plan.shape[P.plan.piece[tile.first_piece + i].shape].rows) * 256u;
      }
      ptx::mbar_arrive_expect_tx(&c.q_full, qbytes);
      for (int g = 0; g < (has_q1 ? 2 : 1); ++g)
        load_window_tile(P, P.map_q, P.plan.tile[ty.first_tile + q_tile0 + g], c.org[0], bh, smem + kSmemQ + g * kTileBytes,
                         &c.q_full);
      KeyIter it{0, 0};
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
          uint32_t bytes = 0;
          if (it.seg <= P.routed_k) {
            const PlanTile &tile = P.plan.tile[P.plan.type[c.wtype[it.seg]].first_tile + it.t];
            for (int i = 0; i < tile.n_pieces; ++i)
              bytes += uint32_t(P.plan.shape[P.plan.piece[tile.first_piece + i].shape].rows) * 256u;
          } else {
            bytes = kTileBytes;
          }
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
      Waiter wt{&c, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_MMA, true};
      Waiter drain{&c, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_MMA, false};
      const uint32_t sQ = ptx::smem_u32(smem + kSmemQ), sP = ptx::smem_u32(smem + kSmemP);
      const uint32_t sR = ptx::smem_u32(smem + kSmemRing);
      const uint32_t tS0 = tmem, tS1 = tmem + 128, tO0 = tmem + 256, tO1 = tmem + 384;
      if (wt.wait(&c.q_full, 0) && wt.wait(&c.full[0], 0)) {
        ptx::tc_fence_after();
        issue_qk(tS0, sQ, sR);
        ptx::mma_commit(&c.s_full[0]);
        if (has_q1) {
          issue_qk(tS1, sQ + kTileBytes, sR);
          ptx::mma_commit(&c.s_full[1]);
        }
        ptx::mma_commit(&c.empty[0]);
        for (int j = 0; j < n_kt; ++j) {
          const int vi = 2 * j + 1, ki = 2 * j + 2;
          const uint32_t vaddr = sR + (vi % kStages) * kTileBytes, kaddr = sR + (ki % kStages) * kTileBytes;
          const bool more = j + 1 < n_kt;
          if (!wt.wait(&c.full[vi % kStages], (vi / kStages) & 1)) break;
          if (!wt.wait(&c.p_full[0], j & 1)) break;
          ptx::tc_fence_after();
          issue_pv(tO0, sP, vaddr, j > 0);
          if (more) {
            if (!wt.wait(&c.full[ki % kStages], (ki / kStages) & 1)) break;
            ptx::tc_fence_after();
            issue_qk(tS0, sQ, kaddr);
            ptx::mma_commit(&c.s_full[0]);
          } else {
            ptx::mma_commit(&c.o_full[0]);
          }
          if (has_q1) {
            if (!wt.wait(&c.p_full[1], j & 1)) break;
            ptx::tc_fence_after();
            issue_pv(tO1, sP + kTileBytes, vaddr, j > 0);
          }
          ptx::mma_commit(&c.empty[vi % kStages]);
          if (more) {
            if (has_q1) {
              issue_qk(tS1, sQ + kTileBytes, kaddr);
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
  } else {
    // ------------------------------------------------------------- softmax
    const int g = (warp - 2) / 4;
    const int sub = warp % 4;  // TMEM lane quarter this warp may access
    const int row = sub * 32 + lane;
    const uint32_t lane_off = uint32_t(sub * 32) << 16;
    const uint32_t tS = tmem + lane_off + g * 128, tO = tmem + lane_off + 256 + g * 128;
    const bool active = g == 0 || has_q1;
    Waiter wt{&c, P.dev_err, P.timeout_ns, BASA_DEVERR_TIMEOUT_SOFTMAX, true};
    uint8_t *p_tile = smem + kSmemP + g * kTileBytes;
    uint8_t *q_tile = smem + kSmemQ + g * kTileBytes;
    const uint32_t p_row = ptx::smem_u32(p_tile) + row * 128;
    const uint32_t swz = row & 7;
    float m = -INFINITY, l = 0.f;
    bool ok = active;
    KeyIter it{0, 0};
    for (int j = 0; ok && j < n_kt; ++j) {
      ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.s_full[g], j & 1));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t s[128];
      ptx::tmem_ld128(tS, s);
      ptx::tmem_ld_wait(s);
      uint32_t mask[4];
      if (!key_tile_mask(P, c, it, mask)) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (!((mask[i >> 5] >> (i & 31)) & 1u)) s[i] = __float_as_uint(-INFINITY);
      }
      float mx0 = __uint_as_float(s[0]), mx1 = __uint_as_float(s[1]), mx2 = __uint_as_float(s[2]),
            mx3 = __uint_as_float(s[3]);
#pragma unroll
      for (int i = 4; i < 128; i += 4) {
        mx0 = fmaxf(mx0, __uint_as_float(s[i]));
        mx1 = fmaxf(mx1, __uint_as_float(s[i + 1]));
        mx2 = fmaxf(mx2, __uint_as_float(s[i + 2]));
        mx3 = fmaxf(mx3, __uint_as_float(s[i + 3]));
      }
      const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
      const float m_new = fmaxf(m, mx * P.scale_log2);
      const float alpha = ptx::ex2(m - m_new);
      const float neg_m = -m_new;
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int i = 0; i < 128; i += 2) {
        const float p0 = ptx::ex2(fmaf(__uint_as_float(s[i]), P.scale_log2, neg_m));
        const float p1 = ptx::ex2(fmaf(__uint_as_float(s[i + 1]), P.scale_log2, neg_m));
        sum0 += p0;
        sum1 += p1;
        s[i] = __float_as_uint(p0);
        s[i + 1] = __float_as_uint(p1);
      }
      l = l * alpha + (sum0 + sum1);
      m = m_new;
      // P row -> shared memory, K-major, 128-byte swizzle (16-byte chunk c of the
      // 128-byte row r sits at chunk position c ^ (r % 8)).
#pragma unroll
      for (int c16 = 0; c16 < 16; ++c16) {
        const int k0 = c16 * 8;
        const uint32_t addr = p_row + (c16 >> 3) * kHalfBytes + (((c16 & 7) ^ swz) << 4);
        ptx::st_shared_v4(addr, ptx::pack_bf16x2(__uint_as_float(s[k0]), __uint_as_float(s[k0 + 1])),
                          ptx::pack_bf16x2(__uint_as_float(s[k0 + 2]), __uint_as_float(s[k0 + 3])),
                          ptx::pack_bf16x2(__uint_as_float(s[k0 + 4]), __uint_as_float(s[k0 + 5])),
                          ptx::pack_bf16x2(__uint_as_float(s[k0 + 6]), __uint_as_float(s[k0 + 7])));
      }
      ptx::fence_proxy_async_smem();
      if (j > 0 && __any_sync(0xFFFFFFFFu, alpha < 1.0f)) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          ptx::tmem_ld32(tO + cc * 32, r);
          ptx::tmem_ld_wait(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          ptx::tmem_st32(tO + cc * 32, r);
        }
        ptx::tmem_st_wait();
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&c.p_full[g]);
      advance(P, c, it);
    }
    if (ok) ok = __all_sync(0xFFFFFFFFu, wt.wait(&c.o_full[g], 0));
    if (ok) {
      ptx::tc_fence_after();
      const float inv = 1.0f / l;
      const uint32_t o_row = ptx::smem_u32(q_tile) + row * 128;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        ptx::tmem_ld32(tO + cc * 32, r);
        ptx::tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c16 = cc * 4 + i;
          const uint32_t addr = o_row + (c16 >> 3) * kHalfBytes + (((c16 & 7) ^ swz) << 4);
          const int b = 8 * i;
          ptx::st_shared_v4(addr, ptx::pack_bf16x2(__uint_as_float(r[b]) * inv, __uint_as_float(r[b + 1]) * inv),
                            ptx::pack_bf16x2(__uint_as_float(r[b + 2]) * inv, __uint_as_float(r[b + 3]) * inv),
                            ptx::pack_bf16x2(__uint_as_float(r[b + 4]) * inv, __uint_as_float(r[b + 5]) * inv),
                            ptx::pack_bf16x2(__uint_as_float(r[b + 6]) * inv, __uint_as_float(r[b + 7]) * inv));
        }
      }
      ptx::fence_proxy_async_smem();
    }
    ptx::named_barrier(1 + g, 128);
    if (active && row == 0 && !*reinterpret_cast<volatile int *>(&c.abort)) {
      const PlanTile &tile = P.plan.tile[ty.first_tile + q_tile0 + g];
      for (int i = 0; i < tile.n_pieces; ++i) {
        const PlanPiece pc = P.plan.piece[tile.first_piece + i];
        const int x = wrap(ox + pc.lx, P.g.W), y = wrap(oy + pc.ly, P.g.H), t = wrap(ot + pc.lt, P.g.T);
        const uint8_t *src = q_tile + uint32_t(pc.dest) * 128u;
        ptx::tma_store_5d(&P.map_o[pc.shape], src, 0, x, y, t, bh);
        ptx::tma_store_5d(&P.map_o[pc.shape], src + kHalfBytes, 64, x, y, t, bh);
      }
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
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map (d, row, b*head) with 128-row boxes; rows past the end read as zero.
bool encode_rows_map(CUtensorMap *m, const void *base, const basa_params &p, long long rows_per_bh) {
  const cuuint64_t e = 2;
  cuuint64_t dims[3] = {cuuint64_t(p.head_dim), cuuint64_t(rows_per_bh), cuuint64_t(p.B) * cuuint64_t(p.heads)};
  cuuint64_t strides[2] = {p.head_dim * e, cuuint64_t(rows_per_bh) * p.head_dim * e};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

basa_status launch_attn_bf16(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                             const int32_t *route_idx, void *out, const basa_params &p, cudaStream_t s) {
  if (!encode_fn()) return BASA_ERR_CUDA;
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
  P.n_pool_tiles = (P.n_pool + kTileRows - 1) / kTileRows;
  P.n_text_tiles = (p.n_text + kTileRows - 1) / kTileRows;
  P.route = route_idx;
  P.dev_err = p.dev_err;
  P.routed_k = p.routed_k;
  P.scale_log2 = float(1.4426950408889634 / std::sqrt(double(p.head_dim)));
  P.flags = p.flags;
  P.timeout_ns = (p.wait_timeout_us ? (unsigned long long)p.wait_timeout_us : 2000000ull) * 1000ull;
  const long long blocks = (long long)p.B * p.heads * P.g.nWin * P.plan.max_pairs;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return BASA_ERR_CUDA;
  attn_bf16_kernel<<<unsigned(blocks), kThreads, kSmemBytes, s>>>(P);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

}  // namespace basa

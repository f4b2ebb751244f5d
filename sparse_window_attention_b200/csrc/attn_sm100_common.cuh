// Pieces shared by the tensor-core attention kernels (forward and backward) for
// sm_100a: the shared-memory operand layout of a 128-row x 128-column bf16 tile,
// the tcgen05 instruction and shared-memory descriptors for it, the TMA box loads
// that assemble a window tile from the tiling plan (the cyclic shift is only
// coordinate arithmetic), the 128 x 128 x 128 MMA sequences, the bounded mbarrier
// wait, and the host-side tensor-map encoders.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "basa_internal.h"
#include "sm100_ptx.cuh"

namespace basa {
namespace sm100 {

// A tile is 128 rows (tokens) x head_dim 128 bf16, stored as two 64-column halves of
// 128 rows x 128 bytes, each 128-byte swizzled (the TMA box's inner extent is 64
// elements, so head_dim 128 is two box loads).
constexpr uint32_t kHalfBytes = 16384;
constexpr uint32_t kTileBytes = 2 * kHalfBytes;

// tcgen05 instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9, 10-12 = 1), N >> 3 at bits 17-22, M >> 4 at bits 24-28; bit 16 marks
// B as MN-major (a token-major tile read with head_dim as the N dimension).
constexpr uint32_t kIdescKMajor = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescBMnMajor = kIdescKMajor | (1u << 16);

// Shared-memory descriptors, split in 32-bit halves. The high half is constant:
// stride byte offset 1024 (8 rows of 128 B), version 1, 128-byte swizzle. The
// low half holds the start address >> 4 (bits 0-13) and the leading byte offset
// (bits 16-29; ignored for K-major swizzled operands, 16 KB between the two
// 64-column halves of an MN-major operand). Stepping the start address is one add.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
constexpr uint32_t kDescLoK = (16u >> 4) << 16;
constexpr uint32_t kDescLoMn = (kHalfBytes >> 4) << 16;
constexpr uint32_t kTileDesc = kTileBytes >> 4;

// D (=) A B^T over head_dim 128 with both operands token-major tiles in shared
// memory (K-major): 8 K-steps of 16; steps 0-3 walk the first 64-column half in
// 32-byte strides, steps 4-7 the second half. D is 128 x 128 fp32 in TMEM.
__device__ __forceinline__ void issue_ss(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
    ptx::mma_bf16_ss2(d_tmem, a_lo + off, kDescHi, b_lo + off, kDescHi, kIdescKMajor, kk > 0);
  }
}

// D (+)= A B with A (bf16, 128 rows x 128 K) in TMEM and B a token-major tile in
// shared memory read MN-major (its 128 tokens are the K dimension, head_dim is N).
// 16 K = 8 TMEM columns per step; K-step kk reads A from column a_col(kk).
// Contiguous layout: A at columns [a, a + 64).
__device__ __forceinline__ void issue_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    ptx::mma_bf16_ts2(d_tmem, a_tmem + kk * 8, b_lo + ((kk * 2048) >> 4), kDescHi, kIdescBMnMajor,
                      (accumulate || kk > 0) ? 1u : 0u);
}
// Split layout: K 0-63 at columns [a, a + 32), K 64-127 at [a + 64, a + 96), so two
// warpgroups that each own 64 columns of a 128-column fp32 buffer can write their
// packed bf16 halves in place without touching the other's inputs.
__device__ __forceinline__ void issue_ts_split(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    ptx::mma_bf16_ts2(d_tmem, a_tmem + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), b_lo + ((kk * 2048) >> 4), kDescHi,
                      kIdescBMnMajor, (accumulate || kk > 0) ? 1u : 0u);
}

// D (=) A B^T over head_dim 128 with A (bf16, 128 rows x 128) in TMEM, 8 columns per
// K-step of 16, and B a token-major tile in shared memory read K-major as in issue_ss.
__device__ __forceinline__ void issue_ts_kmajor(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
    ptx::mma_bf16_ts2(d_tmem, a_tmem + kk * 8, b_lo + off, kDescHi, kIdescKMajor, kk > 0 ? 1u : 0u);
  }
}

// The K-steps of issue_ts_split that read group g's half: K rows [64 g, 64 g + 64)
// of B and A columns [a + 64 g, a + 64 g + 32).
__device__ __forceinline__ void issue_ts_group(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, int g,
                                               bool accumulate) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int kk = 4 * g + i;
    ptx::mma_bf16_ts2(d_tmem, a_tmem + 64 * g + i * 8, b_lo + ((kk * 2048) >> 4), kDescHi, kIdescBMnMajor,
                      (accumulate || i > 0) ? 1u : 0u);
  }
}

__device__ __forceinline__ int wrap(int x, int g) { return x >= g ? x - g : x; }

// Issue the TMA loads of one 128-row tile of a window (query, key or value tile):
// one box per plan piece at coordinates (window origin + piece offset) mod grid,
// two 64-column halves each. Returns the bytes the loads will deliver.
__device__ __forceinline__ uint32_t load_window_tile(const WindowPlan &plan, const Geo &g, const CUtensorMap *maps,
                                                     const PlanTile &tile, const int *org, int bh, uint8_t *dst,
                                                     uint64_t *bar) {
  uint32_t bytes = 0;
  for (int i = 0; i < tile.n_pieces; ++i) {
    const PlanPiece pc = plan.piece[tile.first_piece + i];
    const int x = wrap(org[2] + pc.lx, g.W), y = wrap(org[1] + pc.ly, g.H), t = wrap(org[0] + pc.lt, g.T);
    uint8_t *d = dst + uint32_t(pc.dest) * 128u;
    ptx::tma_load_5d(d, &maps[pc.shape], bar, 0, x, y, t, bh);
    ptx::tma_load_5d(d + kHalfBytes, &maps[pc.shape], bar, 64, x, y, t, bh);
    bytes += uint32_t(plan.shape[pc.shape].rows) * 256u;
  }
  return bytes;
}

// The same boxes over a per-token array of 16-byte records (no swizzle): record r of
// the tile lands at dst + 16 r. Returns the bytes delivered.
__device__ __forceinline__ uint32_t load_window_records(const WindowPlan &plan, const Geo &g, const CUtensorMap *maps,
                                                        const PlanTile &tile, const int *org, int bh, uint8_t *dst,
                                                        uint64_t *bar) {
  uint32_t bytes = 0;
  for (int i = 0; i < tile.n_pieces; ++i) {
    const PlanPiece pc = plan.piece[tile.first_piece + i];
    const int x = wrap(org[2] + pc.lx, g.W), y = wrap(org[1] + pc.ly, g.H), t = wrap(org[0] + pc.lt, g.T);
    ptx::tma_load_5d(dst + uint32_t(pc.dest) * 16u, &maps[pc.shape], bar, 0, x, y, t, bh);
    bytes += uint32_t(plan.shape[pc.shape].rows) * 16u;
  }
  return bytes;
}

// Store a 128-row tile staged in shared memory (the same swizzled layout) back to
// the token positions its plan pieces cover.
__device__ __forceinline__ void store_window_tile(const WindowPlan &plan, const Geo &g, const CUtensorMap *maps,
                                                  const PlanTile &tile, const int *org, int bh, const uint8_t *src) {
  for (int i = 0; i < tile.n_pieces; ++i) {
    const PlanPiece pc = plan.piece[tile.first_piece + i];
    const int x = wrap(org[2] + pc.lx, g.W), y = wrap(org[1] + pc.ly, g.H), t = wrap(org[0] + pc.lt, g.T);
    const uint8_t *s = src + uint32_t(pc.dest) * 128u;
    ptx::tma_store_5d(&maps[pc.shape], s, 0, x, y, t, bh);
    ptx::tma_store_5d(&maps[pc.shape], s + kHalfBytes, 64, x, y, t, bh);
  }
}

// Token (original grid coordinates) held by row `row` of a window tile; false for
// a padding row.
__device__ __forceinline__ bool tile_row_token(const WindowPlan &plan, const Geo &g, const PlanTile &tile,
                                               const int *org, int row, int *t, int *y, int *x) {
  for (int i = 0; i < tile.n_pieces; ++i) {
    const PlanPiece pc = plan.piece[tile.first_piece + i];
    const PlanShape sh = plan.shape[pc.shape];
    const int local = row - int(pc.dest);
    if (local < 0 || local >= sh.rows) continue;
    const int lx = local % sh.cx, ly = (local / sh.cx) % sh.cy, lt = local / (sh.cx * sh.cy);
    *x = wrap(org[2] + pc.lx, g.W) + lx;
    *y = wrap(org[1] + pc.ly, g.H) + ly;
    *t = wrap(org[0] + pc.lt, g.T) + lt;
    return true;
  }
  return false;
}

// Bounded mbarrier wait. Gives up when the shared abort flag is set (if honoured)
// or after `limit` ns; the first waiter that times out sets the flag and ORs `bit`
// into dev_err.
struct Waiter {
  int *abort;
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
        if (honor_abort && *reinterpret_cast<volatile int *>(abort)) return false;
        if (ptx::globaltimer_ns() - t0 > limit) {
          *reinterpret_cast<volatile int *>(abort) = 1;
          if (dev_err) atomicOr(dev_err, bit);
          return false;
        }
      }
    }
  }
};

// Column mask of a run of `valid` rows starting at tile row 0.
__device__ __forceinline__ void prefix_mask(int valid, uint32_t *m) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int v = valid - 32 * i;
    m[i] = v >= 32 ? 0xFFFFFFFFu : (v <= 0 ? 0u : ((1u << v) - 1u));
  }
}

}  // namespace sm100

// ----------------------------------------------------------------- host side
// 5-D map (d, x, y, t, b*head) over the visual rows of a [B, heads, rows, 128] bf16
// tensor, box = one plan shape, 128-byte swizzle.
bool encode_grid_map(CUtensorMap *m, const void *base, const basa_params &p, long long rows_per_bh,
                     const PlanShape &s);
// 3-D map (d, row, b*head) over a [B*heads, rows, 128] bf16 tensor with box_rows-row
// boxes (128 unless given), 128-byte swizzle; rows past the end read as zero and are
// not stored.
bool encode_rows_map(CUtensorMap *m, const void *base, const basa_params &p, long long rows_per_bh,
                     int box_rows = 128);
// 5-D map (4, x, y, t, b*head) over a [B*heads, N, 4] float32 per-token record
// array, box = one plan shape, no swizzle (16-byte records).
bool encode_record_map(CUtensorMap *m, const void *base, const basa_params &p, const PlanShape &s);

}  // namespace basa

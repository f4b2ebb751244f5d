// Fused pre-pass of a BASA layer with routing: one read of Q, K and V yields
//  * the pooled K and V (BASA §3.2 "K/V-pooled global memory": means over the
//    pt x ph x pw patches of the UNSHIFTED grid; §A.1 "regular spatial reduction"),
//  * the window means of Q and K over the shifted windows that routing scores
//    (BASA §3.3 content-adaptive true-window routing),
// followed by the same warp top-k as the unfused path.
//
// Kernel 1 (cell_sum_kernel): the grid is cut into boxes of whole pool patches,
// one CTA per (b*head, box). Inside a box, pool-patch boundaries and window
// boundaries cut every axis into intervals; their products are "cells", each
// inside one pool patch and one window. The CTA
//   1. sums Q, K and V over every cell (one read of each token: threads own a
//      (cell, 16-byte column) pair, split by token rows when cells are few),
//   2. adds the cells of each pool patch -> pooled K and V (complete: a patch
//      never straddles boxes), and the cells of each window it meets -> partial
//      sums of Q and K over box ∩ window, stored in the window's slot for this box.
// Kernel 2 (window_reduce_kernel) adds each window's slots in a fixed order and
// scales by 1 / |window|. Nothing is accumulated with atomics: every sum has a
// fixed order, so the results do not depend on scheduling.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "basa_internal.h"

namespace basa {
namespace {

constexpr int kCellThreads = 256;
constexpr int kMaxAxisRuns = 32;   // windows met by a box along one axis
constexpr int kMaxAxisCells = 64;  // cells along one axis
constexpr int kMaxCells = 96;      // cells of a box
constexpr int kBoxTokens = 512;    // preferred box size (tokens)
constexpr size_t kSmemTwoCtas = 110 * 1024;  // shared memory that still fits two CTAs per SM

// The windows one box meets along one axis: window index j and its (at most
// two) runs of box-local coordinates [lo, hi). Two runs only when the box spans
// the whole axis and the window wraps around its edge.
struct AxisRun {
  int j, lo0, hi0, lo1, hi1;
};

// One interval of an axis inside the box: [lo, hi), the run (window) and the
// pool patch (box-local index) it lies in.
struct AxisCell {
  int16_t lo, hi, run, patch;
};

struct FusedArgs {
  const void *src[3];      // q, k, v
  long long bh_stride[3];  // elements between consecutive (b, head) slices
  void *kp, *vp;
  float *part;
  int d, lpr;              // head_dim; 16-byte chunks per token
  int G[3], e[3], nb[3], pool[3], w[3], s[3], nw[3], K[3];
  int bh;
  float inv_pool;
};

struct CellCtrl {
  int n_runs[3], n_cells[3];
  AxisRun run[3][kMaxAxisRuns];
  AxisCell cell[3][kMaxAxisCells];
};

// Runs of the windows met by the box [o, o + e) along one axis (window extent w,
// shift s, grid extent G): original coordinate c lies in window ((c - s) mod G) / w,
// and window boundaries fall every w coordinates of the shifted axis.
__host__ __device__ void build_runs(int o, int e, int w, int s, int G, AxisRun *runs, int *n_out) {
  int n = 0;
  int c = 0;
  while (c < e && n < kMaxAxisRuns) {
    const int sc = ((o + c - s) % G + G) % G;
    const int j = sc / w;
    const int len = min(e - c, (j + 1) * w - sc);
    if (n > 0 && runs[0].j == j) {  // the first window again, past the wrap
      runs[0].lo1 = c;
      runs[0].hi1 = c + len;
    } else {
      runs[n] = {j, c, c + len, 0, 0};
      ++n;
    }
    c += len;
  }
  *n_out = n;
}

// Cells of one axis in coordinate order: the run intervals cut at pool-patch
// boundaries (multiples of p).
__host__ __device__ void build_cells(const AxisRun *runs, int n_runs, int p, AxisCell *cells, int *n_out) {
  int n = 0;
  // intervals in coordinate order: run 0, 1, ..., n_runs - 1, then run 0's wrapped part
  for (int k = 0; k <= n_runs; ++k) {
    const int r = k < n_runs ? k : 0;
    const int lo = k < n_runs ? runs[r].lo0 : runs[0].lo1, hi = k < n_runs ? runs[r].hi0 : runs[0].hi1;
    for (int c = lo; c < hi && n < kMaxAxisCells;) {
      const int nxt = min(hi, (c / p + 1) * p);
      cells[n++] = {int16_t(c), int16_t(nxt), int16_t(r), int16_t(c / p)};
      c = nxt;
    }
  }
  *n_out = n;
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void add(float *acc, const uint4 &v) {
    acc[0] += __uint_as_float(v.x << 16); acc[1] += __uint_as_float(v.x & 0xFFFF0000u);
    acc[2] += __uint_as_float(v.y << 16); acc[3] += __uint_as_float(v.y & 0xFFFF0000u);
    acc[4] += __uint_as_float(v.z << 16); acc[5] += __uint_as_float(v.z & 0xFFFF0000u);
    acc[6] += __uint_as_float(v.w << 16); acc[7] += __uint_as_float(v.w & 0xFFFF0000u);
  }
  __device__ static void store_mean(void *dst, const float *acc, float scale) {
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r[i]) : "f"(acc[2 * i + 1] * scale), "f"(acc[2 * i] * scale));
    *reinterpret_cast<uint4 *>(dst) = make_uint4(r[0], r[1], r[2], r[3]);
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void add(float *acc, const uint4 &v) {
    acc[0] += __uint_as_float(v.x); acc[1] += __uint_as_float(v.y);
    acc[2] += __uint_as_float(v.z); acc[3] += __uint_as_float(v.w);
  }
  __device__ static void store_mean(void *dst, const float *acc, float scale) {
    *reinterpret_cast<float4 *>(dst) = make_float4(acc[0] * scale, acc[1] * scale, acc[2] * scale, acc[3] * scale);
  }
};

__device__ __forceinline__ uint4 ldg16(const uint8_t *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void decode_box(const FusedArgs &a, int b, int *bh, int *box) {
  box[2] = b % a.nb[2]; b /= a.nb[2];
  box[1] = b % a.nb[1]; b /= a.nb[1];
  box[0] = b % a.nb[0];
  *bh = b / a.nb[0];
}

template <typename T>
__global__ void __launch_bounds__(kCellThreads) cell_sum_kernel(const __grid_constant__ FusedArgs a) {
  constexpr int VEC = Vec<T>::N;
  extern __shared__ float4 smem_f4[];
  CellCtrl &c = *reinterpret_cast<CellCtrl *>(smem_f4);
  float *red = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(smem_f4) + ((sizeof(CellCtrl) + 15) & ~size_t(15)));
  float *cellsum = red + 3 * VEC * kCellThreads;  // [cell][tensor][d]
  const int tid = threadIdx.x;
  int bh, box[3];
  decode_box(a, blockIdx.x, &bh, box);
  if (tid < 3) {
    build_runs(box[tid] * a.e[tid], a.e[tid], a.w[tid], a.s[tid], a.G[tid], c.run[tid], &c.n_runs[tid]);
    build_cells(c.run[tid], c.n_runs[tid], a.pool[tid], c.cell[tid], &c.n_cells[tid]);
  }
  __syncthreads();
  const int nct = c.n_cells[0], ncy = c.n_cells[1], ncx = c.n_cells[2];
  const int row_bytes = a.d * int(sizeof(T));

  // ---- 1. Q, K, V sums over every cell
  {
    const int units = nct * ncy * ncx * a.lpr;
    // splits of a unit take every S-th token of its cell (row-major order)
    const int S = units >= kCellThreads ? 1 : kCellThreads / units;
    const int R = kCellThreads / S;
    for (int u0 = 0; u0 < units; u0 += R) {
      const int unit = u0 + tid % R, split = tid / R;
      const bool valid = unit < units && split < S;
      float acc[3][VEC];
#pragma unroll
      for (int t = 0; t < 3; ++t)
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[t][i] = 0.f;
      const int col = unit % a.lpr, ci = unit / a.lpr;
      if (valid) {
        const AxisCell cx = c.cell[2][ci % ncx], cy = c.cell[1][(ci / ncx) % ncy], ct = c.cell[0][ci / (ncx * ncy)];
        const int lenx = cx.hi - cx.lo, leny = cy.hi - cy.lo;
        const int n = (ct.hi - ct.lo) * leny * lenx;
        const uint8_t *base[3];
#pragma unroll
        for (int t = 0; t < 3; ++t)
          base[t] = static_cast<const uint8_t *>(a.src[t]) + ((long long)bh * a.bh_stride[t]) * int(sizeof(T)) + col * 16;
        // token (lt, ly, lx) of the cell <-> grid row ((t0 + lt) * H + y0 + ly) * W + x0 + lx;
        // positions advance by S tokens with carries, no division per token
        const uint32_t t0 = uint32_t(box[0] * a.e[0] + ct.lo), y0 = uint32_t(box[1] * a.e[1] + cy.lo),
                       x0 = uint32_t(box[2] * a.e[2] + cx.lo);
        const int dx = S % lenx, dyx = S / lenx;
        int lx = split % lenx, lyx = split / lenx;  // lyx = lt * leny + ly
        int ly = lyx % leny, lt = lyx / leny;
        const int dy = dyx % leny, dt = dyx / leny;
        const uint32_t W = uint32_t(a.G[2]), HW = uint32_t(a.G[1]) * W;
        for (int i = split; i < n;) {
          uint32_t off[4];
          int cnt = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (i < n) {
              off[k] = ((t0 + lt) * HW + (y0 + ly) * W + x0 + lx) * uint32_t(row_bytes);
              ++cnt;
              i += S;
              lx += dx;
              ly += dy;
              lt += dt;
              if (lx >= lenx) { lx -= lenx; ++ly; }
              if (ly >= leny) { ly -= leny; ++lt; }
            } else {
              off[k] = off[0];
            }
          }
          uint4 v[3][4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int t = 0; t < 3; ++t) v[t][k] = ldg16(base[t] + off[k]);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k < cnt)
#pragma unroll
              for (int t = 0; t < 3; ++t) Vec<T>::add(acc[t], v[t][k]);
        }
      }
      if (S > 1) {
        // S > 1 means a single round, so every thread reaches every barrier. Tree in
        // a fixed order: split s < cur - half adds split s + half, until one is left.
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
          for (int i = 0; i < VEC; ++i) red[(t * VEC + i) * kCellThreads + tid] = acc[t][i];
        __syncthreads();
        for (int cur = S; cur > 1;) {
          const int half = (cur + 1) / 2;
          if (valid && split < cur - half) {
#pragma unroll
            for (int t = 0; t < 3; ++t)
#pragma unroll
              for (int i = 0; i < VEC; ++i) {
                acc[t][i] += red[(t * VEC + i) * kCellThreads + tid + half * R];
                red[(t * VEC + i) * kCellThreads + tid] = acc[t][i];
              }
          }
          __syncthreads();
          cur = half;
        }
      }
      if (valid && split == 0) {
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          float4 *dst = reinterpret_cast<float4 *>(cellsum + (ci * 3 + t) * a.d + col * VEC);
#pragma unroll
          for (int i = 0; i < VEC; i += 4) dst[i / 4] = make_float4(acc[t][i], acc[t][i + 1], acc[t][i + 2], acc[t][i + 3]);
        }
      }
    }
  }
  __syncthreads();

  // ---- 2. pool patches (K, V) and window partial sums (Q, K) from the cells
  const int np_t = a.e[0] / a.pool[0], np_y = a.e[1] / a.pool[1], np_x = a.e[2] / a.pool[2];
  const int pool_units = np_t * np_y * np_x * 2 * a.lpr;
  const int nrt = c.n_runs[0], nry = c.n_runs[1], nrx = c.n_runs[2];
  const int win_units = nrt * nry * nrx * 2 * a.lpr;
  const long long Np = (long long)(a.G[0] / a.pool[0]) * (a.G[1] / a.pool[1]) * (a.G[2] / a.pool[2]);
  const int nWin = a.nw[0] * a.nw[1] * a.nw[2];
  for (int u = tid; u < pool_units + win_units; u += kCellThreads) {
    const bool is_pool = u < pool_units;
    const int v = is_pool ? u : u - pool_units;
    const int col = v % a.lpr;
    const int which = (v / a.lpr) % 2;  // pool: 0 = K, 1 = V; window: 0 = Q, 1 = K
    int idx = v / (a.lpr * 2);
    int want[3];  // patch indices (pool) or run indices (window) per axis
    const int n2 = is_pool ? np_x : nrx, n1 = is_pool ? np_y : nry;
    want[2] = idx % n2; idx /= n2;
    want[1] = idx % n1;
    want[0] = idx / n1;
    const int tensor = is_pool ? 1 + which : which;
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
    for (int it = 0; it < nct; ++it) {
      const AxisCell &ct = c.cell[0][it];
      if ((is_pool ? ct.patch : ct.run) != want[0]) continue;
      for (int iy = 0; iy < ncy; ++iy) {
        const AxisCell &cy = c.cell[1][iy];
        if ((is_pool ? cy.patch : cy.run) != want[1]) continue;
        for (int ix = 0; ix < ncx; ++ix) {
          const AxisCell &cx = c.cell[2][ix];
          if ((is_pool ? cx.patch : cx.run) != want[2]) continue;
          const float4 *p = reinterpret_cast<const float4 *>(cellsum + (((it * ncy + iy) * ncx + ix) * 3 + tensor) * a.d +
                                                             col * VEC);
#pragma unroll
          for (int i = 0; i < VEC; i += 4) {
            const float4 q = p[i / 4];
            acc[i] += q.x; acc[i + 1] += q.y; acc[i + 2] += q.z; acc[i + 3] += q.w;
          }
        }
      }
    }
    if (is_pool) {
      const long long gt = (long long)box[0] * np_t + want[0], gy = (long long)box[1] * np_y + want[1],
                      gx = (long long)box[2] * np_x + want[2];
      const long long P = (gt * (a.G[1] / a.pool[1]) + gy) * (a.G[2] / a.pool[2]) + gx;
      T *dst = static_cast<T *>(which ? a.vp : a.kp) + ((long long)bh * Np + P) * a.d + col * VEC;
      Vec<T>::store_mean(dst, acc, a.inv_pool);
    } else {
      // slot of this box in the window's run of boxes along each axis
      const int j[3] = {c.run[0][want[0]].j, c.run[1][want[1]].j, c.run[2][want[2]].j};
      int k[3];
#pragma unroll
      for (int ax = 0; ax < 3; ++ax) {
        const int o = (j[ax] * a.w[ax] + a.s[ax]) % a.G[ax];
        k[ax] = (box[ax] - o / a.e[ax] + a.nb[ax]) % a.nb[ax];
      }
      const long long win = ((long long)j[0] * a.nw[1] + j[1]) * a.nw[2] + j[2];
      const long long slot = ((((long long)which * a.bh + bh) * nWin + win) * a.K[0] + k[0]) * a.K[1] * a.K[2] +
                             (long long)k[1] * a.K[2] + k[2];
      float *dst = a.part + slot * a.d + col * VEC;
#pragma unroll
      for (int i = 0; i < VEC; i += 4)
        *reinterpret_cast<float4 *>(dst + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
    }
  }
}

struct ReduceArgs {
  const float *part;
  float *means;  // [2][bh][nWin][d]
  int d, bh;
  int groups;    // threads adding one window's slots per column
  int G[3], e[3], nb[3], w[3], s[3], nw[3], K[3];
  float inv_win;
};

// CTA of 256 threads = `wpc` windows x `groups` x (d/4) float4 columns: thread
// (window, group g, column c4) adds the window's slots g, g + groups, ...; the
// group sums are then added in group order. Windows with few slots take one
// group (several windows per CTA), windows with many slots take up to eight.
__global__ void __launch_bounds__(256) window_reduce_kernel(const __grid_constant__ ReduceArgs a) {
  __shared__ float4 red[256];
  const int d4 = a.d / 4;
  const int groups = a.groups;
  const int wpc = blockDim.x / (d4 * groups);
  const int nWin = a.nw[0] * a.nw[1] * a.nw[2];
  const int local = threadIdx.x / (d4 * groups);
  const int g = (threadIdx.x / d4) % groups, c4 = threadIdx.x % d4;
  const int row = blockIdx.x * wpc + local;  // (tensor, bh, window)
  const bool valid = row < 2 * a.bh * nWin;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (valid) {
    const int win = row % nWin;
    const int j[3] = {win / (a.nw[1] * a.nw[2]), (win / a.nw[2]) % a.nw[1], win % a.nw[2]};
    int n[3];
#pragma unroll
    for (int ax = 0; ax < 3; ++ax) {
      const int o = (j[ax] * a.w[ax] + a.s[ax]) % a.G[ax];
      n[ax] = min((o + a.w[ax] - 1) / a.e[ax] - o / a.e[ax] + 1, a.nb[ax]);
    }
    const float4 *p = reinterpret_cast<const float4 *>(a.part) + (long long)row * a.K[0] * a.K[1] * a.K[2] * d4 + c4;
    const int total = n[0] * n[1] * n[2];
    for (int i = g; i < total; i += groups) {
      const int kx = i % n[2], ky = (i / n[2]) % n[1], kt = i / (n[2] * n[1]);
      const float4 v = p[(((long long)kt * a.K[1] + ky) * a.K[2] + kx) * d4];
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
  }
  if (groups > 1) {
    red[threadIdx.x] = s;
    __syncthreads();
    if (g == 0)
      for (int h = 1; h < groups; ++h) {
        const float4 v = red[threadIdx.x + h * d4];
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
      }
  }
  if (valid && g == 0)
    reinterpret_cast<float4 *>(a.means)[(long long)row * d4 + c4] =
        make_float4(s.x * a.inv_win, s.y * a.inv_win, s.z * a.inv_win, s.w * a.inv_win);
}

}  // namespace

// Largest number of cells (and of window runs) along one axis over the boxes
// [b e, (b + 1) e): one more than the coordinates inside the box where a pool patch
// or a window starts (window starts are the coordinates congruent to s mod w).
static void axis_counts(int G, int e, int p, int w, int s, int *max_cells, int *max_runs) {
  *max_cells = 0;
  *max_runs = 0;
  for (int o = 0; o < G; o += e) {
    int cells = 1, runs = 1;
    for (int x = o + 1; x < o + e; ++x) {
      const bool wstart = ((x - s) % w + w) % w == 0;
      runs += wstart;
      cells += wstart || x % p == 0;
    }
    *max_cells = std::max(*max_cells, cells);
    *max_runs = std::max(*max_runs, runs);
  }
}

static size_t cell_smem_bytes(int cells, int head_dim, basa_dtype dtype) {
  const int vec = dtype == BASA_BF16 ? 8 : 4;
  return ((sizeof(CellCtrl) + 15) & ~size_t(15)) + size_t(3) * vec * kCellThreads * sizeof(float) +
         size_t(cells) * 3 * head_dim * sizeof(float);
}

// Box choice: whole pool patches per axis, extents dividing the grid; the x extent
// is grown first (long contiguous rows), then y, then t, up to kBoxTokens tokens,
// halving the limit while some box would have more than kMaxCells cells or the
// cell sums would keep two CTAs from sharing an SM (one pool patch is the floor).
basa_status plan_fused(const basa_params &p, FusedPlan *fp) {
  const int G[3] = {p.T, p.H, p.W}, P[3] = {p.pt, p.ph, p.pw}, w[3] = {p.wt, p.wh, p.ww}, sh[3] = {p.st, p.sy, p.sx};
  for (int cap = kBoxTokens;; cap /= 2) {
    int e[3] = {P[0], P[1], P[2]};
    const int order[3] = {2, 1, 0};
    for (int oi = 0; oi < 3; ++oi) {
      const int ax = order[oi];
      const int n = G[ax] / P[ax];
      for (int m = n; m >= 1; --m) {
        if (n % m) continue;
        int t[3] = {e[0], e[1], e[2]};
        t[ax] = m * P[ax];
        if ((long long)t[0] * t[1] * t[2] <= cap) {
          e[ax] = t[ax];
          break;
        }
      }
    }
    bool fits = true;
    long long cells = 1;
    for (int ax = 0; ax < 3; ++ax) {
      int ca, ra;
      axis_counts(G[ax], e[ax], P[ax], w[ax], sh[ax], &ca, &ra);
      fits = fits && ca <= kMaxAxisCells && ra <= kMaxAxisRuns;
      cells *= ca;
    }
    fits = fits && cells <= kMaxCells;
    const bool single_patch = e[0] == P[0] && e[1] == P[1] && e[2] == P[2];
    if (fits && !single_patch && cell_smem_bytes(int(cells), p.head_dim, p.dtype) > kSmemTwoCtas) fits = false;
    if (fits) {
      for (int ax = 0; ax < 3; ++ax) {
        fp->e[ax] = e[ax];
        fp->nb[ax] = G[ax] / e[ax];
        // boxes a window meets along the axis: at most ceil((w - 1) / e) + 1
        fp->K[ax] = std::min((w[ax] - 1 + e[ax] - 1) / e[ax] + 1, fp->nb[ax]);
      }
      fp->max_cells = int(cells);
      const size_t nwin = size_t(p.T / p.wt) * (p.H / p.wh) * (p.W / p.ww);
      const size_t bh = size_t(p.B) * p.heads;
      fp->means_bytes = 2 * bh * nwin * p.head_dim * sizeof(float);
      fp->part_bytes = fp->means_bytes * fp->K[0] * fp->K[1] * fp->K[2];
      return BASA_OK;
    }
    if ((long long)P[0] * P[1] * P[2] > cap / 2 || cap <= 1) return BASA_ERR_UNSUPPORTED;
  }
}

basa_status launch_pool_route_fused(const void *q, const void *k, const void *v, void *kp, void *vp, int32_t *route_idx,
                                    float *route_score, void *workspace, const basa_params &p, cudaStream_t s) {
  FusedPlan fp;
  basa_status st = plan_fused(p, &fp);
  if (st != BASA_OK) return st;
  const Geo g = make_geo(p);
  FusedArgs a;
  std::memset(&a, 0, sizeof(a));
  const long long N = g.N;
  a.src[0] = q; a.src[1] = k; a.src[2] = v;
  a.bh_stride[0] = N * p.head_dim;
  a.bh_stride[1] = a.bh_stride[2] = (N + p.n_text) * p.head_dim;
  float *means = static_cast<float *>(workspace);
  float *part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + fp.means_bytes);
  a.kp = kp;
  a.vp = vp;
  a.part = part;
  a.d = p.head_dim;
  const int esz = p.dtype == BASA_BF16 ? 2 : 4;
  a.lpr = p.head_dim * esz / 16;
  const int G[3] = {p.T, p.H, p.W}, P[3] = {p.pt, p.ph, p.pw}, w[3] = {p.wt, p.wh, p.ww}, sh[3] = {p.st, p.sy, p.sx};
  for (int ax = 0; ax < 3; ++ax) {
    a.G[ax] = G[ax];
    a.e[ax] = fp.e[ax];
    a.nb[ax] = fp.nb[ax];
    a.pool[ax] = P[ax];
    a.w[ax] = w[ax];
    a.s[ax] = sh[ax];
    a.nw[ax] = G[ax] / w[ax];
    a.K[ax] = fp.K[ax];
  }
  a.bh = p.B * p.heads;
  a.inv_pool = 1.0f / float(p.pt * p.ph * p.pw);
  if (N * p.head_dim * esz >= (1ll << 32)) return BASA_ERR_UNSUPPORTED;  // 32-bit offsets inside a (b, head) slice
  const long long n_boxes = (long long)a.bh * fp.nb[0] * fp.nb[1] * fp.nb[2];
  if (n_boxes >= (1ll << 31) || 2ll * a.bh * g.nWin >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  const size_t smem = cell_smem_bytes(fp.max_cells, p.head_dim, p.dtype);
  auto kernel = p.dtype == BASA_BF16 ? cell_sum_kernel<__nv_bfloat16> : cell_sum_kernel<float>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return BASA_ERR_CUDA;
  kernel<<<unsigned(n_boxes), kCellThreads, smem, s>>>(a);
  if (cudaGetLastError() != cudaSuccess) return BASA_ERR_CUDA;

  ReduceArgs r;
  std::memset(&r, 0, sizeof(r));
  r.part = part;
  r.means = means;
  r.d = p.head_dim;
  r.bh = a.bh;
  for (int ax = 0; ax < 3; ++ax) {
    r.G[ax] = a.G[ax]; r.e[ax] = a.e[ax]; r.nb[ax] = a.nb[ax]; r.w[ax] = a.w[ax];
    r.s[ax] = a.s[ax]; r.nw[ax] = a.nw[ax]; r.K[ax] = a.K[ax];
  }
  r.inv_win = 1.0f / float(p.wt * p.wh * p.ww);
  // about 8 slots per thread; groups divide 256 / (d/4)
  const int d4 = p.head_dim / 4;
  const int kprod = fp.K[0] * fp.K[1] * fp.K[2];
  r.groups = 1;
  while (r.groups * 2 <= 256 / d4 && r.groups * 8 < kprod) r.groups *= 2;
  const int wpc = 256 / (d4 * r.groups);
  const long long rows = 2ll * a.bh * g.nWin;
  window_reduce_kernel<<<unsigned((rows + wpc - 1) / wpc), 256, 0, s>>>(r);
  if (cudaGetLastError() != cudaSuccess) return BASA_ERR_CUDA;
  const size_t half = fp.means_bytes / 2;
  return launch_topk(means, reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(means) + half), route_idx, route_score,
                     p, s);
}

}  // namespace basa

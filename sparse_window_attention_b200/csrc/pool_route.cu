// Pooled global K/V, window means and top-k window routing (HBM-bound kernels).
//
//  * box_mean_kernel: mean of a tensor over axis-aligned boxes of the token grid.
//    With box = pool patch and offset 0 it is the K/V pooling of BASA §3.2 (pooled
//    global memory over the UNSHIFTED grid); with box = window and offset = shift
//    (boxes wrap around the grid edge) it gives the window means of Q and K used
//    by the routing of BASA §3.3.
//  * route_topk_kernel: score[w,u] = Qm[w] . Km[u] over the candidates u of w (every
//    u != w, or the windows within a window-grid radius) and a warp-level top-k
//    per query window, ties to the lower window id (BASA §3.3 content-adaptive
//    true-window routing; §A.2 candidate-window radius).
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "basa_internal.h"

namespace basa {
namespace {

__device__ __forceinline__ uint32_t ptx_pack(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

constexpr int kMeanThreads = 256;

struct BoxMeanArgs {
  const void *src[2];
  void *dst[2];
  long long src_bh_stride[2];  // elements between consecutive (b, head) slices
  int d;
  int T, H, W;
  int bt, by, bx;     // box extents
  int nbt, nby, nbx;  // boxes per axis
  int ot, oy, ox;     // origin offset of box (0,0,0)
  int nb_cta;         // boxes along x handled by one CTA
  int splits;         // row splits per box (threads per (box, chunk))
  int xgroups;        // CTAs along x = ceil(nbx / nb_cta)
  float inv_count;
};

__device__ __forceinline__ void accumulate(float *acc, const uint4 &v, const __nv_bfloat16 *) {
  // bf16 -> fp32 is a 16-bit shift of the bit pattern
  acc[0] += __uint_as_float(v.x << 16); acc[1] += __uint_as_float(v.x & 0xFFFF0000u);
  acc[2] += __uint_as_float(v.y << 16); acc[3] += __uint_as_float(v.y & 0xFFFF0000u);
  acc[4] += __uint_as_float(v.z << 16); acc[5] += __uint_as_float(v.z & 0xFFFF0000u);
  acc[6] += __uint_as_float(v.w << 16); acc[7] += __uint_as_float(v.w & 0xFFFF0000u);
}
__device__ __forceinline__ void accumulate(float *acc, const uint4 &v, const float *) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}
// Store the VEC means of one 16-byte input column: bfloat16 output (VEC = 8) or
// float32 output (VEC = 8 from bfloat16 input, VEC = 4 from float32 input).
template <int VEC>
__device__ __forceinline__ void store_chunk(__nv_bfloat16 *p, const float *v) {
  static_assert(VEC == 8, "bfloat16 output comes from bfloat16 input");
  uint4 o;
  o.x = ptx_pack(v[0], v[1]); o.y = ptx_pack(v[2], v[3]); o.z = ptx_pack(v[4], v[5]); o.w = ptx_pack(v[6], v[7]);
  *reinterpret_cast<uint4 *>(p) = o;
}
template <int VEC>
__device__ __forceinline__ void store_chunk(float *p, const float *v) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  if (VEC == 8) *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// One CTA per (tensor, b*head, box row (t, y), group of nb_cta boxes along x).
// Thread = (row split s, box i, 16-byte column c of the head dimension): it walks
// rows s, s + splits, ... of its box and the box's x-run in each row with 32-bit
// offsets (a box that wraps around the grid edge is two runs), keeping float32
// sums of its 16 bytes. Adjacent threads read adjacent 16-byte columns, so a warp
// reads whole contiguous token rows. Row splits are summed in shared memory.
template <typename T, typename OutT>
__global__ void __launch_bounds__(kMeanThreads, 2) box_mean_kernel(BoxMeanArgs a) {
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ float red[];
  const int tensor = blockIdx.z;
  const int lpr = a.d / VEC;  // 16-byte columns per token
  int rest = blockIdx.x;
  const int xg = rest % a.xgroups; rest /= a.xgroups;
  const int jy = rest % a.nby; rest /= a.nby;
  const int jt = rest % a.nbt;
  const int bh = rest / a.nbt;
  const int c = threadIdx.x % lpr;
  const int bi = (threadIdx.x / lpr) % a.nb_cta;
  const int sp = threadIdx.x / (lpr * a.nb_cta);
  const int jx = xg * a.nb_cta + bi;
  const bool valid = jx < a.nbx && sp < a.splits;
  // select with conditionals: a dynamic index into the parameter arrays would copy them to local memory
  const void *src = tensor ? a.src[1] : a.src[0];
  const long long stride = tensor ? a.src_bh_stride[1] : a.src_bh_stride[0];
  void *dst = tensor ? a.dst[1] : a.dst[0];
  const uint4 *base = reinterpret_cast<const uint4 *>(static_cast<const T *>(src) + (long long)bh * stride) + c;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  if (valid) {
    const int ot = (jt * a.bt + a.ot) % a.T, oy = (jy * a.by + a.oy) % a.H, ox = (jx * a.bx + a.ox) % a.W;
    const int run0 = min(a.bx, a.W - ox);  // tokens before the grid edge; the rest start at x = 0
    const int nrows = a.bt * a.by;
    int rt = sp / a.by, ry = sp % a.by;
    for (int r = sp; r < nrows; r += a.splits) {
      int t = ot + rt; t -= (t >= a.T) ? a.T : 0;
      int y = oy + ry; y -= (y >= a.H) ? a.H : 0;
      const uint32_t row = uint32_t(t * a.H + y) * uint32_t(a.W);
      const uint4 *p0 = base + (row + uint32_t(ox)) * uint32_t(lpr);
      int xx = 0;
      for (; xx + 4 <= run0; xx += 4) {
        const uint4 v0 = __ldg(p0 + (xx + 0) * lpr), v1 = __ldg(p0 + (xx + 1) * lpr);
        const uint4 v2 = __ldg(p0 + (xx + 2) * lpr), v3 = __ldg(p0 + (xx + 3) * lpr);
        accumulate(acc, v0, static_cast<const T *>(nullptr));
        accumulate(acc, v1, static_cast<const T *>(nullptr));
        accumulate(acc, v2, static_cast<const T *>(nullptr));
        accumulate(acc, v3, static_cast<const T *>(nullptr));
      }
      for (; xx < run0; ++xx) accumulate(acc, __ldg(p0 + xx * lpr), static_cast<const T *>(nullptr));
      const uint4 *p1 = base + row * uint32_t(lpr);  // wrapped part of the run, from x = 0
      const int run1 = a.bx - run0;
      int x1 = 0;
      for (; x1 + 4 <= run1; x1 += 4) {
        const uint4 v0 = __ldg(p1 + (x1 + 0) * lpr), v1 = __ldg(p1 + (x1 + 1) * lpr);
        const uint4 v2 = __ldg(p1 + (x1 + 2) * lpr), v3 = __ldg(p1 + (x1 + 3) * lpr);
        accumulate(acc, v0, static_cast<const T *>(nullptr));
        accumulate(acc, v1, static_cast<const T *>(nullptr));
        accumulate(acc, v2, static_cast<const T *>(nullptr));
        accumulate(acc, v3, static_cast<const T *>(nullptr));
      }
      for (; x1 < run1; ++x1) accumulate(acc, __ldg(p1 + x1 * lpr), static_cast<const T *>(nullptr));
      ry += a.splits;
      while (ry >= a.by) { ry -= a.by; ++rt; }
    }
  }
  if (a.splits > 1) {
    const int slot = threadIdx.x % (lpr * a.nb_cta);
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[(sp * lpr * a.nb_cta + slot) * VEC + e] = acc[e];
    __syncthreads();
    if (sp == 0 && valid)
      for (int q = 1; q < a.splits; ++q)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += red[(q * lpr * a.nb_cta + slot) * VEC + e];
  }
  if (sp == 0 && valid) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] *= a.inv_count;
    const long long box = ((long long)jt * a.nby + jy) * a.nbx + jx;
    const long long nbox = (long long)a.nbt * a.nby * a.nbx;
    OutT *out = static_cast<OutT *>(dst) + ((long long)bh * nbox + box) * a.d + c * VEC;
    store_chunk<VEC>(out, acc);
  }
}

template <typename T, typename OutT>
basa_status run_box_mean(BoxMeanArgs a, int bh, cudaStream_t s) {
  const int lpr = a.d / (16 / int(sizeof(T)));
  a.nb_cta = std::max(1, std::min(a.nbx, kMeanThreads / lpr));
  a.splits = std::max(1, kMeanThreads / (lpr * a.nb_cta));
  a.splits = std::min(a.splits, a.bt * a.by);
  a.xgroups = (a.nbx + a.nb_cta - 1) / a.nb_cta;
  const int threads = lpr * a.nb_cta * a.splits;
  const size_t smem = a.splits > 1 ? size_t(threads) * (16 / sizeof(T)) * sizeof(float) : 0;
  const long long blocks = (long long)bh * a.nbt * a.nby * a.xgroups;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  dim3 grid(unsigned(blocks), 1, 2);
  box_mean_kernel<T, OutT><<<grid, threads, smem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

// ----------------------------------------------------------------- top-k
constexpr int kRouteWarps = 8;
constexpr int kRouteChunk = 128;

struct RouteArgs {
  const float *qm, *km;
  int32_t *idx;
  float *score;
  int nwin, d, k;
  int radius;           // 0 = every other window is a candidate
  int nwy, nwx;         // window grid extents along y and x
};

// Window u is a routing candidate of window w: u != w and, under a radius r >= 1,
// their window-grid coordinates differ by at most r on every axis (no wrap-around).
__device__ __forceinline__ bool route_candidate(const RouteArgs &a, int w, int u) {
  if (u == w) return false;
  if (a.radius == 0) return true;
  const int wx = w % a.nwx, wy = (w / a.nwx) % a.nwy, wt = w / (a.nwx * a.nwy);
  const int ux = u % a.nwx, uy = (u / a.nwx) % a.nwy, ut = u / (a.nwx * a.nwy);
  return abs(wx - ux) <= a.radius && abs(wy - uy) <= a.radius && abs(wt - ut) <= a.radius;
}

// One CTA per (b*head, group of 8 query windows); one warp per query window.
// Km is staged through shared memory in chunks of 128 windows, one warp per row
// with 16-byte loads; rows are padded to d + 4 floats so that the 16-byte reads
// of 8 consecutive rows by a quarter warp hit distinct banks.
__global__ void __launch_bounds__(kRouteWarps * 32) route_topk_kernel(RouteArgs a) {
  extern __shared__ float sm[];
  const int ngroups = (a.nwin + kRouteWarps - 1) / kRouteWarps;
  const int bh = blockIdx.x / ngroups;
  const int group = blockIdx.x % ngroups;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int w = group * kRouteWarps + warp;
  const bool valid = w < a.nwin;
  const int ld = a.d + 4;
  const int d4 = a.d / 4;  // float4 per row
  float *kchunk = sm;                                         // [128][d+4]
  float *qrow = kchunk + kRouteChunk * ld + warp * a.d;       // [8][d]
  float *scores = kchunk + kRouteChunk * ld + kRouteWarps * a.d + warp * a.nwin;  // [8][nwin]
  const float4 *qm = reinterpret_cast<const float4 *>(a.qm + (long long)bh * a.nwin * a.d);
  const float4 *km = reinterpret_cast<const float4 *>(a.km + (long long)bh * a.nwin * a.d);
  if (valid)
    for (int c = lane; c < d4; c += 32) reinterpret_cast<float4 *>(qrow)[c] = qm[(long long)w * d4 + c];
  for (int c0 = 0; c0 < a.nwin; c0 += kRouteChunk) {
    const int rows = min(kRouteChunk, a.nwin - c0);
    __syncthreads();
    // all loads of a thread first (independent), then the shared-memory stores
    constexpr int kPer = kRouteChunk / kRouteWarps;  // rows per warp
    for (int c = lane; c < d4; c += 32) {
      float4 v[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int r = warp + i * kRouteWarps;
        if (r < rows) v[i] = km[(long long)(c0 + r) * d4 + c];
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int r = warp + i * kRouteWarps;
        if (r < rows) reinterpret_cast<float4 *>(kchunk + r * ld)[c] = v[i];
      }
    }
    __syncthreads();
    if (valid)
      for (int r = lane; r < rows; r += 32) {
        const float4 *kr = reinterpret_cast<const float4 *>(kchunk + r * ld);
        const float4 *qr = reinterpret_cast<const float4 *>(qrow);
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        for (int c = 0; c < d4; ++c) {
          const float4 kv = kr[c], qv = qr[c];
          s0 = fmaf(qv.x, kv.x, s0);
          s1 = fmaf(qv.y, kv.y, s1);
          s2 = fmaf(qv.z, kv.z, s2);
          s3 = fmaf(qv.w, kv.w, s3);
        }
        scores[c0 + r] = route_candidate(a, w, c0 + r) ? (s0 + s1) + (s2 + s3) : -INFINITY;
      }
  }
  __syncwarp();
  if (!valid) return;
  for (int r = 0; r < a.k; ++r) {
    float bs = -INFINITY;
    int bi = INT_MAX;
    for (int u = lane; u < a.nwin; u += 32) {
      const float s = scores[u];
      if (s > bs || (s == bs && u < bi)) { bs = s; bi = u; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (os > bs || (os == bs && oi < bi)) { bs = os; bi = oi; }
    }
    if (lane == 0) {
      const long long o = ((long long)bh * a.nwin + w) * a.k + r;
      a.idx[o] = bi;
      if (a.score) a.score[o] = bs;
      scores[bi] = -INFINITY;
    }
    __syncwarp();
  }
}

}  // namespace

basa_status launch_pool_kv(const void *k, const void *v, void *kp, void *vp, const basa_params &p, cudaStream_t s) {
  BoxMeanArgs a{};
  a.src[0] = k; a.src[1] = v;
  a.dst[0] = kp; a.dst[1] = vp;
  const long long N = (long long)p.T * p.H * p.W;
  a.src_bh_stride[0] = a.src_bh_stride[1] = (N + p.n_text) * p.head_dim;
  a.d = p.head_dim;
  a.T = p.T; a.H = p.H; a.W = p.W;
  a.bt = p.pt; a.by = p.ph; a.bx = p.pw;
  a.nbt = p.T / p.pt; a.nby = p.H / p.ph; a.nbx = p.W / p.pw;
  a.ot = a.oy = a.ox = 0;
  a.inv_count = 1.0f / float(p.pt * p.ph * p.pw);
  const int bh = p.B * p.heads;
  if (p.dtype == BASA_BF16) return run_box_mean<__nv_bfloat16, __nv_bfloat16>(a, bh, s);
  return run_box_mean<float, float>(a, bh, s);
}

basa_status launch_route(const void *q, const void *k, int32_t *route_idx, float *route_score, void *workspace,
                         const basa_params &p, cudaStream_t s) {
  const Geo g = make_geo(p);
  const int bh = p.B * p.heads;
  float *qm = static_cast<float *>(workspace);
  float *km = qm + (size_t)bh * g.nWin * p.head_dim;
  BoxMeanArgs a{};
  a.src[0] = q; a.src[1] = k;
  a.dst[0] = qm; a.dst[1] = km;
  a.src_bh_stride[0] = (long long)g.N * p.head_dim;
  a.src_bh_stride[1] = ((long long)g.N + p.n_text) * p.head_dim;
  a.d = p.head_dim;
  a.T = p.T; a.H = p.H; a.W = p.W;
  a.bt = p.wt; a.by = p.wh; a.bx = p.ww;
  a.nbt = g.nWt; a.nby = g.nWy; a.nbx = g.nWx;
  a.ot = p.st; a.oy = p.sy; a.ox = p.sx;
  a.inv_count = 1.0f / float(p.wt * p.wh * p.ww);
  basa_status st = (p.dtype == BASA_BF16) ? run_box_mean<__nv_bfloat16, float>(a, bh, s) : run_box_mean<float, float>(a, bh, s);
  if (st != BASA_OK) return st;
  return launch_topk(qm, km, route_idx, route_score, p, s);
}

basa_status launch_topk(const float *qm, const float *km, int32_t *route_idx, float *route_score, const basa_params &p,
                        cudaStream_t s) {
  const Geo g = make_geo(p);
  const int bh = p.B * p.heads;
  RouteArgs r{qm, km, route_idx, route_score, g.nWin, p.head_dim, p.routed_k, p.route_radius, g.nWy, g.nWx};
  const size_t smem = (size_t(kRouteChunk) * (p.head_dim + 4) + kRouteWarps * p.head_dim + size_t(kRouteWarps) * g.nWin) * sizeof(float);
  // The shared-memory limit is raised once per device; a failed attempt is not
  // recorded, so every later call retries it and reports its own error.
  static std::atomic<int> wide_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BASA_ERR_CUDA;
  if (!wide_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(route_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
      return BASA_ERR_CUDA;
    wide_set[dev].store(1, std::memory_order_release);
  }
  const int ngroups = (g.nWin + kRouteWarps - 1) / kRouteWarps;
  route_topk_kernel<<<unsigned(bh) * unsigned(ngroups), kRouteWarps * 32, smem, s>>>(r);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

// ----------------------------------------------------------------- no-allocation routing
// Window-mean scratch for basa_route_windows_noalloc, for callers that cannot
// allocate device memory themselves. It is part of the library's device image,
// so every GPU that loads the library holds it until the process exits. In host
// code `g_route_scratch` names a host-side stand-in, not a device address: the
// device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_route_scratch[BASA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxScratchDevices] = {};
}  // namespace

basa_status launch_route_noalloc(const void *q, const void *k, int32_t *route_idx, float *route_score,
                                 const basa_params &p, cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BASA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxScratchDevices) return BASA_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
      // `dev` is the current device here, so this is the address on that device.
      void *addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_route_scratch) != cudaSuccess || !addr) return BASA_ERR_CUDA;
      g_scratch_addr[dev] = addr;
    }
    scratch = g_scratch_addr[dev];
  }
  return launch_route(q, k, route_idx, route_score, scratch, p, s);
}

}  // namespace basa

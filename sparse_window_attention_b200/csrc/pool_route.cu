// Pooled global K/V, window means and top-k window routing (HBM-bound kernels).
//
//  * box_mean_kernel: mean of a tensor over axis-aligned boxes of the token grid.
//    With box = pool patch and offset 0 it is the K/V pooling of BASA §3.2 (pooled
//    global memory over the UNSHIFTED grid); with box = window and offset = shift
//    (boxes wrap around the grid edge) it gives the window means of Q and K used
//    by the routing of BASA §3.3.
//  * route_topk_kernel: score[w,u] = Qm[w] . Km[u] (u != w) and a warp-level top-k
//    per query window, ties to the lower window id (BASA §3.3 content-adaptive
//    true-window routing).
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>
#include <mutex>

#include "basa_internal.h"

namespace basa {
namespace {

constexpr int kMeanThreads = 128;
constexpr int kMeanUnroll = 4;

struct BoxMeanArgs {
  const void *src[2];
  void *dst[2];
  long long src_bh_stride[2];  // elements between consecutive (b, head) slices
  int d;
  int T, H, W;
  int bt, by, bx;     // box extents
  int nbt, nby, nbx;  // boxes per axis
  int ot, oy, ox;     // origin offset of box (0,0,0)
  int nbox;
  float inv_count;
};

__device__ __forceinline__ void accumulate(float *acc, const uint4 &v, const __nv_bfloat16 *) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    acc[2 * e] += f.x;
    acc[2 * e + 1] += f.y;
  }
}
__device__ __forceinline__ void accumulate(float *acc, const uint4 &v, const float *) {
  const float *f = reinterpret_cast<const float *>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] += f[e];
}
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store_out(float *p, float x) { *p = x; }

// One CTA per (tensor, b*head, box). A box is walked as rows of bx tokens (one
// row per (t, y)); the row's bx * d elements are cut into 16-byte chunks and the
// CTA's threads take consecutive chunks, so a warp reads contiguous bytes. A
// thread always lands on the same chunk column c (128 is a multiple of the
// chunks per token), keeps float32 sums for it, and the row/column position is
// advanced incrementally (no division per load). Partial sums of the threads
// that share a chunk column are reduced in shared memory at the end.
template <typename T, typename OutT>
__global__ void __launch_bounds__(kMeanThreads) box_mean_kernel(BoxMeanArgs a) {
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ float red[];
  const int tensor = blockIdx.z;
  const int bh = blockIdx.x / a.nbox;
  const int box = blockIdx.x % a.nbox;
  const int lpr = a.d / VEC;                 // chunks per token (8, 16 or 32)
  const int chunk = threadIdx.x % lpr;       // fixed chunk column of this thread
  const int slot = threadIdx.x / lpr;
  const int jx = box % a.nbx, jy = (box / a.nbx) % a.nby, jt = box / (a.nbx * a.nby);
  const int ot = (jt * a.bt + a.ot) % a.T, oy = (jy * a.by + a.oy) % a.H, ox = (jx * a.bx + a.ox) % a.W;
  // select with conditionals: a dynamic index into the parameter arrays would copy them to local memory
  const void *src = tensor ? a.src[1] : a.src[0];
  const long long stride = tensor ? a.src_bh_stride[1] : a.src_bh_stride[0];
  void *dst = tensor ? a.dst[1] : a.dst[0];
  const T *base = static_cast<const T *>(src) + (long long)bh * stride + chunk * VEC;
  const int row_chunks = a.bx * lpr;
  const int nrows = a.bt * a.by;
  const int step_rows = kMeanThreads / row_chunks;  // whole rows advanced per step of 128 chunks
  const int step_rem = kMeanThreads % row_chunks;
  const int lpr_shift = __ffs(lpr) - 1;

  // position of chunk index threadIdx.x: row r = (rt, ry), chunk xc within the row
  int r = threadIdx.x / row_chunks, xc = threadIdx.x % row_chunks;
  int rt = r / a.by, ry = r % a.by;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  auto advance = [&]() {
    xc += step_rem;
    int dr = step_rows;
    if (xc >= row_chunks) { xc -= row_chunks; ++dr; }
    r += dr;
    ry += dr;
    while (ry >= a.by) { ry -= a.by; ++rt; }
  };
  while (r < nrows) {
    uint4 v[kMeanUnroll];
#pragma unroll
    for (int i = 0; i < kMeanUnroll; ++i) {
      if (r < nrows) {
        int t = ot + rt; t -= (t >= a.T) ? a.T : 0;
        int y = oy + ry; y -= (y >= a.H) ? a.H : 0;
        int x = ox + (xc >> lpr_shift); x -= (x >= a.W) ? a.W : 0;
        const long long tok = ((long long)t * a.H + y) * a.W + x;
        v[i] = __ldg(reinterpret_cast<const uint4 *>(base + tok * a.d));
        advance();
      } else {
        v[i] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int i = 0; i < kMeanUnroll; ++i) accumulate(acc, v[i], static_cast<const T *>(nullptr));
  }
  const int slots = kMeanThreads / lpr;
#pragma unroll
  for (int e = 0; e < VEC; ++e) red[slot * a.d + chunk * VEC + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < a.d; c += kMeanThreads) {
    float s = 0.f;
    for (int q = 0; q < slots; ++q) s += red[q * a.d + c];
    OutT *out = static_cast<OutT *>(dst) + ((long long)bh * a.nbox + box) * a.d + c;
    store_out(out, s * a.inv_count);
  }
}

template <typename T, typename OutT>
basa_status run_box_mean(const BoxMeanArgs &a, int bh, cudaStream_t s) {
  const int lpr = a.d / (16 / int(sizeof(T)));
  const size_t smem = size_t(kMeanThreads / lpr) * a.d * sizeof(float);
  dim3 grid(unsigned(bh) * unsigned(a.nbox), 1, 2);
  box_mean_kernel<T, OutT><<<grid, kMeanThreads, smem, s>>>(a);
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
};

// One CTA per (b*head, group of 8 query windows); one warp per query window.
// Km is staged through shared memory in chunks of 128 windows (rows padded by
// one float so the lanes of a warp hit distinct banks).
__global__ void __launch_bounds__(kRouteWarps * 32) route_topk_kernel(RouteArgs a) {
  extern __shared__ float sm[];
  const int ngroups = (a.nwin + kRouteWarps - 1) / kRouteWarps;
  const int bh = blockIdx.x / ngroups;
  const int group = blockIdx.x % ngroups;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int w = group * kRouteWarps + warp;
  const bool valid = w < a.nwin;
  const int ld = a.d + 1;
  float *kchunk = sm;                                        // [128][d+1]
  float *qrow = kchunk + kRouteChunk * ld + warp * a.d;      // [8][d]
  float *scores = kchunk + kRouteChunk * ld + kRouteWarps * a.d + warp * a.nwin;  // [8][nwin]
  const float *qm = a.qm + (long long)bh * a.nwin * a.d;
  const float *km = a.km + (long long)bh * a.nwin * a.d;
  if (valid)
    for (int c = lane; c < a.d; c += 32) qrow[c] = qm[(long long)w * a.d + c];
  for (int c0 = 0; c0 < a.nwin; c0 += kRouteChunk) {
    const int rows = min(kRouteChunk, a.nwin - c0);
    __syncthreads();
    for (int i = threadIdx.x; i < rows * a.d; i += blockDim.x) {
      const int r = i / a.d, c = i % a.d;
      kchunk[r * ld + c] = km[(long long)(c0 + r) * a.d + c];
    }
    __syncthreads();
    if (valid)
      for (int r = lane; r < rows; r += 32) {
        float s = 0.f;
        for (int c = 0; c < a.d; ++c) s = fmaf(qrow[c], kchunk[r * ld + c], s);
        scores[c0 + r] = (c0 + r == w) ? -INFINITY : s;
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
  a.nbox = a.nbt * a.nby * a.nbx;
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
  a.nbox = g.nWin;
  a.inv_count = 1.0f / float(p.wt * p.wh * p.ww);
  basa_status st = (p.dtype == BASA_BF16) ? run_box_mean<__nv_bfloat16, float>(a, bh, s) : run_box_mean<float, float>(a, bh, s);
  if (st != BASA_OK) return st;
  RouteArgs r{qm, km, route_idx, route_score, g.nWin, p.head_dim, p.routed_k};
  const size_t smem = (size_t(kRouteChunk) * (p.head_dim + 1) + kRouteWarps * p.head_dim + size_t(kRouteWarps) * g.nWin) * sizeof(float);
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BASA_ERR_CUDA;
  if (smem > 48 * 1024 && (dev >= 64 || !attr_set[dev])) {
    if (cudaFuncSetAttribute(route_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
      return BASA_ERR_CUDA;
    if (dev < 64) attr_set[dev] = true;
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

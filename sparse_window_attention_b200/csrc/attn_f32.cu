// Shifted-window attention forward in float32 on the CUDA cores (no TF32: its
// 10-bit mantissa cannot meet a 1e-4 tolerance). Same operator as the bfloat16
// tensor-core kernel (BASA §3.1 shifted windows, §3.2 pooled K/V, §3.3 routed
// windows, §A.1 one softmax over the concatenated keys), with an online softmax
// over key tiles staged in shared memory.
#include <cfloat>

#include "basa_internal.h"

namespace basa {
namespace {

constexpr int kThreads = 128;
constexpr int kKeyTile = 32;

struct F32Args {
  const float *q, *k, *v, *kp, *vp;
  const int32_t *route;
  int32_t *dev_err;  // nullable: BASA_DEVERR_BAD_ROUTE on an out-of-range route id
  float *out;
  float *lse;  // nullable [B*heads][N]
  Geo g;
  int heads, d, n_text, n_pool, routed_k, win_tok, q_chunks;
  int n_vis_keys, n_pool_keys, n_text_keys;  // keys taken from each group (0 = group not selected)
  int dense;  // text-query rows: queries are q_text rows, keys are all N + n_text rows of k, v
  float scale;
};

// A route id outside [0, nWin) is reported (BASA_DEVERR_BAD_ROUTE) and replaced by
// the query's own window, so every access stays inside the tensors.
__device__ __forceinline__ int checked_route(const F32Args &a, int u, int w) {
  if (u >= 0 && u < a.g.nWin) return u;
  if (a.dev_err) atomicOr(a.dev_err, BASA_DEVERR_BAD_ROUTE);
  return w;
}

// Row of key j of window w's key list: [own | routed windows | pooled | text],
// restricted to the selected groups.
__device__ __forceinline__ const float *key_row(const F32Args &a, const float *kv, const float *kvp, long long bh,
                                                const int *wins, int j) {
  const int nvis = a.n_vis_keys;
  const long long rows = (long long)a.g.N + a.n_text;
  if (a.dense) return kv + (bh * rows + j) * a.d;
  if (j < nvis) {
    const int u = wins[j / a.win_tok];
    const int l = j % a.win_tok;
    int ot, oy, ox, type;
    window_origin(a.g, u, &ot, &oy, &ox, &type);
    const int lt = l / (a.g.wh * a.g.ww), ly = (l / a.g.ww) % a.g.wh, lx = l % a.g.ww;
    const int t = (ot + lt) % a.g.T, y = (oy + ly) % a.g.H, x = (ox + lx) % a.g.W;
    return kv + (bh * rows + ((long long)t * a.g.H + y) * a.g.W + x) * a.d;
  }
  j -= nvis;
  if (j < a.n_pool_keys) return kvp + (bh * a.n_pool + j) * a.d;
  j -= a.n_pool_keys;
  return kv + (bh * rows + a.g.N + j) * a.d;
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_f32_kernel(F32Args a) {
  constexpr int TPQ = D / 64;          // threads per query
  constexpr int QPB = kThreads / TPQ;  // queries per block
  __shared__ float ks[kKeyTile][D];
  __shared__ float vs[kKeyTile][D];
  __shared__ int wins[1 + kMaxRouted];

  const int n_win = a.dense ? 1 : a.g.nWin;
  const int chunk = blockIdx.x % a.q_chunks;
  const int w = (blockIdx.x / a.q_chunks) % n_win;
  const long long bh = blockIdx.x / (a.q_chunks * n_win);
  if (threadIdx.x == 0) wins[0] = w;
  if (!a.dense && threadIdx.x > 0 && threadIdx.x <= a.routed_k)
    wins[threadIdx.x] = checked_route(a, a.route[(bh * a.g.nWin + w) * a.routed_k + threadIdx.x - 1], w);
  __syncthreads();

  const int half = threadIdx.x % TPQ;
  const int lq = chunk * QPB + threadIdx.x / TPQ;
  const bool active = lq < (a.dense ? a.n_text : a.win_tok);
  // query / output row inside this (b, head): a token of the grid, or a text row
  const long long q_rows = a.dense ? a.n_text : a.g.N;
  long long qtok = 0;
  if (active && a.dense) {
    qtok = lq;
  } else if (active) {
    int ot, oy, ox, type;
    window_origin(a.g, w, &ot, &oy, &ox, &type);
    const int lt = lq / (a.g.wh * a.g.ww), ly = (lq / a.g.ww) % a.g.wh, lx = lq % a.g.ww;
    qtok = ((long long)((ot + lt) % a.g.T) * a.g.H + (oy + ly) % a.g.H) * a.g.W + (ox + lx) % a.g.W;
  }
  float q[64], o[64];
  const float *qp = a.q + (bh * q_rows + qtok) * D;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    q[i] = active ? qp[i * TPQ + half] * a.scale : 0.f;
    o[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int nk = a.dense ? a.g.N + a.n_text : a.n_vis_keys + a.n_pool_keys + a.n_text_keys;
  for (int k0 = 0; k0 < nk; k0 += kKeyTile) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKeyTile * (D / 4); i += kThreads) {
      const int r = i / (D / 4), c4 = i % (D / 4);
      float4 kv4 = make_float4(0.f, 0.f, 0.f, 0.f), vv4 = kv4;
      if (k0 + r < nk) {
        kv4 = reinterpret_cast<const float4 *>(key_row(a, a.k, a.kp, bh, wins, k0 + r))[c4];
        vv4 = reinterpret_cast<const float4 *>(key_row(a, a.v, a.vp, bh, wins, k0 + r))[c4];
      }
      reinterpret_cast<float4 *>(&ks[r][0])[c4] = kv4;
      reinterpret_cast<float4 *>(&vs[r][0])[c4] = vv4;
    }
    __syncthreads();
    float s[kKeyTile];
    float tmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < kKeyTile; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 64; ++i) acc = fmaf(q[i], ks[j][i * TPQ + half], acc);
      if (TPQ == 2) acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      s[j] = (k0 + j < nk) ? acc : -INFINITY;
      tmax = fmaxf(tmax, s[j]);
    }
    const float mn = fmaxf(m, tmax);
    const float alpha = expf(m - mn);
    l *= alpha;
#pragma unroll
    for (int i = 0; i < 64; ++i) o[i] *= alpha;
#pragma unroll
    for (int j = 0; j < kKeyTile; ++j) {
      const float pj = expf(s[j] - mn);
      l += pj;
#pragma unroll
      for (int i = 0; i < 64; ++i) o[i] = fmaf(pj, vs[j][i * TPQ + half], o[i]);
    }
    m = mn;
  }
  if (active) {
    const float inv = 1.0f / l;
    float *op = a.out + (bh * q_rows + qtok) * D;
#pragma unroll
    for (int i = 0; i < 64; ++i) op[i * TPQ + half] = o[i] * inv;
    if (a.lse && half == 0) a.lse[bh * q_rows + qtok] = m + logf(l);
  }
}

}  // namespace

basa_status launch_attn_f32(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                            const int32_t *route_idx, void *out, float *lse, uint32_t keys, const basa_params &p,
                            cudaStream_t s) {
  F32Args a{};
  a.q = static_cast<const float *>(q);
  a.k = static_cast<const float *>(k);
  a.v = static_cast<const float *>(v);
  a.kp = static_cast<const float *>(kp);
  a.vp = static_cast<const float *>(vp);
  a.route = route_idx;
  a.dev_err = p.dev_err;
  a.out = static_cast<float *>(out);
  a.g = make_geo(p);
  a.heads = p.heads;
  a.d = p.head_dim;
  a.n_text = p.n_text;
  a.n_pool = p.pt > 0 ? (p.T / p.pt) * (p.H / p.ph) * (p.W / p.pw) : 0;
  a.routed_k = p.routed_k;
  a.win_tok = p.wt * p.wh * p.ww;
  a.lse = lse;
  a.n_vis_keys = (keys & BASA_KEYS_WINDOWS) ? a.win_tok * (1 + a.routed_k) : 0;
  a.n_pool_keys = (keys & BASA_KEYS_POOLED) ? a.n_pool : 0;
  a.n_text_keys = (keys & BASA_KEYS_TEXT) ? a.n_text : 0;
  const int qpb = kThreads / (p.head_dim / 64);
  a.q_chunks = (a.win_tok + qpb - 1) / qpb;
  a.scale = 1.0f / sqrtf(float(p.head_dim));
  const long long blocks = (long long)p.B * p.heads * a.g.nWin * a.q_chunks;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  if (p.head_dim == 64) attn_f32_kernel<64><<<unsigned(blocks), kThreads, 0, s>>>(a);
  else attn_f32_kernel<128><<<unsigned(blocks), kThreads, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

basa_status launch_attn_text_f32(const void *q_text, const void *k, const void *v, void *out_text,
                                 const basa_params &p, cudaStream_t s) {
  F32Args a{};
  a.q = static_cast<const float *>(q_text);
  a.k = static_cast<const float *>(k);
  a.v = static_cast<const float *>(v);
  a.out = static_cast<float *>(out_text);
  a.g = make_geo(p);
  a.heads = p.heads;
  a.d = p.head_dim;
  a.n_text = p.n_text;
  a.dense = 1;
  const int qpb = kThreads / (p.head_dim / 64);
  a.q_chunks = (p.n_text + qpb - 1) / qpb;
  a.scale = 1.0f / sqrtf(float(p.head_dim));
  const long long blocks = (long long)p.B * p.heads * a.q_chunks;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  if (p.head_dim == 64) attn_f32_kernel<64><<<unsigned(blocks), kThreads, 0, s>>>(a);
  else attn_f32_kernel<128><<<unsigned(blocks), kThreads, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

// ----------------------------------------------------------------- backward
// Gradients of the forward above w.r.t. q, k, v (float32, CUDA cores), written from
// the softmax derivative: with P = softmax(S), S = q K^T / sqrt(d) and the saved
// log-sum-exp L (p = exp(s - L)), D_i = dO_i . O_i:
//   dS = P (dO V^T - D),  dq = dS K / sqrt(d),  dK += dS^T q / sqrt(d),  dV += P^T dO.
// Routing is a selection and gets no gradient; pooled keys collect their gradient
// in dkp, dvp, which a second kernel spreads over the tokens of each patch.
namespace {

constexpr int kBwdThreads = 128;
constexpr int kBwdTPQ = 4;  // threads per query: 32 of the 128 columns each
constexpr int kBwdKeyTile = 16;

struct BwdArgs {
  F32Args f;  // q, k, v, kp, vp, route and geometry as in the forward
  const float *out, *lse, *dout;
  float *dq, *dk, *dv, *dkp, *dvp;
};

// Destination row of key j's gradient: a row of dk/dv (window or text keys) or of
// dkp/dvp (pooled keys, *pooled = true).
__device__ __forceinline__ long long key_dest(const F32Args &a, long long bh, const int *wins, int j, bool *pooled) {
  const int nvis = a.n_vis_keys;
  const long long rows = (long long)a.g.N + a.n_text;
  *pooled = false;
  if (j < nvis) {
    const int u = wins[j / a.win_tok];
    const int l = j % a.win_tok;
    int ot, oy, ox, type;
    window_origin(a.g, u, &ot, &oy, &ox, &type);
    const int lt = l / (a.g.wh * a.g.ww), ly = (l / a.g.ww) % a.g.wh, lx = l % a.g.ww;
    const int t = (ot + lt) % a.g.T, y = (oy + ly) % a.g.H, x = (ox + lx) % a.g.W;
    return bh * rows + ((long long)t * a.g.H + y) * a.g.W + x;
  }
  j -= nvis;
  if (j < a.n_pool_keys) {
    *pooled = true;
    return bh * a.n_pool + j;
  }
  j -= a.n_pool_keys;
  return bh * rows + a.g.N + j;
}

__global__ void __launch_bounds__(kBwdThreads) attn_bwd_f32_kernel(BwdArgs b) {
  const F32Args &a = b.f;
  constexpr int D = 128, C = D / kBwdTPQ, QPB = kBwdThreads / kBwdTPQ;
  __shared__ float ks[kBwdKeyTile][D], vs[kBwdKeyTile][D];
  __shared__ float dks[kBwdKeyTile][D], dvs[kBwdKeyTile][D];
  __shared__ int wins[1 + kMaxRouted];
  const int chunk = blockIdx.x % a.q_chunks;
  const int w = (blockIdx.x / a.q_chunks) % a.g.nWin;
  const long long bh = blockIdx.x / (a.q_chunks * a.g.nWin);
  if (threadIdx.x == 0) wins[0] = w;
  if (threadIdx.x > 0 && threadIdx.x <= a.routed_k)
    wins[threadIdx.x] = checked_route(a, a.route[(bh * a.g.nWin + w) * a.routed_k + threadIdx.x - 1], w);
  __syncthreads();
  const int part = threadIdx.x % kBwdTPQ;  // columns part, part + TPQ, ...
  const int lq = chunk * QPB + threadIdx.x / kBwdTPQ;
  const bool active = lq < a.win_tok;
  long long qtok = 0;
  if (active) {
    int ot, oy, ox, type;
    window_origin(a.g, w, &ot, &oy, &ox, &type);
    const int lt = lq / (a.g.wh * a.g.ww), ly = (lq / a.g.ww) % a.g.wh, lx = lq % a.g.ww;
    qtok = ((long long)((ot + lt) % a.g.T) * a.g.H + (oy + ly) % a.g.H) * a.g.W + (ox + lx) % a.g.W;
  }
  const long long qrow = bh * a.g.N + qtok;
  float q[C], dout[C], dq[C];
  float Dpart = 0.f;
#pragma unroll
  for (int i = 0; i < C; ++i) {
    const int col = i * kBwdTPQ + part;
    q[i] = active ? a.q[qrow * D + col] : 0.f;
    dout[i] = active ? b.dout[qrow * D + col] : 0.f;
    Dpart = fmaf(dout[i], active ? b.out[qrow * D + col] : 0.f, Dpart);
    dq[i] = 0.f;
  }
  // the TPQ threads of a query are adjacent lanes
  float Drow = Dpart + __shfl_xor_sync(0xffffffffu, Dpart, 1);
  Drow += __shfl_xor_sync(0xffffffffu, Drow, 2);
  const float L = active ? b.lse[qrow] : 0.f;
  const int nk = a.n_vis_keys + a.n_pool_keys + a.n_text_keys;
  for (int k0 = 0; k0 < nk; k0 += kBwdKeyTile) {
    __syncthreads();
    for (int i = threadIdx.x; i < kBwdKeyTile * (D / 4); i += kBwdThreads) {
      const int r = i / (D / 4), c4 = i % (D / 4);
      float4 kv4 = make_float4(0.f, 0.f, 0.f, 0.f), vv4 = kv4;
      if (k0 + r < nk) {
        kv4 = reinterpret_cast<const float4 *>(key_row(a, a.k, a.kp, bh, wins, k0 + r))[c4];
        vv4 = reinterpret_cast<const float4 *>(key_row(a, a.v, a.vp, bh, wins, k0 + r))[c4];
      }
      reinterpret_cast<float4 *>(&ks[r][0])[c4] = kv4;
      reinterpret_cast<float4 *>(&vs[r][0])[c4] = vv4;
      reinterpret_cast<float4 *>(&dks[r][0])[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
      reinterpret_cast<float4 *>(&dvs[r][0])[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    for (int j = 0; j < kBwdKeyTile && k0 + j < nk; ++j) {
      float sp = 0.f, dpp = 0.f;
#pragma unroll
      for (int i = 0; i < C; ++i) {
        const int col = i * kBwdTPQ + part;
        sp = fmaf(q[i], ks[j][col], sp);
        dpp = fmaf(dout[i], vs[j][col], dpp);
      }
      sp += __shfl_xor_sync(0xffffffffu, sp, 1);
      sp += __shfl_xor_sync(0xffffffffu, sp, 2);
      dpp += __shfl_xor_sync(0xffffffffu, dpp, 1);
      dpp += __shfl_xor_sync(0xffffffffu, dpp, 2);
      const float p = active ? expf(sp * a.scale - L) : 0.f;
      const float ds = p * (dpp - Drow);
      // the 8 queries of a warp add to the same key row: sum them with shuffles
      // (lanes l, l ^ 4, l ^ 8, l ^ 16 share a column) and let 4 lanes add to shared memory
      const float dsq = active ? ds * a.scale : 0.f, pa = active ? p : 0.f;
#pragma unroll
      for (int i = 0; i < C; ++i) {
        const int col = i * kBwdTPQ + part;
        dq[i] = fmaf(ds, ks[j][col], dq[i]);
        float gk = dsq * q[i], gv = pa * dout[i];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          gk += __shfl_xor_sync(0xffffffffu, gk, off);
          gv += __shfl_xor_sync(0xffffffffu, gv, off);
        }
        if ((threadIdx.x & 31) < kBwdTPQ) {
          atomicAdd(&dks[j][col], gk);
          atomicAdd(&dvs[j][col], gv);
        }
      }
    }
    __syncthreads();
    // this CTA's contributions to the tile's keys -> global accumulators
    for (int i = threadIdx.x; i < kBwdKeyTile * D; i += kBwdThreads) {
      const int r = i / D, col = i % D;
      if (k0 + r >= nk) continue;
      bool pooled;
      const long long dst = key_dest(a, bh, wins, k0 + r, &pooled);
      atomicAdd((pooled ? b.dkp : b.dk) + dst * D + col, dks[r][col]);
      atomicAdd((pooled ? b.dvp : b.dv) + dst * D + col, dvs[r][col]);
    }
  }
  if (active) {
#pragma unroll
    for (int i = 0; i < C; ++i) b.dq[qrow * D + i * kBwdTPQ + part] = dq[i] * a.scale;
  }
}

// dk, dv of every visual token += dkp, dvp of its pool patch / |patch|.
__global__ void __launch_bounds__(256) pool_bwd_kernel(const float *dkp, const float *dvp, float *dk, float *dv,
                                                       Geo g, int pt, int ph, int pw, int n_pool, int n_text, int d,
                                                       long long total, float inv) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // (bh, token, float4 column)
  if (i >= total) return;
  const int d4 = d / 4;
  const int c4 = int(i % d4);
  const long long tok = (i / d4) % g.N, bh = i / (d4 * (long long)g.N);
  const int x = int(tok % g.W), y = int((tok / g.W) % g.H), t = int(tok / ((long long)g.W * g.H));
  const long long P = ((long long)(t / pt) * (g.H / ph) + y / ph) * (g.W / pw) + x / pw;
  const long long src = (bh * n_pool + P) * d4 + c4;
  const long long dst = (bh * ((long long)g.N + n_text) + tok) * d4 + c4;
  const float4 a = reinterpret_cast<const float4 *>(dkp)[src], b2 = reinterpret_cast<const float4 *>(dvp)[src];
  float4 &k4 = reinterpret_cast<float4 *>(dk)[dst];
  float4 &v4 = reinterpret_cast<float4 *>(dv)[dst];
  k4.x += a.x * inv; k4.y += a.y * inv; k4.z += a.z * inv; k4.w += a.w * inv;
  v4.x += b2.x * inv; v4.y += b2.y * inv; v4.z += b2.z * inv; v4.w += b2.w * inv;
}

}  // namespace

size_t attn_bwd_workspace(const basa_params &p) {
  const size_t n_pool = p.pt > 0 ? size_t(p.T / p.pt) * (p.H / p.ph) * (p.W / p.pw) : 0;
  return 2 * size_t(p.B) * p.heads * n_pool * p.head_dim * sizeof(float);
}

basa_status launch_attn_bwd_f32(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                                const int32_t *route_idx, const void *out, const float *lse, const void *dout,
                                void *dq, void *dk, void *dv, void *workspace, const basa_params &p, cudaStream_t s) {
  BwdArgs b{};
  F32Args &a = b.f;
  a.q = static_cast<const float *>(q);
  a.k = static_cast<const float *>(k);
  a.v = static_cast<const float *>(v);
  a.kp = static_cast<const float *>(kp);
  a.vp = static_cast<const float *>(vp);
  a.route = route_idx;
  a.dev_err = p.dev_err;
  a.g = make_geo(p);
  a.heads = p.heads;
  a.d = p.head_dim;
  a.n_text = p.n_text;
  a.n_pool = p.pt > 0 ? (p.T / p.pt) * (p.H / p.ph) * (p.W / p.pw) : 0;
  a.routed_k = p.routed_k;
  a.win_tok = p.wt * p.wh * p.ww;
  a.n_vis_keys = a.win_tok * (1 + a.routed_k);
  a.n_pool_keys = a.n_pool;
  a.n_text_keys = p.n_text;
  a.q_chunks = (a.win_tok + kBwdThreads / kBwdTPQ - 1) / (kBwdThreads / kBwdTPQ);
  a.scale = 1.0f / sqrtf(float(p.head_dim));
  b.out = static_cast<const float *>(out);
  b.lse = lse;
  b.dout = static_cast<const float *>(dout);
  b.dq = static_cast<float *>(dq);
  b.dk = static_cast<float *>(dk);
  b.dv = static_cast<float *>(dv);
  b.dkp = static_cast<float *>(workspace);
  b.dvp = b.dkp + size_t(p.B) * p.heads * a.n_pool * p.head_dim;
  const size_t kv_bytes = size_t(p.B) * p.heads * (size_t(a.g.N) + p.n_text) * p.head_dim * sizeof(float);
  if (cudaMemsetAsync(dk, 0, kv_bytes, s) != cudaSuccess || cudaMemsetAsync(dv, 0, kv_bytes, s) != cudaSuccess)
    return BASA_ERR_CUDA;
  if (a.n_pool > 0 && cudaMemsetAsync(workspace, 0, attn_bwd_workspace(p), s) != cudaSuccess) return BASA_ERR_CUDA;
  const long long blocks = (long long)p.B * p.heads * a.g.nWin * a.q_chunks;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  attn_bwd_f32_kernel<<<unsigned(blocks), kBwdThreads, 0, s>>>(b);
  if (cudaGetLastError() != cudaSuccess) return BASA_ERR_CUDA;
  if (a.n_pool > 0) {
    const long long total = (long long)p.B * p.heads * a.g.N * (p.head_dim / 4);
    pool_bwd_kernel<<<unsigned((total + 255) / 256), 256, 0, s>>>(b.dkp, b.dvp, b.dk, b.dv, a.g, p.pt, p.ph, p.pw,
                                                                 a.n_pool, p.n_text, p.head_dim, total,
                                                                 1.0f / float(p.pt * p.ph * p.pw));
    if (cudaGetLastError() != cudaSuccess) return BASA_ERR_CUDA;
  }
  return BASA_OK;
}

}  // namespace basa

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
  float *out;
  float *lse;  // nullable [B*heads][N]
  Geo g;
  int heads, d, n_text, n_pool, routed_k, win_tok, q_chunks;
  int n_vis_keys, n_pool_keys, n_text_keys;  // keys taken from each group (0 = group not selected)
  int dense;  // text-query rows: queries are q_text rows, keys are all N + n_text rows of k, v
  float scale;
};

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
    wins[threadIdx.x] = a.route[(bh * a.g.nWin + w) * a.routed_k + threadIdx.x - 1];
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

}  // namespace basa

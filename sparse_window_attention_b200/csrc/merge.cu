// Merge of branch results into the joint softmax (BASA §A.1: the local-window and
// text/global-memory branches can be evaluated separately and remain equivalent to
// one softmax over the concatenated K/V). For each query row, with L = log sum_b
// exp(lse_b): out = sum_b exp(lse_b - L) * out_b, and L is the merged log-sum-exp.
#include <cuda_bf16.h>

#include "basa_internal.h"

namespace basa {
namespace {

struct MergeArgs {
  const void *out[kMaxMerge];
  const float *lse[kMaxMerge];
  int n;
  void *dst;
  float *dst_lse;
  long long rows;  // B * heads * N query rows
  int d, lpr;      // head_dim; 16-byte chunks per row
};

__device__ __forceinline__ void load_chunk(const __nv_bfloat16 *p, float *v) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load_chunk(const float *p, float *v) {
  const float4 u = *reinterpret_cast<const float4 *>(p);
  v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
}
__device__ __forceinline__ void store_chunk(__nv_bfloat16 *p, const float *v) {
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r[i]) : "f"(v[2 * i + 1]), "f"(v[2 * i]));
  *reinterpret_cast<uint4 *>(p) = make_uint4(r[0], r[1], r[2], r[3]);
}
__device__ __forceinline__ void store_chunk(float *p, const float *v) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// One thread per (query row, 16-byte column chunk).
template <typename T>
__global__ void __launch_bounds__(256) merge_kernel(const __grid_constant__ MergeArgs a) {
  constexpr int VEC = 16 / sizeof(T);
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = idx / a.lpr;
  const int c = int(idx % a.lpr);
  if (row >= a.rows) return;
  float L[kMaxMerge];
  float m = -INFINITY;
  for (int b = 0; b < a.n; ++b) {
    L[b] = a.lse[b][row];
    m = fmaxf(m, L[b]);
  }
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
  float tot = 0.f;
  for (int b = 0; b < a.n; ++b) {
    const float w = expf(L[b] - m);
    tot += w;
    float v[VEC];
    load_chunk(static_cast<const T *>(a.out[b]) + row * a.d + c * VEC, v);
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = fmaf(w, v[i], acc[i]);
  }
  const float inv = 1.0f / tot;
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] *= inv;
  store_chunk(static_cast<T *>(a.dst) + row * a.d + c * VEC, acc);
  if (a.dst_lse && c == 0) a.dst_lse[row] = m + logf(tot);
}

}  // namespace

basa_status launch_merge_rows(int n, const void *const *outs, const float *const *lses, void *out, float *lse,
                              long long rows, int head_dim, basa_dtype dtype, cudaStream_t s) {
  if (n < 1 || n > kMaxMerge) return BASA_ERR_INVALID_ARG;
  MergeArgs a{};
  for (int b = 0; b < n; ++b) {
    a.out[b] = outs[b];
    a.lse[b] = lses[b];
  }
  a.n = n;
  a.dst = out;
  a.dst_lse = lse;
  a.rows = rows;
  a.d = head_dim;
  a.lpr = head_dim * (dtype == BASA_BF16 ? 2 : 4) / 16;
  const long long threads = a.rows * a.lpr;
  const long long blocks = (threads + 255) / 256;
  if (blocks >= (1ll << 31)) return BASA_ERR_UNSUPPORTED;
  if (dtype == BASA_BF16) merge_kernel<__nv_bfloat16><<<unsigned(blocks), 256, 0, s>>>(a);
  else merge_kernel<float><<<unsigned(blocks), 256, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

basa_status launch_merge(int n, const void *const *outs, const float *const *lses, void *out, float *lse,
                         const basa_params &p, cudaStream_t s) {
  return launch_merge_rows(n, outs, lses, out, lse, (long long)p.B * p.heads * p.T * p.H * p.W, p.head_dim, p.dtype, s);
}

}  // namespace basa

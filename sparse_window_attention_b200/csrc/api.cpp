// C ABI of libbasa: argument checks, then dispatch to the kernel launchers.
// Every check runs on the host before any CUDA call, so an invalid call
// returns its status and launches nothing.
#include <cstdint>
#include <cstring>

#include "basa_internal.h"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool empty_batch(const basa_params *p) { return p->B == 0 || p->heads == 0; }

// Fewest routing candidates of any window under a radius r >= 1: a corner window
// sees min(r, n - 1) + 1 window positions along an axis of n windows.
int64_t min_candidates(const basa_params *p) {
  const int64_t n[3] = {p->T / p->wt, p->H / p->wh, p->W / p->ww};
  int64_t c = 1;
  for (int a = 0; a < 3; ++a) c *= (n[a] - 1 < p->route_radius ? n[a] - 1 : p->route_radius) + 1;
  return c - 1;
}

// Checks shared by every entry point.
basa_status check_common(const basa_params *p) {
  if (!p) return BASA_ERR_INVALID_ARG;
  if (p->B < 0 || p->heads < 0 || p->n_text < 0 || p->routed_k < 0) return BASA_ERR_INVALID_ARG;
  if (p->dtype != BASA_BF16 && p->dtype != BASA_F32) return BASA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return BASA_ERR_UNSUPPORTED;
  if (p->T < 1 || p->H < 1 || p->W < 1) return BASA_ERR_SHAPE;
  if (p->wt < 1 || p->wh < 1 || p->ww < 1) return BASA_ERR_SHAPE;
  if (p->T % p->wt || p->H % p->wh || p->W % p->ww) return BASA_ERR_SHAPE;
  if (p->st < 0 || p->st >= p->T || p->sy < 0 || p->sy >= p->H || p->sx < 0 || p->sx >= p->W) return BASA_ERR_SHAPE;
  const bool no_pool = p->pt == 0 && p->ph == 0 && p->pw == 0;
  if (!no_pool) {
    if (p->pt < 1 || p->ph < 1 || p->pw < 1) return BASA_ERR_SHAPE;
    if (p->T % p->pt || p->H % p->ph || p->W % p->pw) return BASA_ERR_SHAPE;
  }
  const int64_t N = int64_t(p->T) * p->H * p->W;
  const int64_t rows = N + p->n_text;
  if (rows >= (int64_t(1) << 31)) return BASA_ERR_UNSUPPORTED;
  const int64_t bh = int64_t(p->B) * p->heads;
  if (bh >= (int64_t(1) << 31)) return BASA_ERR_UNSUPPORTED;
  const int64_t nwin = N / (int64_t(p->wt) * p->wh * p->ww);
  if (p->route_radius < 0) return BASA_ERR_INVALID_ARG;
  if (p->routed_k > 0) {
    if (p->routed_k > basa::kMaxRouted || p->routed_k > nwin - 1) return BASA_ERR_INVALID_ARG;
    if (p->route_radius > 0 && p->routed_k > min_candidates(p)) return BASA_ERR_INVALID_ARG;
  }
  return BASA_OK;
}

bool has_pool(const basa_params *p) { return p->pt > 0; }

}  // namespace

extern "C" {

const char *basa_status_string(basa_status s) {
  switch (s) {
    case BASA_OK: return "BASA_OK";
    case BASA_ERR_INVALID_ARG: return "BASA_ERR_INVALID_ARG";
    case BASA_ERR_SHAPE: return "BASA_ERR_SHAPE";
    case BASA_ERR_UNSUPPORTED: return "BASA_ERR_UNSUPPORTED";
    case BASA_ERR_CUDA: return "BASA_ERR_CUDA";
    case BASA_ERR_DEVICE_TIMEOUT: return "BASA_ERR_DEVICE_TIMEOUT";
    case BASA_ERR_BAD_INDEX: return "BASA_ERR_BAD_INDEX";
  }
  return "BASA_ERR_UNKNOWN";
}

basa_status basa_device_error_status(int32_t w) {
  if (w == 0) return BASA_OK;
  return (w & BASA_DEVERR_BAD_ROUTE) ? BASA_ERR_BAD_INDEX : BASA_ERR_DEVICE_TIMEOUT;
}

basa_status basa_pool_kv(const void *k, const void *v, void *kp, void *vp, const basa_params *p,
                         basa_stream_t stream) {
  basa_status st = check_common(p);
  if (st != BASA_OK) return st;
  if (!has_pool(p)) return BASA_ERR_INVALID_ARG;
  if (empty_batch(p)) return BASA_OK;
  if (!k || !v || !kp || !vp) return BASA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kp) || !aligned16(vp)) return BASA_ERR_INVALID_ARG;
  return basa::launch_pool_kv(k, v, kp, vp, *p, reinterpret_cast<cudaStream_t>(stream));
}

size_t basa_route_workspace_bytes(const basa_params *p) {
  if (check_common(p) != BASA_OK) return 0;
  const size_t nwin = size_t(p->T / p->wt) * (p->H / p->wh) * (p->W / p->ww);
  return 2 * size_t(p->B) * p->heads * nwin * p->head_dim * sizeof(float);
}

basa_status basa_route_windows(const void *q, const void *k, int32_t *route_idx, float *route_score,
                               void *workspace, const basa_params *p, basa_stream_t stream) {
  basa_status st = check_common(p);
  if (st != BASA_OK) return st;
  if (p->routed_k < 1) return BASA_ERR_INVALID_ARG;
  const int64_t nwin = int64_t(p->T / p->wt) * (p->H / p->wh) * (p->W / p->ww);
  if (nwin > 4096) return BASA_ERR_UNSUPPORTED;
  if (empty_batch(p)) return BASA_OK;
  if (!q || !k || !route_idx || !workspace) return BASA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(workspace) || !aligned4(route_idx)) return BASA_ERR_INVALID_ARG;
  if (route_score && !aligned4(route_score)) return BASA_ERR_INVALID_ARG;
  return basa::launch_route(q, k, route_idx, route_score, workspace, *p, reinterpret_cast<cudaStream_t>(stream));
}

basa_status basa_route_windows_noalloc(const void *q, const void *k, int32_t *route_idx, float *route_score,
                                       const basa_params *p, basa_stream_t stream) {
  basa_status st = check_common(p);
  if (st != BASA_OK) return st;
  if (p->routed_k < 1) return BASA_ERR_INVALID_ARG;
  const int64_t nwin = int64_t(p->T / p->wt) * (p->H / p->wh) * (p->W / p->ww);
  if (nwin > 4096) return BASA_ERR_UNSUPPORTED;
  if (basa_route_workspace_bytes(p) > BASA_NOALLOC_SCRATCH_BYTES) return BASA_ERR_UNSUPPORTED;
  if (empty_batch(p)) return BASA_OK;
  if (!q || !k || !route_idx) return BASA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned4(route_idx)) return BASA_ERR_INVALID_ARG;
  if (route_score && !aligned4(route_score)) return BASA_ERR_INVALID_ARG;
  return basa::launch_route_noalloc(q, k, route_idx, route_score, *p, reinterpret_cast<cudaStream_t>(stream));
}

size_t basa_pool_route_workspace_bytes(const basa_params *p) {
  if (check_common(p) != BASA_OK || !has_pool(p) || p->routed_k < 1) return 0;
  basa::FusedPlan fp;
  if (basa::plan_fused(*p, &fp) != BASA_OK) return 0;
  return fp.means_bytes + fp.part_bytes;
}

basa_status basa_pool_route(const void *q, const void *k, const void *v, void *kp, void *vp, int32_t *route_idx,
                            float *route_score, void *workspace, const basa_params *p, basa_stream_t stream) {
  basa_status st = check_common(p);
  if (st != BASA_OK) return st;
  if (!has_pool(p) || p->routed_k < 1) return BASA_ERR_INVALID_ARG;
  const int64_t nwin = int64_t(p->T / p->wt) * (p->H / p->wh) * (p->W / p->ww);
  if (nwin > 4096) return BASA_ERR_UNSUPPORTED;
  basa::FusedPlan fp;
  st = basa::plan_fused(*p, &fp);
  if (st != BASA_OK) return st;
  if (empty_batch(p)) return BASA_OK;
  if (!q || !k || !v || !kp || !vp || !route_idx || !workspace) return BASA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kp) || !aligned16(vp) || !aligned16(workspace) ||
      !aligned4(route_idx))
    return BASA_ERR_INVALID_ARG;
  if (route_score && !aligned4(route_score)) return BASA_ERR_INVALID_ARG;
  return basa::launch_pool_route_fused(q, k, v, kp, vp, route_idx, route_score, workspace, *p,
                                       reinterpret_cast<cudaStream_t>(stream));
}

static basa_status attn_common(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                               const int32_t *route_idx, void *out, float *lse, uint32_t keys, const basa_params *p,
                               basa_stream_t stream) {
  basa_status st = check_common(p);
  if (st != BASA_OK) return st;
  if (p->dtype == BASA_BF16 && p->head_dim != 128) return BASA_ERR_UNSUPPORTED;
  if (keys & ~BASA_KEYS_ALL) return BASA_ERR_INVALID_ARG;
  // groups the layer does not have add no keys; the selection must leave some
  const bool any = (keys & BASA_KEYS_WINDOWS) || ((keys & BASA_KEYS_POOLED) && has_pool(p)) ||
                   ((keys & BASA_KEYS_TEXT) && p->n_text > 0);
  if (!any) return BASA_ERR_INVALID_ARG;
  if (empty_batch(p)) return BASA_OK;
  if (!q || !k || !v || !out) return BASA_ERR_INVALID_ARG;
  if (has_pool(p) != (kp != nullptr) || has_pool(p) != (vp != nullptr)) return BASA_ERR_INVALID_ARG;
  if ((p->routed_k > 0) != (route_idx != nullptr)) return BASA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return BASA_ERR_INVALID_ARG;
  if (kp && (!aligned16(kp) || !aligned16(vp))) return BASA_ERR_INVALID_ARG;
  if (route_idx && !aligned4(route_idx)) return BASA_ERR_INVALID_ARG;
  if (lse && !aligned4(lse)) return BASA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p->dtype == BASA_F32) return basa::launch_attn_f32(q, k, v, kp, vp, route_idx, out, lse, keys, *p, s);
  return basa::launch_attn_bf16(q, k, v, kp, vp, route_idx, out, lse, keys, *p, s);
}

basa_status basa_window_attn_fwd(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                                 const int32_t *route_idx, void *out, const basa_params *p,
                                 basa_stream_t stream) {
  return attn_common(q, k, v, kp, vp, route_idx, out, nullptr, BASA_KEYS_ALL, p, stream);
}

basa_status basa_window_attn_fwd_lse(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                                     const int32_t *route_idx, void *out, float *lse, uint32_t keys,
                                     const basa_params *p, basa_stream_t stream) {
  return attn_common(q, k, v, kp, vp, route_idx, out, lse, keys, p, stream);
}

size_t basa_text_attn_workspace_bytes(const basa_params *p) {
  if (check_common(p) != BASA_OK || p->n_text < 1 || p->dtype != BASA_BF16) return 0;
  return basa::text_attn_workspace(*p, basa::device_sm_count());
}

basa_status basa_text_attn_fwd(const void *q_text, const void *k, const void *v, void *out_text, void *workspace,
                               const basa_params *p, basa_stream_t stream) {
  basa_status st = check_common(p);
  if (st != BASA_OK) return st;
  if (p->n_text < 1) return BASA_ERR_INVALID_ARG;
  if (p->dtype == BASA_BF16 && p->head_dim != 128) return BASA_ERR_UNSUPPORTED;
  if (empty_batch(p)) return BASA_OK;
  if (!q_text || !k || !v || !out_text) return BASA_ERR_INVALID_ARG;
  if (!aligned16(q_text) || !aligned16(k) || !aligned16(v) || !aligned16(out_text)) return BASA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p->dtype == BASA_F32) return basa::launch_attn_text_f32(q_text, k, v, out_text, *p, s);
  const int sms = basa::device_sm_count();
  if (sms <= 0) return BASA_ERR_CUDA;
  if (basa::text_attn_workspace(*p, sms) > 0 && (!workspace || !aligned16(workspace))) return BASA_ERR_INVALID_ARG;
  return basa::launch_attn_text_bf16(q_text, k, v, out_text, workspace, *p, sms, s);
}

size_t basa_window_attn_bwd_workspace_bytes(const basa_params *p) {
  if (check_common(p) != BASA_OK || p->head_dim != 128) return 0;
  return p->dtype == BASA_BF16 ? basa::attn_bwd_bf16_workspace(*p) : basa::attn_bwd_workspace(*p);
}

basa_status basa_window_attn_bwd(const void *q, const void *k, const void *v, const void *kp, const void *vp,
                                 const int32_t *route_idx, const void *out, const float *lse, const void *dout,
                                 void *dq, void *dk, void *dv, void *workspace, const basa_params *p,
                                 basa_stream_t stream) {
  basa_status st = check_common(p);
  if (st != BASA_OK) return st;
  if (p->head_dim != 128) return BASA_ERR_UNSUPPORTED;
  if (p->dtype == BASA_BF16 && p->routed_k > 0 && int64_t(p->T / p->wt) * (p->H / p->wh) * (p->W / p->ww) > 4096)
    return BASA_ERR_UNSUPPORTED;
  if (empty_batch(p)) return BASA_OK;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return BASA_ERR_INVALID_ARG;
  if (has_pool(p) != (kp != nullptr) || has_pool(p) != (vp != nullptr)) return BASA_ERR_INVALID_ARG;
  if ((p->routed_k > 0) != (route_idx != nullptr)) return BASA_ERR_INVALID_ARG;
  for (const void *x : {q, k, v, out, dout, static_cast<const void *>(dq), static_cast<const void *>(dk),
                        static_cast<const void *>(dv)})
    if (!aligned16(x)) return BASA_ERR_INVALID_ARG;
  if (!aligned4(lse) || (route_idx && !aligned4(route_idx))) return BASA_ERR_INVALID_ARG;
  if (kp && (!aligned16(kp) || !aligned16(vp))) return BASA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p->dtype == BASA_BF16) {
    const size_t need = basa::attn_bwd_bf16_workspace(*p);
    if (need == 0) return BASA_ERR_UNSUPPORTED;  // the tiling plan does not fit the kernel's limits
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return BASA_ERR_INVALID_ARG;
    return basa::launch_attn_bwd_bf16(q, k, v, kp, vp, route_idx, out, lse, dout, dq, dk, dv, workspace, *p, s);
  }
  if (basa::attn_bwd_workspace(*p) > 0 && (!workspace || !aligned16(workspace))) return BASA_ERR_INVALID_ARG;
  return basa::launch_attn_bwd_f32(q, k, v, kp, vp, route_idx, out, lse, dout, dq, dk, dv, workspace, *p, s);
}

basa_status basa_merge_branches(int n, const void *const *outs, const float *const *lses, void *out, float *lse,
                                const basa_params *p, basa_stream_t stream) {
  basa_status st = check_common(p);
  if (st != BASA_OK) return st;
  if (n < 1 || n > BASA_MAX_BRANCHES) return BASA_ERR_INVALID_ARG;
  if (empty_batch(p)) return BASA_OK;
  if (!outs || !lses || !out || !aligned16(out)) return BASA_ERR_INVALID_ARG;
  if (lse && !aligned4(lse)) return BASA_ERR_INVALID_ARG;
  for (int b = 0; b < n; ++b)
    if (!outs[b] || !lses[b] || !aligned16(outs[b]) || !aligned4(lses[b])) return BASA_ERR_INVALID_ARG;
  return basa::launch_merge(n, outs, lses, out, lse, *p, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

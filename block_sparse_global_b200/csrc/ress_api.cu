// C entry points of libress.so: argument validation on the host, then kernel launches on
// the caller's stream.  Validation happens before any CUDA call, so a bad argument is
// reported without touching the device.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/ress.h"
#include "ress_common.cuh"
#include "ress_internal.h"

using ress::Dims;

namespace {

constexpr int32_t kAbiVersion = 5;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every entry point.  On success fills d; *empty = true means
// there is no work (B = 0 or N = 0).
ress_status check_shape(const ress_shape *s, Dims *d, bool *empty) {
  if (s == nullptr) return RESS_ERR_INVALID_ARG;
  if (s->batch < 0 || s->seq_len < 0 || s->heads < 1) return RESS_ERR_INVALID_ARG;
  if (s->head_dim != ress::kHeadDim || s->block != ress::kBlock) return RESS_ERR_UNSUPPORTED;
  if (s->key_block != 0 && s->key_block != ress::kBlock && s->key_block != ress::kBlock / 2)
    return RESS_ERR_UNSUPPORTED;
  if (s->heads > ress::kMaxHeads) return RESS_ERR_UNSUPPORTED;
  d->B = s->batch;
  d->H = s->heads;
  d->N = s->seq_len;
  d->kb = s->key_block == 0 ? ress::kBlock : s->key_block;
  d->nq = (s->seq_len + ress::kBlock - 1) / ress::kBlock;
  d->nk = (s->seq_len + d->kb - 1) / d->kb;
  d->nb = d->nq;
  if (d->nk > ress::kMaxBlocks) return RESS_ERR_UNSUPPORTED;
  if (d->BH() > 65535) return RESS_ERR_UNSUPPORTED;  // grid.y limit of the block kernels
  if (d->BH() * d->nq * (long long)d->nk > 0x7fffffffffffll) return RESS_ERR_UNSUPPORTED;
  if (d->BH() * d->nq > 0x7fffffffll) return RESS_ERR_UNSUPPORTED;
  *empty = (d->B == 0 || d->N == 0);
  return RESS_OK;
}

bool ptr_ok(const void *p) { return p != nullptr && aligned16(p); }

ress_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RESS_OK : RESS_ERR_CUDA; }

}  // namespace

extern "C" {

int32_t ress_abi_version(void) { return kAbiVersion; }

const char *ress_status_string(ress_status status) {
  switch (status) {
    case RESS_OK: return "RESS_OK";
    case RESS_ERR_INVALID_ARG: return "RESS_ERR_INVALID_ARG";
    case RESS_ERR_UNSUPPORTED: return "RESS_ERR_UNSUPPORTED";
    case RESS_ERR_CUDA: return "RESS_ERR_CUDA";
    case RESS_ERR_DEVICE_BOUNDS: return "RESS_ERR_DEVICE_BOUNDS";
    case RESS_ERR_DEVICE_TIMEOUT: return "RESS_ERR_DEVICE_TIMEOUT";
  }
  return "RESS_ERR_UNKNOWN";
}

ress_status ress_head_gram(const ress_shape *shape, int32_t d_model, const float *w_o,
                           float *gram, ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (d_model < 1 || !ptr_ok(w_o) || !ptr_ok(gram)) return RESS_ERR_INVALID_ARG;
  return from_cuda(ress::launch_head_gram(d.H, d_model, w_o, gram, (cudaStream_t)stream));
}

ress_status ress_token_gather(const ress_shape *shape, int32_t views, int32_t specials,
                              int32_t inverse, const void *src, void *dst, ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (views < 1 || (d.N > 0 && d.N % views != 0)) return RESS_ERR_INVALID_ARG;
  if (specials < 0 || specials > d.N / views) return RESS_ERR_INVALID_ARG;
  if (inverse != 0 && inverse != 1) return RESS_ERR_INVALID_ARG;
  if (empty) return RESS_OK;
  if (!ptr_ok(src) || !ptr_ok(dst) || src == dst) return RESS_ERR_INVALID_ARG;
  return from_cuda(ress::launch_token_gather(d, views, specials, inverse != 0, src, dst,
                                             (cudaStream_t)stream));
}

ress_status ress_pool_blocks(const ress_shape *shape, const void *q, const void *k,
                             const void *v, float *q_pool, float *k_pool, float *v_pool,
                             ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (empty) return RESS_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(q_pool) || !ptr_ok(k_pool) ||
      !ptr_ok(v_pool))
    return RESS_ERR_INVALID_ARG;
  return from_cuda(ress::launch_pool(d, q, k, v, q_pool, k_pool, v_pool, (cudaStream_t)stream));
}

ress_status ress_block_scores(const ress_shape *shape, const float *q_pool, const float *k_pool,
                              const float *v_pool, float scale, float *P, float *v_bar,
                              ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (empty) return RESS_OK;
  if (!ptr_ok(q_pool) || !ptr_ok(k_pool) || !ptr_ok(v_pool) || !ptr_ok(P) || !ptr_ok(v_bar))
    return RESS_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return RESS_ERR_INVALID_ARG;
  return from_cuda(
      ress::launch_block_scores(d, q_pool, k_pool, v_pool, scale, P, v_bar, (cudaStream_t)stream));
}

size_t ress_drift_workspace_bytes(const ress_shape *shape) {
  Dims d;
  bool empty;
  if (check_shape(shape, &d, &empty) != RESS_OK || empty) return 0;
  return ress::drift_workspace_bytes(d);
}

ress_status ress_drift_scores(const ress_shape *shape, const float *P, const float *v_pool,
                              const float *v_bar, const float *gram, float *s, void *workspace,
                              size_t workspace_bytes, ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (empty) return RESS_OK;
  if (!ptr_ok(P) || !ptr_ok(v_pool) || !ptr_ok(v_bar) || !ptr_ok(gram) || !ptr_ok(s) ||
      !ptr_ok(workspace))
    return RESS_ERR_INVALID_ARG;
  if (workspace_bytes < ress::drift_workspace_bytes(d)) return RESS_ERR_INVALID_ARG;
  return from_cuda(
      ress::launch_drift(d, P, v_pool, v_bar, gram, s, workspace, (cudaStream_t)stream));
}

ress_status ress_select_blocks(const ress_shape *shape, const ress_select_params *params,
                               const float *P, const float *s, const float *v_pool,
                               const float *v_bar, const float *gram, int32_t *kv_idx,
                               int32_t *kv_cnt, uint8_t *mask, int32_t *dev_err,
                               ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (params == nullptr || params->budgets == nullptr) return RESS_ERR_INVALID_ARG;
  const int m = params->method;
  if (m != RESS_SELECT_MASS && m != RESS_SELECT_DRIFT && m != RESS_SELECT_RANDOM &&
      m != RESS_SELECT_CDF)
    return RESS_ERR_INVALID_ARG;
  if (m == RESS_SELECT_CDF && !(params->top_p > 0.f && params->top_p <= 1.f)) return RESS_ERR_INVALID_ARG;
  for (int h = 0; h < d.H; ++h)
    if (params->budgets[h] < 0 || params->budgets[h] > d.nk) return RESS_ERR_INVALID_ARG;
  const int obj = params->objective;
  if (obj != RESS_DRIFT_MINIMISE && obj != RESS_DRIFT_MAXIMISE_SWAPS && obj != RESS_DRIFT_MAXIMISE_FULL)
    return RESS_ERR_INVALID_ARG;
  if (obj != RESS_DRIFT_MINIMISE && m != RESS_SELECT_DRIFT) return RESS_ERR_INVALID_ARG;
  const bool want_drift = params->drift != nullptr;
  if (m == RESS_SELECT_DRIFT) {
    if (params->rounds < 0 || params->rounds > 64) return RESS_ERR_INVALID_ARG;
    if (!(params->rho > 0.f) || !(params->rho <= 1.f)) return RESS_ERR_INVALID_ARG;
  }
  if ((m == RESS_SELECT_DRIFT || want_drift) && !(params->eps > 0.f)) return RESS_ERR_INVALID_ARG;
  if (empty) return RESS_OK;
  if (!ptr_ok(P) || !ptr_ok(kv_idx) || !ptr_ok(kv_cnt)) return RESS_ERR_INVALID_ARG;
  if (mask != nullptr && !aligned16(mask)) return RESS_ERR_INVALID_ARG;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return RESS_ERR_INVALID_ARG;
  const bool restore = m == RESS_SELECT_DRIFT && params->rounds > 0;
  const bool state = restore || want_drift;  // the kernel tracks g, K and J
  if (m == RESS_SELECT_DRIFT && !ptr_ok(s)) return RESS_ERR_INVALID_ARG;
  if (state && (!ptr_ok(v_pool) || !ptr_ok(v_bar) || !ptr_ok(gram))) return RESS_ERR_INVALID_ARG;
  if (want_drift && !aligned16(params->drift)) return RESS_ERR_INVALID_ARG;
  ress::SelectLaunch a;
  a.method = m;
  a.rounds = m == RESS_SELECT_DRIFT ? params->rounds : 0;
  a.rho = params->rho;
  a.eps = (m == RESS_SELECT_DRIFT || want_drift) ? params->eps : 1e-4f;
  a.objective = obj;
  a.top_p = params->top_p;
  a.drift = params->drift;
  a.seed = params->seed;
  a.budgets = params->budgets;
  a.keep_k = params->keep_k;
  a.dense_q = params->dense_q;
  a.P = P;
  a.s = m == RESS_SELECT_DRIFT ? s : nullptr;
  a.vp = state ? v_pool : nullptr;
  a.vbar = state ? v_bar : nullptr;
  a.gram = state ? gram : nullptr;
  a.kv_idx = kv_idx;
  a.kv_cnt = kv_cnt;
  a.mask = mask;
  a.dev_err = dev_err;
  cudaError_t e = ress::launch_select(d, a, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return RESS_ERR_UNSUPPORTED;
  return from_cuda(e);
}

ress_status ress_scores_select(const ress_shape *shape, const ress_select_params *params,
                               const float *q_pool, const float *k_pool, const float *v_pool,
                               float scale, float *P, float *v_bar, int32_t *kv_idx,
                               int32_t *kv_cnt, uint8_t *mask, int32_t *dev_err,
                               ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (params == nullptr || params->budgets == nullptr) return RESS_ERR_INVALID_ARG;
  const int m = params->method;
  if (m == RESS_SELECT_DRIFT) return RESS_ERR_UNSUPPORTED;
  if (m != RESS_SELECT_MASS && m != RESS_SELECT_RANDOM && m != RESS_SELECT_CDF) return RESS_ERR_INVALID_ARG;
  if (m == RESS_SELECT_CDF && !(params->top_p > 0.f && params->top_p <= 1.f)) return RESS_ERR_INVALID_ARG;
  if (params->objective != RESS_DRIFT_MINIMISE || params->drift != nullptr) return RESS_ERR_INVALID_ARG;
  for (int h = 0; h < d.H; ++h)
    if (params->budgets[h] < 0 || params->budgets[h] > d.nk) return RESS_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return RESS_ERR_INVALID_ARG;
  if (empty) return RESS_OK;
  if (!ptr_ok(q_pool) || !ptr_ok(k_pool) || !ptr_ok(kv_idx) || !ptr_ok(kv_cnt)) return RESS_ERR_INVALID_ARG;
  if (P != nullptr && !aligned16(P)) return RESS_ERR_INVALID_ARG;
  if (v_bar != nullptr && (!aligned16(v_bar) || !ptr_ok(v_pool))) return RESS_ERR_INVALID_ARG;
  if (mask != nullptr && !aligned16(mask)) return RESS_ERR_INVALID_ARG;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return RESS_ERR_INVALID_ARG;
  ress::ScoresSelectLaunch a;
  a.method = m;
  a.seed = params->seed;
  a.top_p = params->top_p;
  a.budgets = params->budgets;
  a.keep_k = params->keep_k;
  a.dense_q = params->dense_q;
  a.qp = q_pool;
  a.kp = k_pool;
  a.vp = v_bar ? v_pool : nullptr;
  a.scale = scale;
  a.P = P;
  a.vbar = v_bar;
  a.kv_idx = kv_idx;
  a.kv_cnt = kv_cnt;
  a.mask = mask;
  return from_cuda(ress::launch_scores_select(d, a, (cudaStream_t)stream));
}

size_t ress_drift_select_workspace_bytes(const ress_shape *shape) {
  Dims d;
  bool empty;
  if (check_shape(shape, &d, &empty) != RESS_OK) return 0;
  return ress::drift_select_workspace_bytes(d);
}

ress_status ress_drift_select(const ress_shape *shape, const ress_select_params *params,
                              const float *q_pool, const float *k_pool, const float *v_pool,
                              const float *gram, float scale, float *P, float *v_bar, float *s,
                              int32_t *kv_idx, int32_t *kv_cnt, uint8_t *mask, int32_t *dev_err,
                              void *workspace, size_t workspace_bytes, ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (params == nullptr || params->budgets == nullptr) return RESS_ERR_INVALID_ARG;
  if (params->method != RESS_SELECT_DRIFT) return RESS_ERR_INVALID_ARG;
  for (int h = 0; h < d.H; ++h)
    if (params->budgets[h] < 0 || params->budgets[h] > d.nk) return RESS_ERR_INVALID_ARG;
  const int obj = params->objective;
  if (obj != RESS_DRIFT_MINIMISE && obj != RESS_DRIFT_MAXIMISE_SWAPS && obj != RESS_DRIFT_MAXIMISE_FULL)
    return RESS_ERR_INVALID_ARG;
  if (params->rounds < 0 || params->rounds > 64) return RESS_ERR_INVALID_ARG;
  if (!(params->rho > 0.f) || !(params->rho <= 1.f) || !(params->eps > 0.f)) return RESS_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return RESS_ERR_INVALID_ARG;
  if (empty) return RESS_OK;
  if (!ptr_ok(q_pool) || !ptr_ok(k_pool) || !ptr_ok(v_pool) || !ptr_ok(gram) || !ptr_ok(kv_idx) ||
      !ptr_ok(kv_cnt) || !ptr_ok(workspace))
    return RESS_ERR_INVALID_ARG;
  if (workspace_bytes < ress::drift_select_workspace_bytes(d)) return RESS_ERR_INVALID_ARG;
  for (const void *o : {(const void *)P, (const void *)v_bar, (const void *)s, (const void *)mask,
                        (const void *)params->drift})
    if (o != nullptr && !aligned16(o)) return RESS_ERR_INVALID_ARG;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return RESS_ERR_INVALID_ARG;
  ress::DriftSelectLaunch a;
  a.sel.method = RESS_SELECT_DRIFT;
  a.sel.rounds = params->rounds;
  a.sel.rho = params->rho;
  a.sel.eps = params->eps;
  a.sel.objective = obj;
  a.sel.top_p = params->top_p;
  a.sel.drift = params->drift;
  a.sel.seed = params->seed;
  a.sel.budgets = params->budgets;
  a.sel.keep_k = params->keep_k;
  a.sel.dense_q = params->dense_q;
  a.sel.P = nullptr;
  a.sel.s = nullptr;
  a.sel.vp = v_pool;
  a.sel.vbar = nullptr;
  a.sel.gram = gram;
  a.sel.kv_idx = kv_idx;
  a.sel.kv_cnt = kv_cnt;
  a.sel.mask = mask;
  a.sel.dev_err = dev_err;
  a.qp = q_pool;
  a.kp = k_pool;
  a.scale = scale;
  a.P_out = P;
  a.s_out = s;
  a.vbar_out = v_bar;
  a.ws = workspace;
  cudaError_t e = ress::launch_drift_select(d, a, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return RESS_ERR_UNSUPPORTED;
  return from_cuda(e);
}

ress_status ress_attn_schedule(const ress_shape *shape, const int32_t *kv_cnt, int32_t *work_order,
                               ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (empty) return RESS_OK;
  if (!ptr_ok(kv_cnt) || !ptr_ok(work_order)) return RESS_ERR_INVALID_ARG;
  return from_cuda(ress::launch_schedule(d, kv_cnt, work_order, (cudaStream_t)stream));
}

ress_status ress_block_sparse_attn(const ress_shape *shape, const void *q, const void *k,
                                   const void *v, const int32_t *kv_idx, const int32_t *kv_cnt,
                                   const int32_t *work_order, float scale, void *out, float *lse,
                                   int32_t *dev_err, ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (empty) return RESS_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(kv_idx) || !ptr_ok(kv_cnt) || !ptr_ok(out))
    return RESS_ERR_INVALID_ARG;
  if (work_order != nullptr && !aligned16(work_order)) return RESS_ERR_INVALID_ARG;
  if (lse != nullptr && !aligned16(lse)) return RESS_ERR_INVALID_ARG;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return RESS_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return RESS_ERR_INVALID_ARG;
  ress::AttnLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.kv_idx = kv_idx;
  a.kv_cnt = kv_cnt;
  a.order = work_order;
  a.scale = scale;
  a.out = out;
  a.lse = lse;
  a.dev_err = dev_err;
  cudaError_t e = ress::launch_attn(d, a, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return RESS_ERR_CUDA;
  return from_cuda(e);
}

ress_status ress_debug_attn_forced_timeout(const ress_shape *shape, const void *q, const void *k,
                                           const void *v, const int32_t *kv_idx,
                                           const int32_t *kv_cnt, float scale, void *out,
                                           int32_t *dev_err, int64_t limit_cycles,
                                           ress_stream_t stream) {
  if (limit_cycles <= 0 || limit_cycles > (int64_t)1 << 32) return RESS_ERR_INVALID_ARG;
  if (dev_err == nullptr || (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return RESS_ERR_INVALID_ARG;
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (empty) return RESS_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(kv_idx) || !ptr_ok(kv_cnt) || !ptr_ok(out))
    return RESS_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return RESS_ERR_INVALID_ARG;
  ress::AttnLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.kv_idx = kv_idx;
  a.kv_cnt = kv_cnt;
  a.order = nullptr;
  a.scale = scale;
  a.out = out;
  a.lse = nullptr;
  a.dev_err = dev_err;
  a.stall_cycles = (long long)limit_cycles;
  cudaError_t e = ress::launch_attn(d, a, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return RESS_ERR_CUDA;
  return from_cuda(e);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// ress_drift_scores_static: the drift score for callers that cannot allocate device
// memory.  Its scratch is this file's static device array; the host looks up the array's
// device address once per device (the array's name in host code is only a stand-in).
#include <mutex>

namespace {

constexpr size_t kDriftStaticBytes = (size_t)8 << 20;  // 8 MiB, see include/ress.h
static __device__ __align__(256) unsigned char g_drift_static_scratch[kDriftStaticBytes];

constexpr int kMaxDevices = 64;
void *g_drift_static_addr[kMaxDevices] = {};
std::mutex g_drift_static_mu;

// Device address of the static scratch on the current device; looked up on the first
// call per device, with that device current.
cudaError_t drift_static_address(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_drift_static_mu);
  if (g_drift_static_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_drift_static_scratch);
    if (e != cudaSuccess) return e;
    g_drift_static_addr[dev] = p;
  }
  *out = g_drift_static_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" ress_status ress_drift_scores_static(const ress_shape *shape, const float *P,
                                                const float *v_pool, const float *v_bar,
                                                const float *gram, float *s,
                                                ress_stream_t stream) {
  Dims d;
  bool empty;
  ress_status st = check_shape(shape, &d, &empty);
  if (st != RESS_OK) return st;
  if (empty) return RESS_OK;
  if (!ptr_ok(P) || !ptr_ok(v_pool) || !ptr_ok(v_bar) || !ptr_ok(gram) || !ptr_ok(s))
    return RESS_ERR_INVALID_ARG;
  if (ress::drift_workspace_bytes(d) > kDriftStaticBytes) return RESS_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  if (drift_static_address(&scratch) != cudaSuccess) return RESS_ERR_CUDA;
  return from_cuda(ress::launch_drift(d, P, v_pool, v_bar, gram, s, scratch, (cudaStream_t)stream));
}

// Host-side launchers shared between the translation units of libress.so.  Arguments
// have been validated by the C entry points (ress_api.cu) before any of these is called.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/ress.h"

namespace ress {

// nq query blocks of 128 tokens, nk key blocks of kb tokens (128, or 64 for the pages'
// grid); nb == nq.
struct Dims {
  int B, H, N, nb, nq, nk, kb;
  long long BH() const { return 1ll * B * H; }
};

cudaError_t launch_head_gram(int H, int d_model, const float *w_o, float *gram, cudaStream_t st);

cudaError_t launch_token_gather(const Dims &d, int views, int specials, bool inverse,
                                const void *src, void *dst, cudaStream_t st);

cudaError_t launch_pool(const Dims &d, const void *q, const void *k, const void *v, float *qp,
                        float *kp, float *vp, cudaStream_t st);

cudaError_t launch_block_scores(const Dims &d, const float *qp, const float *kp, const float *vp,
                                float scale, float *P, float *vbar, cudaStream_t st);

// Block map fused with mass / random selection (P and vbar optional).
struct ScoresSelectLaunch {
  int method;
  float top_p;
  uint64_t seed;
  const int32_t *budgets;  // host [H]
  const uint8_t *keep_k, *dense_q;
  const float *qp, *kp, *vp;
  float scale;
  float *P, *vbar;
  int32_t *kv_idx, *kv_cnt;
  uint8_t *mask;
};
cudaError_t launch_scores_select(const Dims &d, const ScoresSelectLaunch &a, cudaStream_t st);

size_t drift_workspace_bytes(const Dims &d);
cudaError_t launch_drift(const Dims &d, const float *P, const float *vp, const float *vbar,
                         const float *gram, float *s, void *ws, cudaStream_t st);

// Workspace of ress_drift_select: c_j = V_j^T M V_j, [B*H, nk] fp32.
size_t drift_select_workspace_bytes(const Dims &d);
cudaError_t launch_drift_cdiag(const Dims &d, const float *vp, const float *gram, float *c,
                               cudaStream_t st);

struct SelectLaunch {
  int method, rounds, objective;
  float top_p;    // RESS_SELECT_CDF threshold
  float *drift;  // realized J per row, or null
  float rho, eps;
  uint64_t seed;
  const int32_t *budgets;  // host [H]
  const uint8_t *keep_k, *dense_q;
  const float *P, *s, *vp, *vbar, *gram;
  int32_t *kv_idx, *kv_cnt;
  uint8_t *mask;
  int32_t *dev_err;
};
cudaError_t launch_select(const Dims &d, const SelectLaunch &a, cudaStream_t st);

// Fused drift selection: block map, drift score and selection in one kernel.
struct DriftSelectLaunch {
  SelectLaunch sel;               // method DRIFT; P, s, vbar unused
  const float *qp, *kp;           // pooled queries and keys (vp, gram in sel)
  float scale;
  float *P_out, *s_out, *vbar_out;  // optional
  void *ws;                       // drift_select_workspace_bytes
};
cudaError_t launch_drift_select(const Dims &d, const DriftSelectLaunch &a, cudaStream_t st);

cudaError_t launch_schedule(const Dims &d, const int32_t *kv_cnt, int32_t *order, cudaStream_t st);

struct AttnLaunch {
  const void *q, *k, *v;
  const int32_t *kv_idx, *kv_cnt, *order;
  float scale;
  void *out;
  float *lse;
  int32_t *dev_err;
  long long stall_cycles = 0;  // > 0: the diagnostic forced timeout
};
// Returns cudaErrorNotSupported if the driver cannot encode tensor maps.
cudaError_t launch_attn(const Dims &d, const AttnLaunch &a, cudaStream_t st);

}  // namespace ress

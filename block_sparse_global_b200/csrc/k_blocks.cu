// Block-level kernels: head Gram matrices, mean pooling, pooled block map, drift score.
//
// [ReSS] = "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers".
// All of these are small next to the attention itself; pooling is bound by HBM reads of
// Q/K/V, the block map and drift score by fp32 FMA on L2-resident pooled tensors.
#include <cuda_bf16.h>

#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPad = 65;  // padded row of 64 floats: lane-strided rows hit distinct banks

RESS_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
RESS_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ------------------------------------------------------------------ Gram, [ReSS] Eq. 8
// M_h[a][b] = sum_r W[r][64h + a] * W[r][64h + b].  Grid: one CTA per head.
__global__ void __launch_bounds__(kThreads) head_gram_kernel(const float *__restrict__ w_o,
                                                             float *__restrict__ gram,
                                                             int H, int d_model) {
  __shared__ float ws[32][kHeadDim + 1];
  const int h = blockIdx.x, t = threadIdx.x;
  const int a = t >> 2, b0 = (t & 3) * 16;
  float acc[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) acc[c] = 0.f;
  const int ld = H * kHeadDim;
  for (int r0 = 0; r0 < d_model; r0 += 32) {
    __syncthreads();
    for (int idx = t; idx < 32 * kHeadDim; idx += kThreads) {
      int rr = idx / kHeadDim, cc = idx % kHeadDim;
      ws[rr][cc] = (r0 + rr < d_model) ? w_o[(size_t)(r0 + rr) * ld + h * kHeadDim + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int rr = 0; rr < 32; ++rr) {
      float wa = ws[rr][a];
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[c] = fmaf(wa, ws[rr][b0 + c], acc[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) gram[((size_t)h * kHeadDim + a) * kHeadDim + b0 + c] = acc[c];
}

// --------------------------------------------------- mean pooling, [ReSS] §3 step (1)
// One warp per (tensor, b*h, block).  Lane = (token slot ts = lane/8, 16-byte column
// group cg = lane%8): a warp-wide load covers 4 consecutive token rows (512 contiguous
// bytes); 32 such loads cover a 128-token block.
__global__ void __launch_bounds__(kThreads) pool_kernel(const uint4 *__restrict__ q,
                                                        const uint4 *__restrict__ k,
                                                        const uint4 *__restrict__ v,
                                                        float *__restrict__ qp,
                                                        float *__restrict__ kp,
                                                        float *__restrict__ vp, long long BH,
                                                        int N, int nb) {
  const int lane = threadIdx.x & 31;
  const int cg = lane & 7, ts = lane >> 3;
  const long long per_tensor = BH * nb;
  const long long units = 3 * per_tensor;
  for (long long u = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5); u < units;
       u += (long long)gridDim.x * kWarps) {
    const int which = (int)(u / per_tensor);
    const long long rem = u - which * per_tensor;
    const long long bh = rem / nb;
    const int j = (int)(rem - bh * nb);
    const uint4 *src = (which == 0 ? q : which == 1 ? k : v) + (size_t)bh * N * 8;
    float *dst = (which == 0 ? qp : which == 1 ? kp : vp) + ((size_t)bh * nb + j) * kHeadDim;
    const int t0 = j * kBlock, t1 = min(N, t0 + kBlock);
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll 8
    for (int it = 0; it < kBlock / 4; ++it) {
      const int tok = t0 + ts + 4 * it;
      if (tok < t1) {
        uint4 w = __ldg(src + (size_t)tok * 8 + cg);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[2 * c] += __uint_as_float(ww[c] << 16);
          acc[2 * c + 1] += __uint_as_float(ww[c] & 0xffff0000u);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 8);
      acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 16);
    }
    if (ts == 0) {
      const float cnt = (float)(t1 - t0);
      float4 lo = make_float4(__fdiv_rn(acc[0], cnt), __fdiv_rn(acc[1], cnt),
                              __fdiv_rn(acc[2], cnt), __fdiv_rn(acc[3], cnt));
      float4 hi = make_float4(__fdiv_rn(acc[4], cnt), __fdiv_rn(acc[5], cnt),
                              __fdiv_rn(acc[6], cnt), __fdiv_rn(acc[7], cnt));
      reinterpret_cast<float4 *>(dst)[2 * cg] = lo;
      reinterpret_cast<float4 *>(dst)[2 * cg + 1] = hi;
    }
  }
}

// ---------------------------------------- pooled block map and Eq. 1 output, [ReSS] §4.1
// One CTA per (b*h, TQ query blocks).  Logits of the CTA's rows against every key block
// are kept in shared memory ([TQ][nb] floats), so each pooled key / value tile is read
// once per CTA.  Warp w owns rows w, w + 8, ...
template <int TQ>
__global__ void __launch_bounds__(kThreads) block_scores_kernel(
    const float *__restrict__ qp, const float *__restrict__ kp, const float *__restrict__ vp,
    float scale, float *__restrict__ P, float *__restrict__ vbar, int nb) {
  extern __shared__ __align__(16) float sm[];
  float *sq = sm;                     // [TQ][64]
  float *st = sq + TQ * kHeadDim;     // [32][65] key or value tile
  float *sl = st + 32 * kPad;         // [TQ][nb] logits, then probabilities
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * TQ;
  const float *qh = qp + (size_t)bh * nb * kHeadDim;
  const float *kh = kp + (size_t)bh * nb * kHeadDim;
  const float *vh = vp + (size_t)bh * nb * kHeadDim;
  for (int idx = t; idx < TQ * kHeadDim; idx += kThreads) {
    int r = idx / kHeadDim;
    sq[idx] = (i0 + r < nb) ? qh[(size_t)(i0 + r) * kHeadDim + idx % kHeadDim] : 0.f;
  }
  for (int j0 = 0; j0 < nb; j0 += 32) {
    __syncthreads();
    for (int idx = t; idx < 32 * kHeadDim; idx += kThreads) {
      int jj = idx / kHeadDim, c = idx % kHeadDim;
      st[jj * kPad + c] = (j0 + jj < nb) ? kh[(size_t)(j0 + jj) * kHeadDim + c] : 0.f;
    }
    __syncthreads();
    for (int r = warp; r < TQ; r += kWarps) {
      float acc = 0.f;
#pragma unroll 16
      for (int c = 0; c < kHeadDim; ++c) acc = fmaf(sq[r * kHeadDim + c], st[lane * kPad + c], acc);
      if (j0 + lane < nb) sl[r * nb + j0 + lane] = acc * scale;
    }
  }
  __syncthreads();
  for (int r = warp; r < TQ; r += kWarps) {
    const int i = i0 + r;
    if (i >= nb) continue;
    float *row = sl + r * nb;
    float m = -INFINITY;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, row[j]);
    m = warp_max(m);
    float sum = 0.f;
    for (int j = lane; j < nb; j += 32) {
      float e = expf(row[j] - m);
      row[j] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    float *prow = P + ((size_t)bh * nb + i) * nb;
    for (int j = lane; j < nb; j += 32) {
      float p = __fdiv_rn(row[j], sum);
      row[j] = p;
      prow[j] = p;
    }
  }
  // vbar_i = sum_j P_ij V_j, value tiles staged through shared memory.
  float a0[(TQ + kWarps - 1) / kWarps], a1[(TQ + kWarps - 1) / kWarps];
#pragma unroll
  for (int q = 0; q < (TQ + kWarps - 1) / kWarps; ++q) a0[q] = a1[q] = 0.f;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    __syncthreads();
    for (int idx = t; idx < 32 * kHeadDim; idx += kThreads) {
      int jj = idx / kHeadDim, c = idx % kHeadDim;
      st[jj * kPad + c] = (j0 + jj < nb) ? vh[(size_t)(j0 + jj) * kHeadDim + c] : 0.f;
    }
    __syncthreads();
    const int jn = min(32, nb - j0);
#pragma unroll
    for (int q = 0; q < (TQ + kWarps - 1) / kWarps; ++q) {
      const int r = warp + q * kWarps;
      if (r < TQ && i0 + r < nb) {
        const float *row = sl + r * nb + j0;
        for (int jj = 0; jj < jn; ++jj) {
          const float p = row[jj];
          a0[q] = fmaf(p, st[jj * kPad + lane], a0[q]);
          a1[q] = fmaf(p, st[jj * kPad + lane + 32], a1[q]);
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < (TQ + kWarps - 1) / kWarps; ++q) {
    const int r = warp + q * kWarps;
    if (r < TQ && i0 + r < nb) {
      float *o = vbar + ((size_t)bh * nb + i0 + r) * kHeadDim;
      o[lane] = a0[q];
      o[lane + 32] = a1[q];
    }
  }
}

// ------------------------------------------------------- drift score, [ReSS] Eqs. 5-9
// Pass 1: for every pooled vector x of a head (the rows vbar_i and the keys V_j),
// y = M_h x and x . y.  Stores w_i = M vbar_i, a_i = vbar_i^T M vbar_i and
// c_j = V_j^T M V_j in the workspace.
__global__ void __launch_bounds__(kThreads) drift_prep_kernel(
    const float *__restrict__ vp, const float *__restrict__ vbar, const float *__restrict__ gram,
    float *__restrict__ w, float *__restrict__ a, float *__restrict__ c, int H, int nb) {
  __shared__ float sM[kHeadDim][kPad];
  __shared__ float sx[kWarps][kHeadDim];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const long long bh = blockIdx.y;
  const int h = (int)(bh % H);
  const bool rows = blockIdx.z == 0;  // 0: vbar rows -> w, a;  1: pooled keys -> c
  for (int idx = t; idx < kHeadDim * kHeadDim; idx += kThreads)
    sM[idx / kHeadDim][idx % kHeadDim] = gram[(size_t)h * kHeadDim * kHeadDim + idx];
  __syncthreads();
  const float *src = (rows ? vbar : vp) + (size_t)bh * nb * kHeadDim;
  for (int n = blockIdx.x * 32 + warp; n < min(nb, (int)blockIdx.x * 32 + 32); n += kWarps) {
    sx[warp][lane] = src[(size_t)n * kHeadDim + lane];
    sx[warp][lane + 32] = src[(size_t)n * kHeadDim + lane + 32];
    __syncwarp();
    float y0 = 0.f, y1 = 0.f;
#pragma unroll 16
    for (int e = 0; e < kHeadDim; ++e) {
      const float xe = sx[warp][e];
      y0 = fmaf(sM[lane][e], xe, y0);
      y1 = fmaf(sM[lane + 32][e], xe, y1);
    }
    const float dot = warp_sum(sx[warp][lane] * y0 + sx[warp][lane + 32] * y1);
    if (rows) {
      w[((size_t)bh * nb + n) * kHeadDim + lane] = y0;
      w[((size_t)bh * nb + n) * kHeadDim + lane + 32] = y1;
      if (lane == 0) a[(size_t)bh * nb + n] = dot;
    } else if (lane == 0) {
      c[(size_t)bh * nb + n] = dot;
    }
    __syncwarp();
  }
}

// Pass 2: s_ij = P_ij sqrt(max(a_i - 2 w_i . V_j + c_j, 0)).  One CTA per (b*h, 8 rows);
// lane = key within a 32-key tile staged in shared memory.
__global__ void __launch_bounds__(kThreads) drift_kernel(
    const float *__restrict__ P, const float *__restrict__ vp, const float *__restrict__ w,
    const float *__restrict__ a, const float *__restrict__ c, float *__restrict__ s, int nb) {
  __shared__ float sw[kWarps][kHeadDim];
  __shared__ float sv[32][kPad];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const long long bh = blockIdx.y;
  const int i = blockIdx.x * kWarps + warp;
  const bool live = i < nb;
  if (live) {
    sw[warp][lane] = w[((size_t)bh * nb + i) * kHeadDim + lane];
    sw[warp][lane + 32] = w[((size_t)bh * nb + i) * kHeadDim + lane + 32];
  }
  const float ai = live ? a[(size_t)bh * nb + i] : 0.f;
  const float *vh = vp + (size_t)bh * nb * kHeadDim;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    __syncthreads();
    for (int idx = t; idx < 32 * kHeadDim; idx += kThreads) {
      int jj = idx / kHeadDim, cc = idx % kHeadDim;
      sv[jj][cc] = (j0 + jj < nb) ? vh[(size_t)(j0 + jj) * kHeadDim + cc] : 0.f;
    }
    __syncthreads();
    const int j = j0 + lane;
    if (live && j < nb) {
      float dot = 0.f;
#pragma unroll 16
      for (int e = 0; e < kHeadDim; ++e) dot = fmaf(sw[warp][e], sv[lane][e], dot);
      const float q = (ai - 2.f * dot) + c[(size_t)bh * nb + j];
      const size_t o = ((size_t)bh * nb + i) * nb + j;
      s[o] = P[o] * sqrtf(fmaxf(q, 0.f));
    }
  }
}

}  // namespace

cudaError_t launch_head_gram(int H, int d_model, const float *w_o, float *gram, cudaStream_t st) {
  head_gram_kernel<<<H, kThreads, 0, st>>>(w_o, gram, H, d_model);
  return cudaGetLastError();
}

cudaError_t launch_pool(const Dims &d, const void *q, const void *k, const void *v, float *qp,
                        float *kp, float *vp, cudaStream_t st) {
  const long long units = 3 * d.BH() * d.nb;
  long long blocks = (units + kWarps - 1) / kWarps;
  if (blocks > 148 * 64) blocks = 148 * 64;
  pool_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(
      static_cast<const uint4 *>(q), static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
      qp, kp, vp, d.BH(), d.N, d.nb);
  return cudaGetLastError();
}

template <int TQ>
static cudaError_t scores_tq(const Dims &d, const float *qp, const float *kp, const float *vp,
                             float scale, float *P, float *vbar, cudaStream_t st) {
  const size_t smem = sizeof(float) * (TQ * kHeadDim + 32 * kPad + (size_t)TQ * d.nb);
  cudaError_t e = cudaFuncSetAttribute(block_scores_kernel<TQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.nb + TQ - 1) / TQ, (unsigned)d.BH());
  block_scores_kernel<TQ><<<grid, kThreads, smem, st>>>(qp, kp, vp, scale, P, vbar, d.nb);
  return cudaGetLastError();
}

cudaError_t launch_block_scores(const Dims &d, const float *qp, const float *kp, const float *vp,
                                float scale, float *P, float *vbar, cudaStream_t st) {
  // 16 rows per CTA while their logits fit comfortably in shared memory, else 8.
  if ((size_t)16 * d.nb * sizeof(float) <= 160 * 1024)
    return scores_tq<16>(d, qp, kp, vp, scale, P, vbar, st);
  return scores_tq<8>(d, qp, kp, vp, scale, P, vbar, st);
}

size_t drift_workspace_bytes(const Dims &d) {
  const size_t n = (size_t)d.BH() * d.nb;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return up(n * kHeadDim * sizeof(float)) + up(n * sizeof(float)) * 2;
}

cudaError_t launch_drift(const Dims &d, const float *P, const float *vp, const float *vbar,
                         const float *gram, float *s, void *ws, cudaStream_t st) {
  const size_t n = (size_t)d.BH() * d.nb;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char *base = static_cast<char *>(ws);
  float *w = reinterpret_cast<float *>(base);
  float *a = reinterpret_cast<float *>(base + up(n * kHeadDim * sizeof(float)));
  float *c = reinterpret_cast<float *>(base + up(n * kHeadDim * sizeof(float)) + up(n * sizeof(float)));
  dim3 g1((d.nb + 31) / 32, (unsigned)d.BH(), 2);
  drift_prep_kernel<<<g1, kThreads, 0, st>>>(vp, vbar, gram, w, a, c, d.H, d.nb);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2((d.nb + kWarps - 1) / kWarps, (unsigned)d.BH());
  drift_kernel<<<g2, kThreads, 0, st>>>(P, vp, w, a, c, s, d.nb);
  return cudaGetLastError();
}

}  // namespace ress

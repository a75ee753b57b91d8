// Block-level kernels: head Gram matrices, mean pooling, pooled block map, drift score.
//
// [ReSS] = "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers".
// All of these are small next to the attention itself; pooling is bound by HBM reads of
// Q/K/V, the block map and drift score by fp32 FMA on L2-resident pooled tensors.
#include <cuda_bf16.h>

#include "k_tiles.cuh"
#include "k_topk.cuh"
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
// One CTA of two warps per (tensor, b*h, block); warp w reads the w-th half of the
// block's tokens.  Lane = (token slot ts = lane/8, 16-byte column group cg = lane%8): a
// warp-wide load covers 4 consecutive token rows (512 contiguous bytes), and each lane
// issues all 16 of its loads before it adds any, so a warp keeps 8 KB in flight and a
// 128-token block is read by two warps at once.  Within a warp the tokens are added in
// order; the two halves' sums meet in shared memory and are added (first half + second).
constexpr int kPoolWarps = 2;
__global__ void __launch_bounds__(kPoolWarps * 32) pool_kernel(const uint4 *__restrict__ q,
                                                               const uint4 *__restrict__ k,
                                                               const uint4 *__restrict__ v,
                                                               float *__restrict__ qp,
                                                               float *__restrict__ kp,
                                                               float *__restrict__ vp, long long BH,
                                                               int N, int nq, int nk, int kb) {
  __shared__ float part[8][8];  // second half's column sums: [cg][8 columns]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cg = lane & 7, ts = lane >> 3;
  // queries are pooled over nq blocks of 128 tokens, keys and values over nk blocks of kb
  const long long q_units = BH * nq, k_units = BH * nk;
  const long long units = q_units + 2 * k_units;
  for (long long u = blockIdx.x; u < units; u += gridDim.x) {
    int which, nbw, bw;
    long long rem;
    if (u < q_units) {
      which = 0, rem = u, nbw = nq, bw = kBlock;
    } else {
      const long long r2 = u - q_units;
      which = 1 + (int)(r2 / k_units);
      rem = r2 - (which - 1) * k_units, nbw = nk, bw = kb;
    }
    const long long bh = rem / nbw;
    const int j = (int)(rem - bh * nbw);
    const uint4 *src = (which == 0 ? q : which == 1 ? k : v) + (size_t)bh * N * 8;
    float *dst = (which == 0 ? qp : which == 1 ? kp : vp) + ((size_t)bh * nbw + j) * kHeadDim;
    const int t0 = j * bw, t1 = min(N, t0 + bw);
    const int h0 = t0 + warp * (bw / 2), h1 = min(t1, h0 + bw / 2);  // this warp's half
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
    uint4 w[16];
#pragma unroll
    for (int it = 0; it < 16; ++it) {
      const int tok = h0 + ts + 4 * it;
      w[it] = tok < h1 ? __ldg(src + (size_t)tok * 8 + cg) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int it = 0; it < 16; ++it) {
      const uint32_t ww[4] = {w[it].x, w[it].y, w[it].z, w[it].w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[2 * c] += __uint_as_float(ww[c] << 16);
        acc[2 * c + 1] += __uint_as_float(ww[c] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 8);
      acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 16);
    }
    if (warp == 1 && ts == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c) part[cg][c] = acc[c];
    }
    __syncthreads();
    if (warp == 0 && ts == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += part[cg][c];
      const float cnt = (float)(t1 - t0);
      float4 lo = make_float4(__fdiv_rn(acc[0], cnt), __fdiv_rn(acc[1], cnt),
                              __fdiv_rn(acc[2], cnt), __fdiv_rn(acc[3], cnt));
      float4 hi = make_float4(__fdiv_rn(acc[4], cnt), __fdiv_rn(acc[5], cnt),
                              __fdiv_rn(acc[6], cnt), __fdiv_rn(acc[7], cnt));
      reinterpret_cast<float4 *>(dst)[2 * cg] = lo;
      reinterpret_cast<float4 *>(dst)[2 * cg + 1] = hi;
    }
    __syncthreads();  // part[] is free for the next unit
  }
}

// ----------------------------------- special tokens to the tail, [ReSS] Supp. F sink rule
// One warp moves four token rows (8 lanes x 16 bytes each) per step, grid-stride over
// the B*H*N rows.  Row r of a head maps to row perm(r) (forward) or perm^-1(r).
__global__ void __launch_bounds__(kThreads) token_gather_kernel(const uint4 *__restrict__ src,
                                                                uint4 *__restrict__ dst,
                                                                long long rows, int N, int T,
                                                                int S, int V, int inverse) {
  const int lane = threadIdx.x & 31, sub = lane >> 3, cg = lane & 7;
  const int Pv = T - S;
  const long long warps = (long long)gridDim.x * kWarps;
  for (long long base = ((long long)blockIdx.x * kWarps + (threadIdx.x >> 5)) * 4; base < rows;
       base += warps * 4) {
    const long long r = base + sub;
    if (r >= rows) continue;
    const long long head = r / N;
    const int t = (int)(r - head * N);  // token index within the head, view order
    const int v = t / T, w = t - v * T;
    const int tail = w < S ? V * Pv + v * S + w : v * Pv + (w - S);  // its place at the tail layout
    const long long from = head * N + (inverse ? tail : t);
    const long long to = head * N + (inverse ? t : tail);
    dst[to * 8 + cg] = src[from * 8 + cg];
  }
}

// ---------------------------------------- pooled block map and Eq. 1 output, [ReSS] §4.1
// One CTA per (b*h, TQ query blocks); warp w owns rows w*R .. w*R+R-1 (R = TQ/8).  The
// logits of the CTA's rows against every key block stay in shared memory ([TQ][nb]
// floats); the head's pooled keys, then values, stream through two shared-memory tiles
// of 64 blocks (cp.async double buffering), so each is read once per CTA.
//
// With SEL, the same kernel also selects: each warp takes the top-c of its rows'
// probabilities (mass) or SplitMix64 keys (random) straight from shared memory and writes
// the kept list, so P need not go to memory and back (the fused per-row selection; the
// drift method keeps its separate kernels).  P and vbar are then optional outputs.
struct FusedSelect {
  int method, H;
  float top_p;
  uint64_t seed;
  const uint8_t *keep_k, *dense_q;
  int32_t *kv_idx, *kv_cnt;
  uint8_t *mask;
  int budgets[kMaxHeads];
};
constexpr uint8_t kCand = 0, kFixed = 1, kKept = 2;  // per-block state during selection

// per-warp selection scratch: histogram, gather slots, block states, and for the CDF
// method the kept probabilities in rank order
__host__ __device__ __forceinline__ size_t fused_warp_bytes(int nb, bool cdf) {
  return 1024 + 128 + (size_t)((nb + 15) & ~15) + (cdf ? (size_t)((nb + 3) & ~3) * 4 : 0);
}

template <int TQ, bool SEL>
__global__ void __launch_bounds__(kThreads) block_scores_kernel(
    const float *__restrict__ qp, const float *__restrict__ kp, const float *__restrict__ vp,
    float scale, float *__restrict__ P, float *__restrict__ vbar, int nq, int nk,
    const __grid_constant__ FusedSelect fs) {
  constexpr int R = TQ / kWarps;
  extern __shared__ __align__(16) float sm[];
  float *tiles = sm;                      // 2 x [64][68]
  float *sq = tiles + 2 * kTileFloats;    // [TQ][64]
  float *sl = sq + TQ * kHeadDim;         // [TQ][nb] logits, then probabilities
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * TQ;
  const float *qh = qp + (size_t)bh * nq * kHeadDim;
  for (int idx = t; idx < TQ * kHeadDim; idx += kThreads) {
    const int r = idx / kHeadDim;
    sq[idx] = (i0 + r < nq) ? qh[(size_t)(i0 + r) * kHeadDim + idx % kHeadDim] : 0.f;
  }
  // logits: thread t takes a 4-row x (TQ/2)-block micro-tile (row group rg, block group
  // kg) of each 64-block tile over 8 of the 64 dimensions (slice ds: 4ds..4ds+3 and
  // 32+4ds..32+4ds+3), with its rows' pooled-query slices in registers; the 8 slices of
  // a micro-tile sit on 8 consecutive lanes and a transposing butterfly (xor 4, 2, 1)
  // sums them, leaving lane ds the TQ/4 logits of row ds/2, blocks (TQ/4)(ds%2) + i.
  {
    constexpr int KPM = TQ / 2, NV = TQ / 4, NRG = TQ / 4;
    const int ds = t & 7, mt = t >> 3;  // 32 micro-tiles
    const int rg = mt % NRG, kg = mt / NRG;
    __syncthreads();  // pooled queries staged
    float4 qv[4][2];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 *qr = reinterpret_cast<const float4 *>(sq + (rg * 4 + r) * kHeadDim);
      qv[r][0] = qr[ds];
      qv[r][1] = qr[8 + ds];
    }
    const bool b2 = ds & 4, b1 = ds & 2, b0 = ds & 1;
    float *lrow = sl + (rg * 4 + (ds >> 1)) * nk;
    const int jq = kg * KPM + NV * (ds & 1);
    tile_stream(tiles, kp + (size_t)bh * nk * kHeadDim, nk, [&](int tt, const float *tile) {
      float acc[4 * KPM];
#pragma unroll
      for (int kk = 0; kk < KPM; ++kk) {
        const float4 *vk = reinterpret_cast<const float4 *>(tile + (kg * KPM + kk) * kTilePad);
        const float4 a = vk[ds], b = vk[8 + ds];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 x = qv[r][0], y = qv[r][1];
          float d = a.x * x.x;
          d = fmaf(a.y, x.y, d); d = fmaf(a.z, x.z, d); d = fmaf(a.w, x.w, d);
          d = fmaf(b.x, y.x, d); d = fmaf(b.y, y.y, d); d = fmaf(b.z, y.z, d); d = fmaf(b.w, y.w, d);
          acc[r * KPM + kk] = d;
        }
      }
#pragma unroll
      for (int i = 0; i < 2 * KPM; ++i) {
        const float send = b2 ? acc[i] : acc[2 * KPM + i], keep = b2 ? acc[2 * KPM + i] : acc[i];
        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
#pragma unroll
      for (int i = 0; i < KPM; ++i) {
        const float send = b1 ? acc[i] : acc[KPM + i], keep = b1 ? acc[KPM + i] : acc[i];
        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const float send = b0 ? acc[i] : acc[NV + i], keep = b0 ? acc[NV + i] : acc[i];
        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
      }
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int j = tt * kTileKeys + jq + i;
        if (j < nk) lrow[j] = acc[i] * scale;
      }
    });
  }
  // softmax over every key block, per row
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const int r = warp * R + q, i = i0 + r;
    if (i >= nq) continue;
    float *row = sl + r * nk;
    float m = -INFINITY;
    for (int j = lane; j < nk; j += 32) m = fmaxf(m, row[j]);
    m = warp_max(m);
    float sum = 0.f;
    for (int j = lane; j < nk; j += 32) {
      const float e = expf(row[j] - m);
      row[j] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    float *prow = P ? P + ((size_t)bh * nq + i) * nk : nullptr;
    for (int j = lane; j < nk; j += 32) {
      const float pj = __fdiv_rn(row[j], sum);
      row[j] = pj;
      if (prow) prow[j] = pj;
    }
  }
  if constexpr (SEL) {
    // ------------------------------------------------ fused mass / random selection
    // the same decisions as the selection kernel: top-c of the candidates by P (or by
    // the SplitMix64 key), ties to the lower block index; dense rows keep every block
    const bool cdf = fs.method == RESS_SELECT_CDF;
    unsigned char *wb = reinterpret_cast<unsigned char *>(sl + (size_t)TQ * nk) +
                        fused_warp_bytes(nk, cdf) * warp;
    uint32_t *hist = reinterpret_cast<uint32_t *>(wb);
    int *slot = reinterpret_cast<int *>(wb + 1024);
    uint8_t *st = wb + 1152;
    float *sorted = reinterpret_cast<float *>(st + ((nk + 15) & ~15));
    const int h = (int)(bh % fs.H);
#pragma unroll 1
    for (int q = 0; q < R; ++q) {
      const int r = warp * R + q, i = i0 + r;
      if (i >= nq) continue;
      const float *row = sl + r * nk;
      const bool dense = fs.dense_q != nullptr && fs.dense_q[i] != 0;
      int n_cand = 0;
      for (int j = lane; j < nk; j += 32) {
        const bool fixed = fs.keep_k != nullptr && fs.keep_k[j] != 0;
        st[j] = fixed ? kFixed : kCand;
        n_cand += fixed ? 0 : 1;
      }
      n_cand = warp_sum_i(n_cand);
      __syncwarp();
      const int c = min(fs.budgets[h], n_cand);
      if (!dense) {
        auto is_cand = [&](int j) { return st[j] == kCand; };
        auto keep = [&](int j) { st[j] = kKept; };
        if (fs.method == RESS_SELECT_MASS || cdf) {
          warp_select<uint32_t>(nk, c, [&](int j) { return float_key(row[j]); }, is_cand, keep, hist, slot);
          if (cdf) {
            double fixed = 0.0;  // mass of the always-kept blocks
            for (int j = lane; j < nk; j += 32)
              if (st[j] == kFixed) fixed += (double)row[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) fixed += __shfl_xor_sync(0xffffffffu, fixed, o);
            warp_cdf_cut(nk, row, [&](int j) { return st[j] == kKept; }, [&](int j) { st[j] = kCand; },
                         fixed, fs.top_p, sorted);
          }
        } else {
          const uint64_t base = ((uint64_t)bh * nq + (uint64_t)i) * (uint64_t)nk;
          warp_select<uint64_t>(nk, c, [&](int j) { return splitmix64_key(fs.seed, base + (uint64_t)j + 1); },
                               is_cand, keep, hist, slot);
        }
      }
      int32_t *out = fs.kv_idx + ((size_t)bh * nq + i) * nk;
      uint8_t *mrow = fs.mask ? fs.mask + ((size_t)bh * nq + i) * nk : nullptr;
      int total = 0;
      for (int base = 0; base < nk; base += 32) {
        const int j = base + lane;
        const bool k = j < nk && (dense || st[j] != kCand);
        const unsigned bal = __ballot_sync(0xffffffffu, k);
        if (k) out[total + __popc(bal & lanemask_lt())] = j;
        if (mrow && j < nk) mrow[j] = k ? 1 : 0;
        total += __popc(bal);
      }
      if (lane == 0) fs.kv_cnt[(size_t)bh * nq + i] = total;
      __syncwarp();
    }
    if (vbar == nullptr) return;
  }
  // vbar_i = sum_j P_ij V_j.  Warp w takes blocks w, w + 8, ... of each tile for all TQ
  // rows (lane: value dimensions lane and lane + 32), so that one read of a pooled-value
  // row serves every row of the CTA; the eight warps' partial sums then meet in shared
  // memory (the tile buffers, free once the walk is over) and are added in warp order.
  float a0[TQ], a1[TQ];
#pragma unroll
  for (int q = 0; q < TQ; ++q) a0[q] = a1[q] = 0.f;
  tile_stream(tiles, vp + (size_t)bh * nk * kHeadDim, nk, [&](int tt, const float *tile) {
    const int jn = min(kTileKeys, nk - tt * kTileKeys);
    // the tile's blocks warp, warp + 8, ... (at most 8), unrolled so that their loads overlap
#pragma unroll
    for (int it = 0; it < kTileKeys / kWarps; ++it) {
      const int kk = warp + kWarps * it;
      if (kk >= jn) break;
      const float x0 = tile[kk * kTilePad + lane], x1 = tile[kk * kTilePad + lane + 32];
      const float *pc = sl + tt * kTileKeys + kk;
#pragma unroll
      for (int q = 0; q < TQ; ++q) {
        const float pj = pc[q * nk];
        a0[q] = fmaf(pj, x0, a0[q]);
        a1[q] = fmaf(pj, x1, a1[q]);
      }
    }
  });
  float *part = tiles;  // [kWarps][TQ][64], within the two tile buffers
  static_assert(kWarps * TQ * kHeadDim <= 2 * kTileFloats, "partials fit in the tile buffers");
#pragma unroll
  for (int q = 0; q < TQ; ++q) {
    part[(warp * TQ + q) * kHeadDim + lane] = a0[q];
    part[(warp * TQ + q) * kHeadDim + lane + 32] = a1[q];
  }
  __syncthreads();
  for (int idx = t; idx < TQ * kHeadDim; idx += kThreads) {
    const int q = idx / kHeadDim, i = i0 + q;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += part[w * TQ * kHeadDim + idx];
    if (i < nq) vbar[((size_t)bh * nq + i) * kHeadDim + idx % kHeadDim] = v;
  }
}

// ------------------------------------------------------- drift score, [ReSS] Eqs. 5-9
// Pass 1: for every pooled vector x of a head (the rows vbar_i and the keys V_j),
// y = M_h x and x . y.  Stores w_i = M vbar_i, a_i = vbar_i^T M vbar_i and
// c_j = V_j^T M V_j in the workspace.
__global__ void __launch_bounds__(kThreads) drift_prep_kernel(
    const float *__restrict__ vp, const float *__restrict__ vbar, const float *__restrict__ gram,
    float *__restrict__ w, float *__restrict__ a, float *__restrict__ c, int H, int nq, int nk,
    int zbase) {
  __shared__ float sM[kHeadDim][kPad];
  __shared__ float sx[kWarps][kHeadDim];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const long long bh = blockIdx.y;
  const int h = (int)(bh % H);
  const bool rows = blockIdx.z + zbase == 0;  // 0: vbar rows -> w, a;  1: pooled keys -> c
  for (int idx = t; idx < kHeadDim * kHeadDim; idx += kThreads)
    sM[idx / kHeadDim][idx % kHeadDim] = gram[(size_t)h * kHeadDim * kHeadDim + idx];
  __syncthreads();
  const int cnt = rows ? nq : nk;  // vbar has nq rows, the pooled values nk
  const float *src = (rows ? vbar : vp) + (size_t)bh * cnt * kHeadDim;
  const int n_end = min(cnt, (int)blockIdx.x * 32 + 32);
  int n = blockIdx.x * 32 + warp;
  // this warp's rows n, n + 8, ...: the next row's two values are loaded before the
  // current row's product, so that the load latency overlaps it
  float x0 = n < n_end ? src[(size_t)n * kHeadDim + lane] : 0.f;
  float x1 = n < n_end ? src[(size_t)n * kHeadDim + lane + 32] : 0.f;
  for (; n < n_end; n += kWarps) {
    sx[warp][lane] = x0;
    sx[warp][lane + 32] = x1;
    __syncwarp();
    if (n + kWarps < n_end) {
      x0 = src[(size_t)(n + kWarps) * kHeadDim + lane];
      x1 = src[(size_t)(n + kWarps) * kHeadDim + lane + 32];
    }
    float y0 = 0.f, y1 = 0.f;
#pragma unroll 16
    for (int e = 0; e < kHeadDim; ++e) {
      const float xe = sx[warp][e];
      y0 = fmaf(sM[lane][e], xe, y0);
      y1 = fmaf(sM[lane + 32][e], xe, y1);
    }
    const float dot = warp_sum(quad_lane(sx[warp][lane], y0, sx[warp][lane + 32], y1));
    if (rows) {
      w[((size_t)bh * nq + n) * kHeadDim + lane] = y0;
      w[((size_t)bh * nq + n) * kHeadDim + lane + 32] = y1;
      if (lane == 0) a[(size_t)bh * nq + n] = dot;
    } else if (lane == 0) {
      c[(size_t)bh * nk + n] = dot;
    }
    __syncwarp();
  }
}

// Pass 2: s_ij = P_ij sqrt(max(a_i - 2 w_i . V_j + c_j, 0)).  One CTA per (b*h, 16 rows);
// the head's pooled values stream through shared memory in tiles of 64 blocks.  Thread
// t takes a 4-row x 8-block micro-tile of each tile over 8 of the 64 dimensions (slice
// ds: 4ds..4ds+3 and 32+4ds..32+4ds+3), with its rows' w slices in registers; the 8
// slices of a micro-tile sit on 8 consecutive lanes and a transposing butterfly (xor 4,
// 2, 1) sums them, leaving lane ds the inner products of row ds/2 with blocks
// 4(ds%2) .. 4(ds%2)+3, whose scores it writes.
constexpr int kDriftRows = 16;
__global__ void __launch_bounds__(kThreads) drift_kernel(
    const float *__restrict__ P, const float *__restrict__ vp, const float *__restrict__ w,
    const float *__restrict__ a, const float *__restrict__ c, float *__restrict__ s, int nq, int nk) {
  constexpr int KPM = 8, NV = 4, NRG = kDriftRows / 4;
  static_assert(NRG * (kTileKeys / KPM) * 8 == kThreads, "one micro-tile slice per thread");
  __shared__ __align__(16) float tiles[2 * kTileFloats];
  __shared__ __align__(16) float sw[kDriftRows][kHeadDim];
  const int t = threadIdx.x;
  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * kDriftRows;
  for (int idx = t; idx < kDriftRows * kHeadDim; idx += kThreads) {
    const int r = idx / kHeadDim;
    sw[r][idx % kHeadDim] = (i0 + r < nq) ? w[((size_t)bh * nq + i0 + r) * kHeadDim + idx % kHeadDim] : 0.f;
  }
  const int ds = t & 7, mt = t >> 3;
  const int rg = mt % NRG, kg = mt / NRG;
  __syncthreads();  // w rows staged
  float4 wv[4][2];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float4 *wr = reinterpret_cast<const float4 *>(&sw[rg * 4 + r][0]);
    wv[r][0] = wr[ds];
    wv[r][1] = wr[8 + ds];
  }
  const int ie = i0 + rg * 4 + (ds >> 1);  // the row whose scores this lane writes
  const float ae = ie < nq ? a[(size_t)bh * nq + ie] : 0.f;
  const size_t orow = ((size_t)bh * nq + (ie < nq ? ie : 0)) * nk;
  const int jq = kg * KPM + NV * (ds & 1);
  const float *ch = c + (size_t)bh * nk;
  const bool b2 = ds & 4, b1 = ds & 2, b0 = ds & 1;
  // P and c of this lane's NV blocks, fetched one tile ahead
  float pn[NV], cn[NV];
  auto fetch = [&](int tt) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int j = tt * kTileKeys + jq + i;
      const bool ok = ie < nq && j < nk;
      pn[i] = ok ? P[orow + j] : 0.f;
      cn[i] = ok ? ch[j] : 0.f;
    }
  };
  fetch(0);
  tile_stream(tiles, vp + (size_t)bh * nk * kHeadDim, nk, [&](int tt, const float *tile) {
    float pc[NV], cc[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      pc[i] = pn[i];
      cc[i] = cn[i];
    }
    fetch(tt + 1);
    float acc[4 * KPM];
#pragma unroll
    for (int kk = 0; kk < KPM; ++kk) {
      const float4 *vk = reinterpret_cast<const float4 *>(tile + (kg * KPM + kk) * kTilePad);
      const float4 x = vk[ds], y = vk[8 + ds];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 u = wv[r][0], v = wv[r][1];
        float d = u.x * x.x;
        d = fmaf(u.y, x.y, d); d = fmaf(u.z, x.z, d); d = fmaf(u.w, x.w, d);
        d = fmaf(v.x, y.x, d); d = fmaf(v.y, y.y, d); d = fmaf(v.z, y.z, d); d = fmaf(v.w, y.w, d);
        acc[r * KPM + kk] = d;
      }
    }
#pragma unroll
    for (int i = 0; i < 2 * KPM; ++i) {
      const float send = b2 ? acc[i] : acc[2 * KPM + i], keep = b2 ? acc[2 * KPM + i] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int i = 0; i < KPM; ++i) {
      const float send = b1 ? acc[i] : acc[KPM + i], keep = b1 ? acc[KPM + i] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float send = b0 ? acc[i] : acc[NV + i], keep = b0 ? acc[NV + i] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
    if (ie < nq) {
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int j = tt * kTileKeys + jq + i;
        if (j < nk) s[orow + j] = drift_score(pc[i], ae, acc[i], cc[i]);
      }
    }
  });
}

}  // namespace

cudaError_t launch_head_gram(int H, int d_model, const float *w_o, float *gram, cudaStream_t st) {
  head_gram_kernel<<<H, kThreads, 0, st>>>(w_o, gram, H, d_model);
  return cudaGetLastError();
}

cudaError_t launch_token_gather(const Dims &d, int views, int specials, bool inverse,
                                const void *src, void *dst, cudaStream_t st) {
  const long long rows = d.BH() * d.N;
  long long blocks = (rows + 4 * kWarps - 1) / (4 * kWarps);
  if (blocks > 148 * 32) blocks = 148 * 32;
  token_gather_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(
      static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), rows, d.N, d.N / views, specials,
      views, inverse ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_pool(const Dims &d, const void *q, const void *k, const void *v, float *qp,
                        float *kp, float *vp, cudaStream_t st) {
  const long long units = d.BH() * d.nq + 2 * d.BH() * d.nk;  // one CTA per unit
  long long blocks = units;
  if (blocks > 148 * 256) blocks = 148 * 256;
  pool_kernel<<<(unsigned)blocks, kPoolWarps * 32, 0, st>>>(
      static_cast<const uint4 *>(q), static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
      qp, kp, vp, d.BH(), d.N, d.nq, d.nk, d.kb);
  return cudaGetLastError();
}

template <int TQ, bool SEL>
static cudaError_t scores_tq(const Dims &d, const float *qp, const float *kp, const float *vp,
                             float scale, float *P, float *vbar, const FusedSelect &fs,
                             cudaStream_t st) {
  const size_t smem = sizeof(float) * (2 * kTileFloats + TQ * kHeadDim + (size_t)TQ * d.nk) +
                      (SEL ? fused_warp_bytes(d.nk, fs.method == RESS_SELECT_CDF) * kWarps : 0);
  cudaError_t e = cudaFuncSetAttribute(block_scores_kernel<TQ, SEL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.nq + TQ - 1) / TQ, (unsigned)d.BH());
  block_scores_kernel<TQ, SEL><<<grid, kThreads, smem, st>>>(qp, kp, vp, scale, P, vbar, d.nq, d.nk, fs);
  return cudaGetLastError();
}

template <bool SEL>
static cudaError_t scores_any(const Dims &d, const float *qp, const float *kp, const float *vp,
                              float scale, float *P, float *vbar, const FusedSelect &fs,
                              cudaStream_t st) {
  // 16 rows per CTA while their logits fit comfortably in shared memory and the grid
  // still gives every SM two CTAs (296 on a 148-SM B200), else 8.
  const long long ctas16 = (long long)((d.nq + 15) / 16) * d.BH();
  if ((size_t)16 * d.nk * sizeof(float) <= 150 * 1024 && ctas16 >= 2 * 148)
    return scores_tq<16, SEL>(d, qp, kp, vp, scale, P, vbar, fs, st);
  return scores_tq<8, SEL>(d, qp, kp, vp, scale, P, vbar, fs, st);
}

cudaError_t launch_block_scores(const Dims &d, const float *qp, const float *kp, const float *vp,
                                float scale, float *P, float *vbar, cudaStream_t st) {
  FusedSelect fs{};
  return scores_any<false>(d, qp, kp, vp, scale, P, vbar, fs, st);
}

cudaError_t launch_scores_select(const Dims &d, const ScoresSelectLaunch &a, cudaStream_t st) {
  FusedSelect fs{};
  fs.method = a.method;
  fs.top_p = a.top_p;
  fs.H = d.H;
  fs.seed = a.seed;
  fs.keep_k = a.keep_k;
  fs.dense_q = a.dense_q;
  fs.kv_idx = a.kv_idx;
  fs.kv_cnt = a.kv_cnt;
  fs.mask = a.mask;
  for (int h = 0; h < d.H; ++h) fs.budgets[h] = a.budgets[h];
  return scores_any<true>(d, a.qp, a.kp, a.vp, a.scale, a.P, a.vbar, fs, st);
}

// workspace: w [BH, nq, 64] | a [BH, nq] | c [BH, nk], each 256-byte aligned
size_t drift_workspace_bytes(const Dims &d) {
  const size_t nr = (size_t)d.BH() * d.nq, nc = (size_t)d.BH() * d.nk;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return up(nr * kHeadDim * sizeof(float)) + up(nr * sizeof(float)) + up(nc * sizeof(float));
}

size_t drift_select_workspace_bytes(const Dims &d) {
  return ((size_t)d.BH() * d.nk * sizeof(float) + 255) & ~(size_t)255;
}

cudaError_t launch_drift_cdiag(const Dims &d, const float *vp, const float *gram, float *c,
                               cudaStream_t st) {
  dim3 g((d.nk + 31) / 32, (unsigned)d.BH(), 1);
  drift_prep_kernel<<<g, kThreads, 0, st>>>(vp, vp, gram, nullptr, nullptr, c, d.H, d.nq, d.nk, 1);
  return cudaGetLastError();
}

cudaError_t launch_drift(const Dims &d, const float *P, const float *vp, const float *vbar,
                         const float *gram, float *s, void *ws, cudaStream_t st) {
  const size_t nr = (size_t)d.BH() * d.nq;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char *base = static_cast<char *>(ws);
  float *w = reinterpret_cast<float *>(base);
  float *a = reinterpret_cast<float *>(base + up(nr * kHeadDim * sizeof(float)));
  float *c = reinterpret_cast<float *>(base + up(nr * kHeadDim * sizeof(float)) + up(nr * sizeof(float)));
  dim3 g1((max(d.nq, d.nk) + 31) / 32, (unsigned)d.BH(), 2);
  drift_prep_kernel<<<g1, kThreads, 0, st>>>(vp, vbar, gram, w, a, c, d.H, d.nq, d.nk, 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2((d.nq + kDriftRows - 1) / kDriftRows, (unsigned)d.BH());
  drift_kernel<<<g2, kThreads, 0, st>>>(P, vp, w, a, c, s, d.nq, d.nk);
  return cudaGetLastError();
}

}  // namespace ress

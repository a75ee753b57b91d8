// Per-(query block, head) key-block selection and the attention launch order.
//
// [ReSS] = "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers".
// One warp owns one row (b, h, i); a CTA holds T rows of the same head so that the
// pooled value tiles streamed through shared memory during restoration serve T rows.
// Exact top-k is an MSB-first radix select on order-preserving integer keys (8-bit
// digits, a shared-memory histogram per warp), ties to the lower block index.
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {
namespace {

constexpr int kPad = 65;
constexpr uint8_t F_FIXED = 0;    // always-kept block (not a candidate)
constexpr uint8_t F_KEPT = 1;     // candidate, currently kept (S)
constexpr uint8_t F_DROP = 2;     // candidate, currently dropped (D)
constexpr uint8_t F_TO_KEEP = 3;  // chosen for restore this round
constexpr uint8_t F_TO_DROP = 4;  // chosen for drop this round
constexpr uint8_t F_CAND = 5;     // candidate before the initial selection

struct SelectParams {
  int H, nb, method, rounds;
  float rho, eps;
  uint64_t seed;
  const uint8_t *keep_k, *dense_q;
  const float *P, *s, *vp, *vbar, *gram;
  int32_t *kv_idx, *kv_cnt;
  uint8_t *mask;
  int32_t *dev_err;
  int rows_per_cta;
  int budgets[kMaxHeads];
};

RESS_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
RESS_DEV int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
RESS_DEV unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Marks the k valid entries with the largest key (ties: lower index) by calling
// mark(j).  Warp-collective.  hist: 256 words of this warp's shared memory.
template <typename KeyT, typename KeyFn, typename ValidFn, typename MarkFn>
RESS_DEV void warp_top_k(int n, int k, KeyFn key, ValidFn valid, MarkFn mark, uint32_t *hist) {
  const int lane = threadIdx.x & 31;
  int nvalid = 0;
  for (int j = lane; j < n; j += 32) nvalid += valid(j) ? 1 : 0;
  nvalid = warp_sum_i(nvalid);
  if (k <= 0) return;
  if (k >= nvalid) {
    for (int j = lane; j < n; j += 32)
      if (valid(j)) mark(j);
    __syncwarp();
    return;
  }
  constexpr int BITS = sizeof(KeyT) * 8;
  KeyT prefix = 0;
  uint32_t remaining = (uint32_t)k;
#pragma unroll 1
  for (int shift = BITS - 8; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    const KeyT hi_mask = (shift + 8 >= BITS) ? KeyT(0) : (~KeyT(0) << (shift + 8));
    for (int j = lane; j < n; j += 32) {
      if (valid(j)) {
        const KeyT kk = key(j);
        if ((kk & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist[(uint32_t)(kk >> shift) & 255u], 1u);
      }
    }
    __syncwarp();
    // lane l holds bins 255-8l .. 248-8l (highest digits first)
    uint32_t cnt[8], tot = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      cnt[q] = hist[255 - (lane * 8 + q)];
      tot += cnt[q];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - tot;
    const unsigned here = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
    const int src = __ffs(here) - 1;
    int digit = 0;
    uint32_t above = 0;
    if (lane == src) {
      uint32_t acc = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (acc + cnt[q] >= remaining) {
          digit = 255 - (lane * 8 + q);
          above = acc;
          break;
        }
        acc += cnt[q];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    remaining -= above;
    prefix |= KeyT(digit) << shift;
    __syncwarp();
  }
  // prefix is the k-th largest key; take every larger key and the first `remaining`
  // equal keys in ascending index order.
  uint32_t taken = 0;
  for (int base = 0; base < n; base += 32) {
    const int j = base + lane;
    const bool v = j < n && valid(j);
    const KeyT kk = v ? key(j) : KeyT(0);
    const bool gt = v && kk > prefix;
    const bool eq = v && kk == prefix;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    const uint32_t rank = __popc(beq & lanemask_lt()) + taken;
    if (gt || (eq && rank < remaining)) mark(j);
    taken += __popc(beq);
  }
  __syncwarp();
}

// Eq. 17 swap count: max(1, round-half-up(rho c 2^-(r+1))), capped at |D| and c.
RESS_DEV int swap_count(int r, int c, float rho, int n_drop) {
  const double x = (double)rho * (double)c * ldexp(1.0, -(r + 1));
  int m = (int)floor(x + 0.5);
  m = max(m, 1);
  return min(m, min(n_drop, c));
}

// Applies the chosen swaps to the net drift g (lane holds g[lane], g[lane+32]) and K
// (Eq. 13 for restores, its mirror for drops): restores in ascending block order, then
// drops; flags move to KEPT / DROP.
RESS_DEV void apply_swaps(uint8_t *flags, int nb, const float *prow, const float *vph,
                          float vb0, float vb1, float &g0, float &g1, float &K) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const uint8_t target = pass == 0 ? F_TO_KEEP : F_TO_DROP;
    for (int c0 = 0; c0 < nb; c0 += 32) {
      const int j = c0 + lane;
      unsigned bal = __ballot_sync(0xffffffffu, j < nb && flags[j] == target);
      while (bal) {
        int kk[4];
        int n = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          kk[q] = 0;
          if (bal) {
            kk[q] = c0 + __ffs(bal) - 1;
            bal &= bal - 1;
            ++n;
          }
        }
        float pk[4], x0[4], x1[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          pk[q] = q < n ? prow[kk[q]] : 0.f;
          x0[q] = q < n ? vph[(size_t)kk[q] * kHeadDim + lane] : 0.f;
          x1[q] = q < n ? vph[(size_t)kk[q] * kHeadDim + lane + 32] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q < n) {
            const float d0 = __fmul_rn(pk[q], __fsub_rn(vb0, x0[q]));
            const float d1 = __fmul_rn(pk[q], __fsub_rn(vb1, x1[q]));
            if (pass == 0) {
              g0 = __fsub_rn(g0, d0);
              g1 = __fsub_rn(g1, d1);
              K = __fadd_rn(K, pk[q]);
            } else {
              g0 = __fadd_rn(g0, d0);
              g1 = __fadd_rn(g1, d1);
              K = __fsub_rn(K, pk[q]);
            }
          }
        }
      }
      __syncwarp();
      if (j < nb && flags[j] == target) flags[j] = pass == 0 ? F_KEPT : F_DROP;
      __syncwarp();
    }
  }
}

// h = M g (lane computes h[lane], h[lane+32]); returns G = g . h.
RESS_DEV float gram_apply(const float (*sM)[kPad], float g0, float g1, float &h0, float &h1) {
  const int lane = threadIdx.x & 31;
  h0 = 0.f;
  h1 = 0.f;
#pragma unroll 8
  for (int e = 0; e < 32; ++e) {
    const float ge = __shfl_sync(0xffffffffu, g0, e);
    h0 = fmaf(sM[lane][e], ge, h0);
    h1 = fmaf(sM[lane + 32][e], ge, h1);
  }
#pragma unroll 8
  for (int e = 0; e < 32; ++e) {
    const float ge = __shfl_sync(0xffffffffu, g1, e);
    h0 = fmaf(sM[lane][e + 32], ge, h0);
    h1 = fmaf(sM[lane + 32][e + 32], ge, h1);
  }
  return warp_sum(g0 * h0 + g1 * h1);
}

RESS_DEV float objective(float G, float K, float eps) {
  const float Kg = fmaxf(K, eps);
  return __fdiv_rn(G, __fmul_rn(Kg, Kg));
}

__global__ void __launch_bounds__(256) select_kernel(const __grid_constant__ SelectParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int T = p.rows_per_cta, nb = p.nb;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthreads = blockDim.x;
  const bool drift = p.method == RESS_SELECT_DRIFT;
  const bool restore = drift && p.rounds > 0;
  // shared layout
  float(*sM)[kPad] = reinterpret_cast<float(*)[kPad]>(smem_raw);              // 64 x 65
  float(*sV)[kPad] = reinterpret_cast<float(*)[kPad]>(smem_raw + 64 * kPad * 4);  // 32 x 65
  unsigned char *wbase = smem_raw + 96 * kPad * 4;
  const size_t per_warp = 256 * 4 + 64 * 4 + (size_t)nb * 4 + 2 * (size_t)((nb + 15) & ~15);
  unsigned char *mine = wbase + per_warp * warp;
  uint32_t *hist = reinterpret_cast<uint32_t *>(mine);
  float *sh = reinterpret_cast<float *>(mine + 1024);
  float *gain = reinterpret_cast<float *>(mine + 1280);
  uint8_t *flags = mine + 1280 + (size_t)nb * 4;
  uint8_t *best = flags + ((nb + 15) & ~15);

  const long long bh = blockIdx.y;
  const int h = (int)(bh % p.H);
  const int i = blockIdx.x * T + warp;
  const bool row_live = i < nb;
  const bool dense = row_live && p.dense_q != nullptr && p.dense_q[i] != 0;
  const bool active = row_live && !dense;  // takes part in selection
  const float *prow = p.P + ((size_t)bh * nb + (row_live ? i : 0)) * nb;
  const float *srow = p.s ? p.s + ((size_t)bh * nb + (row_live ? i : 0)) * nb : nullptr;
  const float *vph = p.vp ? p.vp + (size_t)bh * nb * kHeadDim : nullptr;

  if (restore) {
    for (int idx = threadIdx.x; idx < 64 * 64; idx += nthreads)
      sM[idx / 64][idx % 64] = p.gram[(size_t)h * 4096 + idx];
  }
  // candidates
  int n_cand = 0;
  for (int j = lane; j < nb; j += 32) {
    const bool fixed = p.keep_k != nullptr && p.keep_k[j] != 0;
    flags[j] = fixed ? F_FIXED : F_CAND;
    n_cand += fixed ? 0 : 1;
  }
  n_cand = warp_sum_i(n_cand);
  __syncwarp();
  const int c = min(p.budgets[h], n_cand);

  if (active) {
    auto is_cand = [&](int j) { return flags[j] == F_CAND; };
    auto keep = [&](int j) { flags[j] = F_KEPT; };
    if (p.method == RESS_SELECT_MASS) {
      warp_top_k<uint32_t>(nb, c, [&](int j) { return float_key(prow[j]); }, is_cand, keep, hist);
    } else if (p.method == RESS_SELECT_RANDOM) {
      const uint64_t base = ((uint64_t)bh * nb + (uint64_t)i) * (uint64_t)nb;
      warp_top_k<uint64_t>(nb, c, [&](int j) { return splitmix64_key(p.seed, base + (uint64_t)j + 1); },
                           is_cand, keep, hist);
    } else {
      // Eq. 7 rank key, staged in `gain`
      for (int j = lane; j < nb; j += 32) {
        const float pj = prow[j];
        gain[j] = __fdiv_rn(srow[j], fmaxf(__fsub_rn(1.f, pj), p.eps));
      }
      __syncwarp();
      warp_top_k<uint32_t>(nb, c, [&](int j) { return float_key(gain[j]); }, is_cand, keep, hist);
    }
    for (int j = lane; j < nb; j += 32)
      if (flags[j] == F_CAND) flags[j] = F_DROP;
    __syncwarp();
  }

  if (restore) {
    const int n_drop = n_cand - c;
    const bool work = active && n_drop > 0 && c > 0;
    float vb0 = 0.f, vb1 = 0.f;
    if (active) {
      const float *vbr = p.vbar + ((size_t)bh * nb + i) * kHeadDim;
      vb0 = vbr[lane];
      vb1 = vbr[lane + 32];
    }
    // initial net drift g and kept mass K (Eq. 10), summed in ascending block order
    float g0 = 0.f, g1 = 0.f, Psum = 0.f;
    for (int j0 = 0; j0 < nb; j0 += 32) {
      __syncthreads();
      for (int idx = threadIdx.x; idx < 32 * 64; idx += nthreads) {
        const int jj = idx >> 6, cc = idx & 63;
        sV[jj][cc] = (j0 + jj < nb) ? vph[(size_t)(j0 + jj) * 64 + cc] : 0.f;
      }
      __syncthreads();
      if (work) {
        const int j = j0 + lane;
        const float pl = j < nb ? prow[j] : 0.f;
        const bool dl = j < nb && flags[j] == F_DROP;
        const unsigned bal = __ballot_sync(0xffffffffu, dl);
        const int jn = min(32, nb - j0);
        for (int jj = 0; jj < jn; ++jj) {
          const float pj = __shfl_sync(0xffffffffu, pl, jj);
          if (bal & (1u << jj)) {
            g0 = __fadd_rn(g0, __fmul_rn(pj, __fsub_rn(vb0, sV[jj][lane])));
            g1 = __fadd_rn(g1, __fmul_rn(pj, __fsub_rn(vb1, sV[jj][lane + 32])));
            Psum = __fadd_rn(Psum, pj);
          }
        }
      }
    }
    float K = __fsub_rn(1.f, Psum);
    float h0 = 0.f, h1 = 0.f;
    float G = work ? gram_apply(sM, g0, g1, h0, h1) : 0.f;
    float J = objective(G, K, p.eps);
    float bestJ = J;
    if (work) {
      for (int j = lane; j < nb; j += 32) best[j] = flags[j];
      __syncwarp();
    }
#pragma unroll 1
    for (int r = 0; r < p.rounds; ++r) {
      const int m = swap_count(r, c, p.rho, n_drop);
      float vh = 0.f, base = 0.f;
      if (work) {
        sh[lane] = h0;
        sh[lane + 32] = h1;
        vh = warp_sum(vb0 * h0 + vb1 * h1);
        const float Kh = fmaxf(K, p.eps);
        base = __fdiv_rn(G, __fmul_rn(Kh, Kh));
        __syncwarp();
      }
      // gains of every candidate from the start-of-round state (Eqs. 14-16)
      for (int j0 = 0; j0 < nb; j0 += 32) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < 32 * 64; idx += nthreads) {
          const int jj = idx >> 6, cc = idx & 63;
          sV[jj][cc] = (j0 + jj < nb) ? vph[(size_t)(j0 + jj) * 64 + cc] : 0.f;
        }
        __syncthreads();
        const int j = j0 + lane;
        if (work && j < nb) {
          const uint8_t f = flags[j];
          if (f == F_KEPT || f == F_DROP) {
            float dot = 0.f;
#pragma unroll 16
            for (int e = 0; e < 64; ++e) dot = fmaf(sV[lane][e], sh[e], dot);
            const float pj = prow[j];
            const float sj = srow[j];
            const float t = __fmul_rn(pj, __fsub_rn(vh, dot));  // d_j^T M g
            const float s2 = __fmul_rn(sj, sj);
            float dG, Kn;
            if (f == F_DROP) {  // restore j
              dG = __fadd_rn(__fmul_rn(-2.f, t), s2);
              Kn = fmaxf(__fadd_rn(K, pj), p.eps);
            } else {            // drop j
              dG = __fadd_rn(__fmul_rn(2.f, t), s2);
              Kn = fmaxf(__fsub_rn(K, pj), p.eps);
            }
            gain[j] = __fsub_rn(base, __fdiv_rn(__fadd_rn(G, dG), __fmul_rn(Kn, Kn)));
          }
        }
      }
      if (work) {
        __syncwarp();
        warp_top_k<uint32_t>(nb, m, [&](int j) { return float_key(gain[j]); },
                             [&](int j) { return flags[j] == F_DROP; },
                             [&](int j) { flags[j] = F_TO_KEEP; }, hist);
        warp_top_k<uint32_t>(nb, m, [&](int j) { return float_key(gain[j]); },
                             [&](int j) { return flags[j] == F_KEPT; },
                             [&](int j) { flags[j] = F_TO_DROP; }, hist);
        apply_swaps(flags, nb, prow, vph, vb0, vb1, g0, g1, K);
        G = gram_apply(sM, g0, g1, h0, h1);
        J = objective(G, K, p.eps);
        if (J < bestJ) {  // track-best
          bestJ = J;
          for (int j = lane; j < nb; j += 32) best[j] = flags[j];
          __syncwarp();
        }
      }
    }
    if (work) {
      for (int j = lane; j < nb; j += 32) flags[j] = best[j];
      __syncwarp();
    }
  }

  // outputs: ascending kept list, count, optional mask
  if (row_live) {
    int32_t *out = p.kv_idx + ((size_t)bh * nb + i) * nb;
    uint8_t *mrow = p.mask ? p.mask + ((size_t)bh * nb + i) * nb : nullptr;
    int total = 0;
    for (int base = 0; base < nb; base += 32) {
      const int j = base + lane;
      const bool k = j < nb && (dense || flags[j] == F_FIXED || flags[j] == F_KEPT);
      const unsigned bal = __ballot_sync(0xffffffffu, k);
      if (k) out[total + __popc(bal & lanemask_lt())] = j;
      if (mrow && j < nb) mrow[j] = k ? 1 : 0;
      total += __popc(bal);
    }
    if (lane == 0) p.kv_cnt[(size_t)bh * nb + i] = total;
  }
}

// Stable descending counting sort of work items by kv_cnt (one CTA).
__global__ void __launch_bounds__(1024) schedule_kernel(const int32_t *__restrict__ kv_cnt,
                                                        int32_t *__restrict__ order,
                                                        long long items, int nb) {
  extern __shared__ int bins[];  // nb + 1
  const int t = threadIdx.x, lane = t & 31;
  for (int b = t; b <= nb; b += blockDim.x) bins[b] = 0;
  __syncthreads();
  for (long long it = t; it < items; it += blockDim.x)
    atomicAdd(&bins[min(max(kv_cnt[it], 0), nb)], 1);
  __syncthreads();
  if (t < 32) {
    // start offset of count value c = items with a larger count
    int running = 0;
    for (int base = 0; base <= nb; base += 32) {
      const int idx = nb - (base + lane);
      const int v = idx >= 0 ? bins[idx] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (idx >= 0) bins[idx] = running + incl - v;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    for (long long base = 0; base < items; base += 32) {
      const long long it = base + lane;
      const int cv = it < items ? min(max(kv_cnt[it], 0), nb) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, cv);
      const int rank = __popc(peers & lanemask_lt());
      const int last = 31 - __clz(peers);
      int pos = 0;
      if (cv >= 0) pos = bins[cv] + rank;
      __syncwarp();
      if (cv >= 0) order[pos] = (int32_t)it;
      if (cv >= 0 && lane == last) bins[cv] += __popc(peers);
      __syncwarp();
    }
  }
}

}  // namespace

static size_t select_smem(int nb, int T) {
  const size_t per_warp = 256 * 4 + 64 * 4 + (size_t)nb * 4 + 2 * (size_t)((nb + 15) & ~15);
  return 96 * kPad * 4 + per_warp * T;
}

cudaError_t launch_select(const Dims &d, const SelectLaunch &a, cudaStream_t st) {
  SelectParams p{};
  p.H = d.H;
  p.nb = d.nb;
  p.method = a.method;
  p.rounds = a.rounds;
  p.rho = a.rho;
  p.eps = a.eps;
  p.seed = a.seed;
  p.keep_k = a.keep_k;
  p.dense_q = a.dense_q;
  p.P = a.P;
  p.s = a.s;
  p.vp = a.vp;
  p.vbar = a.vbar;
  p.gram = a.gram;
  p.kv_idx = a.kv_idx;
  p.kv_cnt = a.kv_cnt;
  p.mask = a.mask;
  p.dev_err = a.dev_err;
  for (int h = 0; h < d.H; ++h) p.budgets[h] = a.budgets[h];
  int T = 8;
  while (T > 1 && select_smem(d.nb, T) > 200 * 1024) --T;
  p.rows_per_cta = T;
  const size_t smem = select_smem(d.nb, T);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.nb + T - 1) / T, (unsigned)d.BH());
  select_kernel<<<grid, 32 * T, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const Dims &d, const int32_t *kv_cnt, int32_t *order, cudaStream_t st) {
  const size_t smem = sizeof(int) * (d.nb + 1);
  cudaError_t e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  schedule_kernel<<<1, 1024, smem, st>>>(kv_cnt, order, d.BH() * d.nb, d.nb);
  return cudaGetLastError();
}

}  // namespace ress

// Per-(query block, head) key-block selection and the attention launch order.
//
// [ReSS] = "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers".
// One warp owns one row (b, h, i).
//   select_kernel        attention mass, CDF threshold or random key; 4 rows per CTA.
//   drift_select_kernel  the drift method (Eq. 7 rank key, then the restoration rounds of
//                        Eqs. 10-17); a CTA holds 4, 8 or 16 rows of one head so that the
//                        pooled value tiles streamed through shared memory (cp.async, three
//                        tiles in flight) serve all of them, and each row keeps its P and s
//                        in tensor memory.  Its fused form also computes P, vbar and s.
// Exact top-k is an MSB-first radix select on order-preserving integer keys (8-bit
// digits, a shared-memory histogram per warp) that finishes by ranking once the
// threshold bucket holds at most 32 keys; ties go to the lower block index.  The
// restoration rounds' top-m (m <= 32) first keeps only the entries at or above the m-th
// largest of the 32 lanes' maxima and ranks them directly when at most 64 remain.
#include "k_tiles.cuh"
#include "k_topk.cuh"
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {
namespace {

constexpr int kPad = 65;
constexpr int kSelStages = 3;  // pooled-value tiles in flight during restoration
constexpr uint8_t F_FIXED = 0;    // always-kept block (not a candidate)
constexpr uint8_t F_KEPT = 1;     // candidate, currently kept (S)
constexpr uint8_t F_DROP = 2;     // candidate, currently dropped (D)
constexpr uint8_t F_TO_KEEP = 3;  // chosen for restore this round
constexpr uint8_t F_TO_DROP = 4;  // chosen for drop this round
constexpr uint8_t F_CAND = 5;     // candidate before the initial selection

struct SelectParams {
  int H, nb, nq, method;  // nb: key blocks per row (nk), nq: query blocks
  float top_p;            // RESS_SELECT_CDF threshold
  float *drift;           // realized J per row, or null
  float eps;
  uint64_t seed;
  const uint8_t *keep_k, *dense_q;
  const float *P, *vp, *vbar, *gram;
  int32_t *kv_idx, *kv_cnt;
  uint8_t *mask;
  int rows_per_cta;
  int budgets[kMaxHeads];
};

RESS_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
RESS_DEV int swap_count(int r, int c, float rho, int n_drop) {
  const double x = (double)rho * (double)c * ldexp(1.0, -(r + 1));
  int m = (int)floor(x + 0.5);
  m = max(m, 1);
  return min(m, min(n_drop, c));
}

// Adds sg * P_k (vbar - V_k) to the net drift g (lane holds dimensions lane and lane+32)
// and sk * P_k to ksum for the listed blocks k, in list order.  Rows are fetched eight
// at a time, and the next eight are requested before the current ones are summed, so
// that two batches of loads overlap the additions.
RESS_DEV void gather_drift(const int *list, int n, const float *prow, const float *vph,
                           float vb0, float vb1, float sg, float sk, float &g0, float &g1,
                           float &ksum) {
  const int lane = threadIdx.x & 31;
  float pk[8], x0[8], x1[8];
  auto load = [&](int q0, float (&p_)[8], float (&a_)[8], float (&b_)[8]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int kk = q0 + q < n ? list[q0 + q] : -1;
      p_[q] = kk >= 0 ? prow[kk] : 0.f;
      a_[q] = kk >= 0 ? vph[(size_t)kk * kHeadDim + lane] : 0.f;
      b_[q] = kk >= 0 ? vph[(size_t)kk * kHeadDim + lane + 32] : 0.f;
    }
  };
  if (n > 0) load(0, pk, x0, x1);
  for (int q0 = 0; q0 < n; q0 += 8) {
    float pn[8], y0[8], y1[8];
    if (q0 + 8 < n) load(q0 + 8, pn, y0, y1);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q0 + q < n) {
        g0 = __fadd_rn(g0, sg * __fmul_rn(pk[q], __fsub_rn(vb0, x0[q])));
        g1 = __fadd_rn(g1, sg * __fmul_rn(pk[q], __fsub_rn(vb1, x1[q])));
        ksum = __fadd_rn(ksum, sk * pk[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      pk[q] = pn[q];
      x0[q] = y0[q];
      x1[q] = y1[q];
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
  return warp_sum(quad_lane(g0, h0, g1, h1));
}

RESS_DEV float objective(float G, float K, float eps) {
  const float Kg = fmaxf(K, eps);
  return __fdiv_rn(G, __fmul_rn(Kg, Kg));
}

// Per-warp shared-memory block of the selection kernel: histogram, gather slots, M g,
// scalars, then the row's gain / key array (nb floats), the flag array (nb bytes) and
// the best drop set of the restoration rounds as a bitmask (bit j = block j kept).  The
// CDF method appends nb floats (the kept probabilities in rank order), the restoration
// rounds an nb-entry list of 16-bit block indices (the kept candidates, ascending).
// The stride is 16 bytes past a multiple of 128: every warp's block starts 16-byte
// aligned (float4 reads of M g), and the M g reads of eight different rows fall on
// distinct banks.
__host__ __device__ __forceinline__ size_t select_flags_bytes(int nb) { return ((size_t)nb + 15) & ~(size_t)15; }
__host__ __device__ __forceinline__ size_t select_best_bytes(int nb) {
  return ((((size_t)nb + 31) / 32) * 4 + 15) & ~(size_t)15;
}
__host__ __device__ __forceinline__ size_t select_warp_bytes(int nb, bool cdf, bool restore) {
  const size_t b = 1024 + 128 + 256 + 32 + (size_t)nb * 4 + select_flags_bytes(nb) +
                   select_best_bytes(nb) + (cdf ? (size_t)nb * 4 : 0) +
                   (restore ? ((2 * (size_t)nb + 15) & ~(size_t)15) : 0);
  return ((b + 127) & ~(size_t)127) + 16;
}

// Selection by attention mass, CDF threshold or random key (the drift method has its own
// kernel, drift_select_kernel below).  One warp per row; with params.drift the realized
// drift J of each row's selection is computed as well (Eqs. 10, 12).
__global__ void __launch_bounds__(512) select_kernel(const __grid_constant__ SelectParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int T = p.rows_per_cta, nb = p.nb, nq = p.nq;  // nb = key blocks (nk)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthreads = blockDim.x;
  const bool want_J = p.drift != nullptr;  // g, K and J are tracked
  // shared layout: [M 64 x 65] (J tracked), then per warp
  float(*sM)[kPad] = reinterpret_cast<float(*)[kPad]>(smem_raw);
  unsigned char *wbase = smem_raw + (want_J ? 64 * kPad * 4 : 0);
  const bool cdf = p.method == RESS_SELECT_CDF;
  const size_t wbytes = select_warp_bytes(nb, cdf, false);
  unsigned char *mine = wbase + wbytes * warp;
  uint32_t *hist = reinterpret_cast<uint32_t *>(mine);
  int *slot = reinterpret_cast<int *>(mine + 1024);
  float *gain = reinterpret_cast<float *>(mine + 1440);
  int *list = reinterpret_cast<int *>(gain);  // block lists reuse the key array
  uint8_t *flags = mine + 1440 + (size_t)nb * 4;
  uint32_t *bestw = reinterpret_cast<uint32_t *>(flags + select_flags_bytes(nb));
  float *sorted = reinterpret_cast<float *>(reinterpret_cast<unsigned char *>(bestw) +
                                            select_best_bytes(nb));  // CDF only

  const long long bh = blockIdx.y;
  const int h = (int)(bh % p.H);
  const int i = blockIdx.x * T + warp;
  const bool row_live = i < nq;
  const bool dense = row_live && p.dense_q != nullptr && p.dense_q[i] != 0;
  const bool active = row_live && !dense;  // takes part in selection
  const float *prow = p.P + ((size_t)bh * nq + (row_live ? i : 0)) * nb;
  const float *vph = p.vp ? p.vp + (size_t)bh * nb * kHeadDim : nullptr;

  if (want_J) {
    for (int idx = threadIdx.x; idx < 64 * 64; idx += nthreads)
      sM[idx / 64][idx % 64] = p.gram[(size_t)h * 4096 + idx];
    __syncthreads();
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
    if (p.method == RESS_SELECT_MASS || cdf) {
      for (int j = lane; j < nb; j += 32) gain[j] = prow[j];
      __syncwarp();
      warp_select<uint32_t>(nb, c, [&](int j) { return float_key(gain[j]); }, is_cand, keep, hist, slot);
      if (cdf) {
        double fixed = 0.0;  // mass of the always-kept blocks
        for (int j = lane; j < nb; j += 32)
          if (flags[j] == F_FIXED) fixed += (double)gain[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) fixed += __shfl_xor_sync(0xffffffffu, fixed, o);
        warp_cdf_cut(nb, gain, [&](int j) { return flags[j] == F_KEPT; },
                     [&](int j) { flags[j] = F_CAND; }, fixed, p.top_p, sorted);
      }
    } else {
      const uint64_t base = ((uint64_t)bh * nq + (uint64_t)i) * (uint64_t)nb;
      warp_select<uint64_t>(nb, c, [&](int j) { return splitmix64_key(p.seed, base + (uint64_t)j + 1); },
                           is_cand, keep, hist, slot);
    }
    for (int j = lane; j < nb; j += 32)
      if (flags[j] == F_CAND) flags[j] = F_DROP;
    __syncwarp();
  }

  // realized drift of the selection ([ReSS] §6.1): Eq. 12 on its drop set, with g and K
  // (Eq. 10) gathered over whichever of the drop set and the kept blocks is smaller (by
  // Eq. 1, sum_D P_j e_j = -sum_kept P_j e_j and K = sum_kept P_j); a dense query block
  // drops nothing
  if (want_J && row_live) {
    float J = 0.f;
    if (active) {
      const float *vbr = p.vbar + ((size_t)bh * nq + i) * kHeadDim;
      const float vb0 = vbr[lane], vb1 = vbr[lane + 32];
      const int n_drop = n_cand - c;
      const bool kept_form = (nb - n_drop) < n_drop;
      int n = 0;
      for (int c0 = 0; c0 < nb; c0 += 32) {
        const int j = c0 + lane;
        const bool sel = j < nb && (kept_form ? flags[j] != F_DROP : flags[j] == F_DROP);
        const unsigned bal = __ballot_sync(0xffffffffu, sel);
        if (sel) list[n + __popc(bal & lanemask_lt())] = j;
        n += __popc(bal);
      }
      __syncwarp();
      float g0 = 0.f, g1 = 0.f, Psum = 0.f;
      gather_drift(list, n, prow, vph, vb0, vb1, 1.f, 1.f, g0, g1, Psum);
      __syncwarp();
      if (kept_form) {
        g0 = -g0;
        g1 = -g1;
      }
      const float K = kept_form ? Psum : __fsub_rn(1.f, Psum);
      float h0, h1;
      const float G = gram_apply(sM, g0, g1, h0, h1);
      J = objective(G, K, p.eps);
    }
    if (lane == 0) p.drift[(size_t)bh * nq + i] = J;
  }

  // outputs: ascending kept list, count, optional mask
  if (row_live) {
    int32_t *out = p.kv_idx + ((size_t)bh * nq + i) * nb;
    uint8_t *mrow = p.mask ? p.mask + ((size_t)bh * nq + i) * nb : nullptr;
    int total = 0;
    for (int base = 0; base < nb; base += 32) {
      const int j = base + lane;
      const bool k = j < nb && (dense || flags[j] == F_FIXED || flags[j] == F_KEPT);
      const unsigned bal = __ballot_sync(0xffffffffu, k);
      if (k) out[total + __popc(bal & lanemask_lt())] = j;
      if (mrow && j < nb) mrow[j] = k ? 1 : 0;
      total += __popc(bal);
    }
    if (lane == 0) p.kv_cnt[(size_t)bh * nq + i] = total;
  }
}

// ------------------------------------------------------------------------------------
// Drift selection with the rows' P and s in tensor memory ([ReSS] §4.2-4.3, Eqs. 7, 10-17).
//
// One warp owns one row (b, h, i); a CTA holds T = 4, 8 or 16 rows of one head.  The rows'
// block maps P and drift scores s are read many times (the rank key, every restoration
// round's gains, the g / K gathers), so each row keeps them in tensor memory, which the
// selection does not otherwise use: the owner warp's lane quarter (lanes 32 (w % 4) ..),
// P at columns [2 tc r, 2 tc r + tc) and s at [2 tc r + tc, 2 (tc) (r + 1)) for the
// warp's slot r = w / 4, block j at lane j % 32 of column j / 32 (tc = columns per array,
// a multiple of 32).
//
// FUSED = false (ress_select_blocks): P and s come from memory, loaded once.
// FUSED = true (ress_drift_select, the fused per-row selection of [ReSS] §4.3 "Fused
// kernel implementation"): the kernel computes them itself from the pooled tensors --
// the logits against every pooled key (Eq. 1's softmax), vbar, w = M vbar, a = vbar^T M
// vbar and s (Eq. 9) -- with the same arithmetic, in the same order, as the separate
// block-map and drift kernels, so both paths select the same blocks bit for bit.  P and s
// never leave the SM unless the caller asks for them.
struct DriftSelectParams {
  int H, nb, nq, rounds, objective;  // nb: key blocks per row (nk), nq: query blocks
  float *drift;                      // realized J per row, or null
  float rho, eps;
  const uint8_t *keep_k, *dense_q;
  const float *P, *s, *vbar;         // unfused inputs
  const float *vp, *gram;
  const float *qp, *kp, *cdiag;      // fused inputs (cdiag = V_j^T M V_j, [B*H, nk])
  float scale;
  float *P_out, *s_out, *vbar_out;   // fused optional outputs
  int32_t *kv_idx, *kv_cnt;
  uint8_t *mask;
  int rows_per_cta, tcols;
  uint32_t tmem_cols;
  int budgets[kMaxHeads];
};

// Loads 16 consecutive tensor-memory columns of the warp's lane quarter; the values are
// usable once the wait has returned (the empty asm ties every value to the wait).
RESS_DEV void tmem_ld16_sync(uint32_t taddr, uint32_t (&r)[16]) {
  tmem_ld16(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < 16; ++q) asm volatile("" : "+r"(r[q]));
}

// P of listed blocks from the row's tensor-memory copy: block k sits at lane k % 32 of
// column k / 32; every lane receives the value.  kk < 0 gives 0.
template <int NB>
RESS_DEV void tmem_gather_p(uint32_t tP, const int (&kk)[NB], float (&out)[NB]) {
  uint32_t raw[NB];
#pragma unroll
  for (int q = 0; q < NB; ++q) raw[q] = tmem_ld1(tP + (uint32_t)(kk[q] >= 0 ? kk[q] >> 5 : 0));
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < NB; ++q) {
    asm volatile("" : "+r"(raw[q]));
    const float v = __shfl_sync(0xffffffffu, __uint_as_float(raw[q]), kk[q] >= 0 ? kk[q] & 31 : 0);
    out[q] = kk[q] >= 0 ? v : 0.f;
  }
}

// gather_drift with P from tensor memory: the same sums in the same order.  The pooled
// value rows of the next eight blocks are requested before the current eight are summed.
// Entries q < n_neg enter with the signs (sg_neg, sk_neg), the rest with (sg, sk).
RESS_DEV void gather_drift_t(const int *list, int n, int n_neg, uint32_t tP, const float *vph,
                             float vb0, float vb1, float sg_neg, float sk_neg, float sg, float sk,
                             float &g0, float &g1, float &ksum) {
  const int lane = threadIdx.x & 31;
  int kk[8];
  float x0[8], x1[8];
  auto load = [&](int q0, int (&k_)[8], float (&a_)[8], float (&b_)[8]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      k_[q] = q0 + q < n ? list[q0 + q] : -1;
      a_[q] = k_[q] >= 0 ? vph[(size_t)k_[q] * kHeadDim + lane] : 0.f;
      b_[q] = k_[q] >= 0 ? vph[(size_t)k_[q] * kHeadDim + lane + 32] : 0.f;
    }
  };
  if (n > 0) load(0, kk, x0, x1);
  for (int q0 = 0; q0 < n; q0 += 8) {
    int kn[8];
    float y0[8], y1[8];
    if (q0 + 8 < n) load(q0 + 8, kn, y0, y1);
    float pk[8];
    tmem_gather_p<8>(tP, kk, pk);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (kk[q] >= 0) {
        const bool neg = q0 + q < n_neg;
        const float a = neg ? sg_neg : sg, b = neg ? sk_neg : sk;
        g0 = __fadd_rn(g0, a * __fmul_rn(pk[q], __fsub_rn(vb0, x0[q])));
        g1 = __fadd_rn(g1, a * __fmul_rn(pk[q], __fsub_rn(vb1, x1[q])));
        ksum = __fadd_rn(ksum, b * pk[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      kk[q] = kn[q];
      x0[q] = y0[q];
      x1[q] = y1[q];
    }
  }
}

// Applies the chosen swaps to the net drift g and K (Eq. 13 for restores, its mirror for
// drops), restores in ascending block order, then drops, with P from tensor memory; flags
// move to KEPT / DROP.  The restores are found among the ascending list rlist (nr entries)
// when given, else by a scan of all nb blocks; the drops among the ascending kept list
// slist.  Both go into one list (this warp's shared memory, room for every block) and
// are gathered in one pass.
RESS_DEV void apply_swaps_t(uint8_t *flags, int nb, const uint16_t *rlist, int nr,
                            const uint16_t *slist, int ns, uint32_t tP, const float *vph, float vb0,
                            float vb1, float &g0, float &g1, float &K, int *list) {
  const int lane = threadIdx.x & 31;
  int n = 0, n_restore = 0;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const uint8_t target = pass == 0 ? F_TO_KEEP : F_TO_DROP;
    const int nscan = pass == 0 ? (rlist ? nr : nb) : ns;
    for (int c0 = 0; c0 < nscan; c0 += 32) {
      const int q = c0 + lane;
      const int j = q < nscan ? (pass == 0 ? (rlist ? (int)rlist[q] : q) : (int)slist[q]) : 0;
      const bool sel = q < nscan && flags[j] == target;
      const unsigned bal = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        list[n + __popc(bal & lanemask_lt())] = j;
        flags[j] = pass == 0 ? F_KEPT : F_DROP;
      }
      n += __popc(bal);
    }
    if (pass == 0) n_restore = n;
  }
  __syncwarp();
  // restore: g -= P_k e_k, K += P_k; drop: g += P_k e_k, K -= P_k
  gather_drift_t(list, n, n_restore, tP, vph, vb0, vb1, -1.f, 1.f, 1.f, -1.f, g0, g1, K);
  __syncwarp();
}

// Products of the CTA's rows with every pooled vector of one 64-block tile, the scheme of
// the restoration gain pass: thread t holds the 8-dimension slices (ds: 4ds..4ds+3 and
// 32+4ds..32+4ds+3) of 4 rows (row group rg) and multiplies them with 4 blocks (block
// group kg); a transposing butterfly (xor 4, 2, 1) over the 8 lanes of a micro-tile leaves
// lane ds the products of row rg*4 + ds/2 with blocks kg*4 + 2(ds%2) + {0, 1}.
// `rows` returns the float4 pointer to a row's 64 values.
struct RowTile {
  float4 v[4][2];
  int ds, rg, kg;
};
template <typename RowPtr>
RESS_DEV void row_tile_load(RowTile &rt, int T, RowPtr rows) {
  rt.ds = threadIdx.x & 7;
  const int mt = threadIdx.x >> 3, ngr = T >> 2;
  rt.rg = mt % ngr;
  rt.kg = mt / ngr;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float4 *x = rows(rt.rg * 4 + r);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    rt.v[r][0] = x ? x[rt.ds] : z;
    rt.v[r][1] = x ? x[8 + rt.ds] : z;
  }
}
RESS_DEV void row_tile_products(const RowTile &rt, const float *tile, float (&out)[2]) {
  float acc[16];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const float4 *vk = reinterpret_cast<const float4 *>(tile + (rt.kg * 4 + kk) * kTilePad);
    const float4 a = vk[rt.ds], b = vk[8 + rt.ds];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 x = rt.v[r][0], y = rt.v[r][1];
      float d = a.x * x.x;
      d = fmaf(a.y, x.y, d); d = fmaf(a.z, x.z, d); d = fmaf(a.w, x.w, d);
      d = fmaf(b.x, y.x, d); d = fmaf(b.y, y.y, d); d = fmaf(b.z, y.z, d); d = fmaf(b.w, y.w, d);
      acc[r * 4 + kk] = d;
    }
  }
  const bool b2 = rt.ds & 4, b1 = rt.ds & 2, b0 = rt.ds & 1;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float send = b2 ? acc[i] : acc[8 + i], keep = b2 ? acc[8 + i] : acc[i];
    acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b1 ? acc[i] : acc[4 + i], keep = b1 ? acc[4 + i] : acc[i];
    acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b0 ? acc[i] : acc[2 + i], keep = b0 ? acc[2 + i] : acc[i];
    acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
  out[0] = acc[0];
  out[1] = acc[1];
}

template <bool FUSED>
__global__ void __launch_bounds__(512) drift_select_kernel(const __grid_constant__ DriftSelectParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ uint32_t s_tmem;
  const int T = p.rows_per_cta, nb = p.nb, nq = p.nq;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthreads = blockDim.x;
  const bool restore = p.rounds > 0;
  const bool want_J = p.drift != nullptr;
  const bool maximise = p.objective != RESS_DRIFT_MINIMISE;
  const bool flip_init = p.objective == RESS_DRIFT_MAXIMISE_FULL;
  const bool stream = FUSED || restore;  // pooled tiles stream through shared memory
  const bool state = restore || want_J;   // g, K and J are tracked
  const size_t tile_bytes = stream ? (size_t)kSelStages * kTileFloats * 4 : 0;
  float *tiles = reinterpret_cast<float *>(smem_raw);
  float(*sM)[kPad] = reinterpret_cast<float(*)[kPad]>(smem_raw + tile_bytes);
  unsigned char *wbase = smem_raw + tile_bytes + 64 * kPad * 4;
  const size_t wbytes = select_warp_bytes(nb, false, restore);
  unsigned char *mine = wbase + wbytes * warp;
  uint32_t *hist = reinterpret_cast<uint32_t *>(mine);
  int *slot = reinterpret_cast<int *>(mine + 1024);
  float *sh = reinterpret_cast<float *>(mine + 1152);    // 64 floats: a row vector
  float *gain = reinterpret_cast<float *>(mine + 1440);  // per-block values of the row
  int *list = reinterpret_cast<int *>(gain);
  uint8_t *flags = mine + 1440 + (size_t)nb * 4;
  uint32_t *bestw = reinterpret_cast<uint32_t *>(flags + select_flags_bytes(nb));
  uint16_t *slist = reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(bestw) +
                                                 select_best_bytes(nb));
  auto warp_block = [&](int w) { return wbase + wbytes * w; };
  auto save_best = [&]() {
    for (int c0 = 0; c0 < nb; c0 += 32) {
      const int j = c0 + lane;
      const unsigned b = __ballot_sync(0xffffffffu, j < nb && flags[j] == F_KEPT);
      if (lane == 0) bestw[c0 >> 5] = b;
    }
    __syncwarp();
  };

  const long long bh = blockIdx.y;
  const int h = (int)(bh % p.H);
  const int i = blockIdx.x * T + warp;
  const bool row_live = i < nq;
  const bool dense = row_live && p.dense_q != nullptr && p.dense_q[i] != 0;
  const bool active = row_live && !dense;
  const float *vph = p.vp ? p.vp + (size_t)bh * nb * kHeadDim : nullptr;
  const int tc = p.tcols;
  const int cu = (nb + 31) >> 5;  // columns that hold blocks (the rest pad to 32-column chunks)

  if (warp == 0) {
    tmem_alloc(&s_tmem, p.tmem_cols);
    tmem_relinquish();
  }
  if (FUSED || state)
    for (int idx = threadIdx.x; idx < 64 * 64; idx += nthreads)
      sM[idx / 64][idx % 64] = p.gram[(size_t)h * 4096 + idx];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tP = s_tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(2 * tc * (warp >> 2));
  const uint32_t tS = tP + (uint32_t)tc;

  float vb0 = 0.f, vb1 = 0.f;  // vbar_i (lane: dimensions lane and lane + 32)
  if constexpr (FUSED) {
    // ---------------------------------------------- logits, the block map P ([ReSS] Eq. 1)
    if (row_live) {
      sh[lane] = p.qp[((size_t)bh * nq + i) * kHeadDim + lane];
      sh[lane + 32] = p.qp[((size_t)bh * nq + i) * kHeadDim + lane + 32];
    }
    __syncthreads();
    {
      RowTile rt;
      row_tile_load(rt, T, [&](int r) -> const float4 * {
        return blockIdx.x * T + r < nq ? reinterpret_cast<const float4 *>(warp_block(r) + 1152) : nullptr;
      });
      const int re = rt.rg * 4 + (rt.ds >> 1);
      float *elog = reinterpret_cast<float *>(warp_block(re) + 1440);
      const bool elive = blockIdx.x * T + re < nq;
      const int jq = rt.kg * 4 + 2 * (rt.ds & 1);
      tile_stream_n<kSelStages>(tiles, p.kp + (size_t)bh * nb * kHeadDim, nb, [&](int tt, const float *tile) {
        float u[2];
        row_tile_products(rt, tile, u);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int j = tt * kTileKeys + jq + q;
          if (elive && j < nb) elog[j] = u[q] * p.scale;
        }
      });
    }
    // softmax over every key block (the block-map kernel's reduction order)
    if (row_live) {
      float m = -INFINITY;
      for (int j = lane; j < nb; j += 32) m = fmaxf(m, gain[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sum = 0.f;
      for (int j = lane; j < nb; j += 32) {
        const float e = expf(gain[j] - m);
        gain[j] = e;
        sum += e;
      }
      sum = warp_sum(sum);
      float *prow = p.P_out ? p.P_out + ((size_t)bh * nq + i) * nb : nullptr;
      for (int j = lane; j < nb; j += 32) {
        const float pj = __fdiv_rn(gain[j], sum);
        gain[j] = pj;
        if (prow) prow[j] = pj;
      }
      __syncwarp();
      for (int c0 = 0; c0 < tc; c0 += 32) {
        uint32_t pv[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int j = lane + 32 * (c0 + q);
          pv[q] = __float_as_uint(j < nb ? gain[j] : 0.f);
        }
        tmem_st32(tP + c0, pv);
      }
      tmem_wait_st();
    }
    __syncthreads();  // every row's P in shared memory
    // ------------------------------------------- vbar_i = sum_j P_ij V_j ([ReSS] Eq. 1)
    // Eight partial sums per row, partial g over the blocks j = g (mod 8) in ascending
    // order, then added in order g = 0..7: the block-map kernel's order.  Warp w computes
    // partial g = w % 8 (T = 16, 8) of rows 8 (w / 8) .. (T = 16: two row halves), or
    // partials g = w and w + 4 of all 4 rows (T = 4).
    {
      constexpr int RB = 8;
      const int rbase = T == 16 ? 8 * (warp >> 3) : 0;
      const int nrows = T == 4 ? 4 : 8;
      const int g0 = T == 4 ? warp : warp & 7;
      const int ng = T == 4 ? 2 : 1;
      float a0[2][RB], a1[2][RB];
#pragma unroll
      for (int gq = 0; gq < 2; ++gq)
#pragma unroll
        for (int q = 0; q < RB; ++q) a0[gq][q] = a1[gq][q] = 0.f;
      tile_stream_n<kSelStages>(tiles, vph, nb, [&](int tt, const float *tile) {
        const int jn = min(kTileKeys, nb - tt * kTileKeys);
#pragma unroll
        for (int gq = 0; gq < 2; ++gq) {
          if (gq >= ng) break;
          const int g = g0 + 4 * gq;
          const float *prow0 = reinterpret_cast<const float *>(warp_block(rbase) + 1440) + tt * kTileKeys;
          const size_t rstride = wbytes / sizeof(float);
          // the tile's blocks g, g + 8, ... (at most 8), unrolled so that their loads overlap
#pragma unroll
          for (int it = 0; it < kTileKeys / 8; ++it) {
            const int kk = g + 8 * it;
            if (kk >= jn) break;
            const float x0 = tile[kk * kTilePad + lane], x1 = tile[kk * kTilePad + lane + 32];
#pragma unroll
            for (int q = 0; q < RB; ++q) {
              if (q >= nrows) break;
              const float pj = prow0[q * rstride + kk];
              a0[gq][q] = fmaf(pj, x0, a0[gq][q]);
              a1[gq][q] = fmaf(pj, x1, a1[gq][q]);
            }
          }
        }
      });
      float *part = tiles;  // [8][T][64]: within the tile buffers, free after the walk
#pragma unroll
      for (int gq = 0; gq < 2; ++gq) {
        if (gq >= ng) break;
        const int g = g0 + 4 * gq;
#pragma unroll
        for (int q = 0; q < RB; ++q) {
          if (q >= nrows) break;
          part[(g * T + rbase + q) * kHeadDim + lane] = a0[gq][q];
          part[(g * T + rbase + q) * kHeadDim + lane + 32] = a1[gq][q];
        }
      }
      __syncthreads();
      if (row_live) {
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          v0 += part[(g * T + warp) * kHeadDim + lane];
          v1 += part[(g * T + warp) * kHeadDim + lane + 32];
        }
        vb0 = v0;
        vb1 = v1;
        if (p.vbar_out) {
          p.vbar_out[((size_t)bh * nq + i) * kHeadDim + lane] = v0;
          p.vbar_out[((size_t)bh * nq + i) * kHeadDim + lane + 32] = v1;
        }
      }
      __syncthreads();  // partials read before the tile buffers are reused
    }
    // ---------------------- w = M vbar, a = vbar^T M vbar (the drift prep kernel's order)
    float a_row = 0.f;
    if (row_live) {
      sh[lane] = vb0;
      sh[lane + 32] = vb1;
      __syncwarp();
      float y0 = 0.f, y1 = 0.f;
#pragma unroll 16
      for (int e = 0; e < kHeadDim; ++e) {
        const float xe = sh[e];
        y0 = fmaf(sM[lane][e], xe, y0);
        y1 = fmaf(sM[lane + 32][e], xe, y1);
      }
      a_row = warp_sum(quad_lane(vb0, y0, vb1, y1));
      __syncwarp();
      sh[lane] = y0;  // w, for the products below
      sh[lane + 32] = y1;
    }
    __syncthreads();
    // ------------------------------ u_ij = w_i . V_j over every pooled value, then s (Eq. 9)
    {
      RowTile rt;
      row_tile_load(rt, T, [&](int r) -> const float4 * {
        return blockIdx.x * T + r < nq ? reinterpret_cast<const float4 *>(warp_block(r) + 1152) : nullptr;
      });
      const int re = rt.rg * 4 + (rt.ds >> 1);
      float *eu = reinterpret_cast<float *>(warp_block(re) + 1440);
      const bool elive = blockIdx.x * T + re < nq;
      const int jq = rt.kg * 4 + 2 * (rt.ds & 1);
      tile_stream_n<kSelStages>(tiles, vph, nb, [&](int tt, const float *tile) {
        float u[2];
        row_tile_products(rt, tile, u);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int j = tt * kTileKeys + jq + q;
          if (elive && j < nb) eu[j] = u[q];
        }
      });
    }
    if (row_live) {
      const float *ch = p.cdiag + (size_t)bh * nb;
      float *srow = p.s_out ? p.s_out + ((size_t)bh * nq + i) * nb : nullptr;
      for (int c0 = 0; c0 < cu; c0 += 16) {
        uint32_t pv[16], sv[16];
        float cj[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int j = lane + 32 * (c0 + q);
          cj[q] = c0 + q < cu && j < nb ? ch[j] : 0.f;
        }
        tmem_ld16_sync(tP + c0, pv);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int j = lane + 32 * (c0 + q);
          float sj = 0.f;
          if (c0 + q < cu && j < nb) {
            sj = drift_score(__uint_as_float(pv[q]), a_row, gain[j], cj[q]);
            if (srow) srow[j] = sj;
          }
          sv[q] = __float_as_uint(sj);
        }
        tmem_st16(tS + c0, sv);
      }
      tmem_wait_st();
    }
    __syncwarp();
  } else {
    // P and s rows from memory into tensor memory; vbar_i into registers
    if (row_live) {
      const float *prow = p.P + ((size_t)bh * nq + i) * nb;
      const float *srow = p.s + ((size_t)bh * nq + i) * nb;
      for (int c0 = 0; c0 < tc; c0 += 32) {
        uint32_t pv[32], sv[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int j = lane + 32 * (c0 + q);
          pv[q] = __float_as_uint(j < nb ? prow[j] : 0.f);
          sv[q] = __float_as_uint(j < nb ? srow[j] : 0.f);
        }
        tmem_st32(tP + c0, pv);
        tmem_st32(tS + c0, sv);
      }
      tmem_wait_st();
      if (state) {
        const float *vbr = p.vbar + ((size_t)bh * nq + i) * kHeadDim;
        vb0 = vbr[lane];
        vb1 = vbr[lane + 32];
      }
    }
  }

  // ---------------------------------------------------------------- candidates, Eq. 7
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
    // rank key s / max(1 - P, eps), negated for the "full" maximising control; the
    // top-c's first radix pass (histogram of the keys' top bytes) is taken on the way
    hist16_clear(hist);
    __syncwarp();
    for (int c0 = 0; c0 < cu; c0 += 16) {
      uint32_t pv[16], sv[16];
      tmem_ld16_sync(tP + c0, pv);
      tmem_ld16_sync(tS + c0, sv);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if (c0 + q >= cu) break;
        const int j = lane + 32 * (c0 + q);
        if (j < nb) {
          const float key = __fdiv_rn(__uint_as_float(sv[q]), fmaxf(__fsub_rn(1.f, __uint_as_float(pv[q])), p.eps));
          const float kf = flip_init ? -key : key;
          gain[j] = kf;
          if (flags[j] == F_CAND) hist16_add(hist, float_key(kf) >> 24);
        }
      }
    }
    __syncwarp();
    warp_top_k16(nb, c, n_cand, [&](int j) { return float_key(gain[j]); },
                 [&](int j) { return flags[j] == F_CAND; }, [&](int j) { flags[j] = F_KEPT; }, hist,
                 slot, true);
    for (int j = lane; j < nb; j += 32)
      if (flags[j] == F_CAND) flags[j] = F_DROP;
    __syncwarp();
  }

  // ------------------------------------------------ restoration rounds, Eqs. 10-17
  const int n_drop = n_cand - c;
  const bool work = restore && active && n_drop > 0 && c > 0;
  const bool gather = active && (work || want_J);
  float g0 = 0.f, g1 = 0.f, Psum = 0.f;
  bool kept_form = false;
  if (gather) {
    // Eq. 10 over whichever set is smaller (see select_kernel), ascending block order
    kept_form = (nb - n_drop) < n_drop;
    int n = 0;
    for (int c0 = 0; c0 < nb; c0 += 32) {
      const int j = c0 + lane;
      const bool sel = j < nb && (kept_form ? flags[j] != F_DROP : flags[j] == F_DROP);
      const unsigned bal = __ballot_sync(0xffffffffu, sel);
      if (sel) list[n + __popc(bal & lanemask_lt())] = j;
      n += __popc(bal);
    }
    __syncwarp();
    gather_drift_t(list, n, 0, tP, vph, vb0, vb1, 1.f, 1.f, 1.f, 1.f, g0, g1, Psum);
    __syncwarp();
    if (kept_form) {
      g0 = -g0;
      g1 = -g1;
    }
  }
  float K = kept_form ? Psum : __fsub_rn(1.f, Psum);
  float h0 = 0.f, h1 = 0.f;
  float G = gather ? gram_apply(sM, g0, g1, h0, h1) : 0.f;
  float J = objective(G, K, p.eps);
  float bestJ = J;
  if (work) save_best();
#pragma unroll 1
  for (int r = 0; r < p.rounds; ++r) {
    const int m = swap_count(r, c, p.rho, n_drop);
    if (work) {
      sh[lane] = h0;
      sh[lane + 32] = h1;
    }
    __syncthreads();  // every row's M g written
    // u_ij = V_j . (M g)_i for every block (CTA-wide, the restoration gain pass)
    {
      RowTile rt;
      row_tile_load(rt, T, [&](int rr) -> const float4 * {
        const bool live = blockIdx.x * T + rr < nq;
        return live ? reinterpret_cast<const float4 *>(warp_block(rr) + 1152) : nullptr;
      });
      const int re = rt.rg * 4 + (rt.ds >> 1);
      float *eu = reinterpret_cast<float *>(warp_block(re) + 1440);
      const bool elive = blockIdx.x * T + re < nq;
      const int jq = rt.kg * 4 + 2 * (rt.ds & 1);
      tile_stream_n<kSelStages>(tiles, vph, nb, [&](int tt, const float *tile) {
        float u[2];
        row_tile_products(rt, tile, u);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int j = tt * kTileKeys + jq + q;
          if (elive && j < nb) eu[j] = u[q];
        }
      });
    }
    if (work) {
      // gains of every candidate from the start-of-round state (Eqs. 14-16)
      const float vh = warp_sum(quad_lane(vb0, h0, vb1, h1));
      const float Kh = fmaxf(K, p.eps);
      const float base = __fdiv_rn(G, __fmul_rn(Kh, Kh));
      auto gkey = [&](int j) { return float_key(maximise ? -gain[j] : gain[j]); };
      // the gains, each lane's largest restore key (for the candidate bound below), and
      // the kept candidates S listed in ascending order for the drop side
      uint32_t lmax = 0u, lmax_s = 0u;  // largest restore / drop key of the lane
      int ns = 0;
      for (int c0 = 0; c0 < cu; c0 += 16) {
        uint32_t pv[16], sv[16];
        tmem_ld16_sync(tP + c0, pv);
        tmem_ld16_sync(tS + c0, sv);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          if (c0 + q >= cu) break;
          const int j = lane + 32 * (c0 + q);
          const uint8_t f = j < nb ? flags[j] : F_FIXED;
          if (f == F_KEPT || f == F_DROP) {
            const float pj = __uint_as_float(pv[q]), sj = __uint_as_float(sv[q]);
            const float t = __fmul_rn(pj, __fsub_rn(vh, gain[j]));  // d_j^T M g
            const float s2 = __fmul_rn(sj, sj);
            float dG, Kn;
            if (f == F_DROP) {  // restore j
              dG = __fadd_rn(__fmul_rn(-2.f, t), s2);
              Kn = fmaxf(__fadd_rn(K, pj), p.eps);
            } else {            // drop j
              dG = __fadd_rn(__fmul_rn(2.f, t), s2);
              Kn = fmaxf(__fsub_rn(K, pj), p.eps);
            }
            const float gj = __fsub_rn(base, __fdiv_rn(__fadd_rn(G, dG), __fmul_rn(Kn, Kn)));
            gain[j] = gj;
            const uint32_t kj = float_key(maximise ? -gj : gj);
            if (f == F_DROP) lmax = max(lmax, kj);
            else lmax_s = max(lmax_s, kj);
          }
          const bool sel = f == F_KEPT;
          const unsigned bal = __ballot_sync(0xffffffffu, sel);
          if (sel) slist[ns + __popc(bal & lanemask_lt())] = (uint16_t)j;
          ns += __popc(bal);
        }
      }
      __syncwarp();
      // Restores: the m largest keys of D.  With m <= 32, the m-th largest of the 32 lanes'
      // maxima is a lower bound theta of the m-th largest key (m different entries reach
      // it), so every entry of the answer has a key >= theta; those entries are listed in
      // ascending order, behind the kept list S (room for nb - ns >= |D| entries), and the
      // top-m is taken among them, with the same order and ties as over all of D (by a
      // direct rank when at most 64 are left).  Drops: the same over S, whose entries at
      // or above its bound go to `slot` when at most 64 of them are.
      auto mth_lane_max = [&](uint32_t v) {
        uint32_t rank = 0;
        for (int l = 0; l < 32; ++l) {
          const uint32_t o = __shfl_sync(0xffffffffu, v, l);
          rank += (o > v || (o == v && l < lane)) ? 1u : 0u;
        }
        const unsigned at = __ballot_sync(0xffffffffu, rank == (uint32_t)(m - 1));
        return __shfl_sync(0xffffffffu, v, __ffs(at) - 1);
      };
      uint16_t *cand = slist + ns;
      int ncand = -1;
      if (m <= 32) {
        const uint32_t theta = mth_lane_max(lmax);
        ncand = 0;
        for (int c0 = 0; c0 < nb; c0 += 32) {
          const int j = c0 + lane;
          const bool sel = j < nb && flags[j] == F_DROP && gkey(j) >= theta;
          const unsigned bal = __ballot_sync(0xffffffffu, sel);
          if (sel) cand[ncand + __popc(bal & lanemask_lt())] = (uint16_t)j;
          ncand += __popc(bal);
        }
        __syncwarp();
      }
      if (ncand >= 0 && ncand <= 64) {
        warp_top_k_small(ncand, m, [&](int q) { return gkey(cand[q]); },
                         [&](int q) { flags[cand[q]] = F_TO_KEEP; });
      } else if (ncand >= 0) {
        warp_top_k16(ncand, m, ncand, [&](int q) { return gkey(cand[q]); },
                     [&](int q) { return true; }, [&](int q) { flags[cand[q]] = F_TO_KEEP; },
                     hist, slot, false);
      } else {
        warp_top_k16(nb, m, n_drop, gkey, [&](int j) { return flags[j] == F_DROP; },
                     [&](int j) { flags[j] = F_TO_KEEP; }, hist, slot, false);
      }
      int nds = -1;
      uint16_t *dcand = reinterpret_cast<uint16_t *>(slot);  // 64 entries
      if (m <= 32) {
        const uint32_t theta = mth_lane_max(lmax_s);
        nds = 0;
        for (int c0 = 0; c0 < ns && nds <= 64; c0 += 32) {
          const int q = c0 + lane;
          const bool sel = q < ns && gkey(slist[q]) >= theta;
          const unsigned bal = __ballot_sync(0xffffffffu, sel);
          const int pos = nds + __popc(bal & lanemask_lt());
          if (sel && pos < 64) dcand[pos] = slist[q];
          nds += __popc(bal);
        }
        __syncwarp();
      }
      if (nds >= 0 && nds <= 64) {
        warp_top_k_small(nds, m, [&](int q) { return gkey(dcand[q]); },
                         [&](int q) { flags[dcand[q]] = F_TO_DROP; });
      } else {
        warp_top_k16(ns, m, ns, [&](int q) { return gkey(slist[q]); },
                     [&](int q) { return flags[slist[q]] == F_KEPT; },
                     [&](int q) { flags[slist[q]] = F_TO_DROP; }, hist, slot, false);
      }
      apply_swaps_t(flags, nb, ncand >= 0 ? cand : nullptr, ncand, slist, ns, tP, vph, vb0, vb1,
                    g0, g1, K, list);
      G = gram_apply(sM, g0, g1, h0, h1);
      J = objective(G, K, p.eps);
      if (maximise ? J > bestJ : J < bestJ) {  // track-best (track-worst when maximising)
        bestJ = J;
        save_best();
      }
    }
  }
  if (work) {
    for (int j = lane; j < nb; j += 32) {
      const uint8_t f = flags[j];
      if (f == F_KEPT || f == F_DROP) flags[j] = (bestw[j >> 5] >> (j & 31)) & 1u ? F_KEPT : F_DROP;
    }
    __syncwarp();
  }
  if (want_J && row_live && lane == 0)
    p.drift[(size_t)bh * nq + i] = active ? (work ? bestJ : J) : 0.f;

  // outputs: ascending kept list, count, optional mask
  if (row_live) {
    int32_t *out = p.kv_idx + ((size_t)bh * nq + i) * nb;
    uint8_t *mrow = p.mask ? p.mask + ((size_t)bh * nq + i) * nb : nullptr;
    int total = 0;
    for (int base = 0; base < nb; base += 32) {
      const int j = base + lane;
      const bool k = j < nb && (dense || flags[j] == F_FIXED || flags[j] == F_KEPT);
      const unsigned bal = __ballot_sync(0xffffffffu, k);
      if (k) out[total + __popc(bal & lanemask_lt())] = j;
      if (mrow && j < nb) mrow[j] = k ? 1 : 0;
      total += __popc(bal);
    }
    if (lane == 0) p.kv_cnt[(size_t)bh * nq + i] = total;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(s_tmem, p.tmem_cols);
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

// The same sort with the scatter spread over all 32 warps: warp w takes the contiguous
// items [w*chunk, (w+1)*chunk), counts them per count value, a scan over the warps gives
// each warp its first position per count value, and each warp then places its items in
// order.  Stable and deterministic like the single-warp version; needs 32 * (nb + 1)
// counters of shared memory.
__global__ void __launch_bounds__(1024) schedule_kernel_par(const int32_t *__restrict__ kv_cnt,
                                                            int32_t *__restrict__ order,
                                                            long long items, int nb) {
  extern __shared__ int wcnt[];  // [32][nb + 1]; row 32 of extra space: bucket starts
  int *start = wcnt + 32 * (nb + 1);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const long long chunk = (items + 31) / 32;
  const long long lo = warp * chunk, hi = min(items, lo + chunk);
  for (int i = t; i < 33 * (nb + 1); i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  int *mine = wcnt + warp * (nb + 1);
  for (long long base = lo; base < hi; base += 32) {
    const long long it = base + lane;
    const int cv = it < hi ? min(max(kv_cnt[it], 0), nb) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, cv);
    if (cv >= 0 && (peers & lanemask_lt()) == 0) mine[cv] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // bucket starts: count values largest first
  if (warp == 0) {
    int running = 0;
    for (int base = 0; base <= nb; base += 32) {
      const int c = nb - (base + lane);
      int v = 0;
      if (c >= 0)
        for (int w = 0; w < 32; ++w) v += wcnt[w * (nb + 1) + c];
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (c >= 0) start[c] = running + incl - v;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncthreads();
  // per warp: its first position for every count value (exclusive scan over the warps)
  for (int c = t; c <= nb; c += blockDim.x) {
    int pos = start[c];
    for (int w = 0; w < 32; ++w) {
      const int n = wcnt[w * (nb + 1) + c];
      wcnt[w * (nb + 1) + c] = pos;
      pos += n;
    }
  }
  __syncthreads();
  for (long long base = lo; base < hi; base += 32) {
    const long long it = base + lane;
    const int cv = it < hi ? min(max(kv_cnt[it], 0), nb) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, cv);
    const int rank = __popc(peers & lanemask_lt());
    if (cv >= 0) order[mine[cv] + rank] = (int32_t)it;
    __syncwarp();
    if (cv >= 0 && rank == 0) mine[cv] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace

static size_t select_smem(int nb, int T, bool state, bool cdf) {
  return (state ? 64 * kPad * 4 : 0) + select_warp_bytes(nb, cdf, false) * T;
}

static size_t drift_select_smem(int nb, int T, bool stream, bool restore) {
  return (stream ? (size_t)kSelStages * kTileFloats * 4 : 0) + 64 * kPad * 4 +
         select_warp_bytes(nb, false, restore) * T;
}
// Tensor-memory columns per array (P or s) of one row: one column per 32 blocks, in
// whole 32-column chunks.
static int drift_select_tcols(int nb) { return (((nb + 31) / 32) + 31) & ~31; }
static int drift_select_tmem_need(int nb, int T) { return ((T + 3) / 4) * 2 * drift_select_tcols(nb); }

// Rows per CTA, tensor-memory allocation and launch of the drift selection kernel.
static cudaError_t run_drift_select(const Dims &d, DriftSelectParams &p, bool fused, cudaStream_t st) {
  const bool restore = p.rounds > 0;
  const bool stream = fused || restore;
  int T = 16;
  while (T > 4 && (drift_select_smem(d.nk, T, stream, restore) > 220 * 1024 ||
                   drift_select_tmem_need(d.nk, T) > 512))
    T >>= 1;
  if (T == 16) {
    // 8 rows per CTA when two CTAs then fit on an SM (shared and tensor memory)
    int dev = 0, per_sm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) ==
            cudaSuccess &&
        2 * (drift_select_smem(d.nk, 8, stream, restore) + 1024) <= (size_t)per_sm &&
        drift_select_tmem_need(d.nk, 8) <= 256)
      T = 8;
  }
  const int need = drift_select_tmem_need(d.nk, T);
  if (need > 512) return cudaErrorNotSupported;
  uint32_t cols = 32;
  while ((int)cols < need) cols <<= 1;
  p.rows_per_cta = T;
  p.tcols = drift_select_tcols(d.nk);
  p.tmem_cols = cols;
  const size_t smem = drift_select_smem(d.nk, T, stream, restore);
  auto kern = fused ? drift_select_kernel<true> : drift_select_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.nq + T - 1) / T, (unsigned)d.BH());
  kern<<<grid, 32 * T, smem, st>>>(p);
  return cudaGetLastError();
}

static DriftSelectParams drift_params(const Dims &d, const SelectLaunch &a) {
  DriftSelectParams p{};
  p.H = d.H;
  p.nb = d.nk;
  p.nq = d.nq;
  p.rounds = a.rounds;
  p.objective = a.objective;
  p.drift = a.drift;
  p.rho = a.rho;
  p.eps = a.eps;
  p.keep_k = a.keep_k;
  p.dense_q = a.dense_q;
  p.P = a.P;
  p.s = a.s;
  p.vbar = a.vbar;
  p.vp = a.vp;
  p.gram = a.gram;
  p.kv_idx = a.kv_idx;
  p.kv_cnt = a.kv_cnt;
  p.mask = a.mask;
  for (int h = 0; h < d.H; ++h) p.budgets[h] = a.budgets[h];
  return p;
}

cudaError_t launch_drift_select(const Dims &d, const DriftSelectLaunch &a, cudaStream_t st) {
  float *cdiag = static_cast<float *>(a.ws);
  cudaError_t e = launch_drift_cdiag(d, a.sel.vp, a.sel.gram, cdiag, st);
  if (e != cudaSuccess) return e;
  DriftSelectParams p = drift_params(d, a.sel);
  p.qp = a.qp;
  p.kp = a.kp;
  p.cdiag = cdiag;
  p.scale = a.scale;
  p.P_out = a.P_out;
  p.s_out = a.s_out;
  p.vbar_out = a.vbar_out;
  return run_drift_select(d, p, true, st);
}

cudaError_t launch_select(const Dims &d, const SelectLaunch &a, cudaStream_t st) {
  if (a.method == RESS_SELECT_DRIFT) {
    DriftSelectParams p = drift_params(d, a);
    return run_drift_select(d, p, false, st);
  }
  SelectParams p{};
  p.H = d.H;
  p.nb = d.nk;
  p.nq = d.nq;
  p.method = a.method;
  p.eps = a.eps;
  p.seed = a.seed;
  p.top_p = a.top_p;
  p.drift = a.drift;
  p.keep_k = a.keep_k;
  p.dense_q = a.dense_q;
  p.P = a.P;
  p.vp = a.vp;
  p.vbar = a.vbar;
  p.gram = a.gram;
  p.kv_idx = a.kv_idx;
  p.kv_cnt = a.kv_cnt;
  p.mask = a.mask;
  for (int h = 0; h < d.H; ++h) p.budgets[h] = a.budgets[h];
  const bool state = a.drift != nullptr;
  const bool cdf = a.method == RESS_SELECT_CDF;
  // 4 rows per CTA: the rows are independent, and small CTAs fill the GPU at small nb
  int T = 4;
  p.rows_per_cta = T;
  const size_t smem = select_smem(d.nk, T, state, cdf);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.nq + T - 1) / T, (unsigned)d.BH());
  select_kernel<<<grid, 32 * T, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const Dims &d, const int32_t *kv_cnt, int32_t *order, cudaStream_t st) {
  const size_t par_smem = sizeof(int) * 33 * (size_t)(d.nk + 1);
  if (par_smem <= 200 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(schedule_kernel_par,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)par_smem);
    if (e != cudaSuccess) return e;
    schedule_kernel_par<<<1, 1024, par_smem, st>>>(kv_cnt, order, d.BH() * d.nq, d.nk);
    return cudaGetLastError();
  }
  const size_t smem = sizeof(int) * (d.nk + 1);
  cudaError_t e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  schedule_kernel<<<1, 1024, smem, st>>>(kv_cnt, order, d.BH() * d.nq, d.nk);
  return cudaGetLastError();
}

}  // namespace ress

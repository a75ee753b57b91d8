// Per-(query block, head) key-block selection and the attention launch order.
//
// [ReSS] = "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers".
// One warp owns one row (b, h, i); a CTA holds 4, 8 or 16 rows of the same head so that
// the pooled value tiles streamed through shared memory during restoration (cp.async,
// three tiles in flight) serve all of them.  Exact top-k is an MSB-first radix select on
// order-preserving integer keys (8-bit digits, a shared-memory histogram per warp) that
// finishes by ranking once the threshold bucket holds at most 32 keys; ties go to the
// lower block index.
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
  int H, nb, nq, method, rounds;  // nb: key blocks per row (nk), nq: query blocks
  int objective;  // ress_drift_objective
  float top_p;    // RESS_SELECT_CDF threshold
  float *drift;   // realized J per row, or null
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

// Applies the chosen swaps to the net drift g and K (Eq. 13 for restores, its mirror
// for drops): restores in ascending block order, then drops; flags move to KEPT / DROP.
// The chosen blocks are first listed in `list` (this warp's shared memory, room for
// every block).  Restores are found by a scan of all nb blocks, drops by a scan of the
// ascending list of kept candidates (slist, ns entries).
RESS_DEV void apply_swaps(uint8_t *flags, int nb, const uint16_t *slist, int ns,
                          const float *prow, const float *vph, float vb0, float vb1, float &g0,
                          float &g1, float &K, int *list) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const uint8_t target = pass == 0 ? F_TO_KEEP : F_TO_DROP;
    const int nscan = pass == 0 ? nb : ns;
    int n = 0;
    for (int c0 = 0; c0 < nscan; c0 += 32) {
      const int q = c0 + lane;
      const int j = q < nscan ? (pass == 0 ? q : (int)slist[q]) : 0;
      const bool sel = q < nscan && flags[j] == target;
      const unsigned bal = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        list[n + __popc(bal & lanemask_lt())] = j;
        flags[j] = pass == 0 ? F_KEPT : F_DROP;
      }
      n += __popc(bal);
    }
    __syncwarp();
    // restore: g -= P_k e_k, K += P_k; drop: g += P_k e_k, K -= P_k
    gather_drift(list, n, prow, vph, vb0, vb1, pass == 0 ? -1.f : 1.f, pass == 0 ? 1.f : -1.f,
                 g0, g1, K);
    __syncwarp();
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

__global__ void __launch_bounds__(512) select_kernel(const __grid_constant__ SelectParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int T = p.rows_per_cta, nb = p.nb, nq = p.nq;  // nb = key blocks (nk)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthreads = blockDim.x;
  const bool drift = p.method == RESS_SELECT_DRIFT;
  const bool restore = drift && p.rounds > 0;
  const bool want_J = p.drift != nullptr;
  const bool state = restore || want_J;  // g, K and J are tracked
  // maximising controls ([ReSS] Fig. 8): flip the rounds' gains, and for "full" the
  // initial rank key too
  const bool maximise = drift && p.objective != RESS_DRIFT_MINIMISE;
  const bool flip_init = drift && p.objective == RESS_DRIFT_MAXIMISE_FULL;
  // shared layout: [tiles kSelStages x 64 x 68] (restoration only), [M 64 x 65] (g, K, J
  // tracked), then per warp
  const size_t tile_bytes = restore ? (size_t)kSelStages * kTileFloats * 4 : 0;
  float *tiles = reinterpret_cast<float *>(smem_raw);
  float(*sM)[kPad] = reinterpret_cast<float(*)[kPad]>(smem_raw + tile_bytes);
  unsigned char *wbase = smem_raw + tile_bytes + (state ? 64 * kPad * 4 : 0);
  const bool cdf = p.method == RESS_SELECT_CDF;
  const size_t wbytes = select_warp_bytes(nb, cdf, restore);
  unsigned char *mine = wbase + wbytes * warp;
  uint32_t *hist = reinterpret_cast<uint32_t *>(mine);
  int *slot = reinterpret_cast<int *>(mine + 1024);
  float *sh = reinterpret_cast<float *>(mine + 1152);
  float *scal = reinterpret_cast<float *>(mine + 1408);  // vh, G/K^2, G, K; int flag at [4]
  float *gain = reinterpret_cast<float *>(mine + 1440);
  int *list = reinterpret_cast<int *>(gain);  // block lists reuse the gain array
  uint8_t *flags = mine + 1440 + (size_t)nb * 4;
  uint32_t *bestw = reinterpret_cast<uint32_t *>(flags + select_flags_bytes(nb));
  unsigned char *tail = reinterpret_cast<unsigned char *>(bestw) + select_best_bytes(nb);
  float *sorted = reinterpret_cast<float *>(tail);      // CDF only
  uint16_t *slist = reinterpret_cast<uint16_t *>(tail);  // restoration rounds only
  // the current selection as the best one (bit j of bestw = candidate block j kept)
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
  const bool active = row_live && !dense;  // takes part in selection
  const float *prow = p.P + ((size_t)bh * nq + (row_live ? i : 0)) * nb;
  const float *srow = p.s ? p.s + ((size_t)bh * nq + (row_live ? i : 0)) * nb : nullptr;
  const float *vph = p.vp ? p.vp + (size_t)bh * nb * kHeadDim : nullptr;

  if (state) {
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
    } else if (p.method == RESS_SELECT_RANDOM) {
      const uint64_t base = ((uint64_t)bh * nq + (uint64_t)i) * (uint64_t)nb;
      warp_select<uint64_t>(nb, c, [&](int j) { return splitmix64_key(p.seed, base + (uint64_t)j + 1); },
                           is_cand, keep, hist, slot);
    } else {
      // Eq. 7 rank key, staged in `gain` (negated for the "full" maximising control:
      // the c candidates with the smallest key are kept)
      for (int j = lane; j < nb; j += 32) {
        const float pj = prow[j];
        const float key = __fdiv_rn(srow[j], fmaxf(__fsub_rn(1.f, pj), p.eps));
        gain[j] = flip_init ? -key : key;
      }
      __syncwarp();
      warp_select<uint32_t>(nb, c, [&](int j) { return float_key(gain[j]); }, is_cand, keep, hist, slot);
    }
    for (int j = lane; j < nb; j += 32)
      if (flags[j] == F_CAND) flags[j] = F_DROP;
    __syncwarp();
  }

  if (state) {
    const int n_drop = n_cand - c;
    const bool work = restore && active && n_drop > 0 && c > 0;  // restoration rounds
    const bool gather = active && (work || want_J);              // initial g and K
    float vb0 = 0.f, vb1 = 0.f;
    if (active) {
      const float *vbr = p.vbar + ((size_t)bh * nq + i) * kHeadDim;
      vb0 = vbr[lane];
      vb1 = vbr[lane + 32];
    }
    // Initial net drift g and kept mass K (Eq. 10).  Gathered over whichever set is
    // smaller: the drop set D itself (g = sum_D P_j e_j, K = 1 - sum_D P_j), or the kept
    // blocks (always-kept and kept candidates): since vbar_i = sum over all j of P_ij V_j
    // (Eq. 1), sum_D P_j e_j = -sum_kept P_j e_j and K = sum_kept P_j.  Ascending block
    // order; rows are fetched eight at a time.
    float g0 = 0.f, g1 = 0.f, Psum = 0.f;
    bool kept_form = false;
    if (gather) {
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
      gather_drift(list, n, prow, vph, vb0, vb1, 1.f, 1.f, g0, g1, Psum);
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
        const float vh = warp_sum(vb0 * h0 + vb1 * h1);
        const float Kh = fmaxf(K, p.eps);
        if (lane == 0) {
          scal[0] = vh;
          scal[1] = __fdiv_rn(G, __fmul_rn(Kh, Kh));
          scal[2] = G;
          scal[3] = K;
          reinterpret_cast<int *>(scal)[4] = 1;
        }
      } else if (lane == 0) {
        reinterpret_cast<int *>(scal)[4] = 0;  // no restoration work in this row
      }
      __syncwarp();
      // Gains of every candidate from the start-of-round state (Eqs. 14-16), computed by
      // the whole CTA against 64-block tiles of the head's pooled values.  The d_j^T M g
      // inner products of a tile form a (rows x 64 blocks) product over 64 dimensions;
      // thread t takes a 4-row x 4-block micro-tile (row group rg, block group kg) over 8
      // of the dimensions (slice ds: 4ds..4ds+3 and 32+4ds..32+4ds+3).  Its rows' M g
      // slices stay in registers for the whole pass, so a tile costs each thread eight
      // 16-byte shared-memory reads for 128 FMAs.  The 8 slices of a micro-tile sit on 8
      // consecutive lanes; a transposing butterfly (xor 4, 2, 1) sums them and leaves lane
      // ds with the products of row ds/2 and blocks 2(ds%2), 2(ds%2)+1, whose gains it
      // writes.
      {
        const int ds = threadIdx.x & 7, mt = threadIdx.x >> 3;
        const int ngr = T >> 2;  // row groups of four (T = 4, 8 or 16)
        const int rg = mt % ngr, kg = mt / ngr;
        __syncthreads();  // every row's M g, scalars and flags of this round are written
        float4 hv[4][2];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const unsigned char *rb = wbase + wbytes * (rg * 4 + r);
          const bool live = reinterpret_cast<const int *>(rb + 1408)[4] == 1;
          const float4 *hh = reinterpret_cast<const float4 *>(rb + 1152);
          const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
          hv[r][0] = live ? hh[ds] : z;
          hv[r][1] = live ? hh[8 + ds] : z;
        }
        // the (row, block) pairs whose gains this lane writes
        const int re = rg * 4 + (ds >> 1);
        unsigned char *eb = wbase + wbytes * re;
        const float *es = reinterpret_cast<const float *>(eb + 1408);
        float *egain = reinterpret_cast<float *>(eb + 1440);
        const uint8_t *eflags = eb + 1440 + (size_t)nb * 4;
        const int ei = blockIdx.x * T + re;
        const bool ework = ei < nq && reinterpret_cast<const int *>(es)[4] == 1;
        const float *ep = p.P + ((size_t)bh * nq + (ework ? ei : 0)) * nb;
        const float *esr = p.s + ((size_t)bh * nq + (ework ? ei : 0)) * nb;
        const float vh = es[0], base = es[1], G = es[2], Kr = es[3];
        const int jq = kg * 4 + 2 * (ds & 1);  // first of the lane's two blocks in a tile
        // P and s of this lane's two blocks, fetched one tile ahead
        float pn[2], sn[2];
        auto fetch = [&](int tt) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int j = tt * kTileKeys + jq + q;
            const bool ok = ework && j < nb;
            pn[q] = ok ? ep[j] : 0.f;
            sn[q] = ok ? esr[j] : 0.f;
          }
        };
        fetch(0);
        const bool b2 = ds & 4, b1 = ds & 2, b0 = ds & 1;
        tile_stream_n<kSelStages>(tiles, vph, nb, [&](int tt, const float *tile) {
          const float pc[2] = {pn[0], pn[1]}, sc[2] = {sn[0], sn[1]};
          fetch(tt + 1);
          float acc[16];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const float4 *vk = reinterpret_cast<const float4 *>(tile + (kg * 4 + kk) * kTilePad);
            const float4 a = vk[ds], b = vk[8 + ds];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const float4 x = hv[r][0], y = hv[r][1];
              float d = a.x * x.x;
              d = fmaf(a.y, x.y, d); d = fmaf(a.z, x.z, d); d = fmaf(a.w, x.w, d);
              d = fmaf(b.x, y.x, d); d = fmaf(b.y, y.y, d); d = fmaf(b.z, y.z, d); d = fmaf(b.w, y.w, d);
              acc[r * 4 + kk] = d;
            }
          }
          // butterfly: after the xor-4 / xor-2 / xor-1 steps lane ds holds the sums of
          // products 2ds and 2ds + 1 (product index = 4 * row + block within the tile)
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
          if (!ework) return;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int j = tt * kTileKeys + jq + q;
            if (j >= nb) continue;
            const uint8_t f = eflags[j];
            if (f != F_KEPT && f != F_DROP) continue;
            const float pj = pc[q], sj = sc[q];
            const float t = __fmul_rn(pj, __fsub_rn(vh, acc[q]));  // d_j^T M g
            const float s2 = __fmul_rn(sj, sj);
            float dG, Kn;
            if (f == F_DROP) {  // restore j
              dG = __fadd_rn(__fmul_rn(-2.f, t), s2);
              Kn = fmaxf(__fadd_rn(Kr, pj), p.eps);
            } else {            // drop j
              dG = __fadd_rn(__fmul_rn(2.f, t), s2);
              Kn = fmaxf(__fsub_rn(Kr, pj), p.eps);
            }
            egain[j] = __fsub_rn(base, __fdiv_rn(__fadd_rn(G, dG), __fmul_rn(Kn, Kn)));
          }
        });
      }
      if (work) {
        __syncwarp();
        // the largest gains (J decreases), or for the maximising controls the largest
        // J increases
        auto gkey = [&](int j) { return float_key(maximise ? -gain[j] : gain[j]); };
        warp_select<uint32_t>(nb, m, gkey, [&](int j) { return flags[j] == F_DROP; },
                             [&](int j) { flags[j] = F_TO_KEEP; }, hist, slot);
        // the kept candidates S as an ascending list: the drop-side select and the drop
        // pass of apply_swaps walk |S| entries instead of nb
        int ns = 0;
        for (int c0 = 0; c0 < nb; c0 += 32) {
          const int j = c0 + lane;
          const bool sel = j < nb && flags[j] == F_KEPT;
          const unsigned bal = __ballot_sync(0xffffffffu, sel);
          if (sel) slist[ns + __popc(bal & lanemask_lt())] = (uint16_t)j;
          ns += __popc(bal);
        }
        __syncwarp();
        warp_select<uint32_t>(ns, m, [&](int q) { return gkey(slist[q]); },
                             [&](int q) { return flags[slist[q]] == F_KEPT; },
                             [&](int q) { flags[slist[q]] = F_TO_DROP; }, hist, slot);
        apply_swaps(flags, nb, slist, ns, prow, vph, vb0, vb1, g0, g1, K, list);
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
    // realized drift of the returned selection ([ReSS] §6.1): the tracked J after the
    // rounds, else the initial one; a dense query block drops nothing
    if (want_J && row_live && lane == 0)
      p.drift[(size_t)bh * nq + i] = active ? (work ? bestJ : J) : 0.f;
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

static size_t select_smem(int nb, int T, bool restore, bool state, bool cdf) {
  return (restore ? (size_t)kSelStages * kTileFloats * 4 : 0) + (state ? 64 * kPad * 4 : 0) +
         select_warp_bytes(nb, cdf, restore) * T;
}

cudaError_t launch_select(const Dims &d, const SelectLaunch &a, cudaStream_t st) {
  SelectParams p{};
  p.H = d.H;
  p.nb = d.nk;
  p.nq = d.nq;
  p.method = a.method;
  p.rounds = a.rounds;
  p.rho = a.rho;
  p.eps = a.eps;
  p.seed = a.seed;
  p.objective = a.objective;
  p.top_p = a.top_p;
  p.drift = a.drift;
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
  const bool restore = a.method == RESS_SELECT_DRIFT && a.rounds > 0;
  const bool state = restore || a.drift != nullptr;
  // rows per CTA: 4, 8 or 16 (the gain pass of the restoration rounds takes micro-tiles
  // of 4 rows); without rounds the rows are independent, and 4 per CTA give a grid that
  // fills the GPU at small nb
  int T = restore ? 16 : 4;
  const bool cdf = a.method == RESS_SELECT_CDF;
  while (T > 4 && select_smem(d.nk, T, restore, state, cdf) > 220 * 1024) T >>= 1;
  if (restore && T == 16) {
    // 8 rows per CTA when that fits two CTAs per SM (small nb): the same 16 warps per SM
    // in finer CTAs, whose barriers and last wave cost less (32 views: -6 %)
    int dev = 0, per_sm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) ==
            cudaSuccess &&
        2 * (select_smem(d.nk, 8, restore, state, cdf) + 1024) <= (size_t)per_sm)
      T = 8;
  }
  p.rows_per_cta = T;
  const size_t smem = select_smem(d.nk, T, restore, state, cdf);
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

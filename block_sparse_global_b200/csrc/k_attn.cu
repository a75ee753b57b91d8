// Block-sparse attention forward on the 5th-generation tensor cores (sm_100a).
//
// [ReSS] = "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers",
// §3 step (3): exact attention over the kept key blocks, softmax renormalised among
// them.  One CTA computes one (batch, head, query block) row of 128 queries against the
// key blocks listed in kv_idx; two CTAs share an SM.  Key blocks are 128 tokens (one
// block per 128 x 128 score tile) or 64 tokens, the grid of ReSS Supp. F: then kept
// blocks 2j and 2j+1 of a row fill the two 64-row halves of tile j, each through its own
// 64-row TMA box, and an odd count leaves the second half of the last tile zero (a box
// that starts past the last token) and masked.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t (tensor-memory lane t).  Reads the
//              S tile from tensor memory, online softmax in the exp2 domain, writes P
//              (bf16) back to tensor memory, rescales O when the running max grows by
//              more than a factor 2^8, and runs the epilogue (O / l -> bf16, LSE).
//   warp 4     TMA producer (one thread): Q once, then K_j of every kept block into a
//              three-slot ring and V_j into a two-slot ring; validates the row first.
//   warp 5     tensor-core issuer (one elected thread): S = Q K^T (M=128, N=128, K=64)
//              and O += P V (M=128, N=64, K=128, A operand read from tensor memory).
//              Also allocates and frees the 256 tensor-memory columns.
// Tensor memory: S columns [0,128), P [128,192) as packed bf16 pairs, O [192,256).  P of
// tile j goes in two halves: keys 0..63 as soon as the first four MMAs of O += P V of tile
// j-1 (which read those columns) are done, keys 64..127 after the whole product.
// Shared memory: Q 16 KB, K 3 x 16 KB, V 2 x 16 KB, all 128-byte swizzled by TMA.
//
// Exponentials: at head_dim 64 the MUFU unit (about 16-21 exp2 per clock per SM) is the
// scarcest resource of the softmax -- a 128 x 128 tile needs 16384 exp2 against roughly
// 700 clock cycles of tensor-core work.  Two of every eight column pairs therefore take
// exp2 on the FMA and integer pipes instead (range reduction plus a fitted polynomial,
// see exp2_pair_fma); the rest use MUFU ex2.approx.f32.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {
namespace {

constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
// lazy rescale: O and l are rescaled only when the row max grows by more than 2^this
constexpr float kRescaleLog2 = 8.0f;
constexpr int kKStages = 3;          // K tiles in flight (S = Q K^T consumes them first)
constexpr int kVStages = 2;          // V tiles in flight (O += P V consumes them later)
constexpr int kTile = 128 * 64 * 2;  // bytes of one 128 x 64 bf16 tile
constexpr int kOffQ = 0;
constexpr int kOffK = kTile;
constexpr int kOffV = kOffK + kKStages * kTile;
constexpr int kOffBar = kOffV + kVStages * kTile;
constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + barriers, alignment slack
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192;

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKStages];
  uint64_t k_empty[kKStages];
  uint64_t v_full[kVStages];
  uint64_t v_empty[kVStages];
  uint64_t s_full;
  uint64_t s_free;
  uint64_t p_full;
  uint64_t o_done;
  uint64_t o_half;  // the first four MMAs of O += P V done: P columns [0, 32) free
  uint64_t drain;
  uint64_t never;  // completed by nobody: the diagnostic stall of stall_cycles waits here
  uint32_t tmem_base;
  int abort;
  int row_state;  // 0 = run, 1 = empty row (kv_cnt == 0), 2 = invalid row
};
static_assert(sizeof(Bars) <= 256, "barriers fit their shared-memory slot");

// Shared-memory matrix descriptor, 128-byte swizzle, 8-row groups 1024 bytes apart.
RESS_DEV uint64_t smem_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// ---------------------------------------------------------------- softmax arithmetic
// Two fp32 values in one 64-bit register, for the packed f32x2 FMA-pipe instructions.
RESS_DEV uint64_t f2(float lo, float hi) {
  return ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}
RESS_DEV float f2lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
RESS_DEV float f2hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
RESS_DEV uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
RESS_DEV uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
RESS_DEV float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair, on the FMA / integer pipes instead of the MUFU unit.  Range reduction
// to nearest: x = j + f with j = round(x) (adding 1.5 * 2^23 rounds to an integer in the
// low mantissa bits), f in [-1/2, 1/2]; 2^f from a degree-3 polynomial fitted here for
// minimax relative error over [-1/2, 1/2] (Lawson's iteratively reweighted least squares,
// max relative error 7.5e-5, far below the bf16 rounding P receives); 2^j enters by
// adding j to the exponent field.  x is clamped at -126 first (masked logits are -inf):
// the polynomial value lies in [0.70, 1.42], so j >= -126 keeps the exponent field >= 0.
constexpr float kPoly0 = 0.99992805719f, kPoly1 = 0.69326096773f, kPoly2 = 0.24261116982f,
                kPoly3 = 0.05517166480f;
constexpr float kRoundMagic = 12582912.0f;
RESS_DEV uint64_t exp2_pair_fma(uint64_t x) {
  const float lo = fmaxf(f2lo(x), -126.0f), hi = fmaxf(f2hi(x), -126.0f);
  x = f2(lo, hi);
  const uint64_t t = fadd2(x, f2(kRoundMagic, kRoundMagic));
  const uint64_t r = fadd2(t, f2(-kRoundMagic, -kRoundMagic));
  const uint64_t f = ffma2(r, f2(-1.0f, -1.0f), x);
  uint64_t q = ffma2(f, f2(kPoly3, kPoly3), f2(kPoly2, kPoly2));
  q = ffma2(q, f, f2(kPoly1, kPoly1));
  q = ffma2(q, f, f2(kPoly0, kPoly0));
  const uint32_t qlo = (uint32_t)q + ((uint32_t)t << 23);
  const uint32_t qhi = (uint32_t)(q >> 32) + ((uint32_t)(t >> 32) << 23);
  return ((uint64_t)qhi << 32) | qlo;
}

// Of every 8 column pairs, how many take exp2 on the FMA pipes (the rest use MUFU).
#ifndef RESS_POLY_PAIRS_PER8
#define RESS_POLY_PAIRS_PER8 2
#endif
constexpr int kPolyPairsPer8 = RESS_POLY_PAIRS_PER8;

// Instruction descriptors, kind::f16: bf16 A and B, fp32 accumulator.
//   S  = Q K^T : M = 128, N = 128, A and B K-major.
//   O += P V   : M = 128, N = 64, A from tensor memory, B (V) MN-major.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((64u >> 3) << 17) | ((128u >> 4) << 24);

struct AttnParams {
  const int32_t *kv_idx, *kv_cnt, *order;
  __nv_bfloat16 *out;
  float *lse;
  int32_t *dev_err;
  int N, nq, nk;  // tokens; query and key blocks per (batch, head)
  long long items;
  float scale_log2;
  long long stall_cycles;  // > 0 only for ress_debug_attn_forced_timeout
};

// KB = tokens per key block (128 or 64); a score tile always spans 128 keys.
template <int KB>
__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars *bar = reinterpret_cast<Bars *>(smem + kOffBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const long long item = p.order ? (long long)p.order[blockIdx.x] : (long long)blockIdx.x;
  const long long bh = item / p.nq;
  const int qi = (int)(item - bh * p.nq);
  const int cnt = p.kv_cnt[item];
  const int32_t *kvrow = p.kv_idx + item * p.nk;
  // score tiles of the row: one per kept block, or one per pair of 64-token blocks
  const int tiles = KB == 128 ? cnt : (cnt + 1) >> 1;

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 4);
    mbar_init(&bar->p_full, 4);
    mbar_init(&bar->o_done, 1);
    mbar_init(&bar->o_half, 1);
    mbar_init(&bar->drain, 1);
    mbar_init(&bar->never, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp) {
    // validate the row before any work: count in range, every entry in [0, nk)
    bool bad = cnt < 0 || cnt > p.nk;
    if (!bad)
      for (int j = lane; j < cnt; j += 32) {
        const int kb = kvrow[j];
        bad |= kb < 0 || kb >= p.nk;
      }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) bar->row_state = bad ? 2 : (cnt == 0 ? 1 : 0);
    if (bad && lane == 0) report_error(p.dev_err, RESS_ERR_DEVICE_BOUNDS);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const int state = bar->row_state;
  volatile int *abort = &bar->abort;

  if (state == 0) {
    if (warp == kProducerWarp) {
      // ------------------------------------------------------------ TMA producer
      // One thread keeps both rings full.  S_j finishes before PV_j, so the slot of K_j
      // frees before that of V_j: waiting in that order never blocks a load that a
      // consumer needs earlier.
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(&bar->q_full, kTile);
        tma_load_3d(smem + kOffQ, &tmQ, &bar->q_full, 0, qi * 128, (int)bh);
        // tile j into one ring slot: one 128-row box, or two 64-row boxes (kept blocks
        // 2j and 2j+1; row N, past the last token, reads as zero when 2j+1 == cnt)
        auto load_tile = [&](const CUtensorMap *tm, unsigned char *dst, uint64_t *full, int j) {
          mbar_arrive_expect_tx(full, kTile);
          if constexpr (KB == 128) {
            tma_load_3d(dst, tm, full, 0, kvrow[j] * 128, (int)bh);
          } else {
            const int r1 = 2 * j + 1 < cnt ? kvrow[2 * j + 1] * 64 : p.N;
            tma_load_3d(dst, tm, full, 0, kvrow[2 * j] * 64, (int)bh);
            tma_load_3d(dst + kTile / 2, tm, full, 0, r1, (int)bh);
          }
        };
        auto load_k = [&](int j) {
          const int s = j % kKStages;
          load_tile(&tmK, smem + kOffK + s * kTile, &bar->k_full[s], j);
        };
        auto load_v = [&](int j) {
          const int s = j % kVStages;
          load_tile(&tmV, smem + kOffV + s * kTile, &bar->v_full[s], j);
        };
        int nk = min(tiles, kKStages), nv = min(tiles, kVStages);
        for (int j = 0; j < nk; ++j) load_k(j);
        for (int j = 0; j < nv; ++j) load_v(j);
        for (int j = 0; j < tiles; ++j) {
          if (j + kKStages < tiles) {
            if (!mbar_wait(&bar->k_empty[j % kKStages], (j / kKStages) & 1, abort)) break;
            load_k(j + kKStages);
            nk = j + kKStages + 1;
          }
          if (j + kVStages < tiles) {
            if (!mbar_wait(&bar->v_empty[j % kVStages], (j / kVStages) & 1, abort)) break;
            load_v(j + kVStages);
            nv = j + kVStages + 1;
          }
        }
        if (*abort == 0 && (nk < tiles || nv < tiles)) {
          report_error(p.dev_err, RESS_ERR_DEVICE_TIMEOUT);
          *abort = 1;
        }
        // never leave the CTA with copies in flight
        for (int j = max(0, nk - kKStages); j < nk; ++j)
          mbar_wait(&bar->k_full[j % kKStages], (j / kKStages) & 1, nullptr);
        for (int j = max(0, nv - kVStages); j < nv; ++j)
          mbar_wait(&bar->v_full[j % kVStages], (j / kVStages) & 1, nullptr);
        mbar_wait(&bar->q_full, 0, nullptr);
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------ tensor-core issuer
      if (lane == 0) {
        const uint32_t sQ = smem_u32(smem + kOffQ);
        const uint32_t sK = smem_u32(smem + kOffK);
        const uint32_t sV = smem_u32(smem + kOffV);
        bool ok = mbar_wait(&bar->q_full, 0, abort);
        tc_fence_after();
        const uint64_t dq = smem_desc(sQ);
        for (int j = 0; ok && j <= tiles; ++j) {
          if (j < tiles) {
            const int s = j % kKStages;
            ok = mbar_wait(&bar->k_full[s], (j / kKStages) & 1, abort);
            if (ok && j > 0) ok = mbar_wait(&bar->s_free, (j - 1) & 1, abort);
            if (!ok) break;
            tc_fence_after();
            const uint64_t dk = smem_desc(sK + s * kTile);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_ss(tmem + kColS, dq + 2 * k, dk + 2 * k, kIdescS, k > 0);
            mma_commit(&bar->s_full);
            mma_commit(&bar->k_empty[s]);
          }
          if (j > 0) {
            const int jp = j - 1, sp = jp % kVStages;
            ok = mbar_wait(&bar->p_full, jp & 1, abort);
            if (ok) ok = mbar_wait(&bar->v_full[sp], (jp / kVStages) & 1, abort);
            if (!ok) break;
            tc_fence_after();
            const uint64_t dv = smem_desc(sV + sp * kTile);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              mma_ts(tmem + kColO, tmem + kColP + 8 * k, dv + 128 * k, kIdescPV, (jp > 0 || k > 0));
              if (k == 3) mma_commit(&bar->o_half);
            }
            mma_commit(&bar->o_done);
            mma_commit(&bar->v_empty[sp]);
          }
        }
        if (!ok) {
          report_error(p.dev_err, RESS_ERR_DEVICE_TIMEOUT);
          *abort = 1;
        }
        // drain: every MMA issued above has finished before the CTA tears down
        mma_commit(&bar->drain);
        mbar_wait(&bar->drain, 0, nullptr);
      }
    } else {
      // ------------------------------------------------------------- softmax
      const int row = tid;  // 0..127, tensor-memory lane
      const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
      const int last_valid = p.N - (p.nk - 1) * KB;  // tokens in the last key block
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      // diagnostics only: wait, with the given limit, on a barrier that nothing
      // completes, so that the CTA takes the bounded-wait timeout path below (error word,
      // producer and MMA warps released through `abort`, copies and MMAs drained)
      if (p.stall_cycles > 0) ok = mbar_wait_for(&bar->never, 0, abort, p.stall_cycles);
      // kept block(s) of the next tile, read ahead of the barrier wait
      int kb_next = kvrow[0];
      int kb2_next = KB == 64 ? (cnt > 1 ? kvrow[1] : -1) : -1;
      for (int j = 0; j < tiles && ok; ++j) {
        const int kb = kb_next, kb2 = kb2_next;
        if constexpr (KB == 128) {
          if (j + 1 < tiles) kb_next = kvrow[j + 1];
        } else {
          if (2 * j + 2 < cnt) kb_next = kvrow[2 * j + 2];
          kb2_next = 2 * j + 3 < cnt ? kvrow[2 * j + 3] : -1;
        }
        ok = mbar_wait(&bar->s_full, j & 1, abort);
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[128];
#pragma unroll
        for (int h = 0; h < 4; ++h)
          tmem_ld32(trow + kColS + 32 * h, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * h]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->s_free);
        if constexpr (KB == 128) {
          if (kb == p.nk - 1 && last_valid < 128) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c >= last_valid) sv[c] = __float_as_uint(-INFINITY);
          }
        } else {
          // valid keys in each 64-column half: the last block is ragged, an absent
          // second block has none
          const int lim0 = kb == p.nk - 1 ? last_valid : 64;
          const int lim1 = kb2 < 0 ? 0 : (kb2 == p.nk - 1 ? last_valid : 64);
          if (lim0 < 64 || lim1 < 64) {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              if (c >= lim0) sv[c] = __float_as_uint(-INFINITY);
              if (c >= lim1) sv[64 + c] = __float_as_uint(-INFINITY);
            }
          }
        }
        // row max: four chains of 3-input max
        float mc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) mc[q] = fmaxf(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1]));
#pragma unroll
        for (int c = 8; c < 128; c += 8) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mc[q] = fmax3(mc[q], __uint_as_float(sv[c + 2 * q]), __uint_as_float(sv[c + 2 * q + 1]));
        }
        const float mx = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        const bool rescale = m_new > m_run + kRescaleLog2;
        const float m_use = rescale ? m_new : m_run;
        const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
        // p = 2^(s * scale_log2 - m_use): packed FMA, exp2 split between MUFU and the FMA
        // pipes, packed row sums in four chains, bf16 pairs for the P tile
        const uint64_t sc2 = f2(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f2(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const uint64_t x = ffma2(f2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), sc2, nm2);
          uint64_t e;
          if ((c & 7) < kPolyPairsPer8) {
            e = exp2_pair_fma(x);
          } else {
            e = f2(ex2_approx(f2lo(x)), ex2_approx(f2hi(x)));
          }
          acc[c & 3] = fadd2(acc[c & 3], e);
          pk[c] = pack_bf16x2(f2lo(e), f2hi(e));
          if (c == 31) {
            // keys 0..63 of P: their columns are free once the first half of the
            // previous tile's O += P V is done
            if (j > 0) ok = mbar_wait(&bar->o_half, (j - 1) & 1, abort);
            if (ok) tmem_st32(trow + kColP, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
          }
        }
        if (!ok) break;
        const uint64_t a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
        const uint64_t a = fadd2(a01, a23);
        l_run = l_run * alpha + (f2lo(a) + f2hi(a));
        if (j > 0) {
          ok = mbar_wait(&bar->o_done, (j - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            uint32_t ov[32];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              tmem_ld32(trow + kColO + 32 * h, ov);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
              tmem_st32(trow + kColO + 32 * h, ov);
            }
          }
        }
        tmem_st32(trow + kColP + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->p_full);
        m_run = m_use;
      }
      if (ok) ok = mbar_wait(&bar->o_done, (tiles - 1) & 1, abort);
      if (!ok) {
        report_error(p.dev_err, RESS_ERR_DEVICE_TIMEOUT);
        *abort = 1;
      } else {
        tc_fence_after();
        uint32_t o[64];
        tmem_ld32(trow + kColO, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
        tmem_ld32(trow + kColO + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
        tmem_wait_ld();
        const int t = qi * 128 + row;
        if (t < p.N) {
          const float inv = 1.0f / l_run;
          uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((size_t)bh * p.N + t) * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
            dst[c] = w;
          }
          if (p.lse) p.lse[(size_t)bh * p.N + t] = (m_run + __log2f(l_run)) * 0.69314718055994530942f;
        }
      }
    }
  } else if (state == 1 && warp < 4) {
    // no kept block: zero rows, LSE = -inf
    const int t = qi * 128 + tid;
    if (t < p.N) {
      uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((size_t)bh * p.N + t) * 64);
#pragma unroll
      for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      if (p.lse) p.lse[(size_t)bh * p.N + t] = -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [B*H, N, 64] bf16 viewed as a 3-D tensor (64, N, B*H); box (64, rows, 1); rows past N
// read as zero.
bool make_map(CUtensorMap *m, const void *base, int N, long long BH, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {128, (cuuint64_t)N * 128};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn(const Dims &d, const AttnLaunch &a, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, d.N, d.BH(), 128) || !make_map(&mk, a.k, d.N, d.BH(), d.kb) ||
      !make_map(&mv, a.v, d.N, d.BH(), d.kb))
    return cudaErrorNotSupported;
  AttnParams p;
  p.kv_idx = a.kv_idx;
  p.kv_cnt = a.kv_cnt;
  p.order = a.order;
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.lse = a.lse;
  p.dev_err = a.dev_err;
  p.N = d.N;
  p.nq = d.nq;
  p.nk = d.nk;
  p.items = d.BH() * d.nq;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.stall_cycles = a.stall_cycles;
  auto kern = d.kb == 64 ? attn_kernel<64> : attn_kernel<128>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)p.items, kThreads, kSmemBytes, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace ress

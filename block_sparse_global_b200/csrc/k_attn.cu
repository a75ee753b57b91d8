// Block-sparse attention forward on the 5th-generation tensor cores (sm_100a).
//
// [ReSS] = "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers",
// §3 step (3): exact attention over the kept key blocks, softmax renormalised among
// them.  One CTA computes one (batch, head, query block) row of 128 queries against the
// key blocks listed in kv_idx; two CTAs share an SM.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t (tensor-memory lane t).  Reads the
//              S tile from tensor memory, online softmax in the exp2 domain, writes P
//              (bf16) back to tensor memory, rescales O when the running max grows by
//              more than 2^8, and runs the epilogue (O / l -> bf16, LSE).
//   warp 4     TMA producer: Q once, then K_j and V_j of every kept block into a
//              two-stage shared-memory ring.
//   warp 5     tensor-core issuer (one elected thread): S = Q K^T (M=128, N=128, K=64)
//              and O += P V (M=128, N=64, K=128, A operand read from tensor memory).
//              Also allocates and frees the 256 tensor-memory columns.
// Tensor memory: S columns [0,128), P [128,192) as packed bf16 pairs, O [192,256).
// Shared memory: Q 16 KB, K 2 x 16 KB, V 2 x 16 KB, all 128-byte swizzled by TMA.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {
namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr int kTile = 128 * 64 * 2;  // bytes of one 128 x 64 bf16 tile
constexpr int kOffQ = 0;
constexpr int kOffK = kTile;
constexpr int kOffV = kOffK + kStages * kTile;
constexpr int kOffBar = kOffV + kStages * kTile;
constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + barriers + alignment slack
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192;

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full;
  uint64_t s_free;
  uint64_t p_full;
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int row_state;  // 0 = run, 1 = empty row (kv_cnt == 0), 2 = invalid row
};

// Shared-memory matrix descriptor, 128-byte swizzle, 8-row groups 1024 bytes apart.
RESS_DEV uint64_t smem_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

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
  int N, nb;
  long long items;
  float scale_log2;
};

__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars *bar = reinterpret_cast<Bars *>(smem + kOffBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const long long item = p.order ? (long long)p.order[blockIdx.x] : (long long)blockIdx.x;
  const long long bh = item / p.nb;
  const int qi = (int)(item - bh * p.nb);
  const int cnt = p.kv_cnt[item];
  const int32_t *kvrow = p.kv_idx + item * p.nb;

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->kv_full[s], 1);
      mbar_init(&bar->kv_empty[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 4);
    mbar_init(&bar->p_full, 4);
    mbar_init(&bar->o_done, 1);
    mbar_init(&bar->drain, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    // validate the row before any work: count in range, every entry in [0, nb)
    bool bad = cnt < 0 || cnt > p.nb;
    if (!bad)
      for (int j = lane; j < cnt; j += 32) {
        const int kb = kvrow[j];
        bad |= kb < 0 || kb >= p.nb;
      }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) bar->row_state = bad ? 2 : (cnt == 0 ? 1 : 0);
    if (bad && lane == 0) report_error(p.dev_err, RESS_ERR_DEVICE_BOUNDS);
  }
  if (warp == 5) {
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
    if (warp == 4) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(&bar->q_full, kTile);
        tma_load_3d(smem + kOffQ, &tmQ, &bar->q_full, 0, qi * 128, (int)bh);
        int issued = 0;
        for (int j = 0; j < cnt; ++j) {
          const int s = j % kStages;
          if (j >= kStages && !mbar_wait(&bar->kv_empty[s], ((j / kStages) - 1) & 1, abort)) {
            report_error(p.dev_err, RESS_ERR_DEVICE_TIMEOUT);
            *abort = 1;
            break;
          }
          const int kb = kvrow[j];
          mbar_arrive_expect_tx(&bar->kv_full[s], 2 * kTile);
          tma_load_3d(smem + kOffK + s * kTile, &tmK, &bar->kv_full[s], 0, kb * 128, (int)bh);
          tma_load_3d(smem + kOffV + s * kTile, &tmV, &bar->kv_full[s], 0, kb * 128, (int)bh);
          issued = j + 1;
        }
        // never leave the CTA with copies in flight
        for (int j = max(0, issued - kStages); j < issued; ++j)
          mbar_wait(&bar->kv_full[j % kStages], (j / kStages) & 1, nullptr);
        mbar_wait(&bar->q_full, 0, nullptr);
      }
    } else if (warp == 5) {
      // ------------------------------------------------------ tensor-core issuer
      if (lane == 0) {
        const uint32_t sQ = smem_u32(smem + kOffQ);
        const uint32_t sK = smem_u32(smem + kOffK);
        const uint32_t sV = smem_u32(smem + kOffV);
        bool ok = mbar_wait(&bar->q_full, 0, abort);
        tc_fence_after();
        const uint64_t dq = smem_desc(sQ);
        for (int j = 0; ok && j <= cnt; ++j) {
          if (j < cnt) {
            const int s = j % kStages;
            ok = mbar_wait(&bar->kv_full[s], (j / kStages) & 1, abort);
            if (ok && j > 0) ok = mbar_wait(&bar->s_free, (j - 1) & 1, abort);
            if (!ok) break;
            tc_fence_after();
            const uint64_t dk = smem_desc(sK + s * kTile);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_ss(tmem + kColS, dq + 2 * k, dk + 2 * k, kIdescS, k > 0);
            mma_commit(&bar->s_full);
          }
          if (j > 0) {
            const int jp = j - 1, sp = jp % kStages;
            ok = mbar_wait(&bar->p_full, jp & 1, abort);
            if (!ok) break;
            tc_fence_after();
            const uint64_t dv = smem_desc(sV + sp * kTile);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ts(tmem + kColO, tmem + kColP + 8 * k, dv + 128 * k, kIdescPV, (jp > 0 || k > 0));
            mma_commit(&bar->o_done);
            mma_commit(&bar->kv_empty[sp]);
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
      const int last_valid = p.N - (p.nb - 1) * 128;  // tokens in the last block
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int j = 0; j < cnt && ok; ++j) {
        ok = mbar_wait(&bar->s_full, j & 1, abort);
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[128];
        tmem_ld32(trow + kColS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(trow + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_ld32(trow + kColS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
        tmem_ld32(trow + kColS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->s_free);
        const int kb = kvrow[j];
        if (kb == p.nb - 1 && last_valid < 128) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= last_valid) sv[c] = __float_as_uint(-INFINITY);
        }
        float mx = __uint_as_float(sv[0]);
#pragma unroll
        for (int c = 1; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sv[c]));
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        const bool rescale = m_new > m_run + 8.0f;
        const float m_use = rescale ? m_new : m_run;
        const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
        float sum = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * c]), p.scale_log2, -m_use));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), p.scale_log2, -m_use));
          sum += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l_run = l_run * alpha + sum;
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
        tmem_st32(trow + kColP, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(trow + kColP + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->p_full);
        m_run = m_use;
      }
      if (ok) ok = mbar_wait(&bar->o_done, (cnt - 1) & 1, abort);
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
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
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

// [B*H, N, 64] bf16 viewed as a 3-D tensor (64, N, B*H); box (64, 128, 1); rows past N
// read as zero.
bool make_map(CUtensorMap *m, const void *base, int N, long long BH) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {128, (cuuint64_t)N * 128};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn(const Dims &d, const AttnLaunch &a, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, d.N, d.BH()) || !make_map(&mk, a.k, d.N, d.BH()) ||
      !make_map(&mv, a.v, d.N, d.BH()))
    return cudaErrorNotSupported;
  AttnParams p;
  p.kv_idx = a.kv_idx;
  p.kv_cnt = a.kv_cnt;
  p.order = a.order;
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.lse = a.lse;
  p.dev_err = a.dev_err;
  p.N = d.N;
  p.nb = d.nb;
  p.items = d.BH() * d.nb;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  cudaError_t e =
      cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_kernel<<<(unsigned)p.items, kThreads, kSmemBytes, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace ress

// Double-buffered streaming of pooled [nb, 64] fp32 tensors through shared memory.
//
// The block-level kernels (block map, drift, selection) all walk the pooled keys or
// values of one head in order, for every row a CTA owns.  The tiles are L2-resident and
// small (64 keys x 64 fp32 = 16 KB); streaming them with cp.async into two buffers lets
// the load of tile t+1 overlap the arithmetic on tile t.  Rows are padded to 68 floats
// (272 bytes, 16-byte aligned) so that 32 lanes reading 16 bytes each from 32 different
// rows hit every bank exactly once per 8-lane group.
#pragma once

#include "ress_common.cuh"

namespace ress {

constexpr int kTileKeys = 64;
constexpr int kTilePad = 68;
constexpr int kTileFloats = kTileKeys * kTilePad;

RESS_DEV void cp_async16(void *smem_dst, const void *gmem_src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src), "r"(valid ? 16 : 0)
               : "memory");
}
RESS_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
RESS_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Issues the copy of keys [t*64, t*64+64) of `src` ([nb, 64] fp32, row-major) into `dst`
// ([64][68] floats); keys >= nb are zero-filled.  Every thread of the CTA takes part.
RESS_DEV void tile_load(float *dst, const float *src, int t, int nb) {
  const int k0 = t * kTileKeys;
  for (int i = threadIdx.x; i < kTileKeys * 16; i += blockDim.x) {
    const int key = i >> 4, c4 = i & 15;
    const bool valid = k0 + key < nb;
    const float *g = src + (size_t)(valid ? k0 + key : 0) * 64 + 4 * c4;
    cp_async16(dst + key * kTilePad + 4 * c4, g, valid);
  }
  cp_async_commit();
}

// Walks all tiles of `src` through `Stages` buffers (Stages * kTileFloats floats at
// `buf`), keeping up to Stages - 1 tile loads in flight, and calls body(t, tile) once
// per tile with the whole CTA synchronised before each call.  One barrier per tile: the
// refill of the buffer that tile t - 1 used is issued only after that barrier, when
// every thread has finished body(t - 1).  Exactly one cp.async group is committed per
// tile slot (empty past the last tile), so waiting for all but the newest Stages - 2
// groups always covers tile t.  body must not write the buffers.
template <int Stages, typename Body>
RESS_DEV void tile_stream_n(float *buf, const float *src, int nb, Body body) {
  static_assert(Stages >= 2, "at least two buffers");
  const int ntiles = (nb + kTileKeys - 1) / kTileKeys;
  __syncthreads();  // buffers free (previous users done)
#pragma unroll
  for (int t = 0; t < Stages - 1; ++t) {
    if (t < ntiles) tile_load(buf + t * kTileFloats, src, t, nb);
    else cp_async_commit();
  }
  for (int t = 0; t < ntiles; ++t) {
    cp_async_wait<Stages - 2>();
    __syncthreads();  // tile t visible to all; everyone is done with tile t - 1
    const int tn = t + Stages - 1;
    if (tn < ntiles) tile_load(buf + (tn % Stages) * kTileFloats, src, tn, nb);
    else cp_async_commit();
    body(t, buf + (t % Stages) * kTileFloats);
  }
  __syncthreads();  // the buffers are free again when the walk returns
}

// Two-buffer form used by the block-map and drift kernels.
template <typename Body>
RESS_DEV void tile_stream(float *buf, const float *src, int nb, Body body) {
  tile_stream_n<2>(buf, src, nb, body);
}

// The per-block drift arithmetic, written with explicit rounding (no contraction) so that
// every kernel that evaluates it -- the separate drift kernels and the fused drift
// selection -- produces the same bits.
// Lane part of x . M x (lane holds x[lane], x[lane + 32] and (M x) at the same indices).
RESS_DEV float quad_lane(float x0, float y0, float x1, float y1) {
  return __fmaf_rn(x1, y1, __fmul_rn(x0, y0));
}
// s_ij = P_ij sqrt(max(a_i - 2 u_ij + c_j, 0)), [ReSS] Eq. 9 with Eq. 5: a_i = vbar^T M vbar,
// u_ij = (M vbar_i) . V_j, c_j = V_j^T M V_j.
RESS_DEV float drift_score(float p, float a, float u, float c) {
  return __fmul_rn(p, sqrtf(fmaxf(__fadd_rn(__fsub_rn(a, __fmul_rn(2.f, u)), c), 0.f)));
}

}  // namespace ress

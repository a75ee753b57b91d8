/*
 * ress.h -- C ABI of the block-sparse global attention library (libress.so).
 *
 * The library computes, on one NVIDIA B200 (sm_100a), the hot path of training-free
 * block-sparse global attention over the concatenated multi-view tokens of a
 * VGGT-style 3D vision transformer:
 *
 *   (1) mean pooling of fixed-size Q/K/V blocks           ress_pool_blocks
 *   (2) pooled block attention map P and its output vbar  ress_block_scores
 *   (3) the ReSS residual-drift score of every block pair  ress_drift_scores
 *   (4) per-head block selection (attention mass, drift    ress_select_blocks
 *       with iterative residual restoration, or random)
 *   (5) exact attention over the kept blocks only          ress_block_sparse_attn
 *
 * plus the head Gram matrices M_h that (3) and (4) need (ress_head_gram, computed once
 * per layer at model load) and a longest-first launch order for (5)
 * (ress_attn_schedule).
 *
 * Sources, cited by page title and section / equation:
 *   [ReSS]       "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers"
 *   [SparseVGGT] "Block-Sparse Global Attention for Efficient Multi-View Geometry
 *                Transformers"
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, unless marked HOST.
 *     The library allocates no memory and keeps no state between calls.
 *   - Work is enqueued on `stream` and the call returns without synchronising.  Calls on
 *     one stream are ordered; calls on different streams may run concurrently as long
 *     as they do not write the same buffers.
 *   - Shapes: B = batch, H = heads, N = tokens, D = head_dim, b = query block,
 *     b_k = key block (shape.key_block; 0 means b), nq = ceil(N / b) query blocks and
 *     nk = ceil(N / b_k) key blocks.  This version supports D = 64, b = 128, b_k = 128
 *     (nq = nk; written nb below where the two are the same) or b_k = 64 (the pages'
 *     grid of 128-token query blocks and 64-token key blocks, [ReSS] Supp. F),
 *     1 <= H <= 128 and nk <= 4096 (the paper's own per-row cap of 4096 key blocks,
 *     [ReSS] Supp. E).  B = 0 or N = 0 is an empty problem: the call returns RESS_OK and
 *     launches nothing.
 *   - Layouts are dense row-major: bf16 Q/K/V/out are [B, H, N, 64]; pooled queries are
 *     fp32 [B, H, nq, 64], pooled keys and values [B, H, nk, 64]; block maps are fp32
 *     [B, H, nq, nk]; the kept-block list is int32 kv_idx [B, H, nq, nk] (row = kept key
 *     blocks of one query block, ascending, entries past kv_cnt unspecified) with int32
 *     kv_cnt [B, H, nq].  Per-query-block outputs (v_bar, drift) are [B, H, nq, ...].
 *   - Every pointer must be 16-byte aligned.
 *   - Errors: arguments are validated on the host before anything is launched; a bad
 *     argument returns RESS_ERR_INVALID_ARG or RESS_ERR_UNSUPPORTED and touches no
 *     memory.  A failed launch returns RESS_ERR_CUDA.  Problems found on the device (a
 *     kv_idx entry >= nk, kv_cnt > nk, an internal wait that timed out) are written to
 *     the optional int32 `dev_err` word with first-writer-wins (0 = none), the affected
 *     work is skipped, and the kernel never traps.  Read dev_err after synchronising.
 */
#ifndef RESS_H_
#define RESS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *ress_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  RESS_OK = 0,
  RESS_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or budget */
  RESS_ERR_UNSUPPORTED = 2,   /* shape outside this version (head_dim != 64, block != 128, ...) */
  RESS_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  RESS_ERR_DEVICE_BOUNDS = 4, /* device code met an out-of-range kv_idx / kv_cnt (dev_err) */
  RESS_ERR_DEVICE_TIMEOUT = 5 /* device code gave up on a bounded internal wait (dev_err) */
} ress_status;

typedef enum {
  RESS_SELECT_MASS = 0,   /* keep the c_h candidate blocks with the largest P_ij
                             (SparseVGGT / HeSS top-k, [ReSS] §3, §4.4)              */
  RESS_SELECT_DRIFT = 1,  /* ReSS: top-c_h by s_ij / max(1 - P_ij, eps) (Eq. 7), then
                             `rounds` rounds of budget-neutral swaps (Eqs. 13-17) with
                             track-best ([ReSS] §4.2-4.3)                            */
  RESS_SELECT_RANDOM = 2, /* c_h candidates chosen at random (the random-selection
                             control of [ReSS] §6.1, Fig. 8)                         */
  RESS_SELECT_CDF = 3     /* SparseVGGT's top-p rule ([ReSS] §2, §4.4, Table 2 "+CDF
                             threshold", Supp. F): candidates by P descending are kept
                             until the kept mass, always-kept blocks included, reaches
                             top_p (float64 partial sums); at most c_h, at least one  */
} ress_method;

/* Sign of the drift objective for RESS_SELECT_DRIFT.  The maximising settings are the
 * control experiment of [ReSS] Fig. 8 ("flip the sign of the objective, either only in the
 * restoration stage (swap only) or from the initial selection (full)", §6.1). */
typedef enum {
  RESS_DRIFT_MINIMISE = 0,       /* the method: keep high-drift blocks, rounds lower J   */
  RESS_DRIFT_MAXIMISE_SWAPS = 1, /* rounds take the moves that raise J most and return
                                    the largest J seen (initial selection unchanged)    */
  RESS_DRIFT_MAXIMISE_FULL = 2   /* as SWAPS, and the initial selection keeps the c_h
                                    candidates with the SMALLEST s / max(1 - P, eps)    */
} ress_drift_objective;

typedef struct {
  int32_t batch;    /* B >= 0 */
  int32_t heads;    /* H, 1..128 */
  int32_t seq_len;  /* N >= 0 */
  int32_t head_dim; /* D, must be 64 */
  int32_t block;    /* b, query block, must be 128 */
  int32_t key_block; /* b_k, key block: 0 (= block), 128 or 64 */
} ress_shape;

typedef struct {
  int32_t method;           /* ress_method */
  const int32_t *budgets;   /* HOST [H]: c_h, candidate blocks kept per row of head h,
                               0 <= c_h <= nk (else INVALID_ARG); a budget above the
                               number of candidate (not always-kept) key blocks keeps
                               every candidate.  The paper keeps at least two key
                               blocks per row ([ReSS] Supp. F); that floor is the
                               caller's choice of budgets.                          */
  const uint8_t *keep_k;    /* DEVICE [nk] or NULL: 1 = key block is always kept (holds
                               special tokens, [ReSS] §3, §4.1); such blocks are never
                               candidates.  NULL = no always-kept block.            */
  const uint8_t *dense_q;   /* DEVICE [nq] or NULL: 1 = this query block keeps every key
                               block (special query tokens are excluded from
                               sparsification, [ReSS] §3).  NULL = none.            */
  int32_t rounds;           /* R, restoration rounds for RESS_SELECT_DRIFT (0 = none);
                               0..64, ignored by the other methods                  */
  float rho;                /* swap budget fraction of Eq. 17 (paper: 0.5), in (0, 1] */
  float eps;                /* guard of Eq. 7 (paper: 1e-4), > 0                      */
  uint64_t seed;            /* RESS_SELECT_RANDOM: key of pair (b,h,i,j) is output number
                               ((b*H + h)*nq + i)*nk + j + 1 of a SplitMix64 generator
                               seeded with `seed` (Steele, Lea, Flood, OOPSLA 2014)   */
  int32_t objective;        /* ress_drift_objective; must be RESS_DRIFT_MINIMISE unless
                               method is RESS_SELECT_DRIFT (else INVALID_ARG)          */
  float top_p;              /* RESS_SELECT_CDF: mass threshold in (0, 1] (else INVALID_ARG);
                               ignored by the other methods                         */
  float *drift;             /* DEVICE fp32 [B,H,nq] output or NULL: the realized drift J
                               of every row's final selection, Eq. 12 on its drop set
                               (Eq. 10) with K guarded by eps, for any method ([ReSS]
                               §6.1, Figs. 7 and 9); 0 for a dense_q row.  Needs
                               v_pool, v_bar and gram, and eps > 0.                 */
} ress_select_params;

/* Version of this ABI (incremented on any change of the exported calls): 5 (version 4:
 * ress_shape gained `key_block`; ress_select_params gained `objective`, `top_p` and
 * `drift`; RESS_SELECT_CDF; version 5: ress_drift_select and its workspace query). */
int32_t ress_abi_version(void);

/* Human-readable name of a status code (static string). */
const char *ress_status_string(ress_status status);

/*
 * ress_token_gather -- the token layout of the sink rule ([ReSS] Supp. F: "the sink rule
 * that always keeps the trailing block holding the special tokens"; §3: special tokens
 * are excluded from sparsification).  A multi-view sequence holds V views of T = S + Pv
 * tokens each, every view's S special tokens (VGGT: camera, then registers) first.
 * Forward (inverse = 0) moves every view's patch tokens, in view order, to the front and
 * every view's special tokens, in view order, to the tail:
 *   dst[.., v*Pv + p, :] = src[.., v*T + S + p, :]      (patch p of view v)
 *   dst[.., V*Pv + v*S + t, :] = src[.., v*T + t, :]    (special token t of view v)
 * so that the trailing key blocks hold every special token (mark them keep_k, and the
 * query blocks that hold them dense_q).  inverse = 1 applies the reverse permutation
 * (to bring the attention output back to the view order).
 *   src, dst  bf16 [B,H,N,64], N = V*T, distinct buffers (else INVALID_ARG).
 *   views V >= 1, specials S with 0 <= S <= T (INVALID_ARG otherwise or if V does not
 *   divide N).  A pure row permutation: bit-exact.
 */
ress_status ress_token_gather(const ress_shape *shape, int32_t views, int32_t specials,
                              int32_t inverse, const void *src, void *dst,
                              ress_stream_t stream);

/*
 * ress_head_gram -- per-head Gram matrices M_h = (W_O^h)^T W_O^h ([ReSS] §4.2, Eq. 8),
 * computed once per layer ("at model load time").
 *   w_o   fp32 [d_model, H*64] row-major: the layer's output projection; head h is the
 *         d_model x 64 column slice 64h .. 64h+63.
 *   gram  fp32 [H, 64, 64] output, row-major, symmetric.
 * Errors: d_model < 1 -> INVALID_ARG.  Accumulates in fp32 over d_model.
 */
ress_status ress_head_gram(const ress_shape *shape, int32_t d_model, const float *w_o,
                           float *gram, ress_stream_t stream);

/*
 * ress_pool_blocks -- block partition and mean pooling ([ReSS] §3 step (1); the pooled
 * values V_j of §4.1).  For every block j of tokens [b j, min(N, b j + b)):
 * x_pool[b,h,j,:] = mean of those tokens' rows; the partial last block divides by its
 * true token count.  Queries are pooled over query blocks (q_pool [B,H,nq,64]), keys and
 * values over key blocks (k_pool, v_pool [B,H,nk,64]).  Reads bf16 q, k, v [B,H,N,64].
 * fp32 accumulation.
 */
ress_status ress_pool_blocks(const ress_shape *shape, const void *q, const void *k,
                             const void *v, float *q_pool, float *k_pool, float *v_pool,
                             ress_stream_t stream);

/*
 * ress_block_scores -- pooled block attention map and dense pooled output
 * ([ReSS] §3 step (1), §4.1 Eq. 1).
 *   P[b,h,i,j] = softmax over ALL key blocks j of (scale * q_pool_i . k_pool_j)
 *   v_bar[b,h,i,:] = sum_j P[b,h,i,j] v_pool[b,h,j,:]
 * scale: logit scale, normally 1/sqrt(64).  Outputs fp32 P [B,H,nq,nk] and
 * v_bar [B,H,nq,64].
 */
ress_status ress_block_scores(const ress_shape *shape, const float *q_pool,
                              const float *k_pool, const float *v_pool, float scale,
                              float *P, float *v_bar, ress_stream_t stream);

/* Bytes of device workspace that ress_drift_scores needs for `shape`. */
size_t ress_drift_workspace_bytes(const ress_shape *shape);

/*
 * ress_drift_scores -- ReSS block drift score ([ReSS] §4.2, Eqs. 5, 6, 9):
 *   e_ij = v_bar_i - v_pool_j,  q_ij = e_ij^T M_h e_ij
 *        = v_bar_i^T M v_bar_i - 2 v_bar_i^T M v_pool_j + v_pool_j^T M v_pool_j  (Eq. 9)
 *   s[b,h,i,j] = P_ij * sqrt(max(q_ij, 0))
 * evaluated through the expansion of Eq. 9 (no per-pair vector is formed).
 *   gram       fp32 [H,64,64] (ress_head_gram).
 *   workspace  DEVICE scratch of at least ress_drift_workspace_bytes(shape) bytes,
 *              owned by the caller, 16-byte aligned; its contents are overwritten and
 *              are meaningless after the call.
 * Output fp32 s [B,H,nq,nk].
 */
ress_status ress_drift_scores(const ress_shape *shape, const float *P, const float *v_pool,
                              const float *v_bar, const float *gram, float *s,
                              void *workspace, size_t workspace_bytes,
                              ress_stream_t stream);

/*
 * ress_drift_scores_static -- the drift score of ress_drift_scores for callers that cannot
 * allocate device memory.  Some callers receive only their inputs and outputs: the
 * plugin interface of an inference engine that offers no workspace, or a runtime that
 * reserves all device memory at start-up and forbids cudaMalloc / cudaFree afterwards
 * (those calls synchronise the device, and can fail or fragment memory in the middle of
 * a run).  This call takes no workspace: its scratch is a fixed 8 MiB buffer inside
 * libress.so, a static device array that every GPU which loads the library holds until
 * the process exits.  The paper has no counterpart to this call; it exists only for
 * such callers.
 *   Arguments, layouts and results are those of ress_drift_scores, minus the workspace.
 *   Limit: the scratch this call needs is ress_drift_workspace_bytes(shape) =
 *   r(B*H*nq*64*4) + r(B*H*nq*4) + r(B*H*nk*4) bytes, each term r(.) rounded up to a
 *   multiple of 256; a shape for which that exceeds 8 MiB (8,388,608 bytes) is rejected
 *   with RESS_ERR_UNSUPPORTED before anything is launched.  That is about 31,700 query
 *   blocks B*H*nq with 128-token key blocks (nk = nq) and about 31,300 with 64-token key
 *   blocks (nk = 2 nq); ress_drift_workspace_bytes gives the exact figure.
 *   The first call on each device looks up the buffer's device address with a CUDA
 *   runtime call, made with that device current; make this first call before any stream
 *   capture.  The address is then kept for the life of the process: calls made after
 *   cudaDeviceReset (or any other teardown of the device's primary context, after which
 *   the library's device code is loaded anew) are not supported.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   All calls on a device share the one buffer, which keeps the last call's contents
 *   (each call writes every part of it that it later reads, so nothing needs clearing).
 *   Calls that overlap on the GPU -- on different streams, or from threads whose calls
 *   are not ordered -- race on the buffer and give wrong results: order them.
 */
ress_status ress_drift_scores_static(const ress_shape *shape, const float *P,
                                     const float *v_pool, const float *v_bar,
                                     const float *gram, float *s, ress_stream_t stream);

/*
 * ress_select_blocks -- per (query block, head) key-block selection ([ReSS] §4.1 Eq. 2,
 * §4.2 Eq. 7, §4.3 Eqs. 10-17; SparseVGGT/HeSS attention-mass top-k).
 * Candidates are the key blocks with keep_k == 0.  A row whose dense_q flag is set
 * keeps every key block.  Any other row keeps the always-kept blocks plus c_h
 * candidates chosen by params->method:
 *   MASS   : largest P_ij;
 *   CDF    : largest P_ij, cut at the top_p mass (see RESS_SELECT_CDF);
 *   RANDOM : largest SplitMix64 key (see ress_select_params.seed);
 *   DRIFT  : largest s_ij / max(1 - P_ij, eps); then for r = 0..R-1, with the drop set
 *            D and its net drift g = sum_D P_ij (v_bar_i - v_pool_j), K = 1 - sum_D P_ij,
 *            G = g^T M g: m_r = max(1, round-half-up(rho c 2^-(r+1))) (capped by |D|
 *            and c) blocks of D with the largest restore gain (Eqs. 14, 16) are kept and
 *            m_r kept candidates with the largest drop gain (Eqs. 15, 16) are dropped,
 *            both chosen from the start-of-round state; g and K move by Eq. 13 and its
 *            mirror; K is guarded as max(K, eps) in Eq. 16.  The drop set with the
 *            smallest J = G / max(K, eps)^2 (Eq. 12) seen, the initial one included, is
 *            returned (track-best).  params->objective flips the sign of J in the rounds
 *            (and, for MAXIMISE_FULL, in the initial selection); the largest J seen is
 *            then returned.
 * Every top-k orders by (score descending, block index ascending).
 *   P       fp32 [B,H,nq,nk] (ress_block_scores).
 *   s       fp32 [B,H,nq,nk] (ress_drift_scores); required for DRIFT, else may be NULL.
 *   v_pool, v_bar, gram: required for DRIFT with rounds > 0 and whenever params->drift
 *           is set, else may be NULL.
 *   kv_idx  int32 [B,H,nq,nk] output; kv_cnt int32 [B,H,nq] output.
 *   mask    uint8 [B,H,nq,nk] output (1 = kept) or NULL.
 *   dev_err int32 device word or NULL.
 */
ress_status ress_select_blocks(const ress_shape *shape, const ress_select_params *params,
                               const float *P, const float *s, const float *v_pool,
                               const float *v_bar, const float *gram, int32_t *kv_idx,
                               int32_t *kv_cnt, uint8_t *mask, int32_t *dev_err,
                               ress_stream_t stream);

/* Bytes of device workspace that ress_drift_select needs for `shape`. */
size_t ress_drift_select_workspace_bytes(const ress_shape *shape);

/*
 * ress_drift_select -- ress_block_scores, ress_drift_scores and ress_select_blocks for the
 * DRIFT method in one pass per row, the fused per-row selection of [ReSS] §4.3 "Fused
 * kernel implementation" (Supp. E; Table 1, "w/o fused kernel" row): each row's block map
 * P (Eq. 1), its drift scores s (Eqs. 5, 6, 9), the rank key (Eq. 7), the top-c and the
 * `rounds` restoration rounds (Eqs. 10-17) stay on chip, so neither P nor s is written
 * to memory and read back.  P, v_bar and s are evaluated with the same arithmetic, in the
 * same order, as the three separate calls, so the kept lists are identical to theirs on
 * the same pooled inputs, bit for bit.
 *   params     as for ress_select_blocks; method must be RESS_SELECT_DRIFT (else
 *              INVALID_ARG); params->drift (realized J per row) may be set.
 *   q_pool [B,H,nq,64], k_pool and v_pool [B,H,nk,64] fp32 (ress_pool_blocks);
 *   gram   fp32 [H,64,64] (ress_head_gram);  scale: logit scale, normally 1/sqrt(64).
 *   P      fp32 [B,H,nq,nk], v_bar fp32 [B,H,nq,64], s fp32 [B,H,nq,nk]: optional
 *          outputs (NULL = not written), equal to the separate calls' outputs.
 *   kv_idx, kv_cnt, mask, dev_err: as for ress_select_blocks.
 *   workspace  DEVICE scratch of at least ress_drift_select_workspace_bytes(shape) bytes
 *              (c_j = V_j^T M V_j of every key block), owned by the caller, 16-byte
 *              aligned; overwritten.
 * Errors as ress_select_blocks; RESS_ERR_UNSUPPORTED if a row's on-chip state does not
 * fit (never for nk <= 4096).
 */
ress_status ress_drift_select(const ress_shape *shape, const ress_select_params *params,
                              const float *q_pool, const float *k_pool, const float *v_pool,
                              const float *gram, float scale, float *P, float *v_bar, float *s,
                              int32_t *kv_idx, int32_t *kv_cnt, uint8_t *mask, int32_t *dev_err,
                              void *workspace, size_t workspace_bytes, ress_stream_t stream);

/*
 * ress_scores_select -- ress_block_scores and ress_select_blocks in one kernel for the
 * MASS and RANDOM methods (the fused per-row selection: each row's block map stays in
 * shared memory from its softmax to its top-c, [ReSS] §4.3 "Fused kernel
 * implementation" on the fusion motive).  The kept lists are identical to those of the
 * two separate calls on the same pooled inputs.
 *   params   as for ress_select_blocks; method must be MASS, CDF or RANDOM (else
 *            UNSUPPORTED: drift selection needs the drift score and restoration of
 *            its own calls), objective MINIMISE and drift NULL (else INVALID_ARG).
 *   q_pool [B,H,nq,64], k_pool [B,H,nk,64] fp32 (ress_pool_blocks); v_pool needed only
 *            with v_bar.
 *   P        fp32 [B,H,nq,nk] output or NULL (not written).
 *   v_bar    fp32 [B,H,nq,64] output or NULL (Eq. 1 output not computed).
 *   kv_idx, kv_cnt, mask, dev_err: as for ress_select_blocks.
 */
ress_status ress_scores_select(const ress_shape *shape, const ress_select_params *params,
                               const float *q_pool, const float *k_pool, const float *v_pool,
                               float scale, float *P, float *v_bar, int32_t *kv_idx,
                               int32_t *kv_cnt, uint8_t *mask, int32_t *dev_err,
                               ress_stream_t stream);

/*
 * ress_attn_schedule -- launch order for ress_block_sparse_attn: a permutation of the
 * B*H*nq (batch, head, query block) work items sorted by kv_cnt descending, ties in
 * ascending item order (item = (b*H + h)*nq + i).  Running the longest rows first keeps
 * rows that keep every block (dense query blocks) off the tail of the launch.
 *   kv_cnt     int32 [B,H,nq];  work_order int32 [B*H*nq] output.
 * Deterministic.  kv_cnt values outside [0, nk] are clamped for ordering only.
 */
ress_status ress_attn_schedule(const ress_shape *shape, const int32_t *kv_cnt,
                               int32_t *work_order, ress_stream_t stream);

/*
 * ress_block_sparse_attn -- exact attention over the kept blocks ([ReSS] §3 step (3):
 * softmax renormalised among the kept blocks, as if the others did not exist;
 * [SparseVGGT] abstract).  For every token t of query block i of head (b,h):
 *   out[b,h,t,:] = sum_u softmax_u(scale * q_t . k_u) v_u,
 *   u over the tokens (< N) of key blocks kv_idx[b,h,i,0 .. kv_cnt[b,h,i]-1]
 * and lse[b,h,t] = ln sum_u exp(scale * q_t . k_u).  A row with kv_cnt = 0 gets zero
 * output and lse = -inf.  kv_idx rows need not be sorted.
 *   q, k, v     bf16 [B,H,N,64];  out bf16 [B,H,N,64];  lse fp32 [B,H,N] or NULL.
 *   work_order  int32 [B*H*nq] permutation from ress_attn_schedule, or NULL for the
 *               natural order.  Outputs do not depend on it.
 *   dev_err     int32 device word or NULL: an entry of kv_idx outside [0, nk) or a
 *               kv_cnt outside [0, nk] sets RESS_ERR_DEVICE_BOUNDS and that row is
 *               left unwritten.
 * Implementation: bf16 tensor-core tiles (tcgen05, accumulators in tensor memory) fed
 * by TMA, fp32 online softmax.
 */
ress_status ress_block_sparse_attn(const ress_shape *shape, const void *q, const void *k,
                                   const void *v, const int32_t *kv_idx,
                                   const int32_t *kv_cnt, const int32_t *work_order,
                                   float scale, void *out, float *lse, int32_t *dev_err,
                                   ress_stream_t stream);

/*
 * ress_debug_attn_forced_timeout -- diagnostics for the device error path; the pages have
 * no counterpart.  Launches the same attention kernel as ress_block_sparse_attn (same
 * arguments, no work_order, no lse), except that every CTA's softmax warps first wait on
 * an internal barrier that nothing ever completes, giving up after `limit_cycles` SM
 * clock cycles (1 .. 2^32; about 0.5 ms per million cycles at 2 GHz).  Each CTA then
 * takes the path a genuinely stuck wait would take: RESS_ERR_DEVICE_TIMEOUT is written to
 * *dev_err (required here), the TMA and MMA warps are released, every copy and MMA
 * already issued is drained, tensor memory is freed, and the CTA exits without trapping;
 * `out` is left unwritten.  The CUDA context stays usable: a following normal call
 * computes normally.  Host validation as for ress_block_sparse_attn, plus
 * RESS_ERR_INVALID_ARG for a NULL or misaligned dev_err or a limit out of range.
 * For tests of the error path; never needed to compute attention.
 */
ress_status ress_debug_attn_forced_timeout(const ress_shape *shape, const void *q,
                                           const void *k, const void *v,
                                           const int32_t *kv_idx, const int32_t *kv_cnt,
                                           float scale, void *out, int32_t *dev_err,
                                           int64_t limit_cycles, ress_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RESS_H_ */

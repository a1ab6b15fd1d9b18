/*
 * sla.h -- C ABI of the B200 (sm_100a) hybrid block-sparse + linear attention
 * library (libsla.so).
 *
 * The method (SLA post, "Selective Linear Attention", list "the idea"; NABLA
 * post, SberAIScience, points 1-4):
 *   1. Q and K are mean-pooled per block (SLA: "a fast mean-pooling step
 *      labels the blocks in advance"; NABLA point 2: Q and K are compressed).
 *   2. The pooled scores softmax(s * Qbar Kbar^T) are formed per query-block
 *      row (NABLA point 2: the softmax's cumulative distribution).
 *   3. Every (query block, key block) pair is labelled critical, marginal or
 *      negligible (SLA: three kinds of attention), either by top-k fractions
 *      or by keeping the smallest top-ranked set whose mass exceeds 1 - thr
 *      (NABLA point 3).
 *   4. Critical pairs get exact softmax attention, marginal pairs get linear
 *      attention with phi = elu + 1 followed by a d x d projection W,
 *      negligible pairs are skipped (SLA: critical -> FlashAttention,
 *      negligible -> skipped, intermediate -> linear attention; NABLA point
 *      4: compute only on the kept blocks):
 *          out = O_s + O_lin W.
 *   5. A backward pass gives dQ, dK, dV, dW for fine-tuning (SLA results
 *      list: a short fine-tune is enough); the mask is not differentiated.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are dense, row-major, [B, H, N, d] for token tensors (q, k, v,
 *   out, dout, o_s, o_lin, dq, dk, dv), [B, H, N] for lse, [d, d] for proj and
 *   dproj (out = o_s + o_lin @ proj, i.e. proj[a][c] maps input channel a to
 *   output channel c).  Nqb = ceil(N / block_q), Nkb = ceil(N / block_k); the
 *   last block of a sequence may be ragged and is pooled and attended over
 *   its real tokens only.
 * - Block masks are int8 [B, H, Nqb, Nkb]: 2 = critical, 1 = marginal,
 *   0 = negligible.
 * - q, k, v, out and dout have the element type p->dtype (fp32 or bf16);
 *   everything else is fp32 or int32 as declared.  Gradients are fp32.
 * - All pointers except `stream` are DEVICE pointers, must be 16-byte aligned
 *   and are owned by the caller.  The library never allocates, frees or
 *   synchronises (except sla_check_device_status), and keeps no state
 *   between calls.
 * - Every call only enqueues work on `stream` (a cudaStream_t; NULL = the
 *   legacy default stream) and returns at once.  Host-side argument errors are
 *   reported before anything is enqueued; no exception crosses the ABI.
 * - `ws` is caller-owned device scratch of at least sla_workspace_size()
 *   bytes for the operation; its first 256 bytes hold a device status word
 *   that sla_check_device_status() reads.  One workspace must not be shared by
 *   calls that may run concurrently.
 */
#ifndef SLA_H_
#define SLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SLA_API __attribute__((visibility("default")))
#else
#define SLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define SLA_ABI_VERSION 1

typedef enum {
  SLA_OK = 0,
  SLA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or fraction */
  SLA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d = 96)      */
  SLA_ERR_WORKSPACE = 3,    /* ws_bytes below sla_workspace_size()          */
  SLA_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, memset)  */
  SLA_ERR_TIMEOUT = 5       /* a device-side wait gave up (status word)     */
} sla_status;

typedef enum { SLA_F32 = 0, SLA_BF16 = 1 } sla_dtype;

typedef enum {
  SLA_MASK_TOPK = 0,  /* n_c = ceil(frac_crit*Nkb), n_m = min(ceil(frac_marg*Nkb), Nkb-n_c) */
  SLA_MASK_CDF = 1    /* keep the smallest top-ranked set with mass > 1 - thr */
} sla_mask_mode;

typedef enum { SLA_OP_MASK = 0, SLA_OP_FORWARD = 1, SLA_OP_BACKWARD = 2 } sla_op;

/* Problem description.  Fractions are applied per query-block row; the count
 * is the smallest integer >= f * Nkb (with a 1e-9 slack against the binary
 * representation error of f).  In CDF mode frac_crit is ignored and
 * frac_marg, if non-zero, marks the next ceil(frac_marg*Nkb) ranks after the
 * kept set as marginal. */
typedef struct {
  int32_t B, H, N, d;        /* d in {64, 128}                              */
  int32_t block_q, block_k;  /* each in {64, 128}                           */
  int32_t dtype;             /* sla_dtype of q, k, v, out, dout             */
  int32_t mask_mode;         /* sla_mask_mode                               */
  double frac_crit;          /* [0, 1]                                      */
  double frac_marg;          /* [0, 1], frac_crit + frac_marg <= 1 (top-k)  */
  double thr;                /* [0, 1), CDF mode                            */
  float scale;               /* softmax scale; 0 selects 1/sqrt(d)          */
  int32_t flags;             /* SLA_FLAG_* bits, 0 by default               */
} sla_params;

/* Force the portable fp32 SIMT kernels even for bf16 inputs, and the fp32
 * FMA pooled logits (testing aid). */
#define SLA_FLAG_SIMT 1
/* Testing aid for the failure path: every bounded device-side wait gives up
 * after ~1.7e7 cycles instead of ~2.1e9, and the first CTA of one tensor-core
 * kernel withholds one tile load, so the call ends with SLA_ERR_TIMEOUT in the
 * status word (read by sla_check_device_status) instead of hanging.  The
 * kernel is chosen with SLA_DEBUG_WITHHOLD(kernel) in the same flags word
 * (default: the attention forward); the flag makes no kernel fault. */
#define SLA_FLAG_DEBUG_TIMEOUT 2
#define SLA_DEBUG_WITHHOLD(kernel) ((kernel) << 8)
typedef enum {
  SLA_WITHHOLD_ATTENTION = 0,  /* sla_forward / sla_attention_combine / sla_sparse_attention */
  SLA_WITHHOLD_LOGITS = 1,     /* sla_build_mask: pooled logits on the tensor cores         */
  SLA_WITHHOLD_SUMMARIES = 2,  /* sla_forward(_prepare): key-block summaries H_j            */
  SLA_WITHHOLD_GATHER = 3,     /* sla_forward(_prepare): marginal sums H^M_i                */
  SLA_WITHHOLD_BWD_DQ = 4,     /* sla_backward: dQ kernel                                   */
  SLA_WITHHOLD_BWD_DKDV = 5    /* sla_backward: dK, dV kernel                               */
} sla_withhold_kernel;

/* Compressed block lists.  Row lists (CSR): for each of the B*H*Nqb query
 * blocks r, crit_cnt[r] critical key-block indices in ascending order at
 * crit_idx[r*Nkb ...], and likewise for marginal.  Column lists (CSC): for
 * each of the B*H*Nkb key blocks c, the query blocks that hold it, ascending,
 * at crit_idx[c*Nqb ...].  All int32, device memory. */
typedef struct {
  int32_t* crit_cnt;
  int32_t* crit_idx;
  int32_t* marg_cnt;
  int32_t* marg_idx;
} sla_block_lists;

/* Library ABI version (SLA_ABI_VERSION). */
SLA_API int32_t sla_abi_version(void);

/* Static description of a status code.  Never NULL. */
SLA_API const char* sla_status_string(sla_status status);

/* Host-side validation of a parameter block (no CUDA call). */
SLA_API sla_status sla_validate(const sla_params* p);

/* Bytes of workspace `op` needs for `p` (0 is possible).  Host only. */
SLA_API sla_status sla_workspace_size(const sla_params* p, int32_t op, size_t* bytes);

/* Steps 1-3: pool, score and classify.
 *   q, k       [B,H,N,d] dtype
 *   mask       [B,H,Nqb,Nkb] int8 out
 *   rows       CSR lists out (required)
 *   cols       CSC lists out (nullable)
 *   scores     [B,H,Nqb,Nkb] fp32 out, row-softmaxed pooled scores (nullable)
 *   tie_count  one int32 out (nullable): rows whose selection sits within
 *              1e-5 of a decision -- a score gap at a cut within 1e-5 of the
 *              higher score, or (CDF) a decisive tail sum within 1e-5 of thr
 * The block means are fp32.  The pooled logits run on the tensor cores as
 * three tf32 products per step (hi.hi + hi.lo + lo.hi of the means split as
 * hi + lo), which keeps fp32 accuracy; SLA_FLAG_SIMT selects fp32 FMAs.  A
 * device-side wait that times out on that path is reported by
 * sla_check_device_status(ws) as SLA_ERR_TIMEOUT. */
SLA_API sla_status sla_build_mask(const sla_params* p, const void* q, const void* k,
                          int8_t* mask, const sla_block_lists* rows,
                          const sla_block_lists* cols, float* scores,
                          int32_t* tie_count, void* ws, size_t ws_bytes,
                          void* stream);

/* Step 3 alone: classify given pooled scores.
 *   scores     [B,H,Nqb,Nkb] fp32 in: each row a softmax over key blocks
 *              (non-negative; the selection rule of p is applied as is)
 *   mask, rows, cols, tie_count as for sla_build_mask.  No workspace. */
SLA_API sla_status sla_classify_scores(const sla_params* p, const float* scores,
                               int8_t* mask, const sla_block_lists* rows,
                               const sla_block_lists* cols, int32_t* tie_count,
                               void* stream);

/* Row (CSR) and/or column (CSC) lists from any block mask (e.g. one made
 * elsewhere).  Either list pointer may be NULL, not both.  No workspace. */
SLA_API sla_status sla_mask_lists(const sla_params* p, const int8_t* mask,
                          const sla_block_lists* rows,
                          const sla_block_lists* cols, void* stream);

/* Step 4: out = O_s + O_lin @ proj.
 *   q, k, v    [B,H,N,d] dtype
 *   proj       [d,d] fp32
 *   rows       CSR lists from sla_build_mask or sla_mask_lists
 *   out        [B,H,N,d] dtype out
 *   lse        [B,H,N] fp32 out: natural-log sum of exp over critical keys,
 *              -inf for rows without critical blocks
 *   o_s        [B,H,N,d] fp32 out (nullable): critical-branch output
 *   o_lin      [B,H,N,d] fp32 out (nullable): linear-branch output before W
 * o_s, lse and o_lin are what sla_backward needs.  With frac_marg = 0 the
 * linear branch is off: marginal entries in `rows` are ignored, out = O_s and
 * o_lin is written as zeros. */
SLA_API sla_status sla_forward(const sla_params* p, const void* q, const void* k,
                       const void* v, const float* proj,
                       const sla_block_lists* rows, void* out, float* lse,
                       float* o_s, float* o_lin, void* ws, size_t ws_bytes,
                       void* stream);

/* sla_forward in two stages (sla_forward = prepare, then combine, on the same
 * workspace and lists).  Prepare: the per-query-tile key-block plan of the
 * tensor-core attention and, with the linear branch on, the key-block
 * summaries H_j, z_j and their per-query-block sums H^M, z^M.  It resets the
 * workspace status word.  Combine: the attention over critical blocks, the
 * linear attention over marginal blocks, the projection and the sum -- for
 * bf16 with d = 128 (or the linear branch off) one fused kernel that writes
 * `out` directly.  Arguments as for sla_forward. */
SLA_API sla_status sla_forward_prepare(const sla_params* p, const void* k, const void* v,
                               const float* proj, const sla_block_lists* rows, void* ws,
                               size_t ws_bytes, void* stream);
SLA_API sla_status sla_attention_combine(const sla_params* p, const void* q, const void* k,
                                 const void* v, const float* proj,
                                 const sla_block_lists* rows, void* out, float* lse,
                                 float* o_s, float* o_lin, void* ws, size_t ws_bytes,
                                 void* stream);

/* Step 4, critical part alone (NABLA-style sparse attention):
 *   o_s        [B,H,N,d] fp32 out: softmax attention over each query block's
 *              critical key blocks (0 where the block has none)
 *   lse        [B,H,N] fp32 out, as for sla_forward
 * Uses the SLA_OP_FORWARD workspace. */
SLA_API sla_status sla_sparse_attention(const sla_params* p, const void* q, const void* k,
                                const void* v, const sla_block_lists* rows,
                                float* o_s, float* lse, void* ws, size_t ws_bytes,
                                void* stream);

/* Step 4, critical part, for callers that cannot allocate device memory.
 * (The pages have no counterpart; this is a deployment variant of
 * sla_sparse_attention with the same arguments minus the workspace.)
 *
 * Some callers get only a stream and their input and output buffers at the
 * point where they run the attention: plugins of inference runtimes that
 * hand no allocator or workspace to their enqueue step, and real-time loops
 * that must not allocate because cudaMalloc synchronises the device and can
 * fail under memory pressure.  This entry point allocates nothing and calls
 * no allocating routine.  Its scratch -- the per-query-tile key-block plan of
 * the tensor-core kernel -- lives in one 16 MiB static device array that
 * every GPU which loads the library holds until the process exits.
 *   q, k, v, rows, o_s, lse  as for sla_sparse_attention
 *   status     one int32 device word (nullable): cleared, then set to
 *              SLA_ERR_TIMEOUT if a bounded device-side wait gave up; read
 *              it after synchronising the stream
 * Returns SLA_ERR_WORKSPACE when the problem needs more than the 16 MiB
 * (bf16 path: about 4 bytes per (128-row query tile, key block) pair,
 * B*H*ceil(N/128)*Nkb*4 bytes; the 1.3B-DiT shape needs 6.3 MB, the
 * 14B-DiT and long-clip shapes are refused).
 * The first call on each device looks up the array's device address (a
 * one-time set-up per device, repeated only when the device's context has
 * changed, e.g. after cudaDeviceReset); make that first call before any
 * stream capture.  All calls share the array and it keeps the last call's
 * contents: calls that may overlap on the GPU (other streams, other host
 * threads) race with each other and must be serialised by the caller. */
SLA_API sla_status sla_sparse_attention_noalloc(const sla_params* p, const void* q,
                                        const void* k, const void* v,
                                        const sla_block_lists* rows, float* o_s,
                                        float* lse, int32_t* status, void* stream);

/* Step 4, marginal part and combine: per-key-block summaries, linear
 * attention over each query block's marginal list, out = o_s + O_lin @ proj.
 *   o_s        [B,H,N,d] fp32 in (from sla_sparse_attention)
 *   out        [B,H,N,d] dtype out;  o_lin  [B,H,N,d] fp32 out (nullable)
 * Uses the SLA_OP_FORWARD workspace. */
SLA_API sla_status sla_linear_combine(const sla_params* p, const void* q, const void* k,
                              const void* v, const float* proj,
                              const sla_block_lists* rows, const float* o_s,
                              void* out, float* o_lin, void* ws, size_t ws_bytes,
                              void* stream);

/* Step 5: gradients of sum(out * dout) with the mask held fixed.
 *   dout               [B,H,N,d] dtype
 *   rows, cols         CSR and CSC lists of the mask used in the forward
 *   o_s, lse, o_lin    as written by sla_forward
 *   dq, dk, dv         [B,H,N,d] fp32 out (overwritten)
 *   dproj              [d,d] fp32 out (overwritten; summed over B, H, N) */
SLA_API sla_status sla_backward(const sla_params* p, const void* q, const void* k,
                        const void* v, const float* proj, const void* dout,
                        const sla_block_lists* rows,
                        const sla_block_lists* cols, const float* o_s,
                        const float* lse, const float* o_lin, float* dq,
                        float* dk, float* dv, float* dproj, void* ws,
                        size_t ws_bytes, void* stream);

/* 1 if sla_forward / sla_sparse_attention would run the tcgen05
 * tensor-core kernel for `p`, 0 if the fp32 SIMT kernel, -1 if `p` is
 * invalid.  Host only. */
SLA_API int32_t sla_forward_uses_tensor_cores(const sla_params* p);

/* Mask quality, step 1 (a measurement, not the hot path): dense attention
 * max-pooled over (query block, key block) tiles -- the reference a block
 * mask is evaluated against (Veda article, section "Контекст" / context).
 *   q, k        [B,H,N,d] dtype, 16-byte aligned
 *   importance  [B,H,Nqb,Nkb] fp32 out: for query block i and key block j,
 *               the largest dense softmax probability between a real token
 *               of block i and a real key of block j, each token's softmax
 *               running over all N keys with p's scale
 * Dense O(N^2 d) work on the SIMT cores, meant for N up to tens of
 * thousands.  No workspace; asynchronous on `stream`. */
SLA_API sla_status sla_block_importance(const sla_params* p, const void* q, const void* k,
                                        float* importance, void* stream);

/* Mask quality, step 2: recall of a mask against an importance map.
 *   mask        [B,H,Nqb,Nkb] int8 in (2 critical, 1 marginal, 0 negligible)
 *   importance  [B,H,Nqb,Nkb] fp32 in, non-negative
 *   counts      4 int32 out, 16-byte aligned (set by the call): critical
 *               hits, critical total, kept hits, kept total.  Per row with c
 *               critical blocks the reference set is the c blocks of largest
 *               importance (ties by lower block index); a hit is a reference
 *               block the mask marks critical.  "Kept" does the same with the
 *               critical-or-marginal set.  recall = hits / total.
 * O(Nkb^2) comparisons per row.  Asynchronous on `stream`. */
SLA_API sla_status sla_mask_recall(const sla_params* p, const int8_t* mask,
                                   const float* importance, int32_t* counts, void* stream);

/* Token order of 3D tiles (Veda article, sections "Что произошло" / what
 * happened and "Контекст" / context: attention is selected over tiles of
 * tokens, with tile shapes fitted per head and layer).  For a latent grid of
 * F frames x R rows x C columns in raster order (token t = (f R + r) C + c),
 * tiles of tf x tr x tc tokens are taken in raster order over the tile grid
 * (tiles at the far edges are partial) and tokens in raster order inside
 * each tile, so that a block of consecutive tokens covers a compact box.
 *   perm   [F*R*C] int32 out (device): perm[n] = raster index of the n-th
 *          token in tile order
 * All sizes >= 1 and F*R*C < 2^31; asynchronous on `stream`. */
SLA_API sla_status sla_tile_order(int32_t F, int32_t R, int32_t C, int32_t tf, int32_t tr,
                                  int32_t tc, int32_t* perm, void* stream);

/* Moves a token tensor [B, H, N, d] (p's B, H, N, d) into or out of another
 * token order:
 *   inverse = 0:  dst[b, h, n, :] = src[b, h, perm[n], :]   (into the order)
 *   inverse = 1:  dst[b, h, perm[n], :] = src[b, h, n, :]   (back to raster)
 *   perm        [N] int32 (device), a permutation of 0..N-1 (e.g. from
 *               sla_tile_order); not checked on the device
 *   elem_bytes  2 (bf16) or 4 (fp32: the gradients, O_s, O_lin)
 * src and dst must not overlap.  Running mask, forward and backward on the
 * permuted q, k, v (and dout) and moving out, dq, dk, dv back gives the
 * hybrid attention of the tiled blocks in raster order.  Asynchronous. */
SLA_API sla_status sla_permute_tokens(const sla_params* p, const void* src, void* dst,
                                      const int32_t* perm, int32_t elem_bytes, int32_t inverse,
                                      void* stream);

/* Synchronises `stream` and returns the status word the last call on `ws`
 * left (SLA_OK, or SLA_ERR_TIMEOUT when a bounded device-side wait gave up),
 * or SLA_ERR_CUDA when a CUDA error is pending. */
SLA_API sla_status sla_check_device_status(void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H_ */

// Internal launch interface of libsla (host side, not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sla.h"

namespace sla {

using i64 = int64_t;

// Everything a launcher needs about one problem, derived from sla_params.
struct Geom {
  int B, H, N, d;
  int bq, bk;          // block sizes
  int nqb, nkb;        // block counts
  int BH;              // B * H
  int dtype;           // sla_dtype
  int mode;            // sla_mask_mode
  int n_c, n_m;        // top-k counts (n_m also used in CDF mode)
  uint64_t thr_fx;     // ceil(thr * 2^62): CDF threshold in 2^-62 fixed point
  double thr;
  float scale;
  int flags;
  bool linear;         // linear branch on (frac_marg > 0)
};

// Bounded device-side waits give up after this many cycles (~1.1 s at
// 1.965 GHz; ~8.5 ms under SLA_FLAG_DEBUG_TIMEOUT).
inline long long wait_limit(const Geom& g) {
  return (g.flags & SLA_FLAG_DEBUG_TIMEOUT) ? (1ll << 24) : (1ll << 31);
}
// Testing aid: true when kernel `k` (sla_withhold_kernel) is the one whose
// first CTA withholds a tile load under SLA_FLAG_DEBUG_TIMEOUT.
inline bool debug_withhold(const Geom& g, int k) {
  return (g.flags & SLA_FLAG_DEBUG_TIMEOUT) != 0 && ((g.flags >> 8) & 0xF) == k;
}

constexpr double kFixedOne = 4611686018427387904.0;  // 2^62
constexpr float kTieEps = 1e-5f;
constexpr int kMaxBlocks = 8192;                     // Nqb, Nkb limit

// TMA descriptors and device queries (tma_host.cu)
bool tma_available();
bool current_context_id(unsigned long long* id);
int sm_count();
bool encode_bf16_map(void* map, const void* ptr, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box);
bool encode_f32_map(void* map, const void* ptr, int rank, const uint64_t* dims,
                    const uint64_t* strides, const uint32_t* box);

// mask path
// block means of Q (blocks of bq tokens) and K (blocks of bk) in one launch;
// with qlo/klo given, split as hi (in qbar/kbar) + lo, both tf32
// zero_words[0, nzero) (nzero <= 128) and *zero_one (if given) are zeroed by
// the first CTA, for the step's later kernels.
cudaError_t launch_pool(const void* q, const void* k, int dtype, float* qbar, float* kbar,
                        float* qlo, float* klo, int BH, int N, int d, int bq, int bk, cudaStream_t s,
                        int32_t* zero_words = nullptr, int nzero = 0, int32_t* zero_one = nullptr);
cudaError_t launch_logits(const float* qbar, const float* kbar, float* logits,
                          const Geom& g, cudaStream_t s);
// the same logits on the tensor cores from the split means (logits_tc.cu)
bool logits_tc_supported(const Geom& g);
cudaError_t launch_logits_tc(const float* qhi, const float* qlo, const float* khi, const float* klo,
                             float* logits, const Geom& g, int32_t* status, cudaStream_t s);
// one warp per row: logits (or row-softmaxed scores, from_prob) of `nrows`
// rows -> mask, row lists, optional scores; near-ties added to *tie_count
// (mask_select.cu)
cudaError_t launch_select_rows(const float* in, int nrows, const Geom& g, int8_t* mask,
                               const sla_block_lists& rows, float* scores, int32_t* tie_count,
                               bool from_prob, cudaStream_t s);
// 3D-tile token order and the row permutation (tile_order.cu)
cudaError_t launch_tile_order(int F, int R, int C, int tf, int tr, int tc, int32_t* perm,
                              cudaStream_t s);
cudaError_t launch_permute_rows(const void* src, void* dst, const int32_t* perm, i64 rows, int N,
                                int row_bytes, bool scatter, cudaStream_t s);
cudaError_t launch_rows_from_mask(const int8_t* mask, const Geom& g,
                                  const sla_block_lists& rows, cudaStream_t s);
cudaError_t launch_cols_from_mask(const int8_t* mask, const Geom& g,
                                  const sla_block_lists& cols, cudaStream_t s);

// mask quality (quality_kernels.cu)
cudaError_t launch_block_importance(const void* q, const void* k, float* imp, const Geom& g,
                                    cudaStream_t s);
cudaError_t launch_mask_recall(const int8_t* mask, const float* imp, const Geom& g, int32_t* counts,
                               cudaStream_t s);

// forward
cudaError_t launch_attn_simt(const void* q, const void* k, const void* v,
                             const Geom& g, const sla_block_lists& rows,
                             float* o_s, float* lse, cudaStream_t s);
bool attn_tc_supported(const Geom& g);
cudaError_t launch_attn_tc(const void* q, const void* k, const void* v,
                           const Geom& g, const sla_block_lists& rows,
                           float* o_s, float* lse, int32_t* status,
                           void* scratch, cudaStream_t s);
size_t attn_tc_scratch_bytes(const Geom& g);
// Tile plan of block lists (the attention kernels' work list): lists of
// `nrb` blocks of `rb` rows (per bh) over `ncb` blocks of `cb` columns are
// grouped into 128-row tiles (one block of 128 or two of 64) whose merged,
// sorted column lists are packed two 16-bit entries per word when cb = 64
// (one otherwise): bit 15 present, bits 13-14 which of the tile's 64-row
// halves the entry holds for, bits 0-12 column block.  cnt[BH * nt] words
// per tile, tiles[BH * nt][ncb], nt = ceil(nrb * rb / 128).
constexpr uint32_t kPlanPresent = 1u << 15;
cudaError_t launch_tile_plan(const sla_block_lists& lists, int BH, int nrb, int ncb, int rb,
                             int cb, int32_t* cnt, uint32_t* tiles, cudaStream_t s);

// Linear-branch inputs of the fused query side of the backward (d = 128).
struct LinBwdIn {
  const void* hm;           // [B*H*Nqb, 128, 128] bf16 H^M (forward prepare)
  const void* wb;           // [128, 128] bf16 W
  const float* zm;          // [B*H*Nqb, 128] z^M
  const int32_t* marg_cnt;  // [B*H*Nqb] marginal counts
  const float* o_lin;       // [B*H, N, 128] saved O_lin
  void* dhm;                // out: [B*H*Nqb, 128, 128] bf16 dH^M
  float* dzm;               // out: [B*H*Nqb, 128] dz^M
};

// Linear-branch inputs of the fused key side (d = 128).
struct LinBwdKIn {
  const void* dh;           // [B*H*Nkb, 128, 128] bf16 dH_j
  const float* dz;          // [B*H*Nkb, 128] dz_j
  const int32_t* marg_cnt;  // [B*H*Nkb] per key block: query blocks holding it
};

// backward of the critical branch on the tensor cores (attn_bwd_tc.cu), in
// two launches.  _dq builds the row and column tile plans in `scratch` and
// writes dq (fp32); with `lin` its epilogue adds the linear branch's dq and
// writes dH^M, dz^M.  _dkdv (same scratch) writes dk, dv; with `lin` its
// epilogue adds the linear branch's dk, dv.
size_t attn_bwd_tc_scratch_bytes(const Geom& g);
cudaError_t launch_attn_bwd_tc_dq(const void* q, const void* k, const void* v, const void* dout,
                                  const float* lse, const float* delta,
                                  const sla_block_lists& rows, const sla_block_lists& cols,
                                  float* dq, const Geom& g, void* scratch, int32_t* status,
                                  cudaStream_t s, const LinBwdIn* lin);
cudaError_t launch_attn_bwd_tc_dkdv(const void* q, const void* k, const void* v,
                                    const void* dout, const float* lse, const float* delta,
                                    float* dk, float* dv, const Geom& g, void* scratch,
                                    int32_t* status, cudaStream_t s, const LinBwdKIn* lin);
// Outputs of the fused tensor-core attention; any pointer may be null.
struct AttnOutputs {
  float* o_s;     // fp32 O_s
  float* lse;     // fp32 LSE (required)
  void* out;      // bf16 out = O_s (+ O_lin W when the linear branch is fused)
  float* o_lin;   // fp32 O_lin
};
// Prepared linear-branch tensors (from launch_lin_tc_prepare).
struct LinInputs {
  const void* hm;          // bf16 H^M [B*H*Nqb, 128, 128]
  const void* wb;          // bf16 W [128, 128]
  const float* zm;         // fp32 z^M [B*H*Nqb, 128]
  const int32_t* marg_cnt; // marginal list counts [B*H*Nqb]
};
// zero_words[0, nzero) (nzero <= 128) are zeroed by the first CTA.
cudaError_t launch_attn_plan(const Geom& g, const sla_block_lists& rows, void* scratch,
                             cudaStream_t s, int32_t* zero_words = nullptr, int nzero = 0);
cudaError_t launch_attn_tc_fused(const void* q, const void* k, const void* v, const Geom& g,
                                 void* scratch, const AttnOutputs& o, const LinInputs* lin,
                                 int32_t* status, cudaStream_t s);
cudaError_t launch_lin_summary(const void* k, const void* v, const Geom& g,
                               float* hsum, float* zsum, cudaStream_t s);
cudaError_t launch_lin_apply(const void* q, const float* hsum,
                             const float* zsum, const sla_block_lists& rows,
                             const float* o_s, const float* proj, void* out,
                             float* o_lin, const Geom& g, cudaStream_t s);

cudaError_t launch_combine_copy(const float* o_s, void* out, float* o_lin, const Geom& g,
                                cudaStream_t s);

// tensor-core linear branch (bf16, d = 128): linear_tc.cu
bool lin_tc_supported(const Geom& g);
size_t lin_tc_scratch_bytes(const Geom& g);
cudaError_t launch_lin_tc(const void* q, const void* k, const void* v, const float* proj,
                          const sla_block_lists& rows, const float* o_s, void* out,
                          float* o_lin, const Geom& g, void* scratch, int32_t* status,
                          cudaStream_t s);
cudaError_t launch_lin_tc_prepare(const void* k, const void* v, const float* proj,
                                  const sla_block_lists& rows, const Geom& g, void* scratch,
                                  int32_t* status, cudaStream_t s);
LinInputs lin_tc_inputs(const Geom& g, void* scratch, const sla_block_lists& rows);
// Indicator GEMM over the marginal part of `lists` (nrow lists over ncol
// blocks per bh): dst_h[bh][r] = sum of src_h[bh][x] (bf16 d x d) and
// dst_z[bh][r] = sum of src_z[bh][x] (fp32 d) over x in list r.  `ind` holds
// BH * nrow * ld bf16 (ld = ncol rounded up to 64).
cudaError_t launch_list_gather(const sla_block_lists& lists, int BH, int nrow, int ncol,
                               const void* src_h, const float* src_z, void* dst_h, float* dst_z,
                               void* ind, int ld, int32_t* status, const Geom& g, cudaStream_t s);

// backward of the linear branch and the projection on the tensor cores
// (lin_bwd_tc.cu): dq, dk, dv are added to; dproj is written.
size_t lin_bwd_tc_scratch_bytes(const Geom& g);
cudaError_t launch_delta(const void* dout, const float* o_s, float* delta, const Geom& g,
                         cudaStream_t s);
// 1. before the attention backward: H^M, z^M, W in bf16 into `scratch`, and
//    the pointers the fused query side needs
cudaError_t launch_lin_bwd_prepare(const void* k, const void* v, const float* proj,
                                   const sla_block_lists& rows, const float* o_lin,
                                   const Geom& g, void* scratch, int32_t* status,
                                   cudaStream_t s, LinBwdIn* lin);
// 2. between the dq and dkdv launches: dH_j, dz_j from dH^M, dz^M (the
//    indicator GEMM over the column lists), and the pointers for the fused
//    key side
cudaError_t launch_lin_bwd_gather(const sla_block_lists& cols, const Geom& g, void* scratch,
                                  int32_t* status, cudaStream_t s, LinBwdKIn* lin);
// 3. dW = O_lin^T dO (zero without a linear branch)
cudaError_t launch_lin_bwd_dw(const void* dout, const float* o_lin, float* dproj, const Geom& g,
                              void* scratch, int32_t* status, cudaStream_t s);

// backward
cudaError_t launch_bwd_prep(const void* dout, const float* o_s,
                            const float* o_lin, const float* proj,
                            float* delta, float* gbuf, float* dw_part,
                            const Geom& g, cudaStream_t s);
cudaError_t launch_bwd_dw_reduce(const float* dw_part, float* dproj,
                                 const Geom& g, cudaStream_t s);
cudaError_t launch_attn_bwd_dq(const void* q, const void* k, const void* v,
                               const void* dout, const float* lse,
                               const float* delta, const sla_block_lists& rows,
                               float* dq, const Geom& g, cudaStream_t s);
cudaError_t launch_attn_bwd_dkdv(const void* q, const void* k, const void* v,
                                 const void* dout, const float* lse,
                                 const float* delta,
                                 const sla_block_lists& cols, float* dk,
                                 float* dv, const Geom& g, cudaStream_t s);
cudaError_t launch_lin_bwd_q(const void* q, const float* hsum,
                             const float* zsum, const sla_block_lists& rows,
                             const float* gbuf, const float* o_lin, float* dq,
                             float* dhm, float* dzm, const Geom& g,
                             cudaStream_t s);
cudaError_t launch_lin_bwd_kv(const void* k, const void* v, const float* dhm,
                              const float* dzm, const sla_block_lists& cols,
                              float* dk, float* dv, const Geom& g,
                              cudaStream_t s);

}  // namespace sla

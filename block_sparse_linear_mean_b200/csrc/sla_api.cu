// C ABI of libsla: argument validation, workspace layout and kernel
// dispatch.  Every entry point only enqueues work on the caller's stream.
#include <math.h>
#include <string.h>

#include <algorithm>

#include "internal.h"

namespace sla {
int bwd_dw_parts(const Geom& g);
}

using sla::Geom;

namespace {

constexpr size_t kStatusBytes = 256;
// The pooled logits of the mask step are produced and classified a group of
// heads at a time through a slab of at most this size, which stays in L2
// (126 MB) between the two kernels: the whole [B, H, Nqb, Nkb] score matrix
// never goes to HBM.  (The largest size measured to stay there: at 74 MB
// the selection kernel already read 9 % of the slab from DRAM.)
constexpr size_t kSlabBytes = size_t(64) << 20;

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int count_from_fraction(double f, int nkb) {
  double c = ceil(f * static_cast<double>(nkb) - 1e-9);
  if (c < 0) c = 0;
  if (c > nkb) c = nkb;
  return static_cast<int>(c);
}

sla_status make_geom(const sla_params* p, Geom* g) {
  if (!p) return SLA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->N < 1 || p->d < 1 || p->block_q < 1 || p->block_k < 1)
    return SLA_ERR_INVALID_ARG;
  if (p->dtype != SLA_F32 && p->dtype != SLA_BF16) return SLA_ERR_INVALID_ARG;
  if (p->mask_mode != SLA_MASK_TOPK && p->mask_mode != SLA_MASK_CDF) return SLA_ERR_INVALID_ARG;
  if (!(p->frac_crit >= 0.0 && p->frac_crit <= 1.0)) return SLA_ERR_INVALID_ARG;
  if (!(p->frac_marg >= 0.0 && p->frac_marg <= 1.0)) return SLA_ERR_INVALID_ARG;
  if (p->mask_mode == SLA_MASK_TOPK && p->frac_crit + p->frac_marg > 1.0 + 1e-9)
    return SLA_ERR_INVALID_ARG;
  if (p->mask_mode == SLA_MASK_CDF && !(p->thr >= 0.0 && p->thr < 1.0)) return SLA_ERR_INVALID_ARG;
  if (!(p->scale >= 0.0f) || !isfinite(p->scale)) return SLA_ERR_INVALID_ARG;
  if (p->flags & ~(SLA_FLAG_SIMT | SLA_FLAG_DEBUG_TIMEOUT | SLA_DEBUG_WITHHOLD(0xF)))
    return SLA_ERR_INVALID_ARG;
  if ((p->flags & SLA_DEBUG_WITHHOLD(0xF)) &&
      (!(p->flags & SLA_FLAG_DEBUG_TIMEOUT) ||
       ((p->flags >> 8) & 0xF) > SLA_WITHHOLD_BWD_DKDV))
    return SLA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return SLA_ERR_UNSUPPORTED;
  if ((p->block_q != 64 && p->block_q != 128) || (p->block_k != 64 && p->block_k != 128))
    return SLA_ERR_UNSUPPORTED;
  g->B = p->B; g->H = p->H; g->N = p->N; g->d = p->d;
  g->bq = p->block_q; g->bk = p->block_k;
  g->nqb = (p->N + p->block_q - 1) / p->block_q;
  g->nkb = (p->N + p->block_k - 1) / p->block_k;
  if (g->nqb > sla::kMaxBlocks || g->nkb > sla::kMaxBlocks) return SLA_ERR_UNSUPPORTED;
  const int64_t bh = static_cast<int64_t>(p->B) * p->H;
  if (bh > 65535) return SLA_ERR_UNSUPPORTED;  // grid y/z dimension limit
  if (bh * g->nqb >= (int64_t(1) << 31) || bh * g->nkb >= (int64_t(1) << 31) ||
      bh * p->N >= (int64_t(1) << 31))
    return SLA_ERR_UNSUPPORTED;
  g->BH = static_cast<int>(bh);
  g->dtype = p->dtype;
  g->mode = p->mask_mode;
  g->n_c = p->mask_mode == SLA_MASK_TOPK ? count_from_fraction(p->frac_crit, g->nkb) : 0;
  g->n_m = count_from_fraction(p->frac_marg, g->nkb);
  if (p->mask_mode == SLA_MASK_TOPK && g->n_m > g->nkb - g->n_c) g->n_m = g->nkb - g->n_c;
  g->thr = p->thr;
  g->thr_fx = static_cast<uint64_t>(ceil(p->thr * sla::kFixedOne));
  g->scale = p->scale > 0.0f ? p->scale : 1.0f / sqrtf(static_cast<float>(p->d));
  g->flags = p->flags;
  g->linear = p->frac_marg > 0.0;
  return SLA_OK;
}

bool has_linear_branch(const Geom& g) { return g.linear; }


// Workspace layouts (each region 256-byte aligned).
struct MaskWs { size_t qbar, kbar, qlo, klo, logits, total; };
struct FwdWs { size_t o_s, hsum, zsum, lintc, tc, total; };
struct BwdWs { size_t delta, gbuf, hsum, zsum, dhm, dzm, dwp, plans, lin, total; };

// Which backward kernels run: the tcgen05 attention backward for bf16
// (unless SLA_FLAG_SIMT), and with it the tcgen05 linear-branch and
// projection backward when d = 128; SIMT fp32 kernels otherwise.
bool bwd_tc_attention(const Geom& g) {
  return g.dtype == SLA_BF16 && !(g.flags & SLA_FLAG_SIMT) && sla::attn_tc_supported(g);
}
bool bwd_tc_linear(const Geom& g) { return bwd_tc_attention(g) && sla::lin_tc_supported(g); }

// Heads per group of the mask step (the slab holds their logits).
int mask_group_heads(const Geom& g) {
  const size_t per_head = sizeof(float) * size_t(g.nqb) * g.nkb;
  const size_t fit = std::max<size_t>(1, kSlabBytes / per_head);
  return static_cast<int>(std::min<size_t>(fit, size_t(g.BH)));
}

MaskWs mask_ws(const Geom& g) {
  MaskWs w;
  size_t off = kStatusBytes;
  w.qbar = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nqb * g.d);
  w.kbar = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nkb * g.d);
  w.qlo = w.klo = off;  // (the tf32 lo parts, for the tensor-core logits)
  if (sla::logits_tc_supported(g)) {
    w.qlo = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nqb * g.d);
    w.klo = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nkb * g.d);
  }
  w.logits = off;
  off = align_up(off + sizeof(float) * size_t(mask_group_heads(g)) * g.nqb * g.nkb);
  w.total = off;
  return w;
}

sla_block_lists lists_from_row(const sla_block_lists& l, size_t row, int width) {
  sla_block_lists r = l;
  r.crit_cnt += row;
  r.marg_cnt += row;
  r.crit_idx += row * width;
  r.marg_idx += row * width;
  return r;
}

FwdWs fwd_ws(const Geom& g) {
  FwdWs w;
  size_t off = kStatusBytes;
  w.o_s = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.N * g.d);
  w.hsum = w.zsum = w.lintc = off;
  if (has_linear_branch(g)) {
    if (sla::lin_tc_supported(g)) {
      w.lintc = off; off = align_up(off + sla::lin_tc_scratch_bytes(g));
    } else {
      w.hsum = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nkb * g.d * g.d);
      w.zsum = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nkb * g.d);
    }
  }
  w.tc = off; off = align_up(off + sla::attn_tc_scratch_bytes(g));
  w.total = off;
  return w;
}

BwdWs bwd_ws(const Geom& g) {
  BwdWs w;
  size_t off = kStatusBytes;
  w.delta = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.N);
  if (bwd_tc_linear(g)) {  // everything else lives in the tensor-core scratch
    w.gbuf = w.hsum = w.zsum = w.dhm = w.dzm = w.dwp = off;
    w.plans = off; off = align_up(off + sla::attn_bwd_tc_scratch_bytes(g));
    w.lin = off; off = align_up(off + sla::lin_bwd_tc_scratch_bytes(g));
    w.total = off;
    return w;
  }
  w.lin = off;
  w.gbuf = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.N * g.d);
  w.hsum = w.zsum = w.dhm = w.dzm = off;
  if (has_linear_branch(g)) {
    w.hsum = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nkb * g.d * g.d);
    w.zsum = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nkb * g.d);
    w.dhm = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nqb * g.d * g.d);
    w.dzm = off; off = align_up(off + sizeof(float) * size_t(g.BH) * g.nqb * g.d);
  }
  w.dwp = off; off = align_up(off + sizeof(float) * size_t(sla::bwd_dw_parts(g)) * g.d * g.d);
  w.plans = off;
  if (bwd_tc_attention(g)) off = align_up(off + sla::attn_bwd_tc_scratch_bytes(g));
  w.total = off;
  return w;
}

bool lists_ok(const sla_block_lists* l) {
  return l && l->crit_cnt && l->crit_idx && l->marg_cnt && l->marg_idx &&
         aligned16(l->crit_cnt) && aligned16(l->crit_idx) && aligned16(l->marg_cnt) &&
         aligned16(l->marg_idx);
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

#define SLA_CUDA(call)                              \
  do {                                              \
    if ((call) != cudaSuccess) return SLA_ERR_CUDA; \
  } while (0)

}  // namespace

extern "C" {

int32_t sla_abi_version(void) { return SLA_ABI_VERSION; }

const char* sla_status_string(sla_status s) {
  switch (s) {
    case SLA_OK: return "ok";
    case SLA_ERR_INVALID_ARG: return "invalid argument";
    case SLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SLA_ERR_WORKSPACE: return "workspace too small";
    case SLA_ERR_CUDA: return "CUDA runtime error";
    case SLA_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

sla_status sla_validate(const sla_params* p) {
  Geom g;
  return make_geom(p, &g);
}

sla_status sla_workspace_size(const sla_params* p, int32_t op, size_t* bytes) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!bytes) return SLA_ERR_INVALID_ARG;
  switch (op) {
    case SLA_OP_MASK: *bytes = mask_ws(g).total; return SLA_OK;
    case SLA_OP_FORWARD: *bytes = fwd_ws(g).total; return SLA_OK;
    case SLA_OP_BACKWARD: *bytes = bwd_ws(g).total; return SLA_OK;
  }
  return SLA_ERR_INVALID_ARG;
}

sla_status sla_build_mask(const sla_params* p, const void* q, const void* k,
                          int8_t* mask, const sla_block_lists* rows,
                          const sla_block_lists* cols, float* scores,
                          int32_t* tie_count, void* ws, size_t ws_bytes,
                          void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!q || !k || !mask || !ws || !aligned16(q) || !aligned16(k) || !aligned16(mask) ||
      !aligned16(ws) || !lists_ok(rows) || (cols && !lists_ok(cols)) ||
      (scores && !aligned16(scores)) ||
      (tie_count && (reinterpret_cast<uintptr_t>(tie_count) & 3u)))
    return SLA_ERR_INVALID_ARG;
  const MaskWs w = mask_ws(g);
  if (ws_bytes < w.total) return SLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* qbar = at<float>(ws, w.qbar);
  float* kbar = at<float>(ws, w.kbar);
  float* logits = at<float>(ws, w.logits);
  // the status words and the near-tie counter are zeroed by the pooling
  // kernel, the first of the step
  int32_t* const zw = at<int32_t>(ws, 0);
  constexpr int kZw = static_cast<int>(kStatusBytes / sizeof(int32_t));
  const size_t rowcols = size_t(g.nqb) * g.nkb;
  if (sla::logits_tc_supported(g)) {
    float* qlo = at<float>(ws, w.qlo);
    float* klo = at<float>(ws, w.klo);
    SLA_CUDA(sla::launch_pool(q, k, g.dtype, qbar, kbar, qlo, klo, g.BH, g.N, g.d, g.bq, g.bk, s, zw, kZw,
                              tie_count));
    // logits and selection a group of heads at a time, through the slab
    const int G = mask_group_heads(g);
    for (int h0 = 0; h0 < g.BH; h0 += G) {
      Geom gg = g;
      gg.BH = std::min(G, g.BH - h0);
      const size_t qo = size_t(h0) * g.nqb * g.d, ko = size_t(h0) * g.nkb * g.d;
      SLA_CUDA(sla::launch_logits_tc(qbar + qo, qlo + qo, kbar + ko, klo + ko, logits, gg,
                                     at<int32_t>(ws, 0), s));
      SLA_CUDA(sla::launch_select_rows(logits, gg.BH * g.nqb, g, mask + h0 * rowcols,
                                       lists_from_row(*rows, size_t(h0) * g.nqb, g.nkb),
                                       scores ? scores + h0 * rowcols : nullptr, tie_count,
                                       false, s));
    }
  } else {
    SLA_CUDA(sla::launch_pool(q, k, g.dtype, qbar, kbar, nullptr, nullptr, g.BH, g.N, g.d, g.bq, g.bk,
                              s, zw, kZw, tie_count));
    const int G = mask_group_heads(g);
    for (int h0 = 0; h0 < g.BH; h0 += G) {
      Geom gg = g;
      gg.BH = std::min(G, g.BH - h0);
      SLA_CUDA(sla::launch_logits(qbar + size_t(h0) * g.nqb * g.d, kbar + size_t(h0) * g.nkb * g.d,
                                  logits, gg, s));
      SLA_CUDA(sla::launch_select_rows(logits, gg.BH * g.nqb, g, mask + h0 * rowcols,
                                       lists_from_row(*rows, size_t(h0) * g.nqb, g.nkb),
                                       scores ? scores + h0 * rowcols : nullptr, tie_count,
                                       false, s));
    }
  }
  if (cols) SLA_CUDA(sla::launch_cols_from_mask(mask, g, *cols, s));
  return SLA_OK;
}

sla_status sla_classify_scores(const sla_params* p, const float* scores,
                               int8_t* mask, const sla_block_lists* rows,
                               const sla_block_lists* cols, int32_t* tie_count,
                               void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!scores || !mask || !aligned16(scores) || !aligned16(mask) || !lists_ok(rows) ||
      (cols && !lists_ok(cols)) || (tie_count && (reinterpret_cast<uintptr_t>(tie_count) & 3u)))
    return SLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tie_count) SLA_CUDA(cudaMemsetAsync(tie_count, 0, sizeof(int32_t), s));
  SLA_CUDA(sla::launch_select_rows(scores, g.BH * g.nqb, g, mask, *rows, nullptr, tie_count, true, s));
  if (cols) SLA_CUDA(sla::launch_cols_from_mask(mask, g, *cols, s));
  return SLA_OK;
}

sla_status sla_mask_lists(const sla_params* p, const int8_t* mask,
                          const sla_block_lists* rows,
                          const sla_block_lists* cols, void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!mask || (!rows && !cols) || (rows && !lists_ok(rows)) || (cols && !lists_ok(cols)))
    return SLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rows) SLA_CUDA(sla::launch_rows_from_mask(mask, g, *rows, s));
  if (cols) SLA_CUDA(sla::launch_cols_from_mask(mask, g, *cols, s));
  return SLA_OK;
}

static bool tensor_ok(const void* x) { return x && aligned16(x); }

sla_status sla_sparse_attention(const sla_params* p, const void* q, const void* k,
                                const void* v, const sla_block_lists* rows,
                                float* o_s, float* lse, void* ws, size_t ws_bytes,
                                void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(o_s) ||
      !tensor_ok(lse) || !tensor_ok(ws) || !lists_ok(rows))
    return SLA_ERR_INVALID_ARG;
  const FwdWs w = fwd_ws(g);
  if (ws_bytes < w.total) return SLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SLA_CUDA(cudaMemsetAsync(ws, 0, kStatusBytes, s));
  const bool tc = g.dtype == SLA_BF16 && !(g.flags & SLA_FLAG_SIMT) && sla::attn_tc_supported(g);
  if (tc)
    SLA_CUDA(sla::launch_attn_tc(q, k, v, g, *rows, o_s, lse, at<int32_t>(ws, 0),
                                 at<void>(ws, w.tc), s));
  else
    SLA_CUDA(sla::launch_attn_simt(q, k, v, g, *rows, o_s, lse, s));
  return SLA_OK;
}

sla_status sla_linear_combine(const sla_params* p, const void* q, const void* k,
                              const void* v, const float* proj,
                              const sla_block_lists* rows, const float* o_s,
                              void* out, float* o_lin, void* ws, size_t ws_bytes,
                              void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(proj) ||
      !tensor_ok(o_s) || !tensor_ok(out) || !tensor_ok(ws) || !lists_ok(rows) ||
      (o_lin && !aligned16(o_lin)))
    return SLA_ERR_INVALID_ARG;
  const FwdWs w = fwd_ws(g);
  if (ws_bytes < w.total) return SLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SLA_CUDA(cudaMemsetAsync(ws, 0, kStatusBytes, s));
  if (!has_linear_branch(g)) {
    SLA_CUDA(sla::launch_combine_copy(o_s, out, o_lin, g, s));
    return SLA_OK;
  }
  if (sla::lin_tc_supported(g)) {
    SLA_CUDA(sla::launch_lin_tc(q, k, v, proj, *rows, o_s, out, o_lin, g, at<void>(ws, w.lintc),
                                at<int32_t>(ws, 0), s));
    return SLA_OK;
  }
  float* hsum = at<float>(ws, w.hsum);
  float* zsum = at<float>(ws, w.zsum);
  SLA_CUDA(sla::launch_lin_summary(k, v, g, hsum, zsum, s));
  SLA_CUDA(sla::launch_lin_apply(q, hsum, zsum, *rows, o_s, proj, out, o_lin, g, s));
  return SLA_OK;
}

static bool tc_attention(const Geom& g) {
  return g.dtype == SLA_BF16 && !(g.flags & SLA_FLAG_SIMT) && sla::attn_tc_supported(g);
}

sla_status sla_forward_prepare(const sla_params* p, const void* k, const void* v,
                               const float* proj, const sla_block_lists* rows, void* ws,
                               size_t ws_bytes, void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!tensor_ok(k) || !tensor_ok(v) || !tensor_ok(proj) || !tensor_ok(ws) || !lists_ok(rows))
    return SLA_ERR_INVALID_ARG;
  const FwdWs w = fwd_ws(g);
  if (ws_bytes < w.total) return SLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tc_attention(g)) {
    // the plan kernel, the first of the step, zeroes the status words
    SLA_CUDA(sla::launch_attn_plan(g, *rows, at<void>(ws, w.tc), s, at<int32_t>(ws, 0),
                                   static_cast<int>(kStatusBytes / sizeof(int32_t))));
  } else {
    SLA_CUDA(cudaMemsetAsync(ws, 0, kStatusBytes, s));
  }
  if (has_linear_branch(g)) {
    if (sla::lin_tc_supported(g))
      SLA_CUDA(sla::launch_lin_tc_prepare(k, v, proj, *rows, g, at<void>(ws, w.lintc),
                                          at<int32_t>(ws, 0), s));
    else
      SLA_CUDA(sla::launch_lin_summary(k, v, g, at<float>(ws, w.hsum), at<float>(ws, w.zsum), s));
  }
  return SLA_OK;
}

sla_status sla_attention_combine(const sla_params* p, const void* q, const void* k,
                                 const void* v, const float* proj,
                                 const sla_block_lists* rows, void* out, float* lse,
                                 float* o_s, float* o_lin, void* ws, size_t ws_bytes,
                                 void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(proj) ||
      !tensor_ok(out) || !tensor_ok(lse) || !tensor_ok(ws) || !lists_ok(rows) ||
      (o_s && !aligned16(o_s)) || (o_lin && !aligned16(o_lin)))
    return SLA_ERR_INVALID_ARG;
  const FwdWs w = fwd_ws(g);
  if (ws_bytes < w.total) return SLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool linear = has_linear_branch(g);
  int32_t* status = at<int32_t>(ws, 0);
  if (tc_attention(g) && (!linear || sla::lin_tc_supported(g))) {
    // one fused kernel: attention, linear apply, projection, combine
    sla::AttnOutputs o;
    o.o_s = o_s;
    o.lse = lse;
    o.out = out;
    o.o_lin = o_lin;
    sla::LinInputs li = sla::lin_tc_inputs(g, at<void>(ws, w.lintc), *rows);
    SLA_CUDA(sla::launch_attn_tc_fused(q, k, v, g, at<void>(ws, w.tc), o, linear ? &li : nullptr,
                                       status, s));
    return SLA_OK;
  }
  float* os = o_s ? o_s : at<float>(ws, w.o_s);
  if (tc_attention(g)) {
    sla::AttnOutputs o;
    o.o_s = os;
    o.lse = lse;
    o.out = nullptr;
    o.o_lin = nullptr;
    SLA_CUDA(sla::launch_attn_tc_fused(q, k, v, g, at<void>(ws, w.tc), o, nullptr, status, s));
  } else {
    SLA_CUDA(sla::launch_attn_simt(q, k, v, g, *rows, os, lse, s));
  }
  if (!linear) {
    SLA_CUDA(sla::launch_combine_copy(os, out, o_lin, g, s));
  } else {
    SLA_CUDA(sla::launch_lin_apply(q, at<float>(ws, w.hsum), at<float>(ws, w.zsum), *rows, os, proj,
                                   out, o_lin, g, s));
  }
  return SLA_OK;
}

sla_status sla_forward(const sla_params* p, const void* q, const void* k,
                       const void* v, const float* proj,
                       const sla_block_lists* rows, void* out, float* lse,
                       float* o_s, float* o_lin, void* ws, size_t ws_bytes,
                       void* stream) {
  sla_status st = sla_forward_prepare(p, k, v, proj, rows, ws, ws_bytes, stream);
  if (st != SLA_OK) return st;
  return sla_attention_combine(p, q, k, v, proj, rows, out, lse, o_s, o_lin, ws, ws_bytes, stream);
}

sla_status sla_backward(const sla_params* p, const void* q, const void* k,
                        const void* v, const float* proj, const void* dout,
                        const sla_block_lists* rows,
                        const sla_block_lists* cols, const float* o_s,
                        const float* lse, const float* o_lin, float* dq,
                        float* dk, float* dv, float* dproj, void* ws,
                        size_t ws_bytes, void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  const void* ptrs[] = {q, k, v, proj, dout, o_s, lse, o_lin, dq, dk, dv, dproj, ws};
  for (const void* x : ptrs)
    if (!x || !aligned16(x)) return SLA_ERR_INVALID_ARG;
  if (!lists_ok(rows) || !lists_ok(cols)) return SLA_ERR_INVALID_ARG;
  const BwdWs w = bwd_ws(g);
  if (ws_bytes < w.total) return SLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SLA_CUDA(cudaMemsetAsync(ws, 0, kStatusBytes, s));
  float* delta = at<float>(ws, w.delta);
  int32_t* status = static_cast<int32_t*>(ws);
  if (bwd_tc_linear(g)) {
    // Delta; the linear branch's H^M, z^M (as in the forward); the critical
    // backward with the linear branch's query side fused into its dq kernel;
    // then the linear branch's key side and dW
    SLA_CUDA(sla::launch_delta(dout, o_s, delta, g, s));
    sla::LinBwdIn lin{};
    const bool linear = has_linear_branch(g);
    if (linear)
      SLA_CUDA(sla::launch_lin_bwd_prepare(k, v, proj, *rows, o_lin, g, at<char>(ws, w.lin), status,
                                           s, &lin));
    SLA_CUDA(sla::launch_attn_bwd_tc_dq(q, k, v, dout, lse, delta, *rows, *cols, dq, g,
                                        at<char>(ws, w.plans), status, s, linear ? &lin : nullptr));
    sla::LinBwdKIn link{};
    if (linear) SLA_CUDA(sla::launch_lin_bwd_gather(*cols, g, at<char>(ws, w.lin), status, s, &link));
    SLA_CUDA(sla::launch_attn_bwd_tc_dkdv(q, k, v, dout, lse, delta, dk, dv, g, at<char>(ws, w.plans),
                                          status, s, linear ? &link : nullptr));
    SLA_CUDA(sla::launch_lin_bwd_dw(dout, o_lin, dproj, g, at<char>(ws, w.lin), status, s));
    return SLA_OK;
  }
  float* gbuf = at<float>(ws, w.gbuf);
  float* dwp = at<float>(ws, w.dwp);
  SLA_CUDA(sla::launch_bwd_prep(dout, o_s, o_lin, proj, delta, gbuf, dwp, g, s));
  if (bwd_tc_attention(g)) {
    SLA_CUDA(sla::launch_attn_bwd_tc_dq(q, k, v, dout, lse, delta, *rows, *cols, dq, g,
                                        at<char>(ws, w.plans), static_cast<int32_t*>(ws), s, nullptr));
    SLA_CUDA(sla::launch_attn_bwd_tc_dkdv(q, k, v, dout, lse, delta, dk, dv, g, at<char>(ws, w.plans),
                                          static_cast<int32_t*>(ws), s, nullptr));
  } else {
    SLA_CUDA(sla::launch_attn_bwd_dq(q, k, v, dout, lse, delta, *rows, dq, g, s));
    SLA_CUDA(sla::launch_attn_bwd_dkdv(q, k, v, dout, lse, delta, *cols, dk, dv, g, s));
  }
  if (has_linear_branch(g)) {
    float* hsum = at<float>(ws, w.hsum);
    float* zsum = at<float>(ws, w.zsum);
    float* dhm = at<float>(ws, w.dhm);
    float* dzm = at<float>(ws, w.dzm);
    SLA_CUDA(sla::launch_lin_summary(k, v, g, hsum, zsum, s));
    SLA_CUDA(sla::launch_lin_bwd_q(q, hsum, zsum, *rows, gbuf, o_lin, dq, dhm, dzm, g, s));
    SLA_CUDA(sla::launch_lin_bwd_kv(k, v, dhm, dzm, *cols, dk, dv, g, s));
  }
  SLA_CUDA(sla::launch_bwd_dw_reduce(dwp, dproj, g, s));
  return SLA_OK;
}

int32_t sla_forward_uses_tensor_cores(const sla_params* p) {
  Geom g;
  if (make_geom(p, &g) != SLA_OK) return -1;
  return (g.dtype == SLA_BF16 && !(g.flags & SLA_FLAG_SIMT) && sla::attn_tc_supported(g)) ? 1 : 0;
}

sla_status sla_block_importance(const sla_params* p, const void* q, const void* k,
                                float* importance, void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!q || !k || !importance || !aligned16(q) || !aligned16(k) || !aligned16(importance))
    return SLA_ERR_INVALID_ARG;
  SLA_CUDA(sla::launch_block_importance(q, k, importance, g, static_cast<cudaStream_t>(stream)));
  return SLA_OK;
}

sla_status sla_mask_recall(const sla_params* p, const int8_t* mask, const float* importance,
                           int32_t* counts, void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!mask || !importance || !counts || !aligned16(mask) || !aligned16(importance) ||
      !aligned16(counts))
    return SLA_ERR_INVALID_ARG;
  SLA_CUDA(sla::launch_mask_recall(mask, importance, g, counts, static_cast<cudaStream_t>(stream)));
  return SLA_OK;
}

sla_status sla_tile_order(int32_t F, int32_t R, int32_t C, int32_t tf, int32_t tr, int32_t tc,
                          int32_t* perm, void* stream) {
  if (F < 1 || R < 1 || C < 1 || tf < 1 || tr < 1 || tc < 1 || !perm ||
      (reinterpret_cast<uintptr_t>(perm) & 3u))
    return SLA_ERR_INVALID_ARG;
  if (int64_t(F) * R * C >= (int64_t(1) << 31)) return SLA_ERR_UNSUPPORTED;
  SLA_CUDA(sla::launch_tile_order(F, R, C, std::min(tf, F), std::min(tr, R), std::min(tc, C), perm,
                                  static_cast<cudaStream_t>(stream)));
  return SLA_OK;
}

sla_status sla_permute_tokens(const sla_params* p, const void* src, void* dst, const int32_t* perm,
                              int32_t elem_bytes, int32_t inverse, void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!tensor_ok(src) || !tensor_ok(dst) || !perm || (reinterpret_cast<uintptr_t>(perm) & 3u) ||
      (elem_bytes != 2 && elem_bytes != 4) || (inverse != 0 && inverse != 1))
    return SLA_ERR_INVALID_ARG;
  const int row_bytes = g.d * elem_bytes;
  const uintptr_t a = reinterpret_cast<uintptr_t>(src), b = reinterpret_cast<uintptr_t>(dst);
  const uintptr_t bytes = static_cast<uintptr_t>(g.BH) * g.N * row_bytes;
  if (a < b + bytes && b < a + bytes) return SLA_ERR_INVALID_ARG;  // overlapping
  SLA_CUDA(sla::launch_permute_rows(src, dst, perm, static_cast<sla::i64>(g.BH) * g.N, g.N, row_bytes,
                                    inverse != 0, static_cast<cudaStream_t>(stream)));
  return SLA_OK;
}

sla_status sla_check_device_status(void* ws, void* stream) {
  if (!ws) return SLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SLA_ERR_CUDA;
  int32_t word = 0;
  if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SLA_ERR_CUDA;
  return word == 0 ? SLA_OK : static_cast<sla_status>(word);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation variant of sla_sparse_attention.
//
// Its scratch (the attention plan, and the status word when the caller gives
// none) lives in one file-scope device array of kNoAllocBytes.  Host code
// only ever sees a host-side stand-in for the array's name, so the device
// address is looked up once per device, with that device current, by the
// first call on it, and cached together with the id of the context it
// belongs to; a later call under another context (after cudaDeviceReset,
// the module is loaded again and the array may move) looks it up again.

#include <mutex>

namespace {
constexpr size_t kNoAllocBytes = size_t(16) << 20;  // 16 MiB
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};
unsigned long long g_noalloc_ctx[kNoAllocMaxDevices] = {};
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

extern "C" sla_status sla_sparse_attention_noalloc(const sla_params* p, const void* q,
                                                   const void* k, const void* v,
                                                   const sla_block_lists* rows, float* o_s,
                                                   float* lse, int32_t* status,
                                                   void* stream) {
  Geom g;
  sla_status st = make_geom(p, &g);
  if (st != SLA_OK) return st;
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(o_s) || !tensor_ok(lse) ||
      !lists_ok(rows) || (status && (reinterpret_cast<uintptr_t>(status) & 3u)))
    return SLA_ERR_INVALID_ARG;
  const bool tc = g.dtype == SLA_BF16 && !(g.flags & SLA_FLAG_SIMT) && sla::attn_tc_supported(g);
  const size_t need = kStatusBytes + (tc ? align_up(sla::attn_tc_scratch_bytes(g)) : 0);
  if (need > kNoAllocBytes) return SLA_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SLA_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return SLA_ERR_UNSUPPORTED;
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    unsigned long long ctx = 0;
    const bool have_ctx = sla::current_context_id(&ctx);
    if (!g_noalloc_addr[dev] || (have_ctx && ctx != g_noalloc_ctx[dev])) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr)
        return SLA_ERR_CUDA;
      g_noalloc_addr[dev] = addr;
      // (the first call creates the context when there is none yet)
      g_noalloc_ctx[dev] = sla::current_context_id(&ctx) ? ctx : 0;
    }
    base = g_noalloc_addr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* word = status ? status : static_cast<int32_t*>(base);
  SLA_CUDA(cudaMemsetAsync(word, 0, sizeof(int32_t), s));  // the only state that must start at 0
  if (tc)
    SLA_CUDA(sla::launch_attn_tc(q, k, v, g, *rows, o_s, lse, word,
                                 static_cast<char*>(base) + kStatusBytes, s));
  else
    SLA_CUDA(sla::launch_attn_simt(q, k, v, g, *rows, o_s, lse, s));
  return SLA_OK;
}

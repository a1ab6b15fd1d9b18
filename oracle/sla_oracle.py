"""Plain, slow, float64 CPU oracle for hybrid block-sparse + linear attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test-suite, the package's
smoke check and the benchmark's CPU-baseline leg may import this module.  It
shares no code, tables or helpers with the CUDA library; it takes plain arrays
and returns plain numpy arrays, computed in float64 with numpy only.

Sources (web pages on the method; they give words, not formulas):

* SLA post ("Selective Linear Attention", machinelearning_books channel,
  list "В чём идея" / "the idea"): attention is split into critical,
  negligible and intermediate (marginal) parts; critical goes through
  FlashAttention (exact softmax attention), negligible is skipped, marginal
  goes through linear attention; a fast mean-pooling step labels the blocks
  in advance.  Same post, list "Результаты" / "results": a short fine-tune
  suffices, so a backward pass is needed.
* NABLA post (SberAIScience channel, numbered points 1-4): Q and K are
  compressed per block, the important blocks are chosen through the
  cumulative distribution function of the softmax, and a block is important
  when the blocks kept sum above the adaptive threshold 1 - thr; compute runs
  only on those blocks.
* The workload statement fixes phi = elu + 1 for the linear branch and a
  d x d output projection W applied to it, top-k fractions for the SLA split
  and the CDF rule for the NABLA split.
* Veda article (mlllm.io, sections "Контекст" / context and the users'
  section): a mask is evaluated by how well it reproduces dense attention,
  max-pooled over tiles, and by its recall; the mask-quality functions at
  the end follow it.

Readings taken where the pages are silent.  Each is the plainest choice the
rest of the pages support; readings 1, 4 (the rounding of the counts), 5 (the
index tie-break) and the diagonal block not being forced critical are
conventions the pages do not fix, so no page value pins them:

1. A block that ends at N (ragged tail) is pooled over its real tokens only.
2. Scores and attention use the scale s = 1/sqrt(d) unless a scale is given.
3. The block-score softmax runs over key blocks, one row per query block.
4. Top-k counts: n_c = ceil(f_c * Nkb), n_m = min(ceil(f_m * Nkb), Nkb - n_c),
   with f * Nkb taken with a 1e-9 slack against the representation error of
   the fraction (0.07 * 100 is 7.000000000000001 in binary64).
5. Ranks order blocks by score descending, ties by block index ascending;
   critical = the first n_c ranks, marginal = the next n_m ranks.
6. CDF rule: walking from the lowest rank upward, a block is dropped while the
   running tail sum including it stays strictly below thr; everything above
   the first block that fails is kept (critical).  This is the smallest prefix
   of ranks whose mass exceeds 1 - thr; at thr = 0 nothing is dropped.  The
   top rank is always kept.  An optional marginal fraction marks the next
   n_m ranks after the kept set.
7. phi(x) = x + 1 for x > 0, exp(x) otherwise; no epsilon in the normaliser
   (phi > 0); an empty marginal set gives a zero linear output; W is applied
   after the normalisation, without bias.
8. Combine: out = O_s + O_lin @ W, with O_s normalised over critical keys only.
9. A row with no critical block has O_s = 0 and LSE = -inf.
10. Backward: the mask is a constant; standard softmax-attention gradients for
    the critical part; chain rule through phi, the normaliser and W for the
    linear part; dW sums over batch, heads and tokens.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Tuple

import numpy as np

CRITICAL = 2
MARGINAL = 1
NEGLIGIBLE = 0

# --------------------------------------------------------------------------
# block geometry


def n_blocks(n: int, block: int) -> int:
    return (n + block - 1) // block


def block_range(i: int, n: int, block: int) -> Tuple[int, int]:
    return i * block, min((i + 1) * block, n)


def f64(x) -> np.ndarray:
    """Upcast anything array-like (numpy, or a CPU torch tensor) to float64."""
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# a1: mean pooling (SLA idea list: "a fast mean-pooling step labels blocks";
# NABLA point 2: "compresses Query and Key")


def pool_blocks(x, block: int) -> np.ndarray:
    """Mean of each block's real tokens: ``[..., N, d] -> [..., Nb, d]``."""
    x = f64(x)
    n = x.shape[-2]
    nb = n_blocks(n, block)
    out = np.empty(x.shape[:-2] + (nb, x.shape[-1]), dtype=np.float64)
    for i in range(nb):
        a, b = block_range(i, n, block)
        out[..., i, :] = x[..., a:b, :].sum(axis=-2) / (b - a)
    return out


# --------------------------------------------------------------------------
# a2: pooled block scores (NABLA point 2: softmax over the compressed QK^T)


def block_scores(qbar, kbar, scale: float) -> np.ndarray:
    """Row softmax over key blocks of ``scale * qbar @ kbar^T``."""
    qbar, kbar = f64(qbar), f64(kbar)
    logits = scale * np.matmul(qbar, np.swapaxes(kbar, -1, -2))
    logits = logits - logits.max(axis=-1, keepdims=True)
    e = np.exp(logits)
    return e / e.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# a3: classification


def topk_counts(frac_crit: float, frac_marg: float, nkb: int) -> Tuple[int, int]:
    """Reading 4: critical and marginal block counts per row."""
    def count(f):
        return max(0, min(nkb, math.ceil(f * nkb - 1e-9)))
    n_c = count(frac_crit)
    n_m = min(nkb - n_c, count(frac_marg))
    return n_c, n_m


def rank_order(p_row: np.ndarray) -> np.ndarray:
    """Reading 5: block indices sorted by score descending, index ascending."""
    idx = np.arange(p_row.shape[0])
    return np.lexsort((idx, -p_row))


def _rel_gap(hi: float, lo: float) -> float:
    """Score gap at a cut, relative to the higher score (0 for equal scores)."""
    return (hi - lo) / hi if hi > 0 else 0.0


def classify_topk_row(p_row, n_c: int, n_m: int) -> Tuple[np.ndarray, float]:
    """Label one row by ranks; also return the row's tie margin: the smallest
    score gap at a cut (last block of a class vs the first block below it),
    relative to the higher of the two scores."""
    p_row = f64(p_row)
    nkb = p_row.shape[0]
    order = rank_order(p_row)
    labels = np.zeros(nkb, dtype=np.int8)
    labels[order[:n_c]] = CRITICAL
    labels[order[n_c:n_c + n_m]] = MARGINAL
    ps = p_row[order]
    margin = math.inf
    for cut in (n_c, n_c + n_m):
        if 0 < cut < nkb and not (cut == n_c + n_m and n_m == 0):
            margin = min(margin, _rel_gap(ps[cut - 1], ps[cut]))
    return labels, margin


def classify_cdf_row(p_row, thr: float, n_m: int = 0) -> Tuple[np.ndarray, float]:
    """Reading 6 (NABLA points 2-3): keep the smallest top-ranked set whose
    mass exceeds 1 - thr.

    Walk from the lowest rank upward; a block is dropped while the tail sum
    including it is strictly below ``thr``.  Returns labels and the row's
    margin: the smaller of the distances of the two decisive tail sums from
    ``thr`` (absolute, on the unit mass scale) and the score gaps at the cut(s)
    (relative to the higher score)."""
    p_row = f64(p_row)
    nkb = p_row.shape[0]
    order = rank_order(p_row)
    ps = p_row[order]
    # Running tail sums of the walk: tails[r] = ps[r] + ps[r+1] + ... summed
    # from the lowest rank upward (np.cumsum adds in exactly that order).  The
    # tail sums never decrease as r falls, so "drop while the tail including
    # the block stays below thr" drops exactly the ranks with tails[r] < thr;
    # the top rank is never dropped.
    tails = np.cumsum(ps[::-1])[::-1]
    kept = max(1, int(np.count_nonzero(tails >= thr)))
    tail = float(tails[kept]) if kept < nkb else 0.0
    # tail sums at the two ranks that decide the cut
    t_kept_last = tail + ps[kept - 1]        # tail sum including last kept
    # at thr <= 0 no tail sum can fall below thr, so no decision is close
    margin = abs(t_kept_last - thr) if (kept > 1 and thr > 0) else math.inf
    if kept < nkb:
        margin = min(margin, abs(thr - tail), _rel_gap(ps[kept - 1], ps[kept]))
    labels = np.zeros(nkb, dtype=np.int8)
    labels[order[:kept]] = CRITICAL
    n_m = min(n_m, nkb - kept)
    labels[order[kept:kept + n_m]] = MARGINAL
    if n_m > 0 and kept + n_m < nkb:
        margin = min(margin, _rel_gap(ps[kept + n_m - 1], ps[kept + n_m]))
    return labels, margin


def classify(p, mode: str, frac_crit=0.0, frac_marg=0.0, thr=0.0
             ) -> Tuple[np.ndarray, np.ndarray]:
    """Label every row of ``p [..., Nqb, Nkb]``; returns (mask int8, margins)."""
    p = f64(p)
    nkb = p.shape[-1]
    rows = p.reshape(-1, nkb)
    mask = np.zeros(rows.shape, dtype=np.int8)
    margins = np.empty(rows.shape[0])
    n_c, n_m = topk_counts(frac_crit, frac_marg, nkb)
    for r in range(rows.shape[0]):
        if mode == "topk":
            mask[r], margins[r] = classify_topk_row(rows[r], n_c, n_m)
        elif mode == "cdf":
            mask[r], margins[r] = classify_cdf_row(rows[r], thr, n_m)
        else:
            raise ValueError(mode)
    return mask.reshape(p.shape), margins.reshape(p.shape[:-1])


def build_mask(q, k, block_q: int, block_k: int, mode: str, frac_crit=0.0,
               frac_marg=0.0, thr=0.0, scale: Optional[float] = None) -> Dict:
    """a1-a3: pool, score, classify.  ``q, k``: ``[B, H, N, d]``."""
    q, k = f64(q), f64(k)
    d = q.shape[-1]
    s = 1.0 / math.sqrt(d) if scale is None else scale
    qbar = pool_blocks(q, block_q)
    kbar = pool_blocks(k, block_k)
    p = block_scores(qbar, kbar, s)
    mask, margins = classify(p, mode, frac_crit, frac_marg, thr)
    return dict(qbar=qbar, kbar=kbar, scores=p, mask=mask, margins=margins)


def mask_lists(mask) -> Tuple[List, List]:
    """Per-row ascending lists of critical and marginal key blocks."""
    mask = np.asarray(mask)
    rows = mask.reshape(-1, mask.shape[-1])
    crit = [np.nonzero(r == CRITICAL)[0] for r in rows]
    marg = [np.nonzero(r == MARGINAL)[0] for r in rows]
    return crit, marg


# --------------------------------------------------------------------------
# a4: exact softmax attention over each query block's critical key blocks
# (SLA idea list: critical -> FlashAttention; negligible -> skipped)


def _block_tokens(blocks, n: int, block: int) -> np.ndarray:
    if len(blocks) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(*block_range(int(j), n, block))
                           for j in blocks])


def sparse_attention_rows(q_rows, k, v, crit_blocks, block_k: int, scale: float):
    """Softmax attention of the query rows ``q_rows [T, d]`` over the keys of
    ``crit_blocks`` (one head).  Returns (O_s [T, d], LSE [T])."""
    q_rows, k, v = f64(q_rows), f64(k), f64(v)
    t = q_rows.shape[0]
    keys = _block_tokens(crit_blocks, k.shape[0], block_k)
    if keys.size == 0:
        return np.zeros((t, v.shape[1])), np.full(t, -np.inf)
    logits = scale * (q_rows @ k[keys].T)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    den = e.sum(axis=1, keepdims=True)
    o = (e / den) @ v[keys]
    lse = (m + np.log(den))[:, 0]
    return o, lse


def sparse_attention(q, k, v, mask, block_q: int, block_k: int,
                     scale: Optional[float] = None):
    """a4 over ``[B, H, N, d]`` with a block mask ``[B, H, Nqb, Nkb]``."""
    q, k, v = f64(q), f64(k), f64(v)
    B, H, N, d = q.shape
    s = 1.0 / math.sqrt(d) if scale is None else scale
    mask = np.asarray(mask)
    o = np.zeros_like(q)
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(n_blocks(N, block_q)):
                a, e = block_range(i, N, block_q)
                crit = np.nonzero(mask[b, h, i] == CRITICAL)[0]
                o[b, h, a:e], lse[b, h, a:e] = sparse_attention_rows(
                    q[b, h, a:e], k[b, h], v[b, h], crit, block_k, s)
    return o, lse


# --------------------------------------------------------------------------
# a5-a7: linear attention on marginal blocks (SLA idea list: marginal ->
# linear attention; phi = elu + 1 and the d x d projection per the workload)


def phi(x):
    x = f64(x)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def dphi(x):
    x = f64(x)
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def linear_summaries(k, v, block_k: int):
    """Per key block j: H_j = sum_t phi(k_t)^T v_t  (d x d) and
    z_j = sum_t phi(k_t).  ``k, v``: ``[..., N, d]``."""
    k, v = f64(k), f64(v)
    n, d = k.shape[-2], k.shape[-1]
    nb = n_blocks(n, block_k)
    hsum = np.empty(k.shape[:-2] + (nb, d, d))
    zsum = np.empty(k.shape[:-2] + (nb, d))
    pk = phi(k)
    for j in range(nb):
        a, b = block_range(j, n, block_k)
        hsum[..., j, :, :] = np.matmul(np.swapaxes(pk[..., a:b, :], -1, -2),
                                       v[..., a:b, :])
        zsum[..., j, :] = pk[..., a:b, :].sum(axis=-2)
    return hsum, zsum


def linear_attention_rows(q_rows, hsum, zsum, marg_blocks):
    """Linear attention of ``q_rows [T, d]`` over the summed summaries of
    ``marg_blocks`` (one head).  Returns O_lin [T, d] (zero if none)."""
    q_rows = f64(q_rows)
    if len(marg_blocks) == 0:
        return np.zeros_like(q_rows)
    hm = hsum[marg_blocks].sum(axis=0)
    zm = zsum[marg_blocks].sum(axis=0)
    f = phi(q_rows)
    return (f @ hm) / (f @ zm)[:, None]


def linear_summaries_of(k, v, blocks, block_k: int):
    """Summaries of the listed key blocks only (one head): ``{j: (H_j, z_j)}``."""
    k, v = f64(k), f64(v)
    n = k.shape[0]
    out = {}
    for j in blocks:
        a, b = block_range(int(j), n, block_k)
        pk = phi(k[a:b])
        out[int(j)] = (pk.T @ v[a:b], pk.sum(axis=0))
    return out


def forward_rows(q, k, v, proj, mask_row, block_i: int, block_q: int,
                 block_k: int, scale: Optional[float] = None) -> Dict:
    """a4-a7 for the tokens of one query block of one head (``q, k, v``:
    ``[N, d]``), from that block's mask row.  Used to check sampled rows of
    workloads too large for the whole oracle."""
    q = f64(q)
    n, d = q.shape
    s = 1.0 / math.sqrt(d) if scale is None else scale
    a, e = block_range(block_i, n, block_q)
    mask_row = np.asarray(mask_row)
    crit = np.nonzero(mask_row == CRITICAL)[0]
    marg = np.nonzero(mask_row == MARGINAL)[0]
    o_s, lse = sparse_attention_rows(q[a:e], k, v, crit, block_k, s)
    if len(marg):
        summ = linear_summaries_of(k, v, marg, block_k)
        hm = sum(summ[int(j)][0] for j in marg)
        zm = sum(summ[int(j)][1] for j in marg)
        f = phi(q[a:e])
        o_lin = (f @ hm) / (f @ zm)[:, None]
    else:
        o_lin = np.zeros_like(q[a:e])
    return dict(out=o_s + o_lin @ f64(proj), o_s=o_s, lse=lse, o_lin=o_lin)


def linear_attention(q, k, v, mask, block_q: int, block_k: int):
    q = f64(q)
    B, H, N, d = q.shape
    hsum, zsum = linear_summaries(k, v, block_k)
    mask = np.asarray(mask)
    o = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            for i in range(n_blocks(N, block_q)):
                a, e = block_range(i, N, block_q)
                marg = np.nonzero(mask[b, h, i] == MARGINAL)[0]
                o[b, h, a:e] = linear_attention_rows(q[b, h, a:e], hsum[b, h],
                                                     zsum[b, h], marg)
    return o


def forward(q, k, v, proj, mask, block_q: int, block_k: int,
            scale: Optional[float] = None) -> Dict:
    """a4-a7: out = O_s + O_lin @ W.  Returns out, o_s, lse, o_lin."""
    o_s, lse = sparse_attention(q, k, v, mask, block_q, block_k, scale)
    o_lin = linear_attention(q, k, v, mask, block_q, block_k)
    out = o_s + o_lin @ f64(proj)
    return dict(out=out, o_s=o_s, lse=lse, o_lin=o_lin)


# --------------------------------------------------------------------------
# a8: backward (SLA results list: a short fine-tune suffices)


def backward(q, k, v, proj, mask, dout, block_q: int, block_k: int,
             scale: Optional[float] = None, saved: Optional[Dict] = None) -> Dict:
    """Gradients of sum(out * dout) w.r.t. q, k, v and W; the mask is fixed."""
    q, k, v, w, dout = f64(q), f64(k), f64(v), f64(proj), f64(dout)
    B, H, N, d = q.shape
    s = 1.0 / math.sqrt(d) if scale is None else scale
    if saved is None:
        saved = forward(q, k, v, w, mask, block_q, block_k, s)
    o_s, lse, o_lin = saved["o_s"], saved["lse"], saved["o_lin"]
    mask = np.asarray(mask)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    # out = o_s + o_lin @ W
    dw = np.einsum("bhta,bhtc->ac", o_lin, dout)
    g = dout @ w.T                      # dL/dO_lin
    hsum, zsum = linear_summaries(k, v, block_k)
    for b in range(B):
        for h in range(H):
            dh = np.zeros_like(hsum[b, h])
            dz = np.zeros_like(zsum[b, h])
            for i in range(n_blocks(N, block_q)):
                a, e = block_range(i, N, block_q)
                # critical part: standard softmax-attention backward
                crit = np.nonzero(mask[b, h, i] == CRITICAL)[0]
                keys = _block_tokens(crit, N, block_k)
                if keys.size:
                    qi = q[b, h, a:e]
                    p = np.exp(s * (qi @ k[b, h, keys].T) - lse[b, h, a:e, None])
                    do = dout[b, h, a:e]
                    dp = do @ v[b, h, keys].T
                    dd = (do * o_s[b, h, a:e]).sum(axis=1, keepdims=True)
                    ds = p * (dp - dd)
                    dq[b, h, a:e] += s * ds @ k[b, h, keys]
                    dk[b, h, keys] += s * ds.T @ qi
                    dv[b, h, keys] += p.T @ do
                # linear part
                marg = np.nonzero(mask[b, h, i] == MARGINAL)[0]
                if len(marg):
                    hm = hsum[b, h][marg].sum(axis=0)
                    zm = zsum[b, h][marg].sum(axis=0)
                    qi = q[b, h, a:e]
                    f = phi(qi)
                    den = f @ zm                           # [T]
                    num = f @ hm                           # [T, d]
                    gi = g[b, h, a:e]
                    dnum = gi / den[:, None]
                    dden = -(gi * num).sum(axis=1) / den ** 2
                    df = dnum @ hm.T + dden[:, None] * zm[None, :]
                    dq[b, h, a:e] += df * dphi(qi)
                    dhm = f.T @ dnum
                    dzm = f.T @ dden
                    dh[marg] += dhm
                    dz[marg] += dzm
            # scatter summary gradients to each key block's tokens
            for j in range(n_blocks(N, block_k)):
                a, e = block_range(j, N, block_k)
                kj = k[b, h, a:e]
                pk = phi(kj)
                dpk = v[b, h, a:e] @ dh[j].T + dz[j][None, :]
                dk[b, h, a:e] += dpk * dphi(kj)
                dv[b, h, a:e] += pk @ dh[j]
    return dict(dq=dq, dk=dk, dv=dv, dproj=dw)


# --------------------------------------------------------------------------
# mask quality: the selection against max-pooled dense attention
#
# Veda article (mlllm.io, section "Контекст" / context): what a block mask
# has to reproduce is the structure of dense attention, and the reference
# it is distilled toward is the dense attention max-pooled over tiles; the
# article's user section reports the predictor's recall.  Below: the pooled
# reference and the share of it a mask keeps.


def max_pooled_attention(q, k, block_q: int, block_k: int,
                         scale: Optional[float] = None) -> np.ndarray:
    """Importance of (query block i, key block j): the largest dense softmax
    probability between a real token of block i and a real key of block j,
    each query token's softmax running over all N keys.
    ``q, k [B, H, N, d] -> [B, H, Nqb, Nkb]``."""
    q, k = f64(q), f64(k)
    B, H, N, d = q.shape
    s = 1.0 / math.sqrt(d) if scale is None else scale
    nqb, nkb = n_blocks(N, block_q), n_blocks(N, block_k)
    out = np.zeros((B, H, nqb, nkb))
    for b in range(B):
        for h in range(H):
            logits = s * (q[b, h] @ k[b, h].T)                  # [N, N]
            e = np.exp(logits - logits.max(axis=1, keepdims=True))
            p = e / e.sum(axis=1, keepdims=True)
            for i in range(nqb):
                t0, t1 = block_range(i, N, block_q)
                col_max = p[t0:t1].max(axis=0)                  # [N]
                for j in range(nkb):
                    s0, s1 = block_range(j, N, block_k)
                    out[b, h, i, j] = col_max[s0:s1].max()
    return out


def mask_recall_counts(mask, importance) -> Tuple[int, int, int, int]:
    """Per row (query block) with c critical blocks, the reference set is the
    c blocks of largest importance (ties by lower index, the order of
    reading 5); hits are the reference blocks the mask marks critical.  The
    same with the kept set (critical or marginal) and its size.  Returns
    (critical hits, critical total, kept hits, kept total) over all rows;
    recall = hits / total."""
    mask = np.asarray(mask)
    imp = np.asarray(importance, dtype=np.float64)
    nkb = mask.shape[-1]
    m2 = mask.reshape(-1, nkb)
    i2 = imp.reshape(-1, nkb)
    ch = ct = kh = kt = 0
    for row in range(m2.shape[0]):
        order = rank_order(i2[row])
        c = int((m2[row] == CRITICAL).sum())
        ck = int((m2[row] != NEGLIGIBLE).sum())
        ch += int((m2[row][order[:c]] == CRITICAL).sum())
        kh += int((m2[row][order[:ck]] != NEGLIGIBLE).sum())
        ct += c
        kt += ck
    return ch, ct, kh, kt


# --------------------------------------------------------------------------
# token order in 3D tiles
#
# Veda article (mlllm.io, sections "Что произошло" / what happened and
# "Контекст" / context): attention is selected over tiles of tokens, with
# tile shapes fitted per head and layer.  Blocks of consecutive tokens then
# cover compact spatio-temporal boxes instead of raster strips.


def tile_order(grid: Tuple[int, int, int], tile: Tuple[int, int, int]) -> np.ndarray:
    """Token order of 3D tiles over a raster grid (F, R, C), token
    t = (f R + r) C + c: tiles in raster order over the tile grid, tokens in
    raster order inside each tile, tiles at the far edges partial.  Returns
    ``perm`` with ``perm[n]`` = raster index of the n-th token in tile order
    (``x[..., perm, :]`` reorders a ``[..., N, d]`` tensor)."""
    F, R, C = grid
    tf, tr, tc = tile
    idx = np.arange(F * R * C).reshape(F, R, C)
    parts = []
    for f0 in range(0, F, tf):
        for r0 in range(0, R, tr):
            for c0 in range(0, C, tc):
                parts.append(idx[f0:f0 + tf, r0:r0 + tr, c0:c0 + tc].reshape(-1))
    return np.concatenate(parts)

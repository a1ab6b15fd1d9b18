"""Token-level brute force for hybrid attention, used only to pin the oracle.

It is written independently of the oracle: the block mask is expanded to a
per-token pair label, and every output is computed token by token from that
label -- softmax over the critical keys, and linear attention as the direct
sum over marginal keys ``sum_u phi(q).phi(k_u) v_u / sum_u phi(q).phi(k_u)``
(no per-block summaries, no pooled lists).  The torch variant is the same
formulation in float64 so that autograd gives reference gradients.
"""

import math

import numpy as np
import torch


def pair_labels(mask_bh, n, block_q, block_k):
    """Expand a ``[Nqb, Nkb]`` block mask to ``[N, N]`` token-pair labels."""
    lab = np.empty((n, n), dtype=np.int8)
    for t in range(n):
        for u in range(n):
            lab[t, u] = mask_bh[t // block_q, u // block_k]
    return lab


def elu1(x):
    return x + 1.0 if x > 0 else math.exp(x)


def brute_forward(q, k, v, w, mask, block_q, block_k, scale):
    """Pure-Python loops over tokens and keys (tiny inputs only)."""
    q, k, v, w = (np.asarray(a, dtype=np.float64) for a in (q, k, v, w))
    B, H, N, d = q.shape
    out = np.zeros_like(q)
    o_s = np.zeros_like(q)
    o_lin = np.zeros_like(q)
    lse = np.full((B, H, N), -np.inf)
    for b in range(B):
        for h in range(H):
            lab = pair_labels(mask[b, h], N, block_q, block_k)
            for t in range(N):
                crit = [u for u in range(N) if lab[t, u] == 2]
                marg = [u for u in range(N) if lab[t, u] == 1]
                if crit:
                    sc = [scale * sum(q[b, h, t, c] * k[b, h, u, c] for c in range(d))
                          for u in crit]
                    m = max(sc)
                    ex = [math.exp(x - m) for x in sc]
                    tot = sum(ex)
                    for c in range(d):
                        o_s[b, h, t, c] = sum(e * v[b, h, u, c]
                                              for e, u in zip(ex, crit)) / tot
                    lse[b, h, t] = m + math.log(tot)
                if marg:
                    fq = [elu1(x) for x in q[b, h, t]]
                    wts = []
                    for u in marg:
                        fk = [elu1(x) for x in k[b, h, u]]
                        wts.append(sum(a * bb for a, bb in zip(fq, fk)))
                    den = sum(wts)
                    for c in range(d):
                        o_lin[b, h, t, c] = sum(wt * v[b, h, u, c]
                                                for wt, u in zip(wts, marg)) / den
                for c in range(d):
                    out[b, h, t, c] = o_s[b, h, t, c] + sum(
                        o_lin[b, h, t, a] * w[a, c] for a in range(d))
    return dict(out=out, o_s=o_s, lse=lse, o_lin=o_lin)


def torch_token_forward(q, k, v, w, mask, block_q, block_k, scale):
    """The same token-level formulation, vectorised in torch float64 so that
    autograd can differentiate it (mask fixed)."""
    B, H, N, d = q.shape
    outs = []
    for b in range(B):
        heads = []
        for h in range(H):
            lab = torch.as_tensor(pair_labels(np.asarray(mask[b, h]), N,
                                              block_q, block_k))
            crit = lab == 2
            marg = (lab == 1).to(torch.float64)
            logits = scale * q[b, h] @ k[b, h].T
            logits = logits.masked_fill(~crit, float("-inf"))
            has_c = crit.any(dim=1, keepdim=True)
            logits = torch.where(has_c, logits, torch.zeros_like(logits))
            p = torch.softmax(logits, dim=1) * has_c
            o_s = p @ v[b, h]
            fq = torch.where(q[b, h] > 0, q[b, h] + 1, torch.exp(q[b, h].clamp(max=0)))
            fk = torch.where(k[b, h] > 0, k[b, h] + 1, torch.exp(k[b, h].clamp(max=0)))
            a = (fq @ fk.T) * marg
            den = a.sum(dim=1, keepdim=True)
            has_m = den > 0
            o_lin = torch.where(has_m, (a @ v[b, h]) / torch.where(has_m, den, torch.ones_like(den)),
                                torch.zeros_like(o_s))
            heads.append(o_s + o_lin @ w)
        outs.append(torch.stack(heads))
    return torch.stack(outs)

"""Python binding of libsla (hybrid block-sparse + linear attention, sm_100a).

Two layers, both argument marshalling only -- every step of the computation
runs in the CUDA kernels of ``libsla.so``:

* ``sla_*`` functions mirror the C entry points of ``include/sla.h`` one to
  one and take raw integers for device pointers and the stream;
* ``build_mask`` / ``forward`` / ``backward`` accept torch CUDA tensors,
  allocate outputs and workspace with torch (device memory and streams are
  the only things torch provides here) and call the C entry points on the
  current torch stream.

There is no fallback: if the library is missing or fails to load, importing
the tensor helpers raises.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

from .synth import Workload

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsla.so")

SLA_OK, SLA_ERR_INVALID_ARG, SLA_ERR_UNSUPPORTED, SLA_ERR_WORKSPACE, SLA_ERR_CUDA, SLA_ERR_TIMEOUT = range(6)
SLA_F32, SLA_BF16 = 0, 1
SLA_MASK_TOPK, SLA_MASK_CDF = 0, 1
SLA_OP_MASK, SLA_OP_FORWARD, SLA_OP_BACKWARD = 0, 1, 2
SLA_FLAG_SIMT = 1
SLA_FLAG_DEBUG_TIMEOUT = 2
# SLA_DEBUG_WITHHOLD(kernel): which tensor-core kernel withholds a load under
# SLA_FLAG_DEBUG_TIMEOUT
(SLA_WITHHOLD_ATTENTION, SLA_WITHHOLD_LOGITS, SLA_WITHHOLD_SUMMARIES, SLA_WITHHOLD_GATHER,
 SLA_WITHHOLD_BWD_DQ, SLA_WITHHOLD_BWD_DKDV) = range(6)


def SLA_DEBUG_WITHHOLD(kernel: int) -> int:
    return kernel << 8
# block labels in the int8 mask
CRITICAL, MARGINAL, NEGLIGIBLE = 2, 1, 0

# Entry points declared in include/sla.h (checked by the test-suite).
EXPORTS = ("sla_abi_version", "sla_status_string", "sla_validate",
           "sla_workspace_size", "sla_build_mask", "sla_classify_scores",
           "sla_mask_lists",
           "sla_forward", "sla_forward_prepare", "sla_attention_combine",
           "sla_sparse_attention", "sla_sparse_attention_noalloc",
           "sla_linear_combine",
           "sla_backward", "sla_forward_uses_tensor_cores",
           "sla_block_importance", "sla_mask_recall",
           "sla_tile_order", "sla_permute_tokens",
           "sla_check_device_status")


class sla_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("block_q", ctypes.c_int32),
                ("block_k", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("mask_mode", ctypes.c_int32), ("frac_crit", ctypes.c_double),
                ("frac_marg", ctypes.c_double), ("thr", ctypes.c_double),
                ("scale", ctypes.c_float), ("flags", ctypes.c_int32)]


class sla_block_lists(ctypes.Structure):
    _fields_ = [("crit_cnt", ctypes.c_void_p), ("crit_idx", ctypes.c_void_p),
                ("marg_cnt", ctypes.c_void_p), ("marg_idx", ctypes.c_void_p)]


class SlaError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


_lib = None


def lib():
    """Load libsla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libsla.so not built at {_LIB_PATH}; run "
                              "`python -m block_sparse_linear_mean_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, VP, SZ = ctypes.POINTER, ctypes.c_void_p, ctypes.c_size_t
        L.sla_abi_version.restype = ctypes.c_int32
        L.sla_status_string.restype = ctypes.c_char_p
        L.sla_status_string.argtypes = [ctypes.c_int]
        L.sla_validate.restype = ctypes.c_int
        L.sla_validate.argtypes = [P(sla_params)]
        L.sla_workspace_size.restype = ctypes.c_int
        L.sla_workspace_size.argtypes = [P(sla_params), ctypes.c_int32, P(SZ)]
        L.sla_build_mask.restype = ctypes.c_int
        L.sla_build_mask.argtypes = [P(sla_params), VP, VP, VP, P(sla_block_lists),
                                     P(sla_block_lists), VP, VP, VP, SZ, VP]
        L.sla_classify_scores.restype = ctypes.c_int
        L.sla_classify_scores.argtypes = [P(sla_params), VP, VP, P(sla_block_lists),
                                          P(sla_block_lists), VP, VP]
        L.sla_mask_lists.restype = ctypes.c_int
        L.sla_mask_lists.argtypes = [P(sla_params), VP, P(sla_block_lists),
                                     P(sla_block_lists), VP]
        L.sla_forward.restype = ctypes.c_int
        L.sla_forward.argtypes = [P(sla_params), VP, VP, VP, VP, P(sla_block_lists),
                                  VP, VP, VP, VP, VP, SZ, VP]
        L.sla_forward_prepare.restype = ctypes.c_int
        L.sla_forward_prepare.argtypes = [P(sla_params), VP, VP, VP, P(sla_block_lists), VP, SZ, VP]
        L.sla_attention_combine.restype = ctypes.c_int
        L.sla_attention_combine.argtypes = [P(sla_params), VP, VP, VP, VP, P(sla_block_lists),
                                            VP, VP, VP, VP, VP, SZ, VP]
        L.sla_sparse_attention.restype = ctypes.c_int
        L.sla_sparse_attention.argtypes = [P(sla_params), VP, VP, VP, P(sla_block_lists),
                                           VP, VP, VP, SZ, VP]
        L.sla_sparse_attention_noalloc.restype = ctypes.c_int
        L.sla_sparse_attention_noalloc.argtypes = [P(sla_params), VP, VP, VP,
                                                   P(sla_block_lists), VP, VP, VP, VP]
        L.sla_linear_combine.restype = ctypes.c_int
        L.sla_linear_combine.argtypes = [P(sla_params), VP, VP, VP, VP, P(sla_block_lists),
                                         VP, VP, VP, VP, SZ, VP]
        L.sla_backward.restype = ctypes.c_int
        L.sla_backward.argtypes = [P(sla_params), VP, VP, VP, VP, VP,
                                   P(sla_block_lists), P(sla_block_lists), VP, VP, VP,
                                   VP, VP, VP, VP, VP, SZ, VP]
        L.sla_forward_uses_tensor_cores.restype = ctypes.c_int32
        L.sla_forward_uses_tensor_cores.argtypes = [P(sla_params)]
        L.sla_block_importance.restype = ctypes.c_int
        L.sla_block_importance.argtypes = [P(sla_params), VP, VP, VP, VP]
        L.sla_mask_recall.restype = ctypes.c_int
        L.sla_mask_recall.argtypes = [P(sla_params), VP, VP, VP, VP]
        I32 = ctypes.c_int32
        L.sla_tile_order.restype = ctypes.c_int
        L.sla_tile_order.argtypes = [I32, I32, I32, I32, I32, I32, VP, VP]
        L.sla_permute_tokens.restype = ctypes.c_int
        L.sla_permute_tokens.argtypes = [P(sla_params), VP, VP, VP, I32, I32, VP]
        L.sla_check_device_status.restype = ctypes.c_int
        L.sla_check_device_status.argtypes = [VP, VP]
        _lib = L
    return _lib


# ------------------------------------------------------------------ C mirror


def sla_abi_version() -> int:
    return lib().sla_abi_version()


def status_string(status: int) -> str:
    return lib().sla_status_string(status).decode()


sla_status_string = status_string


def sla_validate(p: sla_params) -> int:
    return lib().sla_validate(ctypes.byref(p))


def sla_workspace_size(p: sla_params, op: int) -> int:
    n = ctypes.c_size_t(0)
    st = lib().sla_workspace_size(ctypes.byref(p), op, ctypes.byref(n))
    if st != SLA_OK:
        raise SlaError("sla_workspace_size", st)
    return n.value


def sla_build_mask(p, q, k, mask, rows, cols, scores, tie_count, ws, ws_bytes, stream) -> int:
    return lib().sla_build_mask(ctypes.byref(p), q, k, mask, ctypes.byref(rows),
                                ctypes.byref(cols) if cols is not None else None,
                                scores, tie_count, ws, ws_bytes, stream)


def sla_classify_scores(p, scores, mask, rows, cols, tie_count, stream) -> int:
    return lib().sla_classify_scores(ctypes.byref(p), scores, mask, ctypes.byref(rows),
                                     ctypes.byref(cols) if cols is not None else None,
                                     tie_count, stream)


def sla_mask_lists(p, mask, rows, cols, stream) -> int:
    return lib().sla_mask_lists(ctypes.byref(p), mask,
                                ctypes.byref(rows) if rows is not None else None,
                                ctypes.byref(cols) if cols is not None else None, stream)


def sla_forward(p, q, k, v, proj, rows, out, lse, o_s, o_lin, ws, ws_bytes, stream) -> int:
    return lib().sla_forward(ctypes.byref(p), q, k, v, proj, ctypes.byref(rows), out,
                             lse, o_s, o_lin, ws, ws_bytes, stream)


def sla_forward_prepare(p, k, v, proj, rows, ws, ws_bytes, stream) -> int:
    return lib().sla_forward_prepare(ctypes.byref(p), k, v, proj, ctypes.byref(rows), ws,
                                     ws_bytes, stream)


def sla_attention_combine(p, q, k, v, proj, rows, out, lse, o_s, o_lin, ws, ws_bytes,
                          stream) -> int:
    return lib().sla_attention_combine(ctypes.byref(p), q, k, v, proj, ctypes.byref(rows), out,
                                       lse, o_s, o_lin, ws, ws_bytes, stream)


def sla_sparse_attention(p, q, k, v, rows, o_s, lse, ws, ws_bytes, stream) -> int:
    return lib().sla_sparse_attention(ctypes.byref(p), q, k, v, ctypes.byref(rows), o_s,
                                      lse, ws, ws_bytes, stream)


def sla_sparse_attention_noalloc(p, q, k, v, rows, o_s, lse, status, stream) -> int:
    """Workspace-free sparse attention (scratch in a static device array)."""
    return lib().sla_sparse_attention_noalloc(ctypes.byref(p), q, k, v, ctypes.byref(rows),
                                              o_s, lse, status, stream)


def sla_linear_combine(p, q, k, v, proj, rows, o_s, out, o_lin, ws, ws_bytes, stream) -> int:
    return lib().sla_linear_combine(ctypes.byref(p), q, k, v, proj, ctypes.byref(rows),
                                    o_s, out, o_lin, ws, ws_bytes, stream)


def sla_backward(p, q, k, v, proj, dout, rows, cols, o_s, lse, o_lin, dq, dk, dv,
                 dproj, ws, ws_bytes, stream) -> int:
    return lib().sla_backward(ctypes.byref(p), q, k, v, proj, dout, ctypes.byref(rows),
                              ctypes.byref(cols), o_s, lse, o_lin, dq, dk, dv, dproj,
                              ws, ws_bytes, stream)


def sla_forward_uses_tensor_cores(p: sla_params) -> int:
    return lib().sla_forward_uses_tensor_cores(ctypes.byref(p))


def sla_block_importance(p, q, k, importance, stream) -> int:
    return lib().sla_block_importance(ctypes.byref(p), q, k, importance, stream)


def sla_mask_recall(p, mask, importance, counts, stream) -> int:
    return lib().sla_mask_recall(ctypes.byref(p), mask, importance, counts, stream)


def sla_tile_order(F, R, C, tf, tr, tc, perm, stream) -> int:
    return lib().sla_tile_order(F, R, C, tf, tr, tc, perm, stream)


def sla_permute_tokens(p, src, dst, perm, elem_bytes, inverse, stream) -> int:
    return lib().sla_permute_tokens(ctypes.byref(p), src, dst, perm, elem_bytes, inverse, stream)


def sla_check_device_status(ws, stream) -> int:
    return lib().sla_check_device_status(ws, stream)


# ------------------------------------------------------------------ tensors


def params_for(wl: Workload, N: Optional[int] = None, H: Optional[int] = None,
               B: Optional[int] = None, simt: bool = False,
               scale: float = 0.0) -> sla_params:
    """C parameter block for a workload (optionally overriding B, H, N)."""
    return sla_params(
        B=wl.B if B is None else B, H=wl.H if H is None else H,
        N=wl.N if N is None else N, d=wl.d, block_q=wl.block_q, block_k=wl.block_k,
        dtype=SLA_F32 if wl.dtype == "f32" else SLA_BF16,
        mask_mode=SLA_MASK_TOPK if wl.mode == "topk" else SLA_MASK_CDF,
        frac_crit=wl.frac_crit, frac_marg=wl.frac_marg, thr=wl.thr, scale=scale,
        flags=SLA_FLAG_SIMT if simt else 0)


def params_from(q: torch.Tensor, wl: Workload, **kw) -> sla_params:
    B, H, N, d = q.shape
    assert d == wl.d
    return params_for(wl, N=N, H=H, B=B, **kw)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _check(fn: str, st: int):
    if st != SLA_OK:
        raise SlaError(fn, st)


@dataclass
class BlockLists:
    crit_cnt: torch.Tensor
    crit_idx: torch.Tensor
    marg_cnt: torch.Tensor
    marg_idx: torch.Tensor

    @staticmethod
    def empty(nrows: int, width: int, device) -> "BlockLists":
        z = lambda *s: torch.zeros(*s, dtype=torch.int32, device=device)
        return BlockLists(z(nrows), z(nrows, width), z(nrows), z(nrows, width))

    def c(self) -> sla_block_lists:
        return sla_block_lists(self.crit_cnt.data_ptr(), self.crit_idx.data_ptr(),
                               self.marg_cnt.data_ptr(), self.marg_idx.data_ptr())


def workspace(p: sla_params, op: int, device) -> torch.Tensor:
    n = max(sla_workspace_size(p, op), 256)
    return torch.empty(n, dtype=torch.uint8, device=device)


def nblocks(n, b):
    return (n + b - 1) // b


def build_mask(p: sla_params, q: torch.Tensor, k: torch.Tensor, want_scores=False,
               want_cols=False, ws: Optional[torch.Tensor] = None) -> dict:
    """Pool, score and classify.  Returns mask, row lists (and optionally
    column lists, scores) and the near-tie row count (int32 tensor)."""
    dev = q.device
    B, H, N = p.B, p.H, p.N
    nqb, nkb = nblocks(N, p.block_q), nblocks(N, p.block_k)
    mask = torch.empty(B, H, nqb, nkb, dtype=torch.int8, device=dev)
    rows = BlockLists.empty(B * H * nqb, nkb, dev)
    cols = BlockLists.empty(B * H * nkb, nqb, dev) if want_cols else None
    scores = torch.empty(B, H, nqb, nkb, dtype=torch.float32, device=dev) if want_scores else None
    ties = torch.zeros(4, dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(p, SLA_OP_MASK, dev)
    rc = rows.c()
    cc = cols.c() if cols is not None else None
    _check("sla_build_mask", sla_build_mask(p, q.data_ptr(), k.data_ptr(), mask.data_ptr(),
                                            rc, cc, _ptr(scores), ties.data_ptr(),
                                            ws.data_ptr(), ws.numel(), _stream()))
    return dict(mask=mask, rows=rows, cols=cols, scores=scores, ties=ties[:1])


def block_importance(p: sla_params, q: torch.Tensor, k: torch.Tensor) -> torch.Tensor:
    """Dense attention max-pooled over (query block, key block) tiles,
    ``[B,H,Nqb,Nkb]`` fp32 (a mask-quality measurement; dense work)."""
    nqb, nkb = nblocks(p.N, p.block_q), nblocks(p.N, p.block_k)
    imp = torch.empty(p.B, p.H, nqb, nkb, dtype=torch.float32, device=q.device)
    _check("sla_block_importance", sla_block_importance(p, q.data_ptr(), k.data_ptr(),
                                                        imp.data_ptr(), _stream()))
    return imp


def mask_recall(p: sla_params, mask: torch.Tensor, importance: torch.Tensor) -> dict:
    """Recall of ``mask`` against ``importance``: hit and total counts for
    the critical and the kept (critical or marginal) sets, and their
    ratios (reads the four counts back to the host)."""
    counts = torch.empty(4, dtype=torch.int32, device=mask.device)
    _check("sla_mask_recall", sla_mask_recall(p, mask.data_ptr(), importance.data_ptr(),
                                              counts.data_ptr(), _stream()))
    ch, ct, kh, kt = (int(x) for x in counts.cpu().tolist())
    return dict(critical_hits=ch, critical_total=ct, kept_hits=kh, kept_total=kt,
                recall_critical=ch / ct if ct else float("nan"),
                recall_kept=kh / kt if kt else float("nan"))


def flex_block_mask(p: sla_params, mask: torch.Tensor, rows: BlockLists):
    """The critical part of a block mask as a PyTorch Flex Attention
    ``BlockMask`` (NABLA post, SberAIScience channel: the method is fully
    compatible with PyTorch's Flex Attention).  ``kv_num_blocks`` and
    ``kv_indices`` are zero-copy views of the CSR lists (``[B,H,Nqb]``
    counts, ``[B,H,Nqb,Nkb]`` ascending critical key blocks); the block
    sizes are (block_q, block_k); the sequence length N covers the ragged
    tail; the ``mask_mod`` reads the int8 mask (critical = 2), so every Flex
    path, the eager one included, attends to the critical blocks only.  The
    marginal (linear) branch has no Flex counterpart and is not exported.
    ``mask`` must outlive the returned object."""
    from torch.nn.attention.flex_attention import BlockMask
    nqb, nkb = nblocks(p.N, p.block_q), nblocks(p.N, p.block_k)
    bq, bk = p.block_q, p.block_k
    kv_num = rows.crit_cnt.view(p.B, p.H, nqb)
    kv_idx = rows.crit_idx.view(p.B, p.H, nqb, nkb)

    def critical(b, h, q_idx, kv_idx):
        return mask[b, h, q_idx // bq, kv_idx // bk] == CRITICAL

    return BlockMask.from_kv_blocks(kv_num, kv_idx, BLOCK_SIZE=(bq, bk), mask_mod=critical,
                                    seq_lengths=(p.N, p.N))


def classify_scores(p: sla_params, scores: torch.Tensor, want_cols=False) -> dict:
    """Classify given row-softmaxed pooled scores ``[B,H,Nqb,Nkb]`` fp32."""
    dev = scores.device
    B, H, nqb, nkb = scores.shape
    mask = torch.empty(B, H, nqb, nkb, dtype=torch.int8, device=dev)
    rows = BlockLists.empty(B * H * nqb, nkb, dev)
    cols = BlockLists.empty(B * H * nkb, nqb, dev) if want_cols else None
    ties = torch.zeros(4, dtype=torch.int32, device=dev)
    _check("sla_classify_scores", sla_classify_scores(
        p, scores.data_ptr(), mask.data_ptr(), rows.c(), cols.c() if cols else None,
        ties.data_ptr(), _stream()))
    return dict(mask=mask, rows=rows, cols=cols, ties=ties[:1])


def mask_lists(p: sla_params, mask: torch.Tensor, want_rows=True, want_cols=True):
    dev = mask.device
    nqb, nkb = mask.shape[-2], mask.shape[-1]
    nr = p.B * p.H
    rows = BlockLists.empty(nr * nqb, nkb, dev) if want_rows else None
    cols = BlockLists.empty(nr * nkb, nqb, dev) if want_cols else None
    _check("sla_mask_lists", sla_mask_lists(p, mask.data_ptr(),
                                            rows.c() if rows else None,
                                            cols.c() if cols else None, _stream()))
    return rows, cols


def forward(p: sla_params, q, k, v, proj, rows: BlockLists, save_for_backward=False,
            ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> dict:
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)
    o_s = torch.empty(q.shape, dtype=torch.float32, device=dev) if save_for_backward else None
    o_lin = torch.empty(q.shape, dtype=torch.float32, device=dev) if save_for_backward else None
    if ws is None:
        ws = workspace(p, SLA_OP_FORWARD, dev)
    _check("sla_forward", sla_forward(p, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      proj.data_ptr(), rows.c(), out.data_ptr(),
                                      lse.data_ptr(), _ptr(o_s), _ptr(o_lin),
                                      ws.data_ptr(), ws.numel(), _stream()))
    return dict(out=out, lse=lse, o_s=o_s, o_lin=o_lin, ws=ws)


def sparse_attention(p: sla_params, q, k, v, rows: BlockLists,
                     ws: Optional[torch.Tensor] = None) -> dict:
    """Critical part alone (``sla_sparse_attention``): O_s and LSE in fp32."""
    dev = q.device
    o_s = torch.empty(q.shape, dtype=torch.float32, device=dev)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(p, SLA_OP_FORWARD, dev)
    _check("sla_sparse_attention", sla_sparse_attention(
        p, q.data_ptr(), k.data_ptr(), v.data_ptr(), rows.c(), o_s.data_ptr(), lse.data_ptr(),
        ws.data_ptr(), ws.numel(), _stream()))
    return dict(o_s=o_s, lse=lse, ws=ws)


def linear_combine(p: sla_params, q, k, v, proj, rows: BlockLists, o_s: torch.Tensor,
                   save_o_lin=False, ws: Optional[torch.Tensor] = None) -> dict:
    """Marginal part and combine (``sla_linear_combine``): out = o_s +
    O_lin @ proj in the input dtype, O_lin optionally in fp32."""
    dev = q.device
    out = torch.empty_like(q)
    o_lin = torch.empty(q.shape, dtype=torch.float32, device=dev) if save_o_lin else None
    if ws is None:
        ws = workspace(p, SLA_OP_FORWARD, dev)
    _check("sla_linear_combine", sla_linear_combine(
        p, q.data_ptr(), k.data_ptr(), v.data_ptr(), proj.data_ptr(), rows.c(), o_s.data_ptr(),
        out.data_ptr(), _ptr(o_lin), ws.data_ptr(), ws.numel(), _stream()))
    return dict(out=out, o_lin=o_lin, ws=ws)


def backward(p: sla_params, q, k, v, proj, dout, rows: BlockLists, cols: BlockLists,
             saved: dict, ws: Optional[torch.Tensor] = None) -> dict:
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty(q.shape, **f32) for _ in range(3))
    dproj = torch.empty(proj.shape, **f32)
    if ws is None:
        ws = workspace(p, SLA_OP_BACKWARD, dev)
    _check("sla_backward", sla_backward(p, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        proj.data_ptr(), dout.data_ptr(), rows.c(), cols.c(),
                                        saved["o_s"].data_ptr(), saved["lse"].data_ptr(),
                                        saved["o_lin"].data_ptr(), dq.data_ptr(),
                                        dk.data_ptr(), dv.data_ptr(), dproj.data_ptr(),
                                        ws.data_ptr(), ws.numel(), _stream()))
    return dict(dq=dq, dk=dk, dv=dv, dproj=dproj, ws=ws)


def tile_order(grid, tile, device) -> torch.Tensor:
    """``perm [F*R*C]`` int32 on ``device``: perm[n] = raster index of the
    n-th token when the (F, R, C) grid is walked in (tf, tr, tc) tiles."""
    F, R, C = grid
    perm = torch.empty(F * R * C, dtype=torch.int32, device=device)
    _check("sla_tile_order", sla_tile_order(F, R, C, *tile, perm.data_ptr(), _stream()))
    return perm


def permute_tokens(p: sla_params, x: torch.Tensor, perm: torch.Tensor, inverse=False) -> torch.Tensor:
    """``x [B,H,N,d]`` (bf16 or fp32) moved into the order ``perm``
    (``out[..., n, :] = x[..., perm[n], :]``), or back with ``inverse``."""
    out = torch.empty_like(x)
    _check("sla_permute_tokens", sla_permute_tokens(p, x.data_ptr(), out.data_ptr(), perm.data_ptr(),
                                                    x.element_size(), 1 if inverse else 0, _stream()))
    return out


def check_device_status(ws: torch.Tensor) -> int:
    return sla_check_device_status(ws.data_ptr(), _stream())

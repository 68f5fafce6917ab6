"""Torch-facing helpers over the C ABI: allocate outputs and workspaces with
torch (device memory and streams only) and call libusp.so. No arithmetic of
the path happens here.
"""
from __future__ import annotations

import torch

from . import binding as B_


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return B_.USP_BF16
    if t.dtype == torch.float32:
        return B_.USP_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _require_cuda(*ts):
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")


def zigzag_shard(x: torch.Tensor, P_u: int, P_r: int, out=None, stream=None) -> torch.Tensor:
    """global [B, S, H, D] -> rank-major [P, B, S/P, H, D]."""
    _require_cuda(x)
    B, S, H, D = x.shape
    P = P_u * P_r
    out = torch.empty((P, B, S // P, H, D), dtype=x.dtype, device=x.device) if out is None else out
    B_.usp_zigzag_shard(x, out, B, S, H, D, _dt(x), P_u, P_r, stream)
    return out


def zigzag_unshard(x: torch.Tensor, P_u: int, P_r: int, out=None, stream=None) -> torch.Tensor:
    """rank-major [P, B, S/P, H, D] -> global [B, S, H, D]."""
    _require_cuda(x)
    P, B, c2, H, D = x.shape
    S = P * c2
    out = torch.empty((B, S, H, D), dtype=x.dtype, device=x.device) if out is None else out
    B_.usp_zigzag_unshard(x, out, B, S, H, D, _dt(x), P_u, P_r, stream)
    return out


def seq2head(x: torch.Tensor, P_u: int, P_r: int, out=None, stream=None) -> torch.Tensor:
    """rank-major [P, B, S/P, H, D] -> head-sharded [P_r, P_u, B, S/P_r, H/P_u, D]."""
    _require_cuda(x)
    P, B, c2, H, D = x.shape
    S = P * c2
    out = (torch.empty((P_r, P_u, B, S // P_r, H // P_u, D), dtype=x.dtype, device=x.device)
           if out is None else out)
    B_.usp_seq2head_permute(x, out, B, S, H, D, _dt(x), P_u, P_r, stream)
    return out


def head2seq(x: torch.Tensor, P_u: int, P_r: int, out=None, stream=None) -> torch.Tensor:
    """head-sharded [P_r, P_u, B, S/P_r, H/P_u, D] -> rank-major [P, B, S/P, H, D]."""
    _require_cuda(x)
    Pr, Pu, B, L, Hl, D = x.shape
    S = L * P_r
    P = P_u * P_r
    out = torch.empty((P, B, S // P, Hl * P_u, D), dtype=x.dtype, device=x.device) if out is None else out
    B_.usp_head2seq_permute(x, out, B, S, Hl * P_u, D, _dt(x), P_u, P_r, stream)
    return out


def seq2head_many(xs, P_u: int, P_r: int, outs=None, stream=None):
    """The seq->head all-to-all of several rank-major tensors [P, B, S/P, H_x, D_x]
    (e.g. Q, K, V) in one launch; returns the head-sharded tensors."""
    _require_cuda(*xs)
    outs = list(outs) if outs is not None else [None] * len(xs)
    jobs = []
    for x_, (x, o) in enumerate(zip(xs, outs)):
        P, B, c2, H, D = x.shape
        if o is None:
            o = torch.empty((P_r, P_u, B, P * c2 // P_r, H // P_u, D), dtype=x.dtype, device=x.device)
            outs[x_] = o
        jobs.append((x, o, H, D, _dt(x)))
    P, B, c2 = xs[0].shape[:3]
    B_.usp_permute_batch(B_.USP_MAP_SEQ2HEAD, jobs, B, P * c2, P_u, P_r, stream)
    return outs


def head2seq_many(xs, P_u: int, P_r: int, outs=None, stream=None):
    """The head->seq regather of several head-sharded tensors (e.g. dQ, dK, dV)
    in one launch; returns the rank-major tensors [P, B, S/P, H_x, D_x]."""
    _require_cuda(*xs)
    outs = list(outs) if outs is not None else [None] * len(xs)
    jobs = []
    P = P_u * P_r
    for x_, (x, o) in enumerate(zip(xs, outs)):
        Pr, Pu, B, L, Hl, D = x.shape
        if o is None:
            o = torch.empty((P, B, L * P_r // P, Hl * P_u, D), dtype=x.dtype, device=x.device)
            outs[x_] = o
        jobs.append((x, o, Hl * P_u, D, _dt(x)))
    Pr, Pu, B, L = xs[0].shape[:4]
    B_.usp_permute_batch(B_.USP_MAP_HEAD2SEQ, jobs, B, L * P_r, P_u, P_r, stream)
    return outs


def to_head_sharded(x, P_u, P_r, stream=None):
    return seq2head(zigzag_shard(x, P_u, P_r, stream=stream), P_u, P_r, stream=stream)


def from_head_sharded(x, P_u, P_r, stream=None):
    return zigzag_unshard(head2seq(x, P_u, P_r, stream=stream), P_u, P_r, stream=stream)


def workspace(nbytes: int, device) -> torch.Tensor:
    n = max(int(nbytes), 256)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def check_workspace(ws: torch.Tensor, stream=None) -> None:
    """Synchronise the stream and raise UspError(USP_ERR_TIMEOUT) if a kernel that
    used `ws` recorded a timed-out device wait (the word is cleared by the read)."""
    rc, site = B_.usp_workspace_status(ws, stream)
    if rc != B_.USP_OK:
        raise B_.UspError(rc, f"device wait timed out (site {site:#x}): {B_.usp_last_error()}")


def attn_fwd(q, k, v, causal: bool, P_u: int, P_r: int, mode: int = B_.USP_MODE_FUSED,
             ws: torch.Tensor | None = None, out=None, lse=None, stream=None, check_status: bool = False):
    """Forward over head-sharded q [P_r, P_u, B, L, Hq/P_u, D], k/v [..., Hkv/P_u, D].
    Returns (out bf16 like q, lse fp32 [P_r, P_u, B, L, Hq/P_u]). With
    check_status=True the call synchronises and raises on a timed-out device wait."""
    _require_cuda(q, k, v)
    Pr, Pu, B, L, Hql, D = q.shape
    Hkv = k.shape[4] * P_u
    Hq = Hql * P_u
    S = L * P_r
    need = B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, mode, 0)
    if ws is None:
        ws = workspace(need, q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device) if lse is None else lse
    B_.usp_attn_fwd(q, k, v, out, lse, B, S, Hq, Hkv, D, causal, P_u, P_r, mode, ws, ws.numel(), stream)
    if check_status:
        check_workspace(ws, stream)
    return out, lse


def attn_bwd(q, k, v, out, lse, dO, causal: bool, P_u: int, P_r: int, ws=None, dq=None, dk=None, dv=None,
             stream=None, check_status: bool = False, grad_dtype=torch.float32):
    """Backward; returns (dQ bf16 like q, dK like k, dV like v), dK and dV in
    grad_dtype: fp32 (usp_attn_bwd) or bf16 (usp_attn_bwd_prepare, _dkdv_bf16 and
    _dq). With check_status=True the call synchronises and raises on a timed-out
    device wait."""
    if grad_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("grad_dtype must be torch.float32 or torch.bfloat16")
    _require_cuda(q, k, v, out, lse, dO)
    Pr, Pu, B, L, Hql, D = q.shape
    Hkv = k.shape[4] * P_u
    Hq = Hql * P_u
    S = L * P_r
    need = B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, 0, 1)
    if ws is None:
        ws = workspace(need, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty(k.shape, dtype=grad_dtype, device=k.device) if dk is None else dk
    dv = torch.empty(v.shape, dtype=grad_dtype, device=v.device) if dv is None else dv
    if dk.dtype != grad_dtype or dv.dtype != grad_dtype:
        raise ValueError("dk and dv must have dtype grad_dtype")
    if grad_dtype == torch.float32:
        B_.usp_attn_bwd(q, k, v, out, lse, dO, dq, dk, dv, B, S, Hq, Hkv, D, causal, P_u, P_r, ws, ws.numel(),
                        stream)
    else:
        geo = (B, S, Hq, Hkv, D, causal, P_u, P_r)
        B_.usp_attn_bwd_prepare(out, lse, dO, *geo, ws, ws.numel(), stream)
        B_.usp_attn_bwd_dkdv_bf16(q, k, v, dO, dk, dv, *geo, ws, ws.numel(), stream)
        B_.usp_attn_bwd_dq(q, k, v, dO, dq, *geo, ws, ws.numel(), stream)
    if check_status:
        check_workspace(ws, stream)
    return dq, dk, dv


def attn_fwd_masked(q, k, v, causal: bool, P_u: int, P_r: int, block_mask=None, cu_seqlens=None, ws=None, out=None,
                    lse=None, stream=None, check_status: bool = False):
    """usp_attn_fwd (fused) with a block mask [B, Hq, S/128, S/128] (uint8, CUDA)
    and/or document boundaries cu_seqlens [n_docs + 1] (int32, CUDA), both in
    original positions."""
    _require_cuda(q, k, v)
    Pr, Pu, B, L, Hql, D = q.shape
    Hkv = k.shape[4] * P_u
    Hq = Hql * P_u
    S = L * P_r
    n_docs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    if ws is None:
        ws = workspace(B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, 0, 0), q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device) if lse is None else lse
    B_.usp_attn_fwd_masked(q, k, v, out, lse, B, S, Hq, Hkv, D, causal, P_u, P_r, block_mask, cu_seqlens, n_docs, ws,
                           ws.numel(), stream)
    if check_status:
        check_workspace(ws, stream)
    return out, lse


def attn_bwd_masked(q, k, v, out, lse, dO, causal: bool, P_u: int, P_r: int, block_mask=None, cu_seqlens=None,
                    ws=None, stream=None, check_status: bool = False):
    """usp_attn_bwd with the masks of attn_fwd_masked; returns (dQ, dK, dV)."""
    _require_cuda(q, k, v, out, lse, dO)
    Pr, Pu, B, L, Hql, D = q.shape
    Hkv = k.shape[4] * P_u
    Hq = Hql * P_u
    S = L * P_r
    n_docs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    if ws is None:
        ws = workspace(B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, 0, 1), q.device)
    dq = torch.empty_like(q)
    dk = torch.empty(k.shape, dtype=torch.float32, device=k.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=v.device)
    B_.usp_attn_bwd_masked(q, k, v, out, lse, dO, dq, dk, dv, B, S, Hq, Hkv, D, causal, P_u, P_r, block_mask,
                           cu_seqlens, n_docs, ws, ws.numel(), stream)
    if check_status:
        check_workspace(ws, stream)
    return dq, dk, dv


def dilated_attn_fwd(q, k, v, causal: bool, pairs, ws=None, out=None, lse=None, stream=None,
                     check_status: bool = False):
    """LongNet dilated attention over global-layout q [B, S, Hq, D], k/v [B, S, Hkv, D]
    for the (w, r) pairs `pairs`. Returns (out bf16 like q, lse fp32 [B, S, Hq])."""
    _require_cuda(q, k, v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if ws is None:
        ws = workspace(B_.usp_dilated_workspace_size(B, S, Hq, D), q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device) if lse is None else lse
    B_.usp_dilated_attn_fwd(q, k, v, out, lse, B, S, Hq, Hkv, D, causal, pairs, ws, ws.numel(), stream)
    if check_status:
        check_workspace(ws, stream)
    return out, lse


def dilated_attn_bwd(q, k, v, out, lse, dO, causal: bool, pairs, ws=None, stream=None, check_status: bool = False):
    """Backward of dilated_attn_fwd; returns (dQ bf16 like q, dK fp32 like k, dV fp32 like v)."""
    _require_cuda(q, k, v, out, lse, dO)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if ws is None:
        ws = workspace(B_.usp_dilated_bwd_workspace_size(B, S, Hq, D, pairs), q.device)
    dq = torch.empty_like(q)
    dk = torch.empty(k.shape, dtype=torch.float32, device=k.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=v.device)
    B_.usp_dilated_attn_bwd(q, k, v, out, lse, dO, dq, dk, dv, B, S, Hq, Hkv, D, causal, pairs, ws, ws.numel(), stream)
    if check_status:
        check_workspace(ws, stream)
    return dq, dk, dv


def lse_merge(o_parts: torch.Tensor, lse_parts: torch.Tensor, out_dtype=torch.bfloat16, stream=None):
    """o_parts [n, rows, D] fp32, lse_parts [n, rows] fp32 -> (out [rows, D], lse [rows])."""
    _require_cuda(o_parts, lse_parts)
    n, rows, D = o_parts.shape
    out = torch.empty((rows, D), dtype=out_dtype, device=o_parts.device)
    lse = torch.empty(rows, dtype=torch.float32, device=o_parts.device)
    B_.usp_lse_merge(o_parts, lse_parts, n, rows, D, out, _dt(out), lse, stream)
    return out, lse


def bwd_preprocess(out: torch.Tensor, dO: torch.Tensor, stream=None) -> torch.Tensor:
    _require_cuda(out, dO)
    D = out.shape[-1]
    rows = out.numel() // D
    delta = torch.empty(out.shape[:-1], dtype=torch.float32, device=out.device)
    B_.usp_bwd_preprocess(out, dO, delta, rows, D, stream)
    return delta

"""Python face of the fp64 CPU oracle (oracle/usp_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU legs of bench.py, never by the product package. It shares no code with the
CUDA path; both sides receive their inputs from the neutral `usp_inputs`
generators.

Parity status of each function (what pins it is in tests/test_oracle_pins.py):
  attn_fwd_rows / attn_full (forward) -- pinned: closed forms (Q = 0, causal row
      0), torch's fp64 scaled_dot_product_attention, row sums, key-range merge.
  attn_full (backward), attn_dq_rows, attn_dkdv_cols -- pinned: central finite
      differences, torch fp64 autograd, sum_j dK_j = 0, sum_j dV_j = sum_i dO_i.
  lse_merge -- pinned: chunked-and-merged == unchunked, empty partials.
  zigzag_* / seq2head / head2seq -- pinned: hand-written worked examples in
      tests/golden/, bijection and inverse checks.
  dilated_fwd_rows (LongNet dilated attention) -- pinned: a hand-derived worked
      example (tests/golden/dilated_tiny_closed_form.json), one pair (w = S,
      r = 1) against torch's fp64 scaled_dot_product_attention, and torch's fp64
      SDPA with the log of the key multiplicities as an additive mask.
  dilated_attn_full (forward and backward) -- pinned: its forward against the
      pinned dilated_fwd_rows, its gradients against central finite
      differences and against torch fp64 autograd of SDPA with the
      key-multiplicity mask.
  masked_fwd_rows / masked_attn_full (block-sparse and document masks) --
      pinned: a hand-derived worked example (tests/golden/masked_tiny_closed_form.json),
      the all-ones mask against the unmasked pinned oracle, torch fp64 SDPA with
      the boolean mask (forward) and its autograd (backward).
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np
import torch

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        l_ = ctypes.c_long
        i_ = ctypes.c_int
        d_ = ctypes.c_double
        L.oracle_attn_fwd_rows.argtypes = [P, P, P, i_, l_, l_, l_, l_, l_, i_, d_, l_, P, l_, P, P, P, i_]
        L.oracle_attn_full.argtypes = [P, P, P, P, i_, l_, l_, l_, l_, l_, i_, d_, P, P, P, P, P, i_]
        L.oracle_attn_dq_rows.argtypes = [P, P, P, P, i_, l_, l_, l_, l_, l_, i_, d_, l_, P, P, P, P, i_]
        L.oracle_attn_dkdv_cols.argtypes = [P, P, P, P, i_, l_, l_, l_, l_, l_, i_, d_, l_, P, P, P, P, P, i_]
        L.oracle_lse_merge.argtypes = [l_, l_, l_, P, P, P, P, i_]
        L.oracle_dilated_fwd_rows.argtypes = [P, P, P, i_, l_, l_, l_, l_, l_, i_, d_, l_, P, l_, P, P, P, i_]
        L.oracle_dilated_attn_full.argtypes = [P, P, P, P, i_, l_, l_, l_, l_, l_, i_, d_, l_, P, P, P, P, P, P,
                                               i_]
        L.oracle_masked_fwd_rows.argtypes = [P, P, P, i_, l_, l_, l_, l_, l_, i_, d_, P, l_, P, l_, l_, P, P, P,
                                             i_]
        L.oracle_masked_attn_full.argtypes = [P, P, P, P, i_, l_, l_, l_, l_, l_, i_, d_, P, l_, P, l_, P, P, P,
                                              P, P, i_]
        for name in ("oracle_zigzag_shard", "oracle_zigzag_unshard"):
            getattr(L, name).argtypes = [P, P, l_, l_, l_, l_, l_, l_]
        for name in ("oracle_seq2head", "oracle_head2seq"):
            getattr(L, name).argtypes = [P, P, l_, l_, l_, l_, l_, l_, l_]
        for name in ("oracle_attn_fwd_rows", "oracle_attn_full", "oracle_attn_dq_rows",
                     "oracle_attn_dkdv_cols", "oracle_lse_merge", "oracle_zigzag_shard",
                     "oracle_zigzag_unshard", "oracle_seq2head", "oracle_head2seq",
                     "oracle_dilated_fwd_rows", "oracle_masked_fwd_rows", "oracle_masked_attn_full",
                     "oracle_dilated_attn_full"):
            getattr(L, name).restype = ctypes.c_int
        L.oracle_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Contiguous CPU uint16 view of a bf16 tensor (the exact bit patterns)."""
    assert t.dtype == torch.bfloat16
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def _inputs(*ts):
    """Arrays handed to the C oracle: bf16 bit patterns, or float64 when every input is float64."""
    if all(t.dtype == torch.float64 for t in ts):
        return [np.ascontiguousarray(t.detach().to("cpu").numpy()) for t in ts], 1
    return [_bf16_bits(t) for t in ts], 0


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(q, k):
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    return B, S, Hq, Hkv, D


def attn_fwd_rows(q, k, v, causal, rows, ranges=None, scale=None, threads=0):
    """O [n, D] and LSE [n] (float64) of query rows (b, h, i), global layout inputs."""
    B, S, Hq, Hkv, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    (qa, ka, va), f64 = _inputs(q, k, v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.zeros((n, D), np.float64)
    lse = np.zeros(n, np.float64)
    if ranges is None:
        nr, rp = 0, None
    else:
        rg = np.ascontiguousarray(np.asarray(ranges, dtype=np.int64).reshape(-1, 2))
        nr, rp = rg.shape[0], _ptr(rg)
    rc = lib().oracle_attn_fwd_rows(_ptr(qa), _ptr(ka), _ptr(va), f64, B, S, Hq, Hkv, D, int(causal),
                                    scale, n, _ptr(rows), nr, rp, _ptr(o), _ptr(lse), threads)
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd_rows failed ({rc})")
    return o, lse


def dilated_fwd_rows(q, k, v, causal, pairs, rows, scale=None, threads=0):
    """LongNet dilated attention: O [n, D] and LSE [n] (float64) of query rows
    (b, h, i) for the (w, r) pairs `pairs`, global-layout inputs."""
    B, S, Hq, Hkv, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    (qa, ka, va), f64 = _inputs(q, k, v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    n = rows.shape[0]
    o = np.zeros((n, D), np.float64)
    lse = np.zeros(n, np.float64)
    rc = lib().oracle_dilated_fwd_rows(_ptr(qa), _ptr(ka), _ptr(va), f64, B, S, Hq, Hkv, D, int(causal), scale,
                                       pr.shape[0], _ptr(pr), n, _ptr(rows), _ptr(o), _ptr(lse), threads)
    if rc != 0:
        raise ValueError(f"oracle_dilated_fwd_rows failed ({rc})")
    return o, lse


def dilated_attn_full(q, k, v, do, causal, pairs, scale=None, threads=0):
    """Whole-tensor LongNet dilated attention forward and backward: dict of
    float64 o, lse, dq, dk, dv (global layouts)."""
    B, S, Hq, Hkv, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    (qa, ka, va, da), f64 = _inputs(q, k, v, do)
    pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    o = np.zeros((B, S, Hq, D)); lse = np.zeros((B, S, Hq)); dq = np.zeros((B, S, Hq, D))
    dk = np.zeros((B, S, Hkv, D)); dv = np.zeros((B, S, Hkv, D))
    rc = lib().oracle_dilated_attn_full(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), f64, B, S, Hq, Hkv, D, int(causal),
                                        scale, pr.shape[0], _ptr(pr), _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk),
                                        _ptr(dv), threads)
    if rc != 0:
        raise ValueError(f"oracle_dilated_attn_full failed ({rc})")
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def _mask_args(block_mask, block, cu_seqlens):
    bm = None if block_mask is None else np.ascontiguousarray(np.asarray(block_mask, dtype=np.uint8))
    cu = None if cu_seqlens is None else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    return (bm, None if bm is None else _ptr(bm), int(block), cu, None if cu is None else _ptr(cu),
            0 if cu is None else cu.shape[0] - 1)


def masked_fwd_rows(q, k, v, causal, rows, block_mask=None, block=128, cu_seqlens=None, scale=None, threads=0):
    """Masked attention O [n, D], LSE [n] of query rows (b, h, i): block_mask
    [B, Hq, nb, nb] (0/1 per block of `block` positions) and/or document
    boundaries cu_seqlens [n_docs + 1] (shared by the batch)."""
    B, S, Hq, Hkv, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    (qa, ka, va), f64 = _inputs(q, k, v)
    bm, bmp, bs, cu, cup, nd = _mask_args(block_mask, block, cu_seqlens)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.zeros((n, D), np.float64)
    lse = np.zeros(n, np.float64)
    rc = lib().oracle_masked_fwd_rows(_ptr(qa), _ptr(ka), _ptr(va), f64, B, S, Hq, Hkv, D, int(causal), scale,
                                      bmp, bs, cup, nd, n, _ptr(rows), _ptr(o), _ptr(lse), threads)
    if rc != 0:
        raise ValueError(f"oracle_masked_fwd_rows failed ({rc})")
    return o, lse


def masked_attn_full(q, k, v, do, causal, block_mask=None, block=128, cu_seqlens=None, scale=None, threads=0):
    """Whole-tensor masked forward and backward: dict of float64 o, lse, dq, dk, dv."""
    B, S, Hq, Hkv, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    (qa, ka, va, da), f64 = _inputs(q, k, v, do)
    bm, bmp, bs, cu, cup, nd = _mask_args(block_mask, block, cu_seqlens)
    o = np.zeros((B, S, Hq, D)); lse = np.zeros((B, S, Hq)); dq = np.zeros((B, S, Hq, D))
    dk = np.zeros((B, S, Hkv, D)); dv = np.zeros((B, S, Hkv, D))
    rc = lib().oracle_masked_attn_full(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), f64, B, S, Hq, Hkv, D,
                                       int(causal), scale, bmp, bs, cup, nd, _ptr(o), _ptr(lse), _ptr(dq),
                                       _ptr(dk), _ptr(dv), threads)
    if rc != 0:
        raise ValueError(f"oracle_masked_attn_full failed ({rc})")
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def attn_full(q, k, v, do, causal, scale=None, threads=0):
    """Whole-tensor forward and backward: dict of float64 arrays o, lse, dq, dk, dv."""
    B, S, Hq, Hkv, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    (qa, ka, va, da), f64 = _inputs(q, k, v, do)
    o = np.zeros((B, S, Hq, D)); lse = np.zeros((B, S, Hq)); dq = np.zeros((B, S, Hq, D))
    dk = np.zeros((B, S, Hkv, D)); dv = np.zeros((B, S, Hkv, D))
    rc = lib().oracle_attn_full(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), f64, B, S, Hq, Hkv, D,
                                int(causal), scale, _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk),
                                _ptr(dv), threads)
    if rc != 0:
        raise ValueError(f"oracle_attn_full failed ({rc})")
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def attn_dq_rows(q, k, v, do, causal, rows, scale=None, threads=0):
    """dQ [n, D], LSE [n], Delta [n] of query rows (b, h, i)."""
    B, S, Hq, Hkv, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    (qa, ka, va, da), f64 = _inputs(q, k, v, do)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    dq = np.zeros((n, D)); lse = np.zeros(n); delta = np.zeros(n)
    rc = lib().oracle_attn_dq_rows(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), f64, B, S, Hq, Hkv, D,
                                   int(causal), scale, n, _ptr(rows), _ptr(dq), _ptr(lse),
                                   _ptr(delta), threads)
    if rc != 0:
        raise ValueError(f"oracle_attn_dq_rows failed ({rc})")
    return dq, lse, delta


def attn_dkdv_cols(q, k, v, do, causal, cols, lse_tab, delta_tab, scale=None, threads=0):
    """dK [n, D], dV [n, D] of key columns (b, g, j); lse_tab/delta_tab are [B, S, Hq]."""
    B, S, Hq, Hkv, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    (qa, ka, va, da), f64 = _inputs(q, k, v, do)
    cols = np.ascontiguousarray(np.asarray(cols, dtype=np.int64).reshape(-1, 3))
    lt = np.ascontiguousarray(lse_tab, dtype=np.float64)
    dt = np.ascontiguousarray(delta_tab, dtype=np.float64)
    assert lt.shape == (B, S, Hq) and dt.shape == (B, S, Hq)
    n = cols.shape[0]
    dk = np.zeros((n, D)); dv = np.zeros((n, D))
    rc = lib().oracle_attn_dkdv_cols(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), f64, B, S, Hq, Hkv, D,
                                     int(causal), scale, n, _ptr(cols), _ptr(lt), _ptr(dt),
                                     _ptr(dk), _ptr(dv), threads)
    if rc != 0:
        raise ValueError(f"oracle_attn_dkdv_cols failed ({rc})")
    return dk, dv


def lse_merge(o_parts, lse_parts, threads=0):
    """Merge partials o_parts [n, rows, D], lse_parts [n, rows] -> (o [rows, D], lse [rows])."""
    op = np.ascontiguousarray(o_parts, dtype=np.float64)
    lp = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, rows, D = op.shape
    o = np.zeros((rows, D)); lse = np.zeros(rows)
    lib().oracle_lse_merge(n, rows, D, _ptr(op), _ptr(lp), _ptr(o), _ptr(lse), threads)
    return o, lse


def _layout_call(fn, src: torch.Tensor, out_shape, *args):
    a = src.detach().to("cpu").contiguous()
    esize = a.element_size()
    raw = a.view(torch.uint8).numpy() if a.dim() else a.numpy()
    dst = torch.empty(out_shape, dtype=a.dtype)
    draw = dst.view(torch.uint8).numpy()
    rc = fn(_ptr(raw), _ptr(draw), *args[:-1], esize, *args[-1])
    if rc != 0:
        raise ValueError("bad layout arguments")
    return dst


def zigzag_shard(x: torch.Tensor, P: int) -> torch.Tensor:
    """global [B, S, H, D] -> rank-major [P, B, S/P, H, D]."""
    B, S, H, D = x.shape
    return _layout_call(lib().oracle_zigzag_shard, x, (P, B, S // P, H, D), B, S, H, D, (P,))


def zigzag_unshard(x: torch.Tensor, S: int) -> torch.Tensor:
    """rank-major [P, B, S/P, H, D] -> global [B, S, H, D]."""
    P, B, _, H, D = x.shape
    return _layout_call(lib().oracle_zigzag_unshard, x, (B, S, H, D), B, S, H, D, (P,))


def seq2head(x: torch.Tensor, P_u: int, P_r: int) -> torch.Tensor:
    """rank-major [P, B, S/P, H, D] -> head-sharded [P_r, P_u, B, S/P_r, H/P_u, D]."""
    P, B, c2, H, D = x.shape
    S = P * c2
    return _layout_call(lib().oracle_seq2head, x, (P_r, P_u, B, S // P_r, H // P_u, D),
                        B, S, H, D, (P_u, P_r))


def head2seq(x: torch.Tensor, P_u: int, P_r: int) -> torch.Tensor:
    """head-sharded [P_r, P_u, B, S/P_r, H/P_u, D] -> rank-major [P, B, S/P, H, D]."""
    Pr, Pu, B, L, Hl, D = x.shape
    S = L * P_r
    P = P_u * P_r
    return _layout_call(lib().oracle_head2seq, x, (P, B, S // P, Hl * P_u, D),
                        B, S, Hl * P_u, D, (P_u, P_r))


def to_head_sharded(x: torch.Tensor, P_u: int, P_r: int) -> torch.Tensor:
    """global [B, S, H, D] -> head-sharded layout (zigzag shard, then seq->head)."""
    return seq2head(zigzag_shard(x, P_u * P_r), P_u, P_r)


def from_head_sharded(x: torch.Tensor, P_u: int, P_r: int) -> torch.Tensor:
    """head-sharded layout -> global [B, S, H, D] (head->seq, then unshard)."""
    S = x.shape[3] * P_r
    return zigzag_unshard(head2seq(x, P_u, P_r), S)

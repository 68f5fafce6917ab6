"""ctypes binding of libusp.so: one Python function per C entry point of
include/usp.h, with the same name and argument order. Arguments may be torch
tensors (their data pointers are passed) or integers (raw device pointers).
Marshalling only: every step of the path runs in the library's kernels.

Loading fails loudly (ImportError) when libusp.so has not been built; there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libusp.so")

USP_OK = 0
USP_ERR_INVALID_ARG = -1
USP_ERR_UNSUPPORTED = -2
USP_ERR_CUDA = -3
USP_ERR_TIMEOUT = -4
USP_ERR_WORKSPACE = -5
USP_BF16 = 0
USP_F32 = 1
USP_MODE_FUSED = 0
USP_MODE_STEPWISE = 1
USP_MAP_ZIGZAG_SHARD = 0
USP_MAP_ZIGZAG_UNSHARD = 1
USP_MAP_SEQ2HEAD = 2
USP_MAP_HEAD2SEQ = 3
USP_MAX_PERMUTE_JOBS = 4
USP_MAP_PACK_HEADS = 4
USP_MAP_UNPACK_TOKENS = 5
USP_MAP_PACK_TOKENS = 6
USP_MAP_UNPACK_HEADS = 7
USP_DILATED_MAX_PAIRS = 16
USP_MAX_ROWS_JOBS = 16


class AttnMask(ctypes.Structure):
    """usp_attn_mask of include/usp.h."""
    _fields_ = [("block_mask", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p), ("n_docs", ctypes.c_int)]


class RowsJob(ctypes.Structure):
    """usp_rows_job of include/usp.h."""
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("dtype", ctypes.c_int), ("add", ctypes.c_int),
                ("n_b", ctypes.c_int), ("n_k", ctypes.c_int), ("n_j", ctypes.c_int), ("D", ctypes.c_int),
                ("s_b", ctypes.c_longlong), ("s_k", ctypes.c_longlong), ("s_h", ctypes.c_longlong),
                ("s_k0", ctypes.c_int), ("s_kstep", ctypes.c_int), ("s_h0", ctypes.c_int), ("s_hstep", ctypes.c_int),
                ("s_hdiv", ctypes.c_int),
                ("d_b", ctypes.c_longlong), ("d_k", ctypes.c_longlong), ("d_h", ctypes.c_longlong),
                ("d_k0", ctypes.c_int), ("d_kstep", ctypes.c_int), ("d_h0", ctypes.c_int), ("d_hstep", ctypes.c_int),
                ("d_hdiv", ctypes.c_int)]


class PermuteJob(ctypes.Structure):
    """usp_permute_job of include/usp.h."""
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("H", ctypes.c_int), ("D", ctypes.c_int),
                ("dtype", ctypes.c_int)]


# name -> (restype, argtypes); mirrors include/usp.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_LL = ctypes.c_longlong
_SZ = ctypes.c_size_t
_LAYOUT = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P]
SIGNATURES = {
    "usp_version": (_I, []),
    "usp_last_error": (ctypes.c_char_p, []),
    "usp_launch_count": (ctypes.c_ulonglong, []),
    "usp_zigzag_shard": (_I, _LAYOUT),
    "usp_zigzag_unshard": (_I, _LAYOUT),
    "usp_seq2head_permute": (_I, _LAYOUT),
    "usp_head2seq_permute": (_I, _LAYOUT),
    "usp_permute_batch": (_I, [_I, ctypes.POINTER(PermuteJob), _I, _I, _I, _I, _I, _P]),
    "usp_attn_workspace_size": (_SZ, [_I] * 10),
    "usp_ulysses_pack": (_I, [_I, ctypes.POINTER(PermuteJob), _I, _I, _I, _I, _P]),
    "usp_ring_workspace_size": (_SZ, [_I] * 9),
    "usp_ring_fwd_step": (_I, [_P] * 5 + [_I] * 11 + [_P, _SZ, _P]),
    "usp_ring_fwd_accumulate": (_I, [_P] * 5 + [_I] * 11 + [_P, _SZ, _P]),
    "usp_ring_bwd_prepare": (_I, [_P] * 3 + [_I] * 8 + [_P, _SZ, _P]),
    "usp_ring_bwd_step": (_I, [_P] * 8 + [_I] * 11 + [_P, _SZ, _P]),
    "usp_dilated_workspace_size": (_SZ, [_I] * 4),
    "usp_dilated_attn_fwd": (_I, [_P] * 5 + [_I] * 7 + [_P, _P, _P, _SZ, _P]),
    "usp_dilated_bwd_workspace_size": (_SZ, [_I] * 5 + [_P, _P]),
    "usp_dilated_attn_bwd": (_I, [_P] * 9 + [_I] * 7 + [_P, _P, _P, _SZ, _P]),
    "usp_rows_copy": (_I, [ctypes.POINTER(RowsJob), _I, _P]),
    "usp_longnet_rows": (_I, [_I] * 5 + [_P] * 4),
    "usp_longnet_workspace_size": (_SZ, [_I] * 5 + [_P, _P, _I]),
    "usp_longnet_fwd_begin": (_I, [_I] * 4 + [_P, _SZ, _P]),
    "usp_longnet_fwd_local": (_I, [_P] * 3 + [_I] * 8 + [_P, _SZ, _P]),
    "usp_longnet_fwd_cross": (_I, [_P] * 3 + [_I] * 10 + [_P, _SZ, _P]),
    "usp_longnet_fwd_end": (_I, [_P, _P] + [_I] * 4 + [_P, _SZ, _P]),
    "usp_longnet_bwd_begin": (_I, [_P] * 5 + [_I] * 5 + [_P, _SZ, _P]),
    "usp_longnet_bwd_local": (_I, [_P] * 7 + [_I] * 8 + [_P, _SZ, _P]),
    "usp_longnet_bwd_cross": (_I, [_P] * 7 + [_I] * 10 + [_P, _SZ, _P]),
    "usp_longnet_bwd_end": (_I, [_P] + [_I] * 4 + [_P, _SZ, _P]),
    "usp_attn_fwd": (_I, [_P, _P, _P, _P, _P] + [_I] * 9 + [_P, _SZ, _P]),
    "usp_attn_bwd": (_I, [_P] * 9 + [_I] * 8 + [_P, _SZ, _P]),
    "usp_attn_fwd_masked": (_I, [_P] * 5 + [_I] * 8 + [ctypes.POINTER(AttnMask), _P, _SZ, _P]),
    "usp_attn_bwd_masked": (_I, [_P] * 9 + [_I] * 8 + [ctypes.POINTER(AttnMask), _P, _SZ, _P]),
    "usp_attn_bwd_prepare": (_I, [_P, _P, _P] + [_I] * 8 + [_P, _SZ, _P]),
    "usp_attn_bwd_dkdv": (_I, [_P] * 6 + [_I] * 8 + [_P, _SZ, _P]),
    "usp_attn_bwd_dkdv_bf16": (_I, [_P] * 6 + [_I] * 8 + [_P, _SZ, _P]),
    "usp_attn_bwd_dq": (_I, [_P] * 5 + [_I] * 8 + [_P, _SZ, _P]),
    "usp_attn_bwd_noalloc": (_I, [_P] * 9 + [_I] * 8 + [_P]),
    "usp_attn_bwd_noalloc_status": (_I, [_P, _P]),
    "usp_lse_merge": (_I, [_P, _P, _I, _LL, _I, _P, _I, _P, _P]),
    "usp_bwd_preprocess": (_I, [_P, _P, _P, _LL, _I, _P]),
    "usp_workspace_status": (_I, [_P, _P, _P]),
    "usp_set_wait_limit_ns": (None, [ctypes.c_ulonglong]),
    "usp_selftest_wait_timeout": (_I, [_P, _SZ, ctypes.c_ulonglong, _P]),
}

_lib = None


class UspError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"usp status {code}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m long_context_exact_tma_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int) -> int:
    if rc != USP_OK:
        raise UspError(rc, lib().usp_last_error().decode())
    return rc


def usp_version() -> int:
    return lib().usp_version()


def usp_launch_count() -> int:
    return int(lib().usp_launch_count())


def usp_last_error() -> str:
    return lib().usp_last_error().decode()


def _layout(name, src, dst, B, S, H, D, dtype, P_u, P_r, stream=None, check=True):
    rc = getattr(lib(), name)(_ptr(src), _ptr(dst), B, S, H, D, dtype, P_u, P_r, _stream(stream))
    return _check(rc) if check else rc


def usp_zigzag_shard(src, dst, B, S, H, D, dtype, P_u, P_r, stream=None, check=True):
    return _layout("usp_zigzag_shard", src, dst, B, S, H, D, dtype, P_u, P_r, stream, check)


def usp_zigzag_unshard(src, dst, B, S, H, D, dtype, P_u, P_r, stream=None, check=True):
    return _layout("usp_zigzag_unshard", src, dst, B, S, H, D, dtype, P_u, P_r, stream, check)


def usp_seq2head_permute(src, dst, B, S, H, D, dtype, P_u, P_r, stream=None, check=True):
    return _layout("usp_seq2head_permute", src, dst, B, S, H, D, dtype, P_u, P_r, stream, check)


def usp_head2seq_permute(src, dst, B, S, H, D, dtype, P_u, P_r, stream=None, check=True):
    return _layout("usp_head2seq_permute", src, dst, B, S, H, D, dtype, P_u, P_r, stream, check)


def usp_permute_batch(map_, jobs, B, S, P_u, P_r, stream=None, check=True):
    """jobs: sequence of (src, dst, H, D, dtype)."""
    arr = (PermuteJob * max(len(jobs), 1))()
    for x, (src, dst, H, D, dtype) in enumerate(jobs):
        arr[x] = PermuteJob(_ptr(src), _ptr(dst), H, D, dtype)
    rc = lib().usp_permute_batch(map_, arr, len(jobs), B, S, P_u, P_r, _stream(stream))
    return _check(rc) if check else rc


def usp_ulysses_pack(map_, jobs, B, T, G, stream=None, check=True):
    """jobs: sequence of (src, dst, H, D, dtype)."""
    arr = (PermuteJob * max(len(jobs), 1))()
    for x, (src, dst, H, D, dtype) in enumerate(jobs):
        arr[x] = PermuteJob(_ptr(src), _ptr(dst), H, D, dtype)
    rc = lib().usp_ulysses_pack(map_, arr, len(jobs), B, T, G, _stream(stream))
    return _check(rc) if check else rc


def usp_ring_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, bwd) -> int:
    return int(lib().usp_ring_workspace_size(B, S, Hq, Hkv, D, int(causal), P_u, P_r, int(bwd)))


def usp_ring_fwd_step(q, k, v, o_part, lse_part, B, S, Hq, Hkv, D, causal, P_u, P_r, i, u, t, workspace, ws_bytes,
                      stream=None, check=True):
    rc = lib().usp_ring_fwd_step(_ptr(q), _ptr(k), _ptr(v), _ptr(o_part), _ptr(lse_part), B, S, Hq, Hkv, D,
                                 int(causal), P_u, P_r, i, u, t, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_ring_fwd_accumulate(q, k, v, o_run, lse_run, B, S, Hq, Hkv, D, causal, P_u, P_r, i, u, t, workspace,
                            ws_bytes, stream=None, check=True):
    rc = lib().usp_ring_fwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(o_run), _ptr(lse_run), B, S, Hq, Hkv, D,
                                       int(causal), P_u, P_r, i, u, t, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_ring_bwd_prepare(out, lse, dO, B, S, Hq, Hkv, D, causal, P_u, P_r, workspace, ws_bytes, stream=None,
                         check=True):
    rc = lib().usp_ring_bwd_prepare(_ptr(out), _ptr(lse), _ptr(dO), B, S, Hq, Hkv, D, int(causal), P_u, P_r,
                                    _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_ring_bwd_step(q, k, v, dO, dq_acc, dq_out, dk_acc, dv_acc, B, S, Hq, Hkv, D, causal, P_u, P_r, i, u, t,
                      workspace, ws_bytes, stream=None, check=True):
    rc = lib().usp_ring_bwd_step(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dq_acc), _ptr(dq_out), _ptr(dk_acc),
                                 _ptr(dv_acc), B, S, Hq, Hkv, D, int(causal), P_u, P_r, i, u, t, _ptr(workspace),
                                 ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, mode, bwd) -> int:
    return int(lib().usp_attn_workspace_size(B, S, Hq, Hkv, D, int(causal), P_u, P_r, mode, int(bwd)))


def usp_dilated_workspace_size(B, S, Hq, D) -> int:
    return int(lib().usp_dilated_workspace_size(B, S, Hq, D))


def usp_dilated_attn_fwd(q, k, v, out, lse, B, S, Hq, Hkv, D, causal, pairs, workspace, ws_bytes, stream=None,
                         check=True):
    """pairs: sequence of (w, r)."""
    n = len(pairs)
    w = (ctypes.c_int * max(n, 1))(*[int(p[0]) for p in pairs])
    r = (ctypes.c_int * max(n, 1))(*[int(p[1]) for p in pairs])
    rc = lib().usp_dilated_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, S, Hq, Hkv, D, int(causal),
                                    n, w, r, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def _pairs(pairs):
    n = len(pairs)
    return (n, (ctypes.c_int * max(n, 1))(*[int(p[0]) for p in pairs]),
            (ctypes.c_int * max(n, 1))(*[int(p[1]) for p in pairs]))


def usp_dilated_bwd_workspace_size(B, S, Hq, D, pairs) -> int:
    n, w, r = _pairs(pairs)
    return int(lib().usp_dilated_bwd_workspace_size(B, S, Hq, D, n, w, r))


def usp_dilated_attn_bwd(q, k, v, out, lse, dO, dQ, dK, dV, B, S, Hq, Hkv, D, causal, pairs, workspace, ws_bytes,
                         stream=None, check=True):
    n, w, r = _pairs(pairs)
    rc = lib().usp_dilated_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK),
                                    _ptr(dV), B, S, Hq, Hkv, D, int(causal), n, w, r, _ptr(workspace), ws_bytes,
                                    _stream(stream))
    return _check(rc) if check else rc


def usp_rows_copy(jobs, stream=None, check=True):
    """jobs: sequence of dicts with the usp_rows_job fields (src/dst tensors or pointers; omitted strides and
    offsets default to 0, steps and divisors to 1)."""
    arr = (RowsJob * max(len(jobs), 1))()
    for x, j in enumerate(jobs):
        f = dict(add=0, s_k0=0, s_kstep=1, s_h0=0, s_hstep=1, s_hdiv=1, d_k0=0, d_kstep=1, d_h0=0, d_hstep=1,
                 d_hdiv=1, s_b=0, s_k=0, s_h=0, d_b=0, d_k=0, d_h=0)
        f.update(j)
        f["src"], f["dst"] = _ptr(f["src"]), _ptr(f["dst"])
        arr[x] = RowsJob(**f)
    rc = lib().usp_rows_copy(arr, len(jobs), _stream(stream))
    return _check(rc) if check else rc


def usp_longnet_rows(T, w, r, o, g):
    """(lp0, k_lo, n_rows, n_kept) of rank g of a segment at head offset o."""
    out = [ctypes.c_int() for _ in range(4)]
    _check(lib().usp_longnet_rows(T, w, r, o, g, *[ctypes.addressof(x) for x in out]))
    return tuple(x.value for x in out)


def usp_longnet_workspace_size(B, T, Hq, D, pairs, bwd) -> int:
    n, w, r = _pairs(pairs)
    return int(lib().usp_longnet_workspace_size(B, T, Hq, D, n, w, r, int(bwd)))


def usp_longnet_fwd_begin(B, T, Hq, D, workspace, ws_bytes, stream=None, check=True):
    rc = lib().usp_longnet_fwd_begin(B, T, Hq, D, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_longnet_fwd_local(q, k, v, B, T, Hq, Hkv, D, causal, w, r, workspace, ws_bytes, stream=None, check=True):
    rc = lib().usp_longnet_fwd_local(_ptr(q), _ptr(k), _ptr(v), B, T, Hq, Hkv, D, int(causal), w, r, _ptr(workspace),
                                     ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_longnet_fwd_cross(q, kc, vc, B, T, Hq, Hkv, D, causal, w, r, o, g, workspace, ws_bytes, stream=None,
                          check=True):
    rc = lib().usp_longnet_fwd_cross(_ptr(q), _ptr(kc), _ptr(vc), B, T, Hq, Hkv, D, int(causal), w, r, o, g,
                                     _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_longnet_fwd_end(out, lse, B, T, Hq, D, workspace, ws_bytes, stream=None, check=True):
    rc = lib().usp_longnet_fwd_end(_ptr(out), _ptr(lse), B, T, Hq, D, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_longnet_bwd_begin(out, lse, dO, dK, dV, B, T, Hq, Hkv, D, workspace, ws_bytes, stream=None, check=True):
    rc = lib().usp_longnet_bwd_begin(_ptr(out), _ptr(lse), _ptr(dO), _ptr(dK), _ptr(dV), B, T, Hq, Hkv, D,
                                     _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_longnet_bwd_local(q, k, v, dO, lse, dK, dV, B, T, Hq, Hkv, D, causal, w, r, workspace, ws_bytes, stream=None,
                          check=True):
    rc = lib().usp_longnet_bwd_local(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(lse), _ptr(dK), _ptr(dV), B, T, Hq,
                                     Hkv, D, int(causal), w, r, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_longnet_bwd_cross(q, kc, vc, dO, lse, dkc, dvc, B, T, Hq, Hkv, D, causal, w, r, o, g, workspace, ws_bytes,
                          stream=None, check=True):
    rc = lib().usp_longnet_bwd_cross(_ptr(q), _ptr(kc), _ptr(vc), _ptr(dO), _ptr(lse), _ptr(dkc), _ptr(dvc), B, T,
                                     Hq, Hkv, D, int(causal), w, r, o, g, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_longnet_bwd_end(dQ, B, T, Hq, D, workspace, ws_bytes, stream=None, check=True):
    rc = lib().usp_longnet_bwd_end(_ptr(dQ), B, T, Hq, D, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_fwd(q, k, v, out, lse, B, S, Hq, Hkv, D, causal, P_u, P_r, mode, workspace, ws_bytes,
                 stream=None, check=True):
    rc = lib().usp_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, S, Hq, Hkv, D, int(causal),
                            P_u, P_r, mode, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_bwd(q, k, v, out, lse, dO, dQ, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, workspace, ws_bytes,
                 stream=None, check=True):
    rc = lib().usp_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK),
                            _ptr(dV), B, S, Hq, Hkv, D, int(causal), P_u, P_r, _ptr(workspace), ws_bytes,
                            _stream(stream))
    return _check(rc) if check else rc


def _mask(block_mask, cu_seqlens, n_docs):
    return AttnMask(_ptr(block_mask), _ptr(cu_seqlens), int(n_docs))


def usp_attn_fwd_masked(q, k, v, out, lse, B, S, Hq, Hkv, D, causal, P_u, P_r, block_mask, cu_seqlens, n_docs,
                        workspace, ws_bytes, stream=None, check=True):
    m = _mask(block_mask, cu_seqlens, n_docs)
    rc = lib().usp_attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, S, Hq, Hkv, D, int(causal),
                                   P_u, P_r, ctypes.byref(m), _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_bwd_masked(q, k, v, out, lse, dO, dQ, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, block_mask,
                        cu_seqlens, n_docs, workspace, ws_bytes, stream=None, check=True):
    m = _mask(block_mask, cu_seqlens, n_docs)
    rc = lib().usp_attn_bwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK),
                                   _ptr(dV), B, S, Hq, Hkv, D, int(causal), P_u, P_r, ctypes.byref(m),
                                   _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_bwd_prepare(out, lse, dO, B, S, Hq, Hkv, D, causal, P_u, P_r, workspace, ws_bytes, stream=None,
                         check=True):
    rc = lib().usp_attn_bwd_prepare(_ptr(out), _ptr(lse), _ptr(dO), B, S, Hq, Hkv, D, int(causal), P_u, P_r,
                                    _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_bwd_dkdv(q, k, v, dO, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, workspace, ws_bytes, stream=None,
                      check=True):
    rc = lib().usp_attn_bwd_dkdv(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dK), _ptr(dV), B, S, Hq, Hkv, D,
                                 int(causal), P_u, P_r, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_bwd_dkdv_bf16(q, k, v, dO, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, workspace, ws_bytes,
                           stream=None, check=True):
    rc = lib().usp_attn_bwd_dkdv_bf16(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dK), _ptr(dV), B, S, Hq, Hkv, D,
                                      int(causal), P_u, P_r, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_bwd_dq(q, k, v, dO, dQ, B, S, Hq, Hkv, D, causal, P_u, P_r, workspace, ws_bytes, stream=None,
                    check=True):
    rc = lib().usp_attn_bwd_dq(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dQ), B, S, Hq, Hkv, D, int(causal),
                               P_u, P_r, _ptr(workspace), ws_bytes, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_bwd_noalloc(q, k, v, out, lse, dO, dQ, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, stream=None,
                         check=True):
    rc = lib().usp_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dO), _ptr(dQ),
                                    _ptr(dK), _ptr(dV), B, S, Hq, Hkv, D, int(causal), P_u, P_r, _stream(stream))
    return _check(rc) if check else rc


def usp_attn_bwd_noalloc_status(stream=None):
    """(status, site) of the static scratch's status word; clears it."""
    site = ctypes.c_int(0)
    rc = lib().usp_attn_bwd_noalloc_status(ctypes.byref(site), _stream(stream))
    return rc, site.value


def usp_lse_merge(o_parts, lse_parts, n_parts, rows, D, out, out_dtype, lse_out, stream=None, check=True):
    rc = lib().usp_lse_merge(_ptr(o_parts), _ptr(lse_parts), n_parts, rows, D, _ptr(out), out_dtype,
                             _ptr(lse_out), _stream(stream))
    return _check(rc) if check else rc


def usp_bwd_preprocess(out, dO, delta, rows, D, stream=None, check=True):
    rc = lib().usp_bwd_preprocess(_ptr(out), _ptr(dO), _ptr(delta), rows, D, _stream(stream))
    return _check(rc) if check else rc


def usp_workspace_status(workspace, stream=None):
    """(status, site) of the device status word; clears it."""
    site = ctypes.c_int(0)
    rc = lib().usp_workspace_status(_ptr(workspace), ctypes.byref(site), _stream(stream))
    return rc, site.value


def usp_set_wait_limit_ns(ns: int) -> None:
    lib().usp_set_wait_limit_ns(int(ns))


def usp_selftest_wait_timeout(workspace, ws_bytes, limit_ns, stream=None, check=True):
    rc = lib().usp_selftest_wait_timeout(_ptr(workspace), ws_bytes, int(limit_ns), _stream(stream))
    return _check(rc) if check else rc

"""The C ABI loads, exports every symbol include/usp.h declares, and rejects bad
arguments with the documented status codes before launching anything.

Only invalid arguments are passed here (rejected during validation), so these
tests need no GPU and never hand a fake pointer to a kernel.
"""
import ctypes
import os
import re

import pytest

from long_context_exact_tma_b200 import binding as B_

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "usp.h")

FAKE = 1 << 20  # 16-byte aligned, never dereferenced (validation fails first)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(usp_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = B_.lib()
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B_.SIGNATURES), "binding must mirror the header"


def declared_arities():
    """usp_* name -> number of parameters in its include/usp.h prototype."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(usp_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_arities_match_the_header():
    """Every ctypes signature takes exactly the prototype's parameters (a missing
    or extra argument would shift every later one)."""
    ar = declared_arities()
    assert set(ar) == set(B_.SIGNATURES)
    for name, (_, args) in B_.SIGNATURES.items():
        assert len(args) == ar[name], (name, len(args), ar[name])


def test_version_and_empty_error():
    assert B_.usp_version() >= 100
    assert isinstance(B_.usp_last_error(), str)


def test_workspace_size_queries():
    ws = B_.usp_attn_workspace_size
    assert ws(1, 256, 2, 2, 64, 1, 2, 2, 0, 0) == 256
    rows = 1 * 256 * 2
    assert ws(1, 256, 2, 2, 64, 1, 2, 2, 1, 0) == 256 + 2 * rows * (4 * 64 + 4)
    Lp = 128  # S/P_r = 128 already a multiple of 128
    assert ws(1, 256, 2, 2, 64, 1, 2, 2, 0, 1) == 256 + 2 * 4 * (4 * 1 * 1 * Lp)
    assert ws(1, 600, 2, 2, 64, 1, 1, 1, 0, 1) == 256 + 2 * 4 * (1 * 2 * 640)
    assert ws(1, 256, 2, 2, 96, 1, 2, 2, 0, 0) == 0      # D unsupported
    assert ws(1, 250, 2, 2, 64, 1, 2, 2, 0, 0) == 0      # S % 2P != 0
    assert ws(1, 256, 3, 2, 64, 1, 1, 1, 0, 0) == 0      # Hq % Hkv != 0
    assert ws(1, 256, 2, 1, 64, 1, 2, 1, 0, 0) == 0      # Hkv % P_u != 0
    assert ws(1, 256, 2, 2, 64, 1, 1, 1, 7, 0) == 0      # bad mode


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, S=256, Hq=2, Hkv=2, D=64, causal=1, P_u=2,
             P_r=2, mode=0, ws=FAKE, ws_bytes=256)
    a.update(kw)
    return B_.lib().usp_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["S"], a["Hq"], a["Hkv"],
                                 a["D"], a["causal"], a["P_u"], a["P_r"], a["mode"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), B_.USP_ERR_UNSUPPORTED),
    (dict(D=256), B_.USP_ERR_UNSUPPORTED),
    (dict(Hq=3), B_.USP_ERR_UNSUPPORTED),
    (dict(Hkv=1), B_.USP_ERR_UNSUPPORTED),
    (dict(S=250), B_.USP_ERR_UNSUPPORTED),
    (dict(S=0), B_.USP_ERR_INVALID_ARG),
    (dict(B=-1), B_.USP_ERR_INVALID_ARG),
    (dict(causal=2), B_.USP_ERR_INVALID_ARG),
    (dict(mode=5), B_.USP_ERR_INVALID_ARG),
    (dict(q=None), B_.USP_ERR_INVALID_ARG),
    (dict(lse=None), B_.USP_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), B_.USP_ERR_INVALID_ARG),
    (dict(ws=None), B_.USP_ERR_WORKSPACE),
    (dict(ws_bytes=255), B_.USP_ERR_WORKSPACE),
    (dict(mode=1, ws_bytes=4096), B_.USP_ERR_WORKSPACE),
])
def test_fwd_rejects_bad_arguments(kw, code):
    assert _fwd(**kw) == code
    assert B_.usp_last_error() != ""


def test_bwd_rejects_bad_arguments():
    L = B_.lib()
    args = [FAKE] * 9 + [1, 256, 2, 2, 64, 1, 2, 2, FAKE, 256, None]
    assert L.usp_attn_bwd(*args) == B_.USP_ERR_WORKSPACE  # needs the per-head LSE/Delta tables
    bad = list(args)
    bad[13] = 48  # D
    assert L.usp_attn_bwd(*bad) == B_.USP_ERR_UNSUPPORTED
    bad = list(args)
    bad[6] = None  # dQ
    assert L.usp_attn_bwd(*bad) == B_.USP_ERR_INVALID_ARG


def test_bwd_dkdv_bf16_rejects_bad_arguments():
    L = B_.lib()
    args = [FAKE] * 6 + [1, 256, 2, 2, 64, 1, 2, 2, FAKE, 256, None]
    assert L.usp_attn_bwd_dkdv_bf16(*args) == B_.USP_ERR_WORKSPACE  # needs the prepared tables
    bad = list(args)
    bad[10] = 48  # D
    assert L.usp_attn_bwd_dkdv_bf16(*bad) == B_.USP_ERR_UNSUPPORTED
    for i in (4, 5):  # dK, dV
        bad = list(args)
        bad[i] = None
        assert L.usp_attn_bwd_dkdv_bf16(*bad) == B_.USP_ERR_INVALID_ARG


def test_attn_bwd_rejects_other_gradient_types():
    import torch
    from long_context_exact_tma_b200 import api
    x = torch.zeros(1)
    with pytest.raises(ValueError):
        api.attn_bwd(x, x, x, x, x, x, True, 1, 1, grad_dtype=torch.float16)


@pytest.mark.parametrize("name", ["usp_zigzag_shard", "usp_zigzag_unshard", "usp_seq2head_permute",
                                  "usp_head2seq_permute"])
def test_layout_rejects_bad_arguments(name):
    fn = getattr(B_.lib(), name)
    assert fn(FAKE, FAKE, 1, 250, 4, 64, 0, 2, 2, None) == B_.USP_ERR_UNSUPPORTED   # S % 2P
    assert fn(FAKE, FAKE, 1, 256, 3, 64, 0, 2, 2, None) == B_.USP_ERR_UNSUPPORTED   # H % P_u
    assert fn(FAKE, FAKE, 1, 256, 4, 1, 0, 2, 2, None) == B_.USP_ERR_UNSUPPORTED    # D*2 % 4
    assert fn(FAKE, FAKE, 1, 256, 4, 64, 7, 2, 2, None) == B_.USP_ERR_INVALID_ARG   # dtype
    assert fn(None, FAKE, 1, 256, 4, 64, 0, 2, 2, None) == B_.USP_ERR_INVALID_ARG
    assert fn(FAKE + 4, FAKE, 1, 256, 4, 64, 0, 2, 2, None) == B_.USP_ERR_INVALID_ARG
    assert fn(FAKE, FAKE, 0, 256, 4, 64, 0, 2, 2, None) == B_.USP_ERR_INVALID_ARG


def test_merge_and_preprocess_reject_bad_arguments():
    L = B_.lib()
    assert L.usp_lse_merge(FAKE, FAKE, 0, 10, 64, FAKE, 0, FAKE, None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_lse_merge(FAKE, FAKE, 2, 10, 66, FAKE, 0, FAKE, None) == B_.USP_ERR_UNSUPPORTED
    assert L.usp_lse_merge(FAKE, FAKE, 2, 10, 64, FAKE, 3, FAKE, None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_lse_merge(None, FAKE, 2, 10, 64, FAKE, 0, FAKE, None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_bwd_preprocess(FAKE, FAKE, None, 10, 64, None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_bwd_preprocess(FAKE, FAKE, FAKE, 10, 6, None) == B_.USP_ERR_UNSUPPORTED
    assert L.usp_workspace_status(None, None, None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_selftest_wait_timeout(FAKE, 16, 1000, None) == B_.USP_ERR_WORKSPACE


def test_product_package_does_not_import_oracle():
    pkg = os.path.join(ROOT, "long_context_exact_tma_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "usp_oracle" not in text and "liboracle" not in text, f


def test_permute_batch_rejects_bad_arguments():
    L = B_.lib()
    arr = (B_.PermuteJob * 2)(B_.PermuteJob(FAKE, FAKE + 4096, 4, 64, 0), B_.PermuteJob(FAKE, FAKE, 3, 64, 0))
    assert L.usp_permute_batch(2, arr, 2, 1, 256, 2, 2, None) == B_.USP_ERR_UNSUPPORTED  # job 1: H % P_u
    assert "job 1" in B_.usp_last_error()
    assert L.usp_permute_batch(2, arr, 0, 1, 256, 2, 2, None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_permute_batch(2, arr, 5, 1, 256, 2, 2, None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_permute_batch(9, arr, 1, 1, 256, 2, 2, None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_permute_batch(2, None, 1, 1, 256, 2, 2, None) == B_.USP_ERR_INVALID_ARG
    arr[0].dtype = 7
    assert L.usp_permute_batch(2, arr, 1, 1, 256, 2, 2, None) == B_.USP_ERR_INVALID_ARG


def test_dilated_rejects_bad_arguments():
    L = B_.lib()
    import ctypes
    w = (ctypes.c_int * 2)(256, 512)
    r = (ctypes.c_int * 2)(1, 2)

    def call(S=1024, D=128, n=2, ws_bytes=1 << 30, causal=1, Hq=4, Hkv=2, ww=w, rr=r, ws=FAKE):
        return L.usp_dilated_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, S, Hq, Hkv, D, causal, n, ww, rr, ws,
                                      ws_bytes, None)
    assert call(S=1000) == B_.USP_ERR_UNSUPPORTED            # S % w != 0
    assert call(D=96) == B_.USP_ERR_UNSUPPORTED
    assert call(Hq=3) == B_.USP_ERR_UNSUPPORTED
    assert call(n=0) == B_.USP_ERR_INVALID_ARG
    assert call(n=17) == B_.USP_ERR_INVALID_ARG
    assert call(causal=3) == B_.USP_ERR_INVALID_ARG
    assert call(ws_bytes=100) == B_.USP_ERR_WORKSPACE
    assert call(ws=None) == B_.USP_ERR_WORKSPACE
    bad_r = (ctypes.c_int * 2)(1, 600)
    assert call(rr=bad_r) == B_.USP_ERR_UNSUPPORTED          # r > w
    zero_w = (ctypes.c_int * 2)(0, 512)
    assert call(ww=zero_w) == B_.USP_ERR_INVALID_ARG
    assert B_.usp_dilated_workspace_size(1, 1024, 4, 128) == 256 + 1024 * 4 * (4 * 128 + 4)
    assert B_.usp_dilated_workspace_size(1, 1024, 4, 96) == 0


def test_masked_rejects_unaligned_chunks_and_bad_docs():
    L = B_.lib()
    m = B_.AttnMask(FAKE, None, 0)
    # S=768, P=4: chunks of 96 tokens are not whole tiles
    rc = L.usp_attn_fwd_masked(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 768, 4, 4, 128, 1, 2, 2, m, FAKE, 256, None)
    assert rc == B_.USP_ERR_UNSUPPORTED and "128" in B_.usp_last_error()
    m2 = B_.AttnMask(None, FAKE, 0)
    rc = L.usp_attn_fwd_masked(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1024, 4, 4, 128, 1, 2, 2, m2, FAKE, 256, None)
    assert rc == B_.USP_ERR_INVALID_ARG
    rc = L.usp_attn_bwd_masked(*([FAKE] * 9), 1, 768, 4, 4, 128, 1, 2, 2, m, FAKE, 1 << 30, None)
    assert rc == B_.USP_ERR_UNSUPPORTED


def test_rows_copy_rejects_bad_jobs():
    """Validation of usp_rows_copy before any launch (no GPU needed)."""
    L = B_.lib()
    good = dict(src=FAKE, dst=FAKE, dtype=B_.USP_BF16, n_b=1, n_k=4, n_j=2, D=128, s_b=0, s_k=256, s_h=128,
                d_b=0, d_k=256, d_h=128)

    def call(**kw):
        j = dict(good)
        j.update(kw)
        arr = (B_.RowsJob * 1)()
        f = dict(add=0, s_k0=0, s_kstep=1, s_h0=0, s_hstep=1, s_hdiv=1, d_k0=0, d_kstep=1, d_h0=0, d_hstep=1,
                 d_hdiv=1)
        f.update(j)
        arr[0] = B_.RowsJob(**f)
        return L.usp_rows_copy(arr, 1, None)
    assert call(dtype=5) == B_.USP_ERR_INVALID_ARG                 # unknown dtype
    assert call(add=1) == B_.USP_ERR_INVALID_ARG                   # add needs fp32
    assert call(D=12) == B_.USP_ERR_INVALID_ARG                    # 24-byte rows
    assert call(s_hdiv=0) == B_.USP_ERR_INVALID_ARG
    assert call(d_kstep=-1) == B_.USP_ERR_INVALID_ARG
    assert call(src=None) == B_.USP_ERR_INVALID_ARG
    assert call(dst=FAKE + 8) == B_.USP_ERR_INVALID_ARG            # unaligned
    assert call(s_k=100) == B_.USP_ERR_INVALID_ARG                 # rows not 16-byte aligned
    assert call(n_k=0) == B_.USP_OK                                 # nothing to move, nothing launched
    assert L.usp_rows_copy(None, 1, None) == B_.USP_ERR_INVALID_ARG
    arr = (B_.RowsJob * 17)()
    assert L.usp_rows_copy(arr, 17, None) == B_.USP_ERR_INVALID_ARG


def test_longnet_rejects_bad_arguments():
    import ctypes
    L = B_.lib()
    ws = 1 << 30
    # local pairs need w <= T and T % w == 0; gathered ones w > T, w % T == 0
    assert L.usp_longnet_fwd_local(FAKE, FAKE, FAKE, 1, 1024, 4, 4, 128, 1, 2048, 2, FAKE, ws, None) \
        == B_.USP_ERR_UNSUPPORTED
    assert L.usp_longnet_fwd_local(FAKE, FAKE, FAKE, 1, 1024, 4, 4, 128, 1, 384, 2, FAKE, ws, None) \
        == B_.USP_ERR_UNSUPPORTED
    assert L.usp_longnet_fwd_cross(FAKE, FAKE, FAKE, 1, 1024, 4, 4, 128, 1, 512, 2, 0, 0, FAKE, ws, None) \
        == B_.USP_ERR_UNSUPPORTED
    assert L.usp_longnet_fwd_cross(FAKE, FAKE, FAKE, 1, 1024, 4, 4, 128, 1, 3072, 2, 2, 0, FAKE, ws, None) \
        == B_.USP_ERR_INVALID_ARG                                   # offset >= r
    assert L.usp_longnet_fwd_cross(FAKE, FAKE, FAKE, 1, 1024, 4, 4, 128, 1, 3072, 2, 0, 3, FAKE, ws, None) \
        == B_.USP_ERR_INVALID_ARG                                   # rank outside the segment of 3
    assert L.usp_longnet_fwd_cross(FAKE, FAKE, FAKE, 1, 1024, 4, 4, 96, 1, 3072, 2, 0, 0, FAKE, ws, None) \
        == B_.USP_ERR_UNSUPPORTED                                   # D
    assert L.usp_longnet_fwd_begin(1, 1024, 4, 128, FAKE, 100, None) == B_.USP_ERR_WORKSPACE
    assert L.usp_longnet_rows(1024, 1536, 2, 0, 0, None, None, None, None) == B_.USP_ERR_INVALID_ARG
    w = (ctypes.c_int * 2)(512, 4096)
    r = (ctypes.c_int * 2)(1, 3)
    n = B_.usp_longnet_workspace_size(1, 1024, 4, 128, [(512, 1), (4096, 3)], 1)
    assert n > 256 and B_.usp_longnet_workspace_size(1, 1024, 4, 128, [(768, 1)], 1) == 0
    assert L.usp_longnet_workspace_size(1, 1024, 4, 128, 2, w, r, 0) == 256 + 1024 * 4 * (4 * 128 + 4)
    assert L.usp_longnet_bwd_local(*([FAKE] * 7), 1, 1024, 4, 4, 128, 1, 512, 1, FAKE, 1000, None) \
        == B_.USP_ERR_WORKSPACE


def test_ring_accumulate_rejects_bad_arguments():
    L = B_.lib()
    # rank outside the 1 x 4 mesh, then a step past the ring
    assert L.usp_ring_fwd_accumulate(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1024, 4, 4, 128, 1, 1, 4, 4, 0, 0, FAKE, 256,
                                     None) == B_.USP_ERR_INVALID_ARG
    assert L.usp_ring_fwd_accumulate(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1024, 4, 4, 128, 1, 1, 4, 0, 0, 4, FAKE, 256,
                                     None) == B_.USP_ERR_INVALID_ARG

"""usp_attn_bwd_noalloc: the attention backward for callers that cannot
allocate device memory for a workspace (for example while a framework's caching
allocator or a pool reserved at start-up owns the device memory, or in serving
loops that must not allocate after initialisation). It keeps its scratch in a
static device array of the library and must give the results of usp_attn_bwd
with a caller workspace, on consecutive calls that reuse that array.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from long_context_exact_tma_b200 import api
from long_context_exact_tma_b200 import binding as B_
from usp_inputs import workload

from helpers import GRAD_REL_L2, rel_l2

pytestmark = pytest.mark.gpu


def test_noalloc_backward_matches_workspace_backward_on_two_calls(cuda):
    spec = dict(B=1, S=1536, Hq=8, Hkv=2, D=128, causal=True, P_u=2, P_r=2, seed=901, peaky=False)
    B, S, Hq, Hkv, D, P_u, P_r = (spec[k] for k in ("B", "S", "Hq", "Hkv", "D", "P_u", "P_r"))
    t = workload(spec, device=cuda, which=("q", "k", "v", "do"))
    q, k, v, do = (api.to_head_sharded(t[n], P_u, P_r) for n in ("q", "k", "v", "do"))
    out, lse = api.attn_fwd(q, k, v, True, P_u, P_r)
    ref = api.attn_bwd(q, k, v, out, lse, do, True, P_u, P_r)
    torch.cuda.synchronize()
    need = B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, 1, P_u, P_r, 0, 1)
    assert 0 < need <= (32 << 20)
    for call in range(2):  # the second call reuses (and must re-clear) the static scratch
        dq = torch.full_like(q, float("nan"))
        dk = torch.full(k.shape, float("nan"), dtype=torch.float32, device=cuda)
        dv = torch.full(v.shape, float("nan"), dtype=torch.float32, device=cuda)
        B_.usp_attn_bwd_noalloc(q, k, v, out, lse, do, dq, dk, dv, B, S, Hq, Hkv, D, 1, P_u, P_r)
        torch.cuda.synchronize()
        # no bounded device wait gave up during the call (the reader clears the word)
        assert B_.usp_attn_bwd_noalloc_status() == (B_.USP_OK, 0)
        for got, want, name in ((dq, ref[0], "dq"), (dk, ref[1], "dk"), (dv, ref[2], "dv")):
            g = got.double().cpu().numpy()
            w = want.double().cpu().numpy()
            assert np.isfinite(g).all(), (call, name)
            assert rel_l2(g, w) <= GRAD_REL_L2, (call, name, rel_l2(g, w))


def test_noalloc_rejects_problems_beyond_its_scratch(cuda):
    # The call below passes placeholder buffers, so it must be rejected before any
    # launch: check first that this shape's scratch really exceeds the static array.
    B, S, H, D = 4, 262144, 32, 128
    need = B_.usp_attn_workspace_size(B, S, H, H, D, 1, 1, 1, 0, 1)
    assert need > (32 << 20), need
    big = torch.empty(16, dtype=torch.uint8, device=cuda)
    rc = B_.usp_attn_bwd_noalloc(big, big, big, big, big, big, big, big, big, B, S, H, H, D, 1, 1, 1,
                                 check=False)
    assert rc == B_.USP_ERR_WORKSPACE
    msg = B_.usp_last_error()
    assert "static scratch" in msg and "usp_attn_bwd" in msg

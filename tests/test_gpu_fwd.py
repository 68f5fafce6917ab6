"""GPU parity of usp_attn_fwd against the fp64 oracle: whole tensors on small
cases that span several tiles, ragged tails and every mask path; sampled rows
at the full sizes of the five workloads."""
import pytest
import torch

from long_context_exact_tma_b200 import binding as B_
from usp_inputs import WORKLOADS

from helpers import assert_fwd_ok, compare_fwd, gpu_fwd, inputs, make_spec, sample_rows

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_causal_usp2x2": make_spec(**{k: WORKLOADS[1][k] for k in ("B", "S", "Hq", "Hkv", "D", "causal", "P_u", "P_r", "seed")}),
    "causal_ring2_aligned": make_spec(S=1024, Hq=4, Hkv=4, D=128, P_r=2, seed=201),
    "noncausal_ragged": make_spec(S=600, Hq=2, Hkv=2, D=128, seed=202, causal=False),
    "gqa_usp2x2_unaligned": make_spec(S=1536, Hq=8, Hkv=2, D=128, P_u=2, P_r=2, seed=203),
    "d64_ragged_unaligned": make_spec(S=200, Hq=2, Hkv=1, D=64, P_r=2, seed=204),
    "batch2_causal_ring4": make_spec(B=2, S=2048, Hq=2, Hkv=2, D=128, P_r=4, seed=205),
    "noncausal_usp2x2_gqa": make_spec(S=1024, Hq=4, Hkv=2, D=64, P_u=2, P_r=2, seed=206, causal=False),
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("mode", [B_.USP_MODE_FUSED, B_.USP_MODE_STEPWISE])
def test_fwd_small_full_tensors(cuda, name, mode):
    spec = SMALL[name]
    t = inputs(spec)
    o, lse = gpu_fwd(spec, t, mode)
    tc = {k: v.cpu() for k, v in t.items() if k != "spec"}
    assert_fwd_ok(compare_fwd(o, lse, tc, spec))


def test_fwd_peaky_keys_small(cuda):
    spec = make_spec(S=2048, Hq=2, Hkv=2, D=128, P_r=4, seed=207, causal=False, peaky=True)
    t = inputs(spec)
    for mode in (B_.USP_MODE_FUSED, B_.USP_MODE_STEPWISE):
        o, lse = gpu_fwd(spec, t, mode)
        tc = {k: v.cpu() for k, v in t.items() if k not in ("spec", "peaky_positions")}
        assert_fwd_ok(compare_fwd(o, lse, tc, spec))


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_fwd_full_size_sampled_rows(cuda, cfg):
    spec = dict(WORKLOADS[cfg])
    t = inputs(spec)
    mode = B_.USP_MODE_STEPWISE if cfg == 5 else B_.USP_MODE_FUSED
    o, lse = gpu_fwd(spec, t, mode)
    tc = {k: v.cpu() for k, v in t.items() if k not in ("spec", "peaky_positions")}
    del t
    torch.cuda.empty_cache()
    rows = sample_rows(spec, 48 if cfg == 5 else 96, seed=cfg)
    assert_fwd_ok(compare_fwd(o, lse, tc, spec, rows))

"""GPU parity of usp_attn_fwd against the fp64 oracle: whole tensors on small
cases that span several tiles, ragged tails and every mask path; sampled rows
at the full sizes of the five workloads; and an fp32 view of the peaky case
(the merged ring-step partials before the final bf16 rounding), held to the
max-abs bound with no rounding allowance."""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_tma_b200 import api
from long_context_exact_tma_b200 import binding as B_
from usp_inputs import WORKLOADS

from helpers import (assert_fwd_ok, compare_fwd, fwd_stats, gpu_fwd, head_shard_cpu, inputs, make_spec,
                     sample_rows, unshard_cpu)

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
MODES = {B_.USP_MODE_FUSED: "fused", B_.USP_MODE_STEPWISE: "stepwise"}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("mode", [B_.USP_MODE_FUSED, B_.USP_MODE_STEPWISE])
def test_fwd_small_full_tensors(cuda, name, mode):
    spec = SMALL[name]
    t = inputs(spec)
    o, lse = gpu_fwd(spec, t, mode)
    tc = {k: v.cpu() for k, v in t.items() if k != "spec"}
    assert_fwd_ok(compare_fwd(o, lse, tc, spec, name=f"{name}/{MODES[mode]}"))


PEAKY = make_spec(S=2048, Hq=2, Hkv=2, D=128, P_r=4, seed=207, causal=False, peaky=True)


def test_fwd_peaky_keys_small(cuda):
    t = inputs(PEAKY)
    tc = {k: v.cpu() for k, v in t.items() if k not in ("spec", "peaky_positions")}
    for mode in (B_.USP_MODE_FUSED, B_.USP_MODE_STEPWISE):
        o, lse = gpu_fwd(PEAKY, t, mode)
        assert_fwd_ok(compare_fwd(o, lse, tc, PEAKY, name=f"peaky_ring4/{MODES[mode]}"))


@pytest.mark.parametrize("spec_name", ["peaky_ring4", "peaky_ring16_s8k"])
def test_fwd_peaky_fp32_partials_meet_raw_bound(cuda, spec_name):
    """The stepwise forward leaves in its workspace the running merge of ring steps
    0..P_r-2 and the partial of step P_r-1 (fp32). Merging those two with
    usp_lse_merge into an fp32 O gives the attention before its bf16 rounding,
    which must meet max abs <= 1e-2 on every element, with no rounding allowance."""
    spec = PEAKY if spec_name == "peaky_ring4" else make_spec(S=8192, Hq=2, Hkv=2, D=128, P_r=16, seed=208,
                                                              causal=False, peaky=True)
    t = inputs(spec)
    dev = torch.device("cuda")
    P_u, P_r = spec["P_u"], spec["P_r"]
    q, k, v = (head_shard_cpu(t[n], spec).to(dev) for n in ("q", "k", "v"))
    B, S, Hq, Hkv, D = spec["B"], spec["S"], spec["Hq"], spec["Hkv"], spec["D"]
    need = B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, 0, P_u, P_r, B_.USP_MODE_STEPWISE, 0)
    rows = B * S * Hq
    assert need == 256 + 2 * rows * (4 * D + 4)  # two partials, whatever P_r is
    ws = api.workspace(need, dev)
    out, lse = api.attn_fwd(q, k, v, False, P_u, P_r, mode=B_.USP_MODE_STEPWISE, ws=ws, check_status=True)
    body = ws[256:]
    o_parts = body[: 2 * rows * D * 4].view(torch.float32).view(2, rows, D)
    l_parts = body[2 * rows * D * 4:].view(torch.float32).view(2, rows)
    o32, l32 = api.lse_merge(o_parts, l_parts, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(l32, lse.reshape(-1))  # the same merge the forward's last step made
    o32 = unshard_cpu(o32.view(q.shape).cpu(), spec)
    l32 = unshard_cpu(l32.view(lse.shape).unsqueeze(-1).contiguous().cpu(), spec)[..., 0]
    tc = {k_: v_.cpu() for k_, v_ in t.items() if k_ in ("q", "k", "v")}
    rows_all = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(S)]
    o_ref, lse_ref = oracle.attn_fwd_rows(tc["q"], tc["k"], tc["v"], False, rows_all)
    idx = np.array(rows_all)
    st = fwd_stats(o32.numpy()[idx[:, 0], idx[:, 2], idx[:, 1]], l32.numpy()[idx[:, 0], idx[:, 2], idx[:, 1]],
                   o_ref, lse_ref, name=f"{spec_name}/fp32", bf16_out=False)
    assert st["o_max"] <= 1e-2, st
    assert st["o_mean"] <= 1e-3 and st["lse_max"] <= 1e-3, st


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
    assert_fwd_ok(compare_fwd(o, lse, tc, spec, rows, name=f"{spec['name']}/{MODES[mode]}/sampled"))

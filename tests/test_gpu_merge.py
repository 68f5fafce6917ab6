"""GPU parity of the log-sum-exp merge and of the backward preprocess."""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_tma_b200 import api
from usp_inputs import normal_bf16, uniform_f32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,rows,D,out_dtype", [
    (2, 1000, 64, torch.bfloat16), (16, 4099, 128, torch.float32), (5, 333, 128, torch.bfloat16),
    (1, 64, 64, torch.float32)])
def test_lse_merge_matches_oracle(cuda, n, rows, D, out_dtype):
    o = normal_bf16(20 + n, (n, rows, D), device=cuda).float()
    lse = (normal_bf16(40 + n, (n, rows), device=cuda).float() * 4.0).contiguous()
    # empty partials (no visible key) and one row with no partial at all
    drop = uniform_f32(60 + n, (n, rows), device=cuda) < 0.3
    lse = torch.where(drop, torch.full_like(lse, float("-inf")), lse)
    lse[:, 0] = float("-inf")
    o = torch.where(drop.unsqueeze(-1), torch.zeros_like(o), o).contiguous()
    out, lse_out = api.lse_merge(o, lse, out_dtype=out_dtype)
    ref_o, ref_l = oracle.lse_merge(o.double().cpu().numpy(), lse.double().cpu().numpy())
    got_o = out.float().cpu().numpy()
    got_l = lse_out.cpu().numpy()
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isneginf(got_l), ~fin)
    assert np.abs(got_l[fin] - ref_l[fin]).max() < 1e-5
    # fp32 output: fp32 arithmetic error; bf16 output: one rounding to bf16 (half an ulp, 2^-9 relative)
    rel = 1e-6 if out_dtype == torch.float32 else 2.0 ** -8
    assert np.all(np.abs(got_o - ref_o) <= rel * np.abs(ref_o) + 1e-5)
    assert np.all(got_o[~fin] == 0)


def test_bwd_preprocess_matches_definition(cuda):
    rows, D = 5000, 128
    o = normal_bf16(90, (rows, D), device=cuda)
    do = normal_bf16(91, (rows, D), device=cuda)
    delta = api.bwd_preprocess(o, do)
    ref = (o.double() * do.double()).sum(-1)
    assert (delta.double() - ref).abs().max().item() < 1e-4

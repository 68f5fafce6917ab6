"""GPU parity of the layout gathers (zigzag shard/unshard, seq->head, head->seq):
bit-exact against the oracle's push-style maps, called through the C ABI."""
import pytest
import torch

import oracle
from long_context_exact_tma_b200 import api
from usp_inputs import normal_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,S,H,D,P_u,P_r,dtype", [
    (1, 256, 2, 64, 2, 2, torch.bfloat16),     # the tiny causal case
    (2, 1536, 8, 128, 2, 3, torch.bfloat16),
    (1, 960, 4, 64, 4, 1, torch.bfloat16),
    (1, 640, 6, 1, 2, 2, torch.float32),       # LSE rows (D = 1)
    (2, 512, 8, 1, 4, 2, torch.float32),
    (1, 400, 3, 16, 1, 5, torch.float32),
])
def test_layout_bit_exact(cuda, B, S, H, D, P_u, P_r, dtype):
    if dtype == torch.bfloat16:
        x = normal_bf16(7, (B, S, H, D), device=cuda)
    else:
        x = normal_bf16(8, (B, S, H, D), device=cuda).float()
    xc = x.cpu()
    rm = api.zigzag_shard(x, P_u, P_r)
    assert torch.equal(rm.cpu(), oracle.zigzag_shard(xc, P_u * P_r))
    hs = api.seq2head(rm, P_u, P_r)
    hs_ref = oracle.seq2head(rm.cpu(), P_u, P_r)
    assert torch.equal(hs.cpu(), hs_ref)
    back = api.head2seq(hs, P_u, P_r)
    assert torch.equal(back.cpu(), oracle.head2seq(hs_ref, P_u, P_r))
    assert torch.equal(api.zigzag_unshard(back, P_u, P_r).cpu(), xc)


@pytest.mark.parametrize("cfg", [3])
def test_layout_full_size_config3(cuda, cfg):
    """The GQA USP 4x2 workload at full size: Q [1, 131072, 32, 128] and K [.., 8, ..]."""
    from usp_inputs import WORKLOADS
    w = WORKLOADS[cfg]
    P_u, P_r = w["P_u"], w["P_r"]
    for H, seed in ((w["Hq"], 3000), (w["Hkv"], 3001)):
        x = normal_bf16(seed, (w["B"], w["S"], H, w["D"]), device=cuda)
        hs = api.to_head_sharded(x, P_u, P_r)
        ref = oracle.to_head_sharded(x.cpu(), P_u, P_r)
        assert torch.equal(hs.cpu(), ref)
        assert torch.equal(api.from_head_sharded(hs, P_u, P_r), x)
        del x, hs, ref


@pytest.mark.parametrize("B,S,P_u,P_r,lse_hl", [(1, 1536, 2, 3, 4), (2, 512, 4, 2, 4), (1, 256, 1, 2, 4),
                                                (1, 640, 2, 2, 3)])
def test_permute_batch_bit_exact_mixed_jobs(cuda, B, S, P_u, P_r, lse_hl):
    """usp_permute_batch moves Q, K, V (different head counts) and an fp32 LSE-like
    tensor in one launch exactly as the oracle's maps do, in both directions. With
    3 LSE heads per rank (12-byte runs) the whole batch takes the 4-byte path."""
    from long_context_exact_tma_b200 import binding as B_
    H = 4 * P_u
    shapes = [((B, S, H, 128), torch.bfloat16), ((B, S, P_u, 128), torch.bfloat16),
              ((B, S, 2 * P_u, 64), torch.bfloat16), ((B, S, lse_hl * P_u, 1), torch.float32)]
    xs = [(normal_bf16(50 + n, shp, device=cuda).to(dt)) for n, (shp, dt) in enumerate(shapes)]
    rms = [api.zigzag_shard(x, P_u, P_r) for x in xs]
    hs = api.seq2head_many(rms, P_u, P_r)
    for rm, h in zip(rms, hs):
        assert torch.equal(h.cpu(), oracle.seq2head(rm.cpu(), P_u, P_r))
    back = api.head2seq_many(hs, P_u, P_r)
    for rm, bk in zip(rms, back):
        assert torch.equal(bk.cpu(), rm.cpu())
    # the zigzag maps batched too
    P = P_u * P_r
    outs = [torch.empty_like(r) for r in rms]
    B_.usp_permute_batch(B_.USP_MAP_ZIGZAG_SHARD, [(x, o, x.shape[2], x.shape[3], api._dt(x))
                                                   for x, o in zip(xs, outs)], B, S, P_u, P_r)
    for o, x in zip(outs, xs):
        assert torch.equal(o.cpu(), oracle.zigzag_shard(x.cpu(), P))

"""GPU parity of usp_dilated_attn_fwd (LongNet dilated attention) against the
fp64 oracle: whole tensors on small cases (segments that are and are not
multiples of the dilation, head offsets, GQA, causal and not, ragged kept-row
counts below a tile), and sampled rows at the LongNet segment/dilation schedule
w = {2048, 4096, 8192, 16384, 32768}, r = {1, 2, 4, 6, 12} on a 32K sequence."""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_tma_b200 import api
from usp_inputs import normal_bf16

from helpers import assert_fwd_ok, fwd_stats

pytestmark = pytest.mark.gpu

LONGNET_PAIRS = [(2048, 1), (4096, 2), (8192, 4), (16384, 6), (32768, 12)]

CASES = {
    # name: (B, S, Hq, Hkv, D, causal, pairs)
    "longnet_scaled_s6k": (1, 6144, 4, 4, 128, True, [(512, 1), (1024, 2), (2048, 4), (3072, 6), (6144, 12)]),
    "noncausal_gqa_d64": (2, 2048, 8, 2, 64, False, [(256, 1), (1024, 3), (2048, 8)]),
    "single_pair_full": (1, 1024, 2, 2, 128, True, [(1024, 1)]),
    "tiny_segments": (1, 768, 4, 2, 128, True, [(96, 1), (192, 5), (768, 7)]),
    "sparse_rows_only": (1, 1536, 6, 6, 64, True, [(1536, 4), (512, 2)]),
    # the r = 1 pair (which writes the running result) listed last, with GQA
    "r1_pair_listed_last": (1, 1024, 4, 2, 128, True, [(512, 2), (1024, 3), (256, 1)]),
}


def _inputs(B, S, Hq, Hkv, D, seed, device):
    q = normal_bf16(seed, (B, S, Hq, D), device=device)
    k = normal_bf16(seed + 1, (B, S, Hkv, D), device=device)
    v = normal_bf16(seed + 2, (B, S, Hkv, D), device=device)
    return q, k, v


def _compare(o, lse, q, k, v, causal, pairs, rows, name):
    o_ref, lse_ref = oracle.dilated_fwd_rows(q.cpu(), k.cpu(), v.cpu(), causal, pairs, rows)
    idx = np.array(rows)
    o_g = o.float().cpu().numpy()[idx[:, 0], idx[:, 2], idx[:, 1]]
    l_g = lse.cpu().numpy()[idx[:, 0], idx[:, 2], idx[:, 1]]
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(l_g), empty), name  # rows that no pair keeps
    assert np.all(o_g[empty] == 0), name
    keep = ~empty
    st = fwd_stats(o_g[keep], l_g[keep], o_ref[keep], lse_ref[keep], name=name)
    assert_fwd_ok(st)


@pytest.mark.parametrize("name", list(CASES))
def test_dilated_small_full_tensors(cuda, name):
    B, S, Hq, Hkv, D, causal, pairs = CASES[name]
    q, k, v = _inputs(B, S, Hq, Hkv, D, 700 + len(name), cuda)
    o, lse = api.dilated_attn_fwd(q, k, v, causal, pairs, check_status=True)
    rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(S)]
    _compare(o, lse, q, k, v, causal, pairs, rows, f"dilated/{name}")


def test_dilated_longnet_schedule_sampled_rows(cuda):
    B, S, Hq, Hkv, D = 1, 32768, 16, 16, 128
    q, k, v = _inputs(B, S, Hq, Hkv, D, 750, cuda)
    o, lse = api.dilated_attn_fwd(q, k, v, True, LONGNET_PAIRS, check_status=True)
    rng = np.random.default_rng(5)
    rows = [(0, int(rng.integers(Hq)), int(rng.integers(S))) for _ in range(192)]
    rows += [(0, 0, 0), (0, Hq - 1, S - 1), (0, 11, 32767), (0, 5, 16389)]
    _compare(o, lse, q, k, v, True, LONGNET_PAIRS, rows, "dilated/longnet_s32k/sampled")


def test_dilated_two_calls_reuse_workspace(cuda):
    """The running result is re-initialised on every call: a second call on the
    same workspace gives bit for bit the first call's result."""
    B, S, Hq, Hkv, D, causal, pairs = CASES["noncausal_gqa_d64"]
    q, k, v = _inputs(B, S, Hq, Hkv, D, 760, cuda)
    from long_context_exact_tma_b200 import binding as B_
    ws = api.workspace(B_.usp_dilated_workspace_size(B, S, Hq, D), cuda)
    o1, l1 = api.dilated_attn_fwd(q, k, v, causal, pairs, ws=ws)
    o2, l2 = api.dilated_attn_fwd(q, k, v, causal, pairs, ws=ws, check_status=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


BWD_CASES = {
    # name: (B, S, Hq, Hkv, D, causal, pairs) -- whole-tensor oracle in seconds
    "longnet_scaled_s768": (1, 768, 4, 4, 128, True, [(64, 1), (128, 2), (256, 4), (384, 6), (768, 12)]),
    "noncausal_gqa_d64": (2, 512, 8, 2, 64, False, [(128, 1), (256, 3), (512, 8)]),
    "tiny_segments_gqa": (1, 384, 4, 2, 128, True, [(96, 1), (192, 5), (384, 7)]),
    # r a multiple of the group size: each dK/dV launch walks only its offset's kv heads
    "gqa_r_multiple_of_group": (1, 512, 8, 4, 128, True, [(128, 2), (256, 4), (512, 8)]),
    # no r = 1 pair (the gradients start from zero) / the r = 1 pair (which writes them) listed last
    "no_r1_pair": (1, 512, 4, 4, 128, True, [(256, 2), (512, 4)]),
    "r1_pair_listed_last_gqa": (1, 512, 4, 2, 128, True, [(256, 2), (512, 3), (128, 1)]),
}


@pytest.mark.parametrize("name", list(BWD_CASES))
def test_dilated_backward_full_tensors(cuda, name):
    from helpers import GRAD_REL_L2, GRAD_STATS, rel_l2
    B, S, Hq, Hkv, D, causal, pairs = BWD_CASES[name]
    q, k, v = _inputs(B, S, Hq, Hkv, D, 770 + len(name), cuda)
    do = normal_bf16(790 + len(name), (B, S, Hq, D), device=cuda)
    o, lse = api.dilated_attn_fwd(q, k, v, causal, pairs, check_status=True)
    dq, dk, dv = api.dilated_attn_bwd(q, k, v, o, lse, do, causal, pairs, check_status=True)
    torch.cuda.synchronize()
    ref = oracle.dilated_attn_full(q.cpu(), k.cpu(), v.cpu(), do.cpu(), causal, pairs)
    errs = {n: rel_l2(g.double().cpu().numpy(), ref[n]) for n, g in (("dq", dq), ("dk", dk), ("dv", dv))}
    GRAD_STATS.append((f"dilated/{name}", errs))
    assert all(e <= GRAD_REL_L2 for e in errs.values()), errs


@pytest.mark.parametrize("Hkv", [16, 4])
def test_dilated_backward_longnet_s32k_invariants(cuda, Hkv):
    """The LongNet schedule at S=32K (the bench's dilated workload, and its GQA
    form with 4 query heads per kv head), backward at full size through
    size-independent properties. The backward uses the merged LSE, so a query's
    weights over all its pairs' keys sum to 1 (keys counted once per pair): per
    kv head sum_j dK_j = 0 and sum_j dV_j = the sum of dO_i over the group's
    query heads. A kv head or a pair's rows left out, counted twice, or an add
    lost between the head offsets' launches (which run side by side) breaks them."""
    from helpers import GRAD_REL_L2, GRAD_STATS, sum_invariants
    B, S, H, D = 1, 32768, 16, 128
    q, k, v = _inputs(B, S, H, Hkv, D, 820, cuda)
    do = normal_bf16(821, (B, S, H, D), device=cuda)
    o, lse = api.dilated_attn_fwd(q, k, v, True, LONGNET_PAIRS, check_status=True)
    dq, dk, dv = api.dilated_attn_bwd(q, k, v, o, lse, do, True, LONGNET_PAIRS, check_status=True)
    torch.cuda.synchronize()
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()
    ek, ev = sum_invariants(dk.cpu(), dv.cpu(), do.cpu(), H // Hkv)
    GRAD_STATS.append((f"dilated/longnet_s32k_hkv{Hkv}/invariants", {"sum_dk": ek, "sum_dv": ev}))
    assert ek <= GRAD_REL_L2 and ev <= GRAD_REL_L2, (ek, ev)

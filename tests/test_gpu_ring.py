"""GPU parity of the per-rank calls of a real multi-GPU USP mesh (usp_ring_*,
usp_ulysses_pack), with every rank of the mesh run in turn on the one GPU: the
Ulysses pack/unpack around an (emulated) all-to-all are bit-exact against the
oracle's layout maps, and the ring schedule of per-rank steps -- each rank's
queries against the K/V block it holds at step t, partials merged by
usp_lse_merge, gradients of a block accumulated as it travels -- matches the
fp64 oracle, forward and backward."""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_tma_b200 import api
from long_context_exact_tma_b200 import binding as B_

from helpers import GRAD_REL_L2, GRAD_STATS, assert_fwd_ok, compare_fwd, inputs, make_spec, rel_l2

pytestmark = pytest.mark.gpu

CASES = {
    "causal_usp2x2_gqa": make_spec(B=2, S=1024, Hq=8, Hkv=4, D=128, P_u=2, P_r=2, seed=601),
    "causal_ring4_d64": make_spec(B=1, S=1536, Hq=2, Hkv=2, D=64, P_u=1, P_r=4, seed=602),
    "noncausal_usp2x3_ragged": make_spec(B=1, S=600, Hq=4, Hkv=2, D=128, P_u=2, P_r=3, seed=603, causal=False),
}


def _dt(t):
    return B_.USP_BF16 if t.dtype == torch.bfloat16 else B_.USP_F32


def test_ulysses_pack_around_all_to_all_bit_exact(cuda):
    """Per rank: pack heads, all-to-all (emulated by indexing), unpack tokens gives
    the rank's slice of the head-sharded layout; the way back restores the
    rank-local tensor (bf16 and fp32 rows)."""
    B, S, P_u, P_r = 2, 1536, 2, 3
    P, T = P_u * P_r, S // (P_u * P_r)
    for H, D, dt in ((8, 128, torch.bfloat16), (4, 1, torch.float32)):
        x = torch.randn(B, S, H, D).to(dt)
        rm = oracle.zigzag_shard(x, P).to(cuda)  # [P, B, T, H, D]: the rank-local tensors
        hs_ref = oracle.to_head_sharded(x, P_u, P_r)
        G, Hl = P_u, H // P_u
        for i in range(P_r):
            sends = []
            for u in range(P_u):
                s = torch.empty((G, B, T, Hl, D), dtype=dt, device=cuda)
                B_.usp_ulysses_pack(B_.USP_MAP_PACK_HEADS, [(rm[i * P_u + u], s, H, D, _dt(s))], B, T, G)
                sends.append(s)
            backs = []
            for u in range(P_u):
                recv = torch.stack([sends[up][u] for up in range(P_u)])  # the all-to-all
                got = torch.empty((B, G * T, Hl, D), dtype=dt, device=cuda)
                B_.usp_ulysses_pack(B_.USP_MAP_UNPACK_TOKENS, [(recv, got, H, D, _dt(got))], B, T, G)
                assert torch.equal(got.cpu(), hs_ref[i, u])
                # and back: pack tokens, all-to-all, unpack heads
                back_s = torch.empty((G, B, T, Hl, D), dtype=dt, device=cuda)
                B_.usp_ulysses_pack(B_.USP_MAP_PACK_TOKENS, [(got, back_s, H, D, _dt(got))], B, T, G)
                backs.append(back_s)
            for u in range(P_u):
                recv = torch.stack([backs[up][u] for up in range(P_u)])
                out = torch.empty((B, T, H, D), dtype=dt, device=cuda)
                B_.usp_ulysses_pack(B_.USP_MAP_UNPACK_HEADS, [(recv, out, H, D, _dt(out))], B, T, G)
                assert torch.equal(out, rm[i * P_u + u])


def _ring_all_ranks(spec, hs, do_hs, accumulate=False):
    """Run every rank's ring schedule with the per-rank calls (one GPU, ranks in turn):
    each step's partial merged by usp_lse_merge, or (accumulate) folded into one
    running partial by usp_ring_fwd_accumulate."""
    B, S, Hq, Hkv, D = (spec[k] for k in ("B", "S", "Hq", "Hkv", "D"))
    P_u, P_r, causal = spec["P_u"], spec["P_r"], spec["causal"]
    geo = (B, S, Hq, Hkv, D, causal, P_u, P_r)
    q, k, v = hs["q"], hs["k"], hs["v"]
    dev = q.device
    ws_f = api.workspace(B_.usp_ring_workspace_size(*geo, 0), dev)
    ws_b = api.workspace(B_.usp_ring_workspace_size(*geo, 1), dev)
    out, lse = torch.empty_like(q), torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)
    L, Hl = q.shape[3], q.shape[4]
    rows = B * L * Hl
    for i in range(P_r):
        for u in range(P_u):
            o_parts = torch.empty((2, rows, D), dtype=torch.float32, device=dev)
            l_parts = torch.empty((2, rows), dtype=torch.float32, device=dev)
            for t in range(P_r):
                j = (i - t) % P_r
                if accumulate:
                    B_.usp_ring_fwd_accumulate(q[i, u], k[j, u], v[j, u], o_parts[0], l_parts[0], *geo, i, u, t,
                                               ws_f, ws_f.numel())
                    continue
                s = 0 if t == 0 else 1
                B_.usp_ring_fwd_step(q[i, u], k[j, u], v[j, u], o_parts[s], l_parts[s], *geo, i, u, t, ws_f,
                                     ws_f.numel())
                if t > 0:
                    B_.usp_lse_merge(o_parts, l_parts, 2, rows, D, o_parts[0], B_.USP_F32, l_parts[0])
            B_.usp_lse_merge(o_parts, l_parts, 1, rows, D, out[i, u], B_.USP_BF16, lse[i, u])
    assert B_.usp_workspace_status(ws_f)[0] == 0
    dq = torch.empty_like(q)
    dk = torch.zeros(k.shape, dtype=torch.float32, device=dev)
    dv = torch.zeros(v.shape, dtype=torch.float32, device=dev)
    for i in range(P_r):
        for u in range(P_u):
            B_.usp_ring_bwd_prepare(out[i, u], lse[i, u], do_hs[i, u], *geo, ws_b, ws_b.numel())
            dq_acc = torch.zeros(q.shape[2:], dtype=torch.float32, device=dev)
            for t in range(P_r):
                j = (i - t) % P_r  # the block this rank holds at step t; its gradients travel with it
                B_.usp_ring_bwd_step(q[i, u], k[j, u], v[j, u], do_hs[i, u], dq_acc,
                                     dq[i, u] if t == P_r - 1 else None, dk[j, u], dv[j, u], *geo, i, u, t, ws_b,
                                     ws_b.numel())
            assert B_.usp_workspace_status(ws_b)[0] == 0
    torch.cuda.synchronize()
    return out, lse, dq, dk, dv


@pytest.mark.parametrize("accumulate", [False, True], ids=["merged", "accumulated"])
@pytest.mark.parametrize("name", list(CASES))
def test_ring_steps_of_every_rank_match_oracle(cuda, name, accumulate):
    spec = CASES[name]
    t = inputs(spec, which=("q", "k", "v", "do"))
    P_u, P_r = spec["P_u"], spec["P_r"]
    hs = {n: oracle.to_head_sharded(t[n].cpu(), P_u, P_r).to(cuda) for n in ("q", "k", "v", "do")}
    out, lse, dq, dk, dv = _ring_all_ranks(spec, hs, hs["do"], accumulate)
    name = f"{name}/accumulated" if accumulate else name
    to_g = lambda x: oracle.from_head_sharded(x.cpu(), P_u, P_r)  # noqa: E731
    tc = {n: t[n].cpu() for n in ("q", "k", "v", "do")}
    o_g = to_g(out)
    l_g = oracle.from_head_sharded(lse.cpu().unsqueeze(-1).contiguous(), P_u, P_r)[..., 0]
    assert_fwd_ok(compare_fwd(o_g, l_g, tc, spec, name=f"ring_steps/{name}"))
    ref = oracle.attn_full(tc["q"], tc["k"], tc["v"], tc["do"], spec["causal"])
    errs = {n: rel_l2(to_g(g).double().numpy(), ref[n]) for n, g in (("dq", dq), ("dk", dk), ("dv", dv))}
    GRAD_STATS.append((f"ring_steps/{name}", errs))
    assert all(e <= GRAD_REL_L2 for e in errs.values()), errs

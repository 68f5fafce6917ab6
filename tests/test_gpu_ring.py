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

from helpers import GRAD_REL_L2, GRAD_STATS, assert_fwd_ok, compare_fwd, fwd_stats, inputs, make_spec, rel_l2

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


def test_rank_full_size_s128k_usp4x2_sampled(cuda):
    """Rank (0, 0) of the S=128K GQA USP 4x2 mesh in the launch configuration of
    its per-rank measurement: its 2 forward ring steps folded by
    usp_ring_fwd_accumulate into one running partial, then its 2 backward steps.
    O, LSE and dQ of sampled rows of the rank (complete after every ring step)
    against the oracle over the whole sequence."""
    from usp_inputs import WORKLOADS
    spec = dict(WORKLOADS[3])
    B, S, Hq, Hkv, D, P_u, P_r = (spec[n] for n in ("B", "S", "Hq", "Hkv", "D", "P_u", "P_r"))
    causal, L, Hl = spec["causal"], S // P_r, Hq // P_u
    t = inputs(spec, which=("q", "k", "v", "do"))
    hs = {n: api.to_head_sharded(t[n], P_u, P_r) for n in ("q", "k", "v", "do")}
    tc = {n: x.cpu() for n, x in t.items() if n in ("q", "k", "v", "do")}
    del t
    q, do = hs["q"][0, 0].contiguous(), hs["do"][0, 0].contiguous()
    ks = [hs["k"][j, 0].contiguous() for j in range(P_r)]
    vs = [hs["v"][j, 0].contiguous() for j in range(P_r)]
    del hs
    torch.cuda.empty_cache()
    rows = B * L * Hl
    wsf = torch.zeros(B_.usp_ring_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, 0), dtype=torch.uint8,
                      device=cuda)
    wsb = torch.zeros(B_.usp_ring_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, 1), dtype=torch.uint8,
                      device=cuda)
    o_run = torch.empty((1, rows, D), dtype=torch.float32, device=cuda)
    l_run = torch.empty((1, rows), dtype=torch.float32, device=cuda)
    for s in range(P_r):
        B_.usp_ring_fwd_accumulate(q, ks[(0 - s) % P_r], vs[(0 - s) % P_r], o_run[0], l_run[0], B, S, Hq, Hkv, D,
                                   causal, P_u, P_r, 0, 0, s, wsf, wsf.numel())
    out = torch.empty_like(q)
    lse = torch.empty((B, L, Hl), dtype=torch.float32, device=cuda)
    B_.usp_lse_merge(o_run, l_run, 1, rows, D, out, B_.USP_BF16, lse)
    dq_acc = torch.zeros((B, L, Hl, D), dtype=torch.float32, device=cuda)
    dq = torch.empty_like(q)
    dk = torch.zeros((B, L, Hkv // P_u, D), dtype=torch.float32, device=cuda)
    dv = torch.zeros_like(dk)
    B_.usp_ring_bwd_prepare(out, lse, do, B, S, Hq, Hkv, D, causal, P_u, P_r, wsb, wsb.numel())
    for s in range(P_r):
        B_.usp_ring_bwd_step(q, ks[(0 - s) % P_r], vs[(0 - s) % P_r], do, dq_acc, dq if s == P_r - 1 else None, dk,
                             dv, B, S, Hq, Hkv, D, causal, P_u, P_r, 0, 0, s, wsb, wsb.numel())
    torch.cuda.synchronize()
    for ws in (wsf, wsb):
        assert B_.usp_workspace_status(ws)[0] == B_.USP_OK
    # the rank's rows in original positions, through the oracle's own layout map
    pos = torch.arange(S, dtype=torch.float32).view(1, S, 1, 1).expand(B, S, P_u, 1).contiguous()
    pos0 = oracle.to_head_sharded(pos, P_u, P_r)[0, 0, 0, :, 0, 0].long().numpy()
    rng = np.random.default_rng(33)
    loc = [(int(rng.integers(B)), int(rng.integers(Hl)), int(rng.integers(L))) for _ in range(40)]
    loc += [(0, 0, 0), (B - 1, Hl - 1, L - 1)]
    glob = [(b, h, int(pos0[x])) for b, h, x in loc]  # rank (i, u) = (0, 0): local head = global head
    o_ref, lse_ref = oracle.attn_fwd_rows(tc["q"], tc["k"], tc["v"], causal, glob)
    o_g = np.stack([out[b, x, h].float().cpu().numpy() for b, h, x in loc])
    l_g = np.array([float(lse[b, x, h]) for b, h, x in loc])
    assert_fwd_ok(fwd_stats(o_g, l_g, o_ref, lse_ref, name="ring_rank/s128k_usp4x2/sampled"))
    dq_ref, _, _ = oracle.attn_dq_rows(tc["q"], tc["k"], tc["v"], tc["do"], causal, glob)
    dq_g = np.stack([dq[b, x, h].double().cpu().numpy() for b, h, x in loc])
    err = rel_l2(dq_g, dq_ref)
    GRAD_STATS.append(("ring_rank/s128k_usp4x2/sampled", {"dq": err}))
    assert err <= GRAD_REL_L2, err

"""GPU parity of usp_attn_bwd against the fp64 oracle: whole tensors on small
cases (several tiles, ragged tails, GQA, USP meshes, every mask path), sampled
rows/columns and size-independent invariants at the full sizes."""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_tma_b200 import api
from usp_inputs import WORKLOADS

from helpers import GRAD_REL_L2, GRAD_STATS, head_shard_cpu, inputs, make_spec, rel_l2, unshard_cpu, sum_invariants

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_causal_usp2x2": make_spec(**{k: WORKLOADS[1][k] for k in ("B", "S", "Hq", "Hkv", "D", "causal", "P_u", "P_r", "seed")}),
    "causal_ring2_aligned": make_spec(S=1024, Hq=4, Hkv=4, D=128, P_r=2, seed=301),
    "noncausal_ragged": make_spec(S=600, Hq=2, Hkv=2, D=128, seed=302, causal=False),
    "gqa_usp2x2_unaligned": make_spec(S=1536, Hq=8, Hkv=2, D=128, P_u=2, P_r=2, seed=303),
    "d64_ragged_unaligned": make_spec(S=200, Hq=2, Hkv=1, D=64, P_r=2, seed=304),
    "batch2_causal_ring4": make_spec(B=2, S=2048, Hq=2, Hkv=2, D=128, P_r=4, seed=305),
    "noncausal_usp2x2_gqa_d64": make_spec(S=1024, Hq=4, Hkv=2, D=64, P_u=2, P_r=2, seed=306, causal=False),
    "peaky_noncausal_ring4": make_spec(S=2048, Hq=2, Hkv=2, D=128, P_r=4, seed=307, causal=False, peaky=True),
    # the code paths of the S=256K peaky workload (non-causal, ring of 16, chunks of
    # 512 = 4 key tiles, 8 key tiles per rank, 128 key tiles per query tile) at a size
    # whose whole-tensor fp64 oracle takes about a minute
    "peaky_noncausal_ring16_s16k_gqa": make_spec(S=16384, Hq=2, Hkv=1, D=128, P_r=16, seed=310, causal=False,
                                                 peaky=True),
}


def gpu_fwd_bwd(spec, t):
    dev = torch.device("cuda")
    P_u, P_r, causal = spec["P_u"], spec["P_r"], spec["causal"]
    q, k, v, do = (head_shard_cpu(t[n], spec).to(dev) for n in ("q", "k", "v", "do"))
    out, lse = api.attn_fwd(q, k, v, causal, P_u, P_r, check_status=True)
    dq, dk, dv = api.attn_bwd(q, k, v, out, lse, do, causal, P_u, P_r, check_status=True)
    torch.cuda.synchronize()
    return unshard_cpu(dq, spec), unshard_cpu(dk, spec), unshard_cpu(dv, spec)


def oracle_grads(tc, spec):
    """Whole-tensor dQ, dK, dV from the oracle: attn_full for small cases; for the
    larger ones its row form (dQ, LSE, Delta of every query row) and column form
    (dK, dV of every key), which parallelise over rows and columns."""
    B, S, Hq, Hkv = spec["B"], spec["S"], spec["Hq"], spec["Hkv"]
    causal = spec["causal"]
    if S * Hq <= 8192:
        return oracle.attn_full(tc["q"], tc["k"], tc["v"], tc["do"], causal)
    rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(S)]
    dq, lse, delta = oracle.attn_dq_rows(tc["q"], tc["k"], tc["v"], tc["do"], causal, rows)
    # rows are enumerated b-major, then h, then i: reshape straight into [B, Hq, S]
    lse_tab = np.ascontiguousarray(lse.reshape(B, Hq, S).transpose(0, 2, 1))
    delta_tab = np.ascontiguousarray(delta.reshape(B, Hq, S).transpose(0, 2, 1))
    cols = [(b, g, j) for b in range(B) for g in range(Hkv) for j in range(S)]
    dk, dv = oracle.attn_dkdv_cols(tc["q"], tc["k"], tc["v"], tc["do"], causal, cols, lse_tab, delta_tab)
    D = spec["D"]
    return dict(dq=dq.reshape(B, Hq, S, D).transpose(0, 2, 1, 3), dk=dk.reshape(B, Hkv, S, D).transpose(0, 2, 1, 3),
                dv=dv.reshape(B, Hkv, S, D).transpose(0, 2, 1, 3))


@pytest.mark.parametrize("name", list(SMALL))
def test_bwd_small_full_tensors(cuda, name):
    spec = SMALL[name]
    t = inputs(spec, which=("q", "k", "v", "do"))
    dq, dk, dv = gpu_fwd_bwd(spec, t)
    tc = {n: t[n].cpu() for n in ("q", "k", "v", "do")}
    ref = oracle_grads(tc, spec)
    errs = {n: rel_l2(g.double().numpy(), ref[n]) for n, g in (("dq", dq), ("dk", dk), ("dv", dv))}
    GRAD_STATS.append((name, errs))
    assert all(e <= GRAD_REL_L2 for e in errs.values()), errs


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_bwd_full_size_sampled(cuda, cfg):
    spec = dict(WORKLOADS[cfg])
    t = inputs(spec, which=("q", "k", "v", "do"))
    dq, dk, dv = gpu_fwd_bwd(spec, t)
    tc = {n: t[n].cpu() for n in ("q", "k", "v", "do")}
    del t
    torch.cuda.empty_cache()
    B, S, Hq, Hkv = spec["B"], spec["S"], spec["Hq"], spec["Hkv"]
    G = Hq // Hkv
    causal = spec["causal"]
    # dQ on sampled rows
    rng = np.random.default_rng(cfg)
    rows = [(int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(S))) for _ in range(24)]
    rows += [(0, 0, 0), (B - 1, Hq - 1, S - 1)]
    dq_ref, lse_r, delta_r = oracle.attn_dq_rows(tc["q"], tc["k"], tc["v"], tc["do"], causal, rows)
    idx = np.array(rows)
    dq_g = dq.double().numpy()[idx[:, 0], idx[:, 2], idx[:, 1]]
    errs = {"dq_rows": rel_l2(dq_g, dq_ref)}
    # size-independent invariants of dK, dV
    ek, ev = sum_invariants(dk, dv, tc["do"], G)
    errs.update(sum_dk=ek, sum_dv=ev)
    GRAD_STATS.append((spec["name"], errs))
    if causal:
        # dK/dV of keys near the end: only the last queries see them, so the
        # oracle needs LSE/Delta of those rows only
        tail = 48
        need = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(S - tail, S)]
        _, lse_t, delta_t = oracle.attn_dq_rows(tc["q"], tc["k"], tc["v"], tc["do"], causal, need)
        lse_tab = np.full((B, S, Hq), np.nan)
        delta_tab = np.full((B, S, Hq), np.nan)
        for r, (b, h, i) in enumerate(need):
            lse_tab[b, i, h] = lse_t[r]
            delta_tab[b, i, h] = delta_t[r]
        cols = [(b, g, S - 1 - int(o)) for b in range(B) for g in range(Hkv) for o in rng.choice(tail, 4, replace=False)]
        dk_ref, dv_ref = oracle.attn_dkdv_cols(tc["q"], tc["k"], tc["v"], tc["do"], causal, cols, lse_tab, delta_tab)
        ci = np.array(cols)
        dk_g = dk.double().numpy()[ci[:, 0], ci[:, 2], ci[:, 1]]
        dv_g = dv.double().numpy()[ci[:, 0], ci[:, 2], ci[:, 1]]
        errs.update(dk_cols=rel_l2(dk_g, dk_ref), dv_cols=rel_l2(dv_g, dv_ref))
    assert all(e <= GRAD_REL_L2 for e in errs.values()), errs


def test_bwd_ignores_stale_workspace_contents(cuda):
    """A workspace full of NaN bytes (a reused scratch) gives the same gradients as
    a fresh one, on a ragged causal case whose padded query rows read it."""
    from long_context_exact_tma_b200 import binding as B_
    spec = make_spec(S=600, Hq=4, Hkv=2, D=128, P_u=1, P_r=3, seed=308)
    t = inputs(spec, which=("q", "k", "v", "do"))
    P_u, P_r = spec["P_u"], spec["P_r"]
    q, k, v, do = (head_shard_cpu(t[n], spec).to(cuda) for n in ("q", "k", "v", "do"))
    out, lse = api.attn_fwd(q, k, v, True, P_u, P_r)
    clean = api.attn_bwd(q, k, v, out, lse, do, True, P_u, P_r)
    need = B_.usp_attn_workspace_size(1, 600, 4, 2, 128, 1, P_u, P_r, 0, 1)
    dirty_ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=cuda)
    dirty = api.attn_bwd(q, k, v, out, lse, do, True, P_u, P_r, ws=dirty_ws)
    torch.cuda.synchronize()
    for a_, b_ in zip(clean, dirty):
        assert torch.isfinite(b_.float()).all()
        assert rel_l2(b_.double().cpu().numpy(), a_.double().cpu().numpy()) <= 1e-5


def test_bwd_phases_compose_to_usp_attn_bwd(cuda):
    """prepare, then the dQ kernel before the dK/dV kernel, gives bit for bit what
    usp_attn_bwd gives (both kernels only read the prepared workspace)."""
    from long_context_exact_tma_b200 import binding as B_
    spec = make_spec(S=1536, Hq=8, Hkv=2, D=128, P_u=2, P_r=2, seed=309)
    t = inputs(spec, which=("q", "k", "v", "do"))
    P_u, P_r = spec["P_u"], spec["P_r"]
    q, k, v, do = (head_shard_cpu(t[n], spec).to(cuda) for n in ("q", "k", "v", "do"))
    out, lse = api.attn_fwd(q, k, v, True, P_u, P_r)
    whole = api.attn_bwd(q, k, v, out, lse, do, True, P_u, P_r)
    geo = (1, 1536, 8, 2, 128, 1, P_u, P_r)
    need = B_.usp_attn_workspace_size(*geo, 0, 1)
    ws = api.workspace(need, cuda)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(whole[1]), torch.empty_like(whole[2])
    B_.usp_attn_bwd_prepare(out, lse, do, *geo, ws, need)
    B_.usp_attn_bwd_dq(q, k, v, do, dq, *geo, ws, need)
    B_.usp_attn_bwd_dkdv(q, k, v, do, dk, dv, *geo, ws, need)
    torch.cuda.synchronize()
    assert B_.usp_workspace_status(ws)[0] == 0
    for a_, b_ in zip(whole, (dq, dk, dv)):
        assert torch.equal(a_, b_)


BF16_GRAD_CASES = ["tiny_causal_usp2x2", "gqa_usp2x2_unaligned", "d64_ragged_unaligned", "batch2_causal_ring4",
                   "noncausal_usp2x2_gqa_d64"]


def _bf16_vs_f32(spec, t, dev):
    P_u, P_r, causal = spec["P_u"], spec["P_r"], spec["causal"]
    q, k, v, do = (head_shard_cpu(t[n], spec).to(dev) for n in ("q", "k", "v", "do"))
    out, lse = api.attn_fwd(q, k, v, causal, P_u, P_r, check_status=True)
    g32 = api.attn_bwd(q, k, v, out, lse, do, causal, P_u, P_r, check_status=True)
    g16 = api.attn_bwd(q, k, v, out, lse, do, causal, P_u, P_r, check_status=True, grad_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert g16[1].dtype == torch.bfloat16 and g16[2].dtype == torch.bfloat16
    # the same fp32 sums, rounded once to the nearest bf16 (ties to even), as torch rounds
    assert torch.equal(g16[0], g32[0])
    assert torch.equal(g16[1], g32[1].to(torch.bfloat16))
    assert torch.equal(g16[2], g32[2].to(torch.bfloat16))
    return g16


@pytest.mark.parametrize("name", BF16_GRAD_CASES)
def test_bwd_bf16_grads_small(cuda, name):
    """usp_attn_bwd_dkdv_bf16: dK, dV in bf16 are the fp32 call's values rounded to
    bf16 element by element, and stay within the gradient bound of the oracle."""
    spec = SMALL[name]
    t = inputs(spec, which=("q", "k", "v", "do"))
    dq, dk, dv = (unshard_cpu(x, spec) for x in _bf16_vs_f32(spec, t, cuda))
    ref = oracle_grads({n: t[n].cpu() for n in ("q", "k", "v", "do")}, spec)
    errs = {n: rel_l2(g.double().numpy(), ref[n]) for n, g in (("dq", dq), ("dk", dk), ("dv", dv))}
    GRAD_STATS.append((f"bf16 grads/{name}", errs))
    assert all(e <= GRAD_REL_L2 for e in errs.values()), errs


def test_bwd_bf16_grads_s16k_ring8(cuda):
    """The same element-wise rounding identity on the S=16K ring-8 workload, in
    the launch configuration the bench step times."""
    spec = dict(WORKLOADS[2])
    t = inputs(spec, which=("q", "k", "v", "do"))
    _bf16_vs_f32(spec, t, cuda)

"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare.

Inputs are generated once (usp_inputs, on the GPU for speed) and the SAME bf16
bytes go to both sides. Layout changes on the oracle side use the oracle's own
push-style permutes, so a GPU permute bug cannot hide an attention bug.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from long_context_exact_tma_b200 import api
from long_context_exact_tma_b200 import binding as B_
from usp_inputs import workload

# Acceptance bounds on bf16-rounded inputs with fp32 accumulation.
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 2e-2


def make_spec(**kw):
    spec = dict(B=1, S=256, Hq=2, Hkv=2, D=64, causal=True, P_u=1, P_r=1, seed=100, peaky=False)
    spec.update(kw)
    return spec


def inputs(spec, which=("q", "k", "v"), device="cuda"):
    return workload(spec, device=device, which=which)


def head_shard_cpu(x_global: torch.Tensor, spec) -> torch.Tensor:
    """Oracle-side layout: global [B,S,H,D] -> head-sharded (CPU)."""
    return oracle.to_head_sharded(x_global.cpu(), spec["P_u"], spec["P_r"])


def unshard_cpu(x_hs: torch.Tensor, spec) -> torch.Tensor:
    return oracle.from_head_sharded(x_hs.cpu(), spec["P_u"], spec["P_r"])


def lse_to_global(lse_hs: torch.Tensor, spec) -> torch.Tensor:
    """head-sharded LSE [P_r,P_u,B,L,Hl] -> global [B,S,H] (via the D=1 layout)."""
    return unshard_cpu(lse_hs.unsqueeze(-1).contiguous(), spec)[..., 0]


def gpu_fwd(spec, tensors, mode=B_.USP_MODE_FUSED):
    """Head-shard on the CPU (oracle permutes), run usp_attn_fwd, map back to global."""
    dev = torch.device("cuda")
    q = head_shard_cpu(tensors["q"], spec).to(dev)
    k = head_shard_cpu(tensors["k"], spec).to(dev)
    v = head_shard_cpu(tensors["v"], spec).to(dev)
    out, lse = api.attn_fwd(q, k, v, spec["causal"], spec["P_u"], spec["P_r"], mode=mode, check_status=True)
    torch.cuda.synchronize()
    return unshard_cpu(out, spec), lse_to_global(lse, spec)


def sample_rows(spec, n, seed):
    rng = np.random.default_rng(seed)
    B, S, H = spec["B"], spec["S"], spec["Hq"]
    rows = [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(S))) for _ in range(n)]
    # always include the first and last positions of a head
    rows += [(0, 0, 0), (B - 1, H - 1, S - 1)]
    return rows


def compare_fwd(o_gpu, lse_gpu, tensors, spec, rows=None, name=None):
    """Compare global-layout GPU O/LSE with the oracle at `rows` (all rows if None).

    The max-abs bound on O is applied raw to every element whose reference value
    has |O_ref| < 4. O is delivered in bf16, and for |O_ref| >= 4 the spacing of
    bf16 is 2^-5, so rounding the exact value alone may move it by half of that,
    2^-6 = 0.0156 > 1e-2: only there is the error beyond that half-ulp held to the
    bound. (For |O_ref| in [2, 4) the half-ulp is 2^-7 = 0.0078, which still fits
    inside 1e-2, so those elements get no allowance.)
    """
    B, S, H = spec["B"], spec["S"], spec["Hq"]
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(S)]
    o_ref, lse_ref = oracle.attn_fwd_rows(tensors["q"], tensors["k"], tensors["v"], spec["causal"], rows)
    idx = np.array(rows)
    o_g = o_gpu.float().numpy()[idx[:, 0], idx[:, 2], idx[:, 1]].astype(np.float64)
    l_g = lse_gpu.float().numpy()[idx[:, 0], idx[:, 2], idx[:, 1]].astype(np.float64)
    return fwd_stats(o_g, l_g, o_ref, lse_ref, name=name)


def fwd_stats(o_g, l_g, o_ref, lse_ref, name=None, bf16_out=True):
    """Error statistics of a forward result against the oracle (see compare_fwd).
    With bf16_out=False (an fp32 O) no rounding allowance applies anywhere."""
    err = np.abs(np.asarray(o_g, np.float64) - o_ref)
    lerr = np.abs(np.asarray(l_g, np.float64) - lse_ref)
    big = np.abs(o_ref) >= 4.0
    allow = np.where(big, half_ulp_bf16(o_ref), 0.0) if bf16_out else np.zeros_like(o_ref)
    excess = np.maximum(err - allow, 0.0)
    st = dict(o_max=float(err.max()), o_max_below4=float(err[~big].max()) if (~big).any() else 0.0,
              o_max_excess=float(excess.max()), n_big=int(big.sum()), o_mean=float(err.mean()),
              lse_max=float(lerr.max()))
    if name is not None:
        FWD_STATS.append((name, st))
    return st


# (case name, stats) of every forward comparison made in this process; printed by
# the terminal summary hook in conftest.py.
FWD_STATS: list = []
# (case name, {gradient: relative L2 error}) of every backward comparison.
GRAD_STATS: list = []


def half_ulp_bf16(x):
    """Half the bf16 spacing at |x| (bf16 keeps 8 significant bits)."""
    ax = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 8)


def assert_fwd_ok(stats):
    assert stats["o_max_below4"] <= O_MAX_ABS, stats
    assert stats["o_max_excess"] <= O_MAX_ABS, stats
    assert stats["o_mean"] <= O_MEAN_ABS, stats
    assert stats["lse_max"] <= LSE_MAX_ABS, stats


def rel_l2(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def sum_invariants(dk, dv, do, G):
    """sum_j dK_j = 0 and sum_j dV_j = sum over the group of sum_i dO_i, per (b, kv-head).

    The dV invariant compares the vector sum_j dV_j with its reference sum_i dO_i
    by relative L2 against that reference (the relative L2 of the readings, over
    the compared elements). The dK invariant's reference is 0, so its error is
    measured against the size of dK itself, ||dK||_F."""
    dk = dk.double()
    dv = dv.double()
    B, S, Hkv, D = dk.shape
    sk = dk.sum(1)
    nk = dk.pow(2).sum(1).sum(-1).sqrt()
    dsum = do.double().sum(1).view(B, Hkv, G, D).sum(2)
    sv = dv.sum(1) - dsum
    return (sk.norm(dim=-1) / nk).max().item(), (sv.norm(dim=-1) / dsum.norm(dim=-1)).max().item()

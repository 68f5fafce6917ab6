"""GPU parity of the masked attention (usp_attn_fwd_masked / usp_attn_bwd_masked:
block-sparse masks and packed variable-length documents, in original token
positions, under USP meshes) against the fp64 oracle: whole tensors, forward
and backward, on random block masks, ragged documents (one of a single token),
both together, and a mask that leaves some rows with no visible key; sampled
forward rows at S=16K on a ring of 8."""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_tma_b200 import api

from helpers import GRAD_REL_L2, GRAD_STATS, assert_fwd_ok, fwd_stats, head_shard_cpu, inputs, make_spec, rel_l2, \
    unshard_cpu, lse_to_global

pytestmark = pytest.mark.gpu


def _block_mask(B, H, nb, density, seed, empty_rows=False):
    rng = np.random.default_rng(seed)
    bm = (rng.random((B, H, nb, nb)) < density).astype(np.uint8)
    if empty_rows:
        bm[0, 0, 1, :] = 0  # every query of block 1, head 0, batch 0 sees nothing
    return bm


CASES = {
    # name: spec, block-mask density (None = no block mask), documents (None = none), empty rows
    "block_causal_usp2x2": (make_spec(B=2, S=1024, Hq=4, Hkv=2, D=128, P_u=2, P_r=2, seed=401), 0.5, None, False),
    "docs_causal_ring2": (make_spec(B=2, S=1024, Hq=4, Hkv=2, D=128, P_u=1, P_r=2, seed=402), None,
                          [0, 300, 301, 700, 1024], False),
    "both_noncausal_d64": (make_spec(B=2, S=1024, Hq=4, Hkv=4, D=64, P_u=2, P_r=2, seed=403, causal=False), 0.6,
                           [0, 129, 640, 1024], False),
    "block_empty_rows": (make_spec(B=2, S=1024, Hq=2, Hkv=2, D=128, P_u=1, P_r=4, seed=404), 0.7, None, True),
    "docs_noncausal_gqa_usp4x1": (make_spec(B=2, S=1024, Hq=8, Hkv=4, D=128, P_u=4, P_r=1, seed=405,
                                            causal=False), None, [0, 1, 2, 500, 1023, 1024], False),
}


def _run(spec, t, bm, cu):
    dev = torch.device("cuda")
    P_u, P_r, causal = spec["P_u"], spec["P_r"], spec["causal"]
    q, k, v, do = (head_shard_cpu(t[n], spec).to(dev) for n in ("q", "k", "v", "do"))
    bmd = None if bm is None else torch.tensor(bm, device=dev)
    cud = None if cu is None else torch.tensor(cu, dtype=torch.int32, device=dev)
    out, lse = api.attn_fwd_masked(q, k, v, causal, P_u, P_r, block_mask=bmd, cu_seqlens=cud, check_status=True)
    dq, dk, dv = api.attn_bwd_masked(q, k, v, out, lse, do, causal, P_u, P_r, block_mask=bmd, cu_seqlens=cud,
                                     check_status=True)
    torch.cuda.synchronize()
    return (unshard_cpu(out, spec), lse_to_global(lse, spec), unshard_cpu(dq, spec), unshard_cpu(dk, spec),
            unshard_cpu(dv, spec))


@pytest.mark.parametrize("name", list(CASES))
def test_masked_small_full_tensors(cuda, name):
    spec, density, cu, empty_rows = CASES[name]
    B, S, Hq = spec["B"], spec["S"], spec["Hq"]
    bm = None if density is None else _block_mask(B, Hq, S // 128, density, spec["seed"], empty_rows)
    t = inputs(spec, which=("q", "k", "v", "do"))
    o, lse, dq, dk, dv = _run(spec, t, bm, cu)
    tc = {n: t[n].cpu() for n in ("q", "k", "v", "do")}
    ref = oracle.masked_attn_full(tc["q"], tc["k"], tc["v"], tc["do"], spec["causal"], block_mask=bm, block=128,
                                  cu_seqlens=cu)
    empty = np.isneginf(ref["lse"])
    if empty_rows:
        assert empty.any()
    assert np.array_equal(np.isneginf(lse.numpy()), empty)
    og = o.float().numpy()
    assert np.all(og[empty] == 0)
    st = fwd_stats(og[~empty], lse.numpy()[~empty], ref["o"][~empty], ref["lse"][~empty], name=f"masked/{name}")
    assert_fwd_ok(st)
    errs = {n: rel_l2(g.double().numpy(), ref[n]) for n, g in (("dq", dq), ("dk", dk), ("dv", dv))}
    GRAD_STATS.append((f"masked/{name}", errs))
    assert all(np.isfinite(g.double().numpy()).all() for g in (dq, dk, dv))
    assert all(e <= GRAD_REL_L2 for e in errs.values()), errs


def test_masked_sampled_rows_s16k_ring8(cuda):
    spec = make_spec(B=1, S=16384, Hq=8, Hkv=8, D=128, P_u=1, P_r=8, seed=410)
    B, S, Hq = spec["B"], spec["S"], spec["Hq"]
    bm = _block_mask(B, Hq, S // 128, 0.5, 410)
    cu = [0, 1000, 1001, 5000, 5120, 12000, 16384]
    t = inputs(spec, which=("q", "k", "v"))
    dev = torch.device("cuda")
    q, k, v = (head_shard_cpu(t[n], spec).to(dev) for n in ("q", "k", "v"))
    out, lse = api.attn_fwd_masked(q, k, v, True, 1, 8, block_mask=torch.tensor(bm, device=dev),
                                   cu_seqlens=torch.tensor(cu, dtype=torch.int32, device=dev), check_status=True)
    o, l = unshard_cpu(out, spec), lse_to_global(lse, spec)
    rng = np.random.default_rng(11)
    rows = [(0, int(rng.integers(Hq)), int(rng.integers(S))) for _ in range(96)] + [(0, 3, 1000), (0, 5, 5119)]
    tc = {n: t[n].cpu() for n in ("q", "k", "v")}
    o_ref, l_ref = oracle.masked_fwd_rows(tc["q"], tc["k"], tc["v"], True, rows, block_mask=bm, block=128,
                                          cu_seqlens=cu)
    idx = np.array(rows)
    og = o.float().numpy()[idx[:, 0], idx[:, 2], idx[:, 1]]
    lg = l.numpy()[idx[:, 0], idx[:, 2], idx[:, 1]]
    empty = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(lg), empty) and np.all(og[empty] == 0)
    assert_fwd_ok(fwd_stats(og[~empty], lg[~empty], o_ref[~empty], l_ref[~empty], name="masked/s16k_ring8/sampled"))


def test_block_sparse_bench_config_s16k(cuda):
    """The block-sparse line's configuration: the S=16K ring-8 workload (32 heads)
    with its seeded half-dense 128x128 block mask, causal. Forward on sampled rows
    against the oracle; backward at full size through sum_j dK_j = 0 and
    sum_j dV_j = sum_i dO_i per head, the latter over the rows that see a key."""
    from helpers import sum_invariants
    from usp_inputs import WORKLOADS
    spec = dict(WORKLOADS[2])
    B, S, Hq, Hkv, P_u, P_r = (spec[n] for n in ("B", "S", "Hq", "Hkv", "P_u", "P_r"))
    nb = S // 128
    bm = (np.random.default_rng(17).random((B, Hq, nb, nb)) < 0.5).astype(np.uint8)
    t = inputs(spec, which=("q", "k", "v", "do"))
    qh, kh, vh, doh = (api.to_head_sharded(t[n], P_u, P_r) for n in ("q", "k", "v", "do"))
    tc = {n: t[n].cpu() for n in ("q", "k", "v", "do")}
    del t
    bmd = torch.tensor(bm, device=cuda)
    out, lse = api.attn_fwd_masked(qh, kh, vh, True, P_u, P_r, block_mask=bmd, check_status=True)
    dq, dk, dv = api.attn_bwd_masked(qh, kh, vh, out, lse, doh, True, P_u, P_r, block_mask=bmd, check_status=True)
    torch.cuda.synchronize()
    o, l = unshard_cpu(out, spec), lse_to_global(lse, spec)
    rng = np.random.default_rng(12)
    rows = [(0, int(rng.integers(Hq)), int(rng.integers(S))) for _ in range(64)] + [(0, 0, 0), (0, Hq - 1, S - 1)]
    o_ref, l_ref = oracle.masked_fwd_rows(tc["q"], tc["k"], tc["v"], True, rows, block_mask=bm, block=128)
    idx = np.array(rows)
    og = o.float().numpy()[idx[:, 0], idx[:, 2], idx[:, 1]]
    lg = l.numpy()[idx[:, 0], idx[:, 2], idx[:, 1]]
    empty = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(lg), empty) and np.all(og[empty] == 0)
    assert_fwd_ok(fwd_stats(og[~empty], lg[~empty], o_ref[~empty], l_ref[~empty], name="masked/bench_s16k/sampled"))
    # a row sees a key iff one of its query block's blocks up to the diagonal is kept
    sees = np.cumsum(bm, axis=-1)[..., np.arange(nb), np.arange(nb)] > 0  # [B, Hq, nb]
    row_sees = torch.tensor(np.repeat(sees, 128, axis=-1)).permute(0, 2, 1)  # [B, S, Hq]
    do_seen = tc["do"].double() * row_sees.unsqueeze(-1)
    ek, ev = sum_invariants(unshard_cpu(dk, spec), unshard_cpu(dv, spec), do_seen, Hq // Hkv)
    GRAD_STATS.append(("masked/bench_s16k/invariants", {"sum_dk": ek, "sum_dv": ev}))
    assert torch.isfinite(dq.float()).all()
    assert ek <= GRAD_REL_L2 and ev <= GRAD_REL_L2, (ek, ev)

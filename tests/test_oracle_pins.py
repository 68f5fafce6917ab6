"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
hand-computed worked examples (tests/golden/), closed forms, torch's fp64
library routines (scaled_dot_product_attention and autograd), central finite
differences, and invariants of softmax attention and of the layout maps.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from usp_inputs import normal_bf16

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rand(seed, shape):
    return normal_bf16(seed, shape)


def _sdpa64(q, k, v, causal):
    """torch fp64 SDPA on [B, S, H, D] tensors, GQA by repeating K/V heads."""
    G = q.shape[2] // k.shape[2]
    qt = q.double().transpose(1, 2)
    kt = k.double().repeat_interleave(G, dim=2).transpose(1, 2)
    vt = v.double().repeat_interleave(G, dim=2).transpose(1, 2)
    return F.scaled_dot_product_attention(qt, kt, vt, is_causal=causal).transpose(1, 2)


def _all_rows(B, S, H):
    return [(b, h, i) for b in range(B) for h in range(H) for i in range(S)]


def test_golden_tiny_closed_form():
    g = json.load(open(os.path.join(GOLD, "attn_tiny_closed_form.json")))
    q = torch.tensor(g["q"], dtype=torch.float64).view(1, 3, 1, 2)
    k = torch.tensor(g["k"], dtype=torch.float64).view(1, 3, 1, 2)
    v = torch.tensor(g["v"], dtype=torch.float64).view(1, 3, 1, 2)
    for dt in (torch.float64, torch.bfloat16):  # these integers are exact in bf16
        o, lse = oracle.attn_fwd_rows(q.to(dt), k.to(dt), v.to(dt), True, _all_rows(1, 3, 1))
        np.testing.assert_allclose(o, np.array(g["o"]), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, np.array(g["lse"]), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [True, False])
def test_q_zero_gives_mean_of_visible_v(causal):
    B, S, H, D = 2, 37, 3, 16
    q = torch.zeros(B, S, H, D, dtype=torch.bfloat16)
    k, v = _rand(11, (B, S, H, D)), _rand(12, (B, S, H, D))
    rows = _all_rows(B, S, H)
    o, lse = oracle.attn_fwd_rows(q, k, v, causal, rows)
    vd = v.double().numpy()
    for r, (b, h, i) in enumerate(rows):
        n = i + 1 if causal else S
        np.testing.assert_allclose(o[r], vd[b, :n, h].mean(0), atol=1e-13)
        assert abs(lse[r] - math.log(n)) < 1e-13


def test_causal_row0_is_v0():
    B, S, Hq, Hkv, D = 1, 20, 4, 2, 32
    q, k, v = _rand(1, (B, S, Hq, D)), _rand(2, (B, S, Hkv, D)), _rand(3, (B, S, Hkv, D))
    rows = [(0, h, 0) for h in range(Hq)]
    o, lse = oracle.attn_fwd_rows(q, k, v, True, rows)
    for h in range(Hq):
        g = h // 2
        np.testing.assert_array_equal(o[h], v[0, 0, g].double().numpy())
        s00 = float((q[0, 0, h].double() * k[0, 0, g].double()).sum()) / math.sqrt(D)
        assert abs(lse[h] - s00) < 1e-13


def test_v_ones_rows_sum_to_one():
    B, S, H, D = 1, 50, 2, 8
    q, k = _rand(5, (B, S, H, D)), _rand(6, (B, S, H, D))
    v = torch.ones(B, S, H, D, dtype=torch.bfloat16)
    for causal in (True, False):
        o, _ = oracle.attn_fwd_rows(q, k, v, causal, _all_rows(B, S, H))
        np.testing.assert_allclose(o, 1.0, atol=1e-14)


@pytest.mark.parametrize("causal,Hq,Hkv", [(True, 4, 4), (False, 4, 2), (True, 6, 2)])
def test_fwd_matches_torch_sdpa_fp64(causal, Hq, Hkv):
    B, S, D = 2, 45, 16
    q, k, v = _rand(21, (B, S, Hq, D)), _rand(22, (B, S, Hkv, D)), _rand(23, (B, S, Hkv, D))
    rows = _all_rows(B, S, Hq)
    o, lse = oracle.attn_fwd_rows(q, k, v, causal, rows)
    ref = _sdpa64(q, k, v, causal).numpy()
    G = Hq // Hkv
    s = torch.einsum("bihd,bjhd->bhij", q.double(), k.double().repeat_interleave(G, 2)) / math.sqrt(D)
    if causal:
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    lse_ref = torch.logsumexp(s, dim=-1).numpy()  # [B, H, S]
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(o[r], ref[b, i, h], atol=1e-12)
        assert abs(lse[r] - lse_ref[b, h, i]) < 1e-12


@pytest.mark.parametrize("causal", [True, False])
def test_key_ranges_merge_to_full(causal):
    """Partials over a partition of the keys, LSE-merged, equal the unchunked result."""
    B, S, H, D = 1, 64, 2, 16
    q, k, v = _rand(31, (B, S, H, D)), _rand(32, (B, S, H, D)), _rand(33, (B, S, H, D))
    rows = _all_rows(B, S, H)
    full_o, full_lse = oracle.attn_fwd_rows(q, k, v, causal, rows)
    rng = np.random.default_rng(7)
    cuts = np.sort(rng.choice(np.arange(1, S), size=5, replace=False))
    bounds = [0, *cuts.tolist(), S]
    parts = [oracle.attn_fwd_rows(q, k, v, causal, rows, ranges=[(bounds[t], bounds[t + 1])])
             for t in range(len(bounds) - 1)]
    o_parts = np.stack([p[0] for p in parts])
    lse_parts = np.stack([p[1] for p in parts])
    if causal:
        assert np.isneginf(lse_parts).any()  # early rows see nothing of later pieces
    o, lse = oracle.lse_merge(o_parts, lse_parts)
    np.testing.assert_allclose(o, full_o, atol=1e-12)
    np.testing.assert_allclose(lse, full_lse, atol=1e-12)


def test_merge_special_cases():
    rows, D = 5, 4
    o_parts = np.random.default_rng(1).standard_normal((3, rows, D))
    lse_parts = np.full((3, rows), -np.inf)
    o, lse = oracle.lse_merge(o_parts, lse_parts)
    assert np.all(o == 0) and np.all(np.isneginf(lse))
    lse_parts[1] = np.linspace(-3, 3, rows)
    o, lse = oracle.lse_merge(o_parts, lse_parts)
    np.testing.assert_allclose(o, o_parts[1], atol=1e-15)
    np.testing.assert_allclose(lse, lse_parts[1], atol=1e-15)
    # two equal partials: LSE + log 2, O = their average
    lse_parts[0] = lse_parts[1]
    o, lse = oracle.lse_merge(o_parts, lse_parts)
    np.testing.assert_allclose(lse, lse_parts[1] + math.log(2), atol=1e-14)
    np.testing.assert_allclose(o, 0.5 * (o_parts[0] + o_parts[1]), atol=1e-14)


def _loss(q, k, v, w, causal):
    """L = sum over rows of O_i . W_i, evaluated with the oracle's forward."""
    B, S, Hq, D = q.shape
    rows = _all_rows(B, S, Hq)
    o, _ = oracle.attn_fwd_rows(q, k, v, causal, rows)
    wn = w.numpy()
    return float(sum((o[r] * wn[b, i, h]).sum() for r, (b, h, i) in enumerate(rows)))


@pytest.mark.parametrize("causal", [True, False])
def test_backward_central_finite_differences(causal):
    """dQ, dK, dV of L = sum(O * W) with dO = W against central differences (h = 1e-6)."""
    B, S, Hq, Hkv, D = 1, 6, 2, 1, 4
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, S, Hq, D, dtype=torch.float64, generator=g)
    k = torch.randn(B, S, Hkv, D, dtype=torch.float64, generator=g)
    v = torch.randn(B, S, Hkv, D, dtype=torch.float64, generator=g)
    w = torch.randn(B, S, Hq, D, dtype=torch.float64, generator=g)
    res = oracle.attn_full(q, k, v, w, causal)
    h = 1e-6
    for name, x, grad in (("q", q, res["dq"]), ("k", k, res["dk"]), ("v", v, res["dv"])):
        fd = np.zeros(x.shape)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.clone(), x.clone()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], w, causal)
                       - _loss(args_m["q"], args_m["k"], args_m["v"], w, causal)) / (2 * h)
        err = np.abs(fd - grad).max() / max(np.abs(fd).max(), 1e-30)
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("causal,Hq,Hkv", [(True, 4, 2), (False, 2, 2)])
def test_backward_matches_torch_autograd_fp64(causal, Hq, Hkv):
    B, S, D = 2, 33, 8
    q, k, v, do = (_rand(41, (B, S, Hq, D)), _rand(42, (B, S, Hkv, D)),
                   _rand(43, (B, S, Hkv, D)), _rand(44, (B, S, Hq, D)))
    res = oracle.attn_full(q, k, v, do, causal)
    qd, kd, vd = (t.double().requires_grad_() for t in (q, k, v))
    out = _sdpa64(qd, kd, vd, causal)
    out.backward(do.double())
    np.testing.assert_allclose(res["o"], out.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(res["dq"], qd.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(res["dk"], kd.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(res["dv"], vd.grad.numpy(), atol=1e-11)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_sum_invariants(causal):
    """sum_j dK_j = 0 (softmax Jacobian rows sum to 0); sum_j dV_j = sum over the group of sum_i dO_i."""
    B, S, Hq, Hkv, D = 2, 40, 4, 2, 8
    q, k, v, do = (_rand(51, (B, S, Hq, D)), _rand(52, (B, S, Hkv, D)),
                   _rand(53, (B, S, Hkv, D)), _rand(54, (B, S, Hq, D)))
    res = oracle.attn_full(q, k, v, do, causal)
    np.testing.assert_allclose(res["dk"].sum(1), 0.0, atol=1e-11)
    dsum = do.double().numpy().sum(1).reshape(B, Hkv, Hq // Hkv, D).sum(2)
    np.testing.assert_allclose(res["dv"].sum(1), dsum, atol=1e-11)


def test_gqa_equals_mha_with_repeated_kv():
    B, S, Hq, Hkv, D = 1, 24, 6, 2, 8
    q, k, v, do = (_rand(61, (B, S, Hq, D)), _rand(62, (B, S, Hkv, D)),
                   _rand(63, (B, S, Hkv, D)), _rand(64, (B, S, Hq, D)))
    G = Hq // Hkv
    gqa = oracle.attn_full(q, k, v, do, True)
    mha = oracle.attn_full(q, k.repeat_interleave(G, 2), v.repeat_interleave(G, 2), do, True)
    np.testing.assert_allclose(gqa["o"], mha["o"], atol=1e-13)
    np.testing.assert_allclose(gqa["dq"], mha["dq"], atol=1e-12)
    np.testing.assert_allclose(gqa["dk"], mha["dk"].reshape(B, S, Hkv, G, D).sum(3), atol=1e-12)
    np.testing.assert_allclose(gqa["dv"], mha["dv"].reshape(B, S, Hkv, G, D).sum(3), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_row_and_column_backward_agree_with_full(causal):
    B, S, Hq, Hkv, D = 1, 30, 4, 2, 8
    q, k, v, do = (_rand(71, (B, S, Hq, D)), _rand(72, (B, S, Hkv, D)),
                   _rand(73, (B, S, Hkv, D)), _rand(74, (B, S, Hq, D)))
    full = oracle.attn_full(q, k, v, do, causal)
    rows = [(0, 1, 0), (0, 3, 17), (0, 0, 29)]
    dq, lse, delta = oracle.attn_dq_rows(q, k, v, do, causal, rows)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(dq[r], full["dq"][b, i, h], atol=1e-13)
        assert abs(lse[r] - full["lse"][b, i, h]) < 1e-13
    lse_tab = full["lse"]
    delta_tab = (do.double().numpy() * full["o"]).sum(-1)
    cols = [(0, 0, 0), (0, 1, 13), (0, 1, 29)]
    dk, dv = oracle.attn_dkdv_cols(q, k, v, do, causal, cols, lse_tab, delta_tab)
    for c, (b, g, j) in enumerate(cols):
        np.testing.assert_allclose(dk[c], full["dk"][b, j, g], atol=1e-13)
        np.testing.assert_allclose(dv[c], full["dv"][b, j, g], atol=1e-13)
    bad = np.full_like(lse_tab, np.nan)
    with pytest.raises(ValueError):
        oracle.attn_dkdv_cols(q, k, v, do, causal, cols, bad, delta_tab)


def _token_ids(S, H, D=1):
    """Tensor whose element (b, s, h, d) encodes the token s and head h exactly (float32)."""
    t = torch.arange(S, dtype=torch.float32).view(1, S, 1, 1) * 16 + torch.arange(H).view(1, 1, H, 1)
    return t.expand(1, S, H, D).contiguous()


def test_zigzag_golden_ring_only():
    g = json.load(open(os.path.join(GOLD, "zigzag_ring2_s8.json")))
    x = _token_ids(g["S"], 1)
    sh = oracle.zigzag_shard(x, g["P"])
    got = (sh[:, 0, :, 0, 0] // 16).long().tolist()
    assert got == g["rank_major_tokens"]
    assert torch.equal(oracle.zigzag_unshard(sh, g["S"]), x)


def test_zigzag_and_seq2head_golden_usp():
    g = json.load(open(os.path.join(GOLD, "zigzag_usp2x2_s16.json")))
    S, H, P_u, P_r = g["S"], g["H"], g["P_u"], g["P_r"]
    x = _token_ids(S, H, D=3)
    rm = oracle.zigzag_shard(x, P_u * P_r)
    assert (rm[:, 0, :, 0, 0] // 16).long().tolist() == g["rank_major_tokens"]
    hs = oracle.seq2head(rm, P_u, P_r)
    for i in range(P_r):
        for u in range(P_u):
            want = g["head_sharded"][f"i{i}_u{u}"]
            blk = hs[i, u, 0]  # [L, H_l, D]
            assert (blk[:, 0, 0] // 16).long().tolist() == want["tokens"]
            assert (blk[0, :, 0] % 16).long().tolist() == want["heads"]
    assert torch.equal(oracle.head2seq(hs, P_u, P_r), rm)
    assert torch.equal(oracle.from_head_sharded(hs, P_u, P_r), x)


@pytest.mark.parametrize("P_u,P_r,H", [(1, 4, 3), (2, 2, 4), (4, 2, 8), (2, 3, 2)])
def test_layout_maps_are_bijections(P_u, P_r, H):
    B, D = 2, 2
    S = 2 * P_u * P_r * 5
    x = torch.arange(B * S * H * D, dtype=torch.float32).view(B, S, H, D)
    hs = oracle.to_head_sharded(x, P_u, P_r)
    assert torch.equal(torch.sort(hs.flatten()).values, torch.sort(x.flatten()).values)
    assert torch.equal(oracle.from_head_sharded(hs, P_u, P_r), x)
    # bf16 and a D=1 fp32 tensor (the LSE layout) go through the same maps
    xb = normal_bf16(9, (B, S, H, 8))
    assert torch.equal(oracle.from_head_sharded(oracle.to_head_sharded(xb, P_u, P_r), P_u, P_r), xb)


def test_attention_result_is_split_invariant():
    """The attention result, mapped back to token order, does not depend on (P_u, P_r)."""
    B, S, H, D = 1, 48, 4, 8
    q, k, v = _rand(81, (B, S, H, D)), _rand(82, (B, S, H, D)), _rand(83, (B, S, H, D))
    ref_o, ref_lse = oracle.attn_fwd_rows(q, k, v, True, _all_rows(B, S, H))
    for P_u, P_r in ((1, 2), (2, 2), (4, 1), (2, 3)):
        # permute to the head-sharded layout and back: the rows the oracle is asked
        # about keep their global positions, so the answer must not move
        qs = oracle.from_head_sharded(oracle.to_head_sharded(q, P_u, P_r), P_u, P_r)
        o, lse = oracle.attn_fwd_rows(qs, k, v, True, _all_rows(B, S, H))
        np.testing.assert_array_equal(o, ref_o)
        np.testing.assert_array_equal(lse, ref_lse)

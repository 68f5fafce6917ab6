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


@pytest.mark.parametrize("P_u,P_r", [(1, 2), (2, 2), (4, 1), (2, 3), (1, 4)])
def test_ring_steps_of_every_rank_merge_to_the_unsplit_result(P_u, P_r):
    """The USP computation done rank by rank and ring step by ring step: ring rank
    i's queries at step t attend the keys held by owner j = (i - t) mod P_r, the
    P_r partials merge (oracle.lse_merge) to the unsplit attention of those rows.

    The positions a rank holds are read off the oracle's own layout maps applied
    to a tensor of token ids, and checked against the zigzag reading (rank r holds
    chunks r and 2P-1-r), so a wrong chunk assignment, a ring schedule that misses
    or repeats a key block, or a wrong merge all fail here."""
    B, H, D = 1, 2 * P_u, 8
    P = P_u * P_r
    c = 3
    S = 2 * P * c
    q, k, v = _rand(81, (B, S, H, D)), _rand(82, (B, S, H, D)), _rand(83, (B, S, H, D))
    ids = torch.arange(S, dtype=torch.float32).view(1, S, 1, 1).expand(B, S, H, 1).contiguous()
    hs = oracle.to_head_sharded(ids, P_u, P_r)  # [P_r, P_u, B, L, H/P_u, 1]
    L, Hl = S // P_r, H // P_u

    def chunks_of(r):
        return [r, 2 * P - 1 - r]

    def positions(i):  # original positions held by ring rank i (any u), in local order
        return [ch * c + x for up in range(P_u) for ch in chunks_of(i * P_u + up) for x in range(c)]

    for i in range(P_r):
        for u in range(P_u):
            assert hs[i, u, 0, :, 0, 0].long().tolist() == positions(i)
    for i in range(P_r):
        for u in range(P_u):
            heads = range(u * Hl, (u + 1) * Hl)
            rows = [(0, h, pos) for h in heads for pos in positions(i)]
            ref_o, ref_lse = oracle.attn_fwd_rows(q, k, v, True, rows)
            o_parts, l_parts, seen = [], [], []
            for t in range(P_r):
                j = (i - t) % P_r
                ranges = [(ch * c, ch * c + c) for up in range(P_u) for ch in chunks_of(j * P_u + up)]
                seen += [x for a, e in ranges for x in range(a, e)]
                o_t, l_t = oracle.attn_fwd_rows(q, k, v, True, rows, ranges=ranges)
                o_parts.append(o_t)
                l_parts.append(l_t)
            assert sorted(seen) == list(range(S))  # every key block exactly once per ring
            o, lse = oracle.lse_merge(np.stack(o_parts), np.stack(l_parts))
            np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- LongNet dilated attention
def test_dilated_golden_tiny_closed_form():
    g = json.load(open(os.path.join(GOLD, "dilated_tiny_closed_form.json")))
    S = g["S"]
    q = torch.zeros(1, S, 2, 2, dtype=torch.bfloat16)
    v = torch.zeros(1, S, 2, 2, dtype=torch.float64)
    for j in range(S):
        v[0, j, 0] = torch.tensor([j, 1.0])
        v[0, j, 1] = torch.tensor([10 - j, 2.0])
    v = v.to(torch.bfloat16)  # small integers: exact in bf16
    k = _rand(5, (1, S, 2, 2))  # irrelevant when Q = 0
    for c in g["cases"]:
        o, lse = oracle.dilated_fwd_rows(q, k, v, True, c["pairs"], [(0, c["head"], c["row"])])
        np.testing.assert_allclose(o[0], c["o"], rtol=0, atol=1e-13)
        want = -math.inf if c["lse"] == "-inf" else c["lse"]
        if want == -math.inf:
            assert lse[0] == -math.inf
        else:
            assert abs(lse[0] - want) < 1e-13


@pytest.mark.parametrize("causal", [True, False])
def test_dilated_one_pair_w_s_r1_is_full_attention(causal):
    B, S, Hq, Hkv, D = 2, 48, 4, 2, 16
    q, k, v = _rand(61, (B, S, Hq, D)), _rand(62, (B, S, Hkv, D)), _rand(63, (B, S, Hkv, D))
    o, lse = oracle.dilated_fwd_rows(q, k, v, causal, [(S, 1)], _all_rows(B, S, Hq))
    ref = _sdpa64(q, k, v, causal).numpy()
    rows = _all_rows(B, S, Hq)
    idx = np.array(rows)
    np.testing.assert_allclose(o, ref[idx[:, 0], idx[:, 2], idx[:, 1]], rtol=0, atol=1e-12)


def _multiplicity_mask(S, H, pairs, causal):
    """[H, S, S] count of the pairs through which query i sees key j (from the
    reading: segments of w, rows s*w + (h mod r) + m*r kept, causal within)."""
    C = np.zeros((H, S, S))
    for w, r in pairs:
        for h in range(H):
            off = h % r
            for s0 in range(0, S, w):
                kept = list(range(s0 + off, min(s0 + w, S), r))
                for i in kept:
                    for j in kept:
                        if not causal or j <= i:
                            C[h, i, j] += 1
    return C


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("pairs", [[(8, 1), (16, 2), (32, 4)], [(12, 3), (24, 6)], [(10, 1), (40, 4), (40, 12)]])
def test_dilated_matches_sdpa_with_multiplicity_mask(causal, pairs):
    """Dilated attention is softmax attention in which key j counts C_ij times for
    query i (C = the number of pairs that show it): torch fp64 SDPA with the
    additive mask log C (-inf where C = 0) gives the same O."""
    B, S, Hq, Hkv, D = 1, 40, 4, 2, 8
    q, k, v = _rand(71, (B, S, Hq, D)), _rand(72, (B, S, Hkv, D)), _rand(73, (B, S, Hkv, D))
    rows = _all_rows(B, S, Hq)
    o, lse = oracle.dilated_fwd_rows(q, k, v, causal, pairs, rows)
    C = _multiplicity_mask(S, Hq, pairs, causal)
    with np.errstate(divide="ignore"):
        mask = torch.tensor(np.log(C))
    G = Hq // Hkv
    qt = q.double().transpose(1, 2)
    kt = k.double().repeat_interleave(G, dim=2).transpose(1, 2)
    vt = v.double().repeat_interleave(G, dim=2).transpose(1, 2)
    idx = np.array(rows)
    seen = C.sum(-1)[idx[:, 1], idx[:, 2]] > 0
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask.unsqueeze(0)).transpose(1, 2).numpy()
    ref = ref[idx[:, 0], idx[:, 2], idx[:, 1]]
    np.testing.assert_allclose(o[seen], ref[seen], rtol=0, atol=1e-12)
    # rows no pair keeps: empty result
    assert np.all(o[~seen] == 0) and np.all(np.isneginf(lse[~seen]))
    # LSE = log sum_j C_ij exp(s_ij)
    s = torch.einsum("bhid,bhjd->bhij", qt, kt).numpy()[0] / math.sqrt(D)
    with np.errstate(divide="ignore"):
        lref = np.log((C * np.exp(s)).sum(-1))[idx[:, 1], idx[:, 2]]
    np.testing.assert_allclose(lse[seen], lref[seen], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- block-sparse / document masks
def test_masked_golden_tiny_closed_form():
    g = json.load(open(os.path.join(GOLD, "masked_tiny_closed_form.json")))
    S = g["S"]
    q = torch.zeros(1, S, 1, 2, dtype=torch.bfloat16)
    v = torch.tensor([[j, 1.0] for j in range(S)], dtype=torch.float64).view(1, S, 1, 2).to(torch.bfloat16)
    k = _rand(6, (1, S, 1, 2))
    for c in g["cases"]:
        bm = None if c["mask"] is None else np.array(g["masks"][c["mask"]], np.uint8).reshape(1, 1, 3, 3)
        o, lse = oracle.masked_fwd_rows(q, k, v, c["causal"], [(0, 0, c["row"])], block_mask=bm, block=g["block"],
                                        cu_seqlens=g["cu_seqlens"])
        np.testing.assert_allclose(o[0], c["o"], rtol=0, atol=1e-13)
        if c["lse"] == "-inf":
            assert lse[0] == -math.inf
        else:
            assert abs(lse[0] - c["lse"]) < 1e-13


def _bool_mask(B, S, H, causal, bm, bs, cu):
    """[B, H, S, S] visibility from the reading: causal, block bit, same document."""
    vis = np.ones((B, H, S, S), bool)
    if causal:
        vis &= np.tril(np.ones((S, S), bool))
    if bm is not None:
        vis &= np.repeat(np.repeat(bm.astype(bool), bs, axis=2), bs, axis=3)[:, :, :S, :S]
    if cu is not None:
        doc = np.searchsorted(np.asarray(cu), np.arange(S), side="right") - 1
        vis &= doc[:, None] == doc[None, :]
    return vis


def _sdpa_masked(q, k, v, vis):
    G = q.shape[2] // k.shape[2]
    qt = q.double().transpose(1, 2)
    kt = k.double().repeat_interleave(G, dim=2).transpose(1, 2)
    vt = v.double().repeat_interleave(G, dim=2).transpose(1, 2)
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.tensor(vis)).transpose(1, 2)


@pytest.mark.parametrize("causal", [True, False])
def test_masked_all_ones_is_unmasked(causal):
    B, S, Hq, Hkv, D, bs = 1, 40, 4, 2, 8, 8
    q, k, v, do = (_rand(90 + n, (B, S, h, D)) for n, h in enumerate((Hq, Hkv, Hkv, Hq)))
    bm = np.ones((B, Hq, 5, 5), np.uint8)
    m = oracle.masked_attn_full(q, k, v, do, causal, block_mask=bm, block=bs, cu_seqlens=[0, S])
    u = oracle.attn_full(q, k, v, do, causal)
    for n in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(m[n], u[n], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("kind", ["block", "docs", "both"])
def test_masked_matches_sdpa_forward_and_autograd(causal, kind):
    """Forward against torch fp64 SDPA with the boolean mask, gradients against
    its autograd; rows whose visible set is empty are checked to be O = 0,
    LSE = -inf and are left out of the SDPA comparison (SDPA gives NaN there)."""
    B, S, Hq, Hkv, D, bs = 2, 36, 4, 2, 8, 6
    q, k, v, do = (_rand(95 + n, (B, S, h, D)).double() for n, h in enumerate((Hq, Hkv, Hkv, Hq)))
    rng = np.random.default_rng(3)
    bm = (rng.random((B, Hq, 6, 6)) < 0.6).astype(np.uint8) if kind in ("block", "both") else None
    cu = [0, 5, 13, 14, 30, 36] if kind in ("docs", "both") else None
    vis = _bool_mask(B, S, Hq, causal, bm, bs, cu)
    m = oracle.masked_attn_full(q, k, v, do, causal, block_mask=bm, block=bs, cu_seqlens=cu)
    empty = ~vis.any(-1)  # [B, H, S]
    e_bsh = empty.transpose(0, 2, 1)
    assert np.all(np.isneginf(m["lse"][e_bsh])) and np.all(m["o"][e_bsh] == 0)
    qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
    vis_safe = vis | empty[..., None]  # SDPA needs one visible key per row; those rows are dropped below
    o = _sdpa_masked(qr, kr, vr, vis_safe)
    keep = torch.tensor(~e_bsh)[..., None].double()
    (o * do * keep).sum().backward()
    on = o.detach().numpy()
    np.testing.assert_allclose(m["o"][~e_bsh], on[~e_bsh], rtol=0, atol=1e-12)
    for n, t in (("dq", qr), ("dk", kr), ("dv", vr)):
        np.testing.assert_allclose(m[n], t.grad.numpy(), rtol=0, atol=1e-11)


@pytest.mark.parametrize("causal", [True, False])
def test_dilated_full_forward_matches_rows_and_grads_match_autograd(causal):
    """The whole-tensor dilated oracle: its forward equals the row form (pinned
    above); its gradients equal torch fp64 autograd of SDPA with the additive
    log-multiplicity mask."""
    B, S, Hq, Hkv, D = 1, 24, 4, 2, 8
    pairs = [(6, 1), (12, 2), (24, 4)]
    q, k, v, do = (_rand(120 + n, (B, S, h, D)).double() for n, h in enumerate((Hq, Hkv, Hkv, Hq)))
    full = oracle.dilated_attn_full(q, k, v, do, causal, pairs)
    rows = _all_rows(B, S, Hq)
    o_r, l_r = oracle.dilated_fwd_rows(q, k, v, causal, pairs, rows)
    idx = np.array(rows)
    np.testing.assert_allclose(full["o"][idx[:, 0], idx[:, 2], idx[:, 1]], o_r, rtol=0, atol=1e-12)
    np.testing.assert_allclose(full["lse"][idx[:, 0], idx[:, 2], idx[:, 1]], l_r, rtol=0, atol=1e-12)
    C = _multiplicity_mask(S, Hq, pairs, causal)
    with np.errstate(divide="ignore"):
        mask = torch.tensor(np.log(C)).unsqueeze(0)
    G = Hq // Hkv
    qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = F.scaled_dot_product_attention(qr.transpose(1, 2), kr.repeat_interleave(G, dim=2).transpose(1, 2),
                                       vr.repeat_interleave(G, dim=2).transpose(1, 2), attn_mask=mask).transpose(1, 2)
    (o * do).sum().backward()
    for n, t in (("dq", qr), ("dk", kr), ("dv", vr)):
        np.testing.assert_allclose(full[n], t.grad.numpy(), rtol=0, atol=1e-11)


def test_dilated_full_backward_central_finite_differences():
    B, S, Hq, Hkv, D = 1, 12, 2, 1, 4
    pairs = [(4, 1), (12, 3)]
    q, k, v = (_rand(130 + n, (B, S, h, D)).double() for n, h in enumerate((Hq, Hkv, Hkv)))
    wgt = _rand(133, (B, S, Hq, D)).double()
    full = oracle.dilated_attn_full(q, k, v, wgt, True, pairs)

    def loss(q_, k_, v_):
        return float((oracle.dilated_attn_full(q_, k_, v_, wgt, True, pairs)["o"] * wgt.numpy()).sum())

    h = 1e-6
    rng = np.random.default_rng(2)
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        for _ in range(6):
            idx = tuple(int(rng.integers(n)) for n in t.shape)
            tp, tm = t.clone(), t.clone()
            tp[idx] += h
            tm[idx] -= h
            args_p = [tp if x is t else x for x in (q, k, v)]
            args_m = [tm if x is t else x for x in (q, k, v)]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - full[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, full[name][idx])

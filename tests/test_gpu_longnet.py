"""GPU parity of LongNet's distributed layout: the per-rank kernels of
usp_longnet_* and usp_rows_copy, driven by the schedule of
long_context_exact_tma_b200.dist, for M ranks emulated on one GPU (one host
thread per rank; the all-gathers and reduce-scatters are copies between the
threads' buffers behind host barriers, so no kernel ever waits on another
rank's). The slices the ranks return, put together, are compared with the
oracle's dilated attention over the whole sequence (forward and backward)."""
import threading

import numpy as np
import pytest
import torch

import oracle
from helpers import GRAD_REL_L2, GRAD_STATS, assert_fwd_ok, fwd_stats, rel_l2
from long_context_exact_tma_b200 import dist as udist
from usp_inputs import normal_bf16

pytestmark = pytest.mark.gpu


class ThreadComm:
    """All-gather and reduce-scatter among threads that each play one rank; the
    group is the list of its ranks (every rank makes the same sequence of calls)."""

    def __init__(self, world):
        self.bar = threading.Barrier(world, timeout=120)
        self.slots = {}
        self.lock = threading.Lock()
        self.local = threading.local()

    def _post(self, x):
        n = getattr(self.local, "n", 0)
        self.local.n = n + 1
        torch.cuda.synchronize()  # the posted buffer is complete
        with self.lock:
            self.slots[(n, self.local.rank)] = x
        self.bar.wait()
        return n

    def _done(self, n):
        torch.cuda.synchronize()  # this rank has read what it needs
        self.bar.wait()
        with self.lock:
            self.slots.pop((n, self.local.rank))

    def all_gather(self, recv, send, group):
        n = self._post(send)
        for x, rk in enumerate(group):
            recv[x].copy_(self.slots[(n, rk)])
        self._done(n)

    def reduce_scatter(self, recv, send, group):
        n = self._post(send)
        me = group.index(self.local.rank)
        recv.zero_()
        for rk in group:
            recv += self.slots[(n, rk)][me]
        self._done(n)


CASES = {
    # name: (world, B, T, Hq, Hkv, D, causal, pairs): local pairs (w <= T) and gathered ones
    "w4_longnet_scaled_causal": (4, 1, 384, 4, 4, 128, True, [(192, 1), (384, 2), (768, 4), (1536, 6)]),
    "w2_gqa_noncausal_d64": (2, 2, 256, 8, 2, 64, False, [(128, 1), (512, 3)]),
    "w4_ragged_rows_gqa": (4, 1, 320, 6, 3, 128, True, [(320, 3), (640, 5), (1280, 7)]),
}


def _run(name, device):
    world, B, T, Hq, Hkv, D, causal, pairs = CASES[name]
    S = world * T
    seed = 1300 + 17 * len(name)
    g = {n: normal_bf16(seed + x, (B, S, h, D), device=device) for x, (n, h) in
         enumerate((("q", Hq), ("k", Hkv), ("v", Hkv), ("do", Hq)))}
    comm = ThreadComm(world)
    res, errs = {}, []

    def rank_main(rank):
        try:
            comm.local.rank = rank
            torch.cuda.set_device(device)
            mine = slice(rank * T, (rank + 1) * T)
            q, k, v, do = (g[n][:, mine].contiguous() for n in ("q", "k", "v", "do"))
            lm = udist.LongNetMesh(S, pairs, rank=rank, world=world, make_groups=False)
            ops = udist.CudaLongNetOps(B, T, Hq, Hkv, D, pairs, device=device)
            out, lse = udist.longnet_attn_fwd(q, k, v, pairs, causal, lm, ops, comm)
            dq, dk, dv = udist.longnet_attn_bwd(q, k, v, out, lse, do, pairs, causal, lm, ops, comm)
            torch.cuda.synchronize()
            ops.check()
            res[rank] = (out, lse, dq, dk, dv)
        except BaseException as e:  # noqa: BLE001 -- reported by the main thread
            errs.append(e)
            comm.bar.abort()

    threads = [threading.Thread(target=rank_main, args=(x,)) for x in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    if errs:
        raise errs[0]
    parts = list(zip(*(res[x] for x in range(world))))
    out, lse, dq, dk, dv = (torch.cat(p, dim=1).cpu() for p in parts)
    ref = oracle.dilated_attn_full(g["q"].cpu(), g["k"].cpu(), g["v"].cpu(), g["do"].cpu(), causal, pairs)
    return out, lse, dq, dk, dv, ref


@pytest.mark.parametrize("name", list(CASES))
def test_longnet_distributed_matches_whole_sequence_oracle(cuda, name):
    out, lse, dq, dk, dv, ref = _run(name, cuda)
    o_g, l_g = out.double().numpy().reshape(-1, out.shape[-1]), lse.double().numpy().reshape(-1)
    o_r, l_r = ref["o"].reshape(-1, out.shape[-1]), ref["lse"].reshape(-1)
    empty = np.isneginf(l_r)  # rows that no pair keeps
    assert np.array_equal(np.isneginf(l_g), empty)
    assert np.all(o_g[empty] == 0)
    st = fwd_stats(o_g[~empty], l_g[~empty], o_r[~empty], l_r[~empty], name=f"longnet_dist/{name}")
    assert_fwd_ok(st)
    errs = {n: rel_l2(x.double().numpy(), ref[n]) for n, x in (("dq", dq), ("dk", dk), ("dv", dv))}
    GRAD_STATS.append((f"longnet_dist/{name}", errs))
    assert all(e <= GRAD_REL_L2 for e in errs.values()), errs


def test_rows_copy_bit_exact(cuda):
    """usp_rows_copy against plain index arithmetic: a strided, head-mapped bf16
    gather and an fp32 scatter-add whose GQA heads share destination rows."""
    from long_context_exact_tma_b200 import binding as B_
    B, T, H, Hkv, D = 2, 40, 6, 3, 128
    src = normal_bf16(77, (B, T, Hkv, D), device=cuda)
    r, o, lp0, n = 3, 1, 2, 12
    ns = (H - o + r - 1) // r
    dst = torch.zeros((B, n, ns, D), dtype=torch.bfloat16, device=cuda)
    B_.usp_rows_copy([dict(src=src, dst=dst, dtype=B_.USP_BF16, n_b=B, n_k=n, n_j=ns, D=D, s_b=T * Hkv * D,
                           s_k=Hkv * D, s_h=D, s_k0=lp0, s_kstep=r, s_h0=o, s_hstep=r, s_hdiv=H // Hkv,
                           d_b=n * ns * D, d_k=ns * D, d_h=D)])
    want = torch.stack([torch.stack([src[:, lp0 + r * k, (o + j * r) // (H // Hkv)] for j in range(ns)], 1)
                        for k in range(n)], 1)
    assert torch.equal(dst, want)
    # every query head of a group added into its kv head (j = 0..H-1 -> kv head j // 2)
    acc = torch.ones((B, T, Hkv, D), dtype=torch.float32, device=cuda)
    add = normal_bf16(78, (B, n, H, D), device=cuda).float()
    B_.usp_rows_copy([dict(src=add, dst=acc, dtype=B_.USP_F32, add=1, n_b=B, n_k=n, n_j=H, D=D, s_b=n * H * D,
                           s_k=H * D, s_h=D, d_b=T * Hkv * D, d_k=Hkv * D, d_h=D, d_k0=lp0, d_kstep=r, d_h0=0,
                           d_hstep=1, d_hdiv=H // Hkv)])
    ref = torch.ones((B, T, Hkv, D), dtype=torch.float32, device=cuda)
    for k in range(n):
        for j in range(H):
            ref[:, lp0 + r * k, j // (H // Hkv)] += add[:, k, j]
    torch.cuda.synchronize()
    assert torch.equal(acc, ref)


def test_longnet_rank_full_size_s32k_sampled(cuda):
    """Rank 0 of 4 on the S=32K LongNet schedule in the launch configuration of
    its per-rank measurement: local pairs on its slice, and for the gathered
    pairs every head offset's cross attention (on side streams) against the
    segment's kept K/V rows gathered from the whole sequence. O and LSE of
    sampled rows of the slice against the oracle's dilated attention."""
    from long_context_exact_tma_b200 import binding as B_
    B, S, H, D, M = 1, 32768, 16, 128, 4
    T = S // M
    pairs = [(2048, 1), (4096, 2), (8192, 4), (16384, 6), (32768, 12)]
    qg, kg, vg = (normal_bf16(900 + x, (B, S, H, D), device=cuda) for x in range(3))
    q, k, v = (x[:, :T].contiguous() for x in (qg, kg, vg))
    ops = udist.CudaLongNetOps(B, T, H, H, D, pairs, device=cuda)
    ops.fwd_begin()
    for w, r in pairs:
        if w <= T:
            ops.fwd_local(q, k, v, True, w, r)
            continue
        for o in range(min(r, H)):
            ns = (H - o + r - 1) // r
            n_kept = (w - o + r - 1) // r
            kc = torch.empty((B, n_kept, ns, D), dtype=torch.bfloat16, device=cuda)
            vc = torch.empty_like(kc)
            B_.usp_rows_copy([dict(src=x, dst=y, dtype=B_.USP_BF16, n_b=B, n_k=n_kept, n_j=ns, D=D, s_b=S * H * D,
                                   s_k=H * D, s_h=D, s_k0=o, s_kstep=r, s_h0=o, s_hstep=r, d_b=n_kept * ns * D,
                                   d_k=ns * D, d_h=D) for x, y in ((kg, kc), (vg, vc))])
            ops.fwd_cross(q, kc, vc, True, w, r, o, 0)
        ops.cross_join()
    out, lse = ops.fwd_end()
    torch.cuda.synchronize()
    ops.check()
    rng = np.random.default_rng(34)
    rows = [(0, int(rng.integers(H)), int(rng.integers(T))) for _ in range(40)] + [(0, 0, 0), (0, H - 1, T - 1)]
    o_ref, l_ref = oracle.dilated_fwd_rows(qg.cpu(), kg.cpu(), vg.cpu(), True, pairs, rows)
    o_g = np.stack([out[b, i, h].float().cpu().numpy() for b, h, i in rows])
    l_g = np.array([float(lse[b, i, h]) for b, h, i in rows])
    assert_fwd_ok(fwd_stats(o_g, l_g, o_ref, l_ref, name="longnet_rank/s32k_rank0_of_4/sampled"))

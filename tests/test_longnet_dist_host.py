"""LongNet's distributed layout (long_context_exact_tma_b200.dist, the LongNet
slides' "LONGNET as a Distributed Trainer") on CPU: world-size 2 and 4 gloo
process groups run the real all-gathers and reduce-scatters of the schedule,
with the per-rank compute (the affine row copies, the local and the cross
attention of one pair, their backward) supplied by a plain fp64 torch
implementation of the same operations. Every rank's output, LSE and gradients
for its own slice must equal the oracle's dilated attention over the whole
sequence -- which checks the kept-row arithmetic, the pack / gather / compact
steps, that the gathered segments hold every kept row exactly once and in
order, and that the gradients of gathered rows come home to their owner."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rows_copy(jobs):
    """fp64 torch form of usp_rows_copy (any dtype, in place)."""
    for J in jobs:
        src, dst = J["src"].reshape(-1), J["dst"].reshape(-1)
        D = J["D"]
        g = dict(add=0, s_k0=0, s_kstep=1, s_h0=0, s_hstep=1, s_hdiv=1, d_k0=0, d_kstep=1, d_h0=0, d_hstep=1,
                 d_hdiv=1)
        g.update(J)
        for b in range(g["n_b"]):
            for k in range(g["n_k"]):
                for j in range(g["n_j"]):
                    s = (b * g["s_b"] + (g["s_k0"] + k * g["s_kstep"]) * g["s_k"]
                         + ((g["s_h0"] + j * g["s_hstep"]) // g["s_hdiv"]) * g["s_h"])
                    d = (b * g["d_b"] + (g["d_k0"] + k * g["d_kstep"]) * g["d_k"]
                         + ((g["d_h0"] + j * g["d_hstep"]) // g["d_hdiv"]) * g["d_h"])
                    if g["add"]:
                        dst[d:d + D] += src[s:s + D]
                    else:
                        dst[d:d + D] = src[s:s + D]


class TorchLongNetOps:
    """fp64 torch implementation of the per-rank operations of dist.CudaLongNetOps."""
    BF16, F32 = 0, 1

    def __init__(self, B, T, Hq, Hkv, D):
        self.B, self.T, self.Hq, self.Hkv, self.D = B, T, Hq, Hkv, D
        self.scale = 1.0 / math.sqrt(D)

    def rows_copy(self, jobs):
        _rows_copy(jobs)

    # forward: a running (O, LSE) folded by the log-sum-exp merge
    def fwd_begin(self):
        self.o = torch.zeros(self.B, self.T, self.Hq, self.D, dtype=torch.float64)
        self.l = torch.full((self.B, self.T, self.Hq), -math.inf, dtype=torch.float64)

    def _attend(self, Q, K, V, qidx, kidx, causal):
        s = Q @ K.T * self.scale
        if causal:
            s = s.masked_fill(kidx[None, :] > qidx[:, None], -math.inf)
        lse = torch.logsumexp(s, dim=-1)
        p = torch.exp(s - lse[:, None]).nan_to_num(0.0)
        return p @ V, lse

    def _fold(self, b, rows, h, O, L):
        lo, oo = self.l[b, rows, h], self.o[b, rows, h]
        m = torch.maximum(lo, L)
        ms = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
        a, c = torch.exp(lo - ms), torch.exp(L - ms)
        tot = a + c
        self.o[b, rows, h] = torch.where(tot[:, None] > 0, (a[:, None] * oo + c[:, None] * O) / tot.clamp_min(1e-300)[:, None], oo)
        self.l[b, rows, h] = torch.where(tot > 0, ms + torch.log(tot.clamp_min(1e-300)), lo)

    def _local_blocks(self, w, r):
        """(segment rows, query head, kv head) of a local pair on this slice."""
        G = self.Hq // self.Hkv
        for o in range(min(r, self.Hq)):
            kept = torch.arange(o, w, r)
            for s in range(self.T // w):
                for h in range(o, self.Hq, r):
                    yield s * w + kept, h, h // G

    def fwd_local(self, q, k, v, causal, w, r):
        for b in range(self.B):
            for rows, h, kh in self._local_blocks(w, r):
                idx = torch.arange(len(rows))
                O, L = self._attend(q[b, rows, h].double(), k[b, rows, kh].double(), v[b, rows, kh].double(), idx,
                                    idx, causal)
                self._fold(b, rows, h, O, L)

    def _cross_blocks(self, w, r, o, g):
        from long_context_exact_tma_b200.dist import longnet_rows
        lp0, k_lo, n_rows, n_kept = longnet_rows(self.T, w, r, o, g)
        rows = lp0 + r * torch.arange(n_rows)
        qidx = k_lo + torch.arange(n_rows)
        for j, h in enumerate(range(o, self.Hq, r)):
            yield rows, qidx, torch.arange(n_kept), j, h

    def fwd_cross(self, q, kc, vc, causal, w, r, o, g):
        for b in range(self.B):
            for rows, qidx, kidx, j, h in self._cross_blocks(w, r, o, g):
                O, L = self._attend(q[b, rows, h].double(), kc[b, :, j].double(), vc[b, :, j].double(), qidx, kidx,
                                    causal)
                self._fold(b, rows, h, O, L)

    def cross_join(self):
        pass

    def fwd_end(self):
        return self.o.clone(), self.l.clone()

    # backward: P from the final LSE, the five products of the attention gradient
    def bwd_begin(self, out, lse, dO, dK, dV):
        self.lse = lse.double()
        self.delta = (dO.double() * out.double()).sum(-1)
        self.dq = torch.zeros(self.B, self.T, self.Hq, self.D, dtype=torch.float64)
        dK.zero_()
        dV.zero_()

    def _grads(self, Q, K, V, dO, lse, delta, qidx, kidx, causal):
        s = Q @ K.T * self.scale
        if causal:
            s = s.masked_fill(kidx[None, :] > qidx[:, None], -math.inf)
        p = torch.exp(s - lse[:, None]).nan_to_num(0.0)
        ds = p * (dO @ V.T - delta[:, None])
        return ds @ K * self.scale, ds.T @ Q * self.scale, p.T @ dO

    def bwd_local(self, q, k, v, dO, lse, dK, dV, causal, w, r):
        for b in range(self.B):
            for rows, h, kh in self._local_blocks(w, r):
                idx = torch.arange(len(rows))
                dq, dk, dv = self._grads(q[b, rows, h].double(), k[b, rows, kh].double(), v[b, rows, kh].double(),
                                         dO[b, rows, h].double(), self.lse[b, rows, h], self.delta[b, rows, h], idx,
                                         idx, causal)
                self.dq[b, rows, h] += dq
                dK[b, rows, kh] += dk.to(dK.dtype)
                dV[b, rows, kh] += dv.to(dV.dtype)

    def bwd_cross(self, q, kc, vc, dO, lse, dkc, dvc, causal, w, r, o, g):
        dkc.zero_()
        dvc.zero_()
        for b in range(self.B):
            for rows, qidx, kidx, j, h in self._cross_blocks(w, r, o, g):
                dq, dk, dv = self._grads(q[b, rows, h].double(), kc[b, :, j].double(), vc[b, :, j].double(),
                                         dO[b, rows, h].double(), self.lse[b, rows, h], self.delta[b, rows, h], qidx,
                                         kidx, causal)
                self.dq[b, rows, h] += dq
                dkc[b, :, j] += dk.to(dkc.dtype)
                dvc[b, :, j] += dv.to(dvc.dtype)

    def bwd_end(self):
        return self.dq.clone()


CASES = {
    # name: (world, T, Hq, Hkv, causal, pairs)
    "w2_causal": (2, 24, 4, 2, True, [(8, 1), (24, 3), (48, 6)]),
    "w4_causal_gqa": (4, 12, 4, 2, True, [(6, 1), (12, 2), (24, 3), (48, 5)]),
    "w4_noncausal": (4, 12, 3, 3, False, [(12, 1), (48, 4)]),
}


def _worker(rank, world, port, name, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from long_context_exact_tma_b200 import dist as udist
        from usp_inputs import normal_bf16
        _, T, Hq, Hkv, causal, pairs = CASES[name]
        B, D = 1, 8
        S = world * T
        g = {n: normal_bf16(900 + x, (B, S, h, D)).double() for x, (n, h) in
             enumerate((("q", Hq), ("k", Hkv), ("v", Hkv), ("do", Hq)))}
        mine = slice(rank * T, (rank + 1) * T)
        local = {n: x[:, mine].contiguous() for n, x in g.items()}
        lm = udist.LongNetMesh(S, pairs)
        ops = TorchLongNetOps(B, T, Hq, Hkv, D)
        out, lse = udist.longnet_attn_fwd(local["q"], local["k"], local["v"], pairs, causal, lm, ops)
        dq, dk, dv = udist.longnet_attn_bwd(local["q"], local["k"], local["v"], out, lse, local["do"], pairs, causal,
                                            lm, ops)
        ref = oracle.dilated_attn_full(g["q"], g["k"], g["v"], g["do"], causal, pairs)
        got = {"o": out, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
        results[rank] = {n: float(np.abs(got[n].numpy() - ref[n][:, mine]).max()) for n in got}
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("name", list(CASES))
def test_longnet_schedule_on_gloo(name):
    world = CASES[name][0]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), name, results), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(results)
    assert len(res) == world
    for rank, errs in res.items():
        # dK, dV travel in fp32 buffers (the reduce-scatter's), as in the library
        assert all(errs[n] <= 1e-9 for n in ("o", "lse", "dq")), (rank, errs)
        assert all(errs[n] <= 1e-5 for n in ("dk", "dv")), (rank, errs)


@pytest.mark.parametrize("T,w,r", [(12, 24, 5), (12, 48, 7), (10, 40, 3), (8, 8, 3), (6, 36, 4)])
def test_longnet_rows_against_brute_force_and_the_library(T, w, r):
    """Each rank's kept rows of offset o are those positions of its slice that
    are = o (mod r), contiguous in kept order; the ranks' shares tile the
    segment's kept list exactly once. The library's usp_longnet_rows (a host
    function, no GPU needed) gives the same numbers."""
    from long_context_exact_tma_b200 import binding as B_
    from long_context_exact_tma_b200.dist import longnet_rows
    G = w // T
    for o in range(r):
        kept = [p for p in range(w) if p % r == o]
        seen = []
        for g in range(G):
            lp0, k_lo, n_rows, n_kept = longnet_rows(T, w, r, o, g)
            assert B_.usp_longnet_rows(T, w, r, o, g) == (lp0, k_lo, n_rows, n_kept)
            assert n_kept == len(kept)
            mine = [p for p in kept if g * T <= p < (g + 1) * T]
            assert [g * T + lp0 + r * x for x in range(n_rows)] == mine
            assert kept[k_lo:k_lo + n_rows] == mine
            seen += mine
        assert seen == kept


def _worker_peer_lost(rank, world, port, results):
    """Rank 1 leaves between steps; rank 0 runs the forward, whose first gathered
    pair all-gathers kept K/V rows over the segment, and must get an error from
    the process group within its timeout instead of waiting for ever."""
    import datetime
    import time
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    from long_context_exact_tma_b200 import dist as udist
    _, T, Hq, Hkv, causal, pairs = CASES["w2_causal"]
    B, D = 1, 8
    lm = udist.LongNetMesh(world * T, pairs)
    if rank == 1:
        results[rank] = "left"
        os._exit(0)  # gone without a goodbye: no destroy_process_group
    q = torch.zeros((B, T, Hq, D), dtype=torch.float64)
    kv = torch.zeros((B, T, Hkv, D), dtype=torch.float64)
    t0 = time.monotonic()
    try:
        udist.longnet_attn_fwd(q, kv, kv, pairs, causal, lm, TorchLongNetOps(B, T, Hq, Hkv, D))
        results[rank] = ("no error", time.monotonic() - t0)
    except Exception as e:  # the process group's error for the lost peer
        results[rank] = ("error", time.monotonic() - t0, type(e).__name__)
    os._exit(0)


@pytest.mark.timeout(180)
def test_longnet_lost_peer_raises_instead_of_hanging():
    """Failure detection on the host for LongNet's layout: with one rank gone, the
    survivor's all-gather of a segment's kept rows ends with an error within the
    process group's 5 s timeout."""
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker_peer_lost, args=(2, _free_port(), results), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(results)
    assert res.get(1) == "left"
    assert res[0][0] == "error", res[0]
    assert res[0][1] < 60, res[0]

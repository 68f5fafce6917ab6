"""The exchange schedule of the multi-GPU USP mesh (long_context_exact_tma_b200.dist)
on CPU: world-size 2 and 4 gloo process groups run the real all-to-alls and
ring send/receives of dist.py, with the per-rank compute supplied by a plain
fp64 torch implementation of the same operations (positions from the zigzag
reading). Each rank's output and gradients, for its own tokens, must equal the
oracle's unsplit attention -- which checks the Ulysses layout, that every rank
sees every K/V block exactly once, the merge, and that each block's gradients
come home to their owner."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _positions(i, P_u, P_r, S):
    """Original positions of the L local tokens of ring rank i (the reading:
    rank r holds chunks r and 2P-1-r; ring rank i concatenates its P_u ranks)."""
    P = P_u * P_r
    c = S // (2 * P)
    pos = []
    for up in range(P_u):
        r = i * P_u + up
        pos += list(range(r * c, r * c + c)) + list(range((2 * P - 1 - r) * c, (2 * P - r) * c))
    return torch.tensor(pos)


class TorchOps:
    """fp64 torch implementation of the per-rank operations of dist.CudaOps."""

    def __init__(self, geo, mesh):
        self.geo, self.mesh = geo, mesh
        self.scale = 1.0 / math.sqrt(geo.D)

    def pack(self, map_, xs, outs, T):
        G = self.geo.P_u
        for (x, H), o in zip(xs, outs):
            if map_ == 4:    # [B, T, H, D] -> [G, B, T, H/G, D]
                o.copy_(x.view(x.shape[0], T, G, H // G, x.shape[-1]).permute(2, 0, 1, 3, 4))
            elif map_ == 5:  # [G, B, T, Hl, D] -> [B, G*T, Hl, D]
                o.copy_(x.permute(1, 0, 2, 3, 4).reshape(o.shape))
            elif map_ == 6:  # [B, G*T, Hl, D] -> [G, B, T, Hl, D]
                o.copy_(x.view(x.shape[0], G, T, x.shape[2], x.shape[3]).permute(1, 0, 2, 3, 4))
            else:            # [G, B, T, Hl, D] -> [B, T, G*Hl, D]
                o.copy_(x.permute(1, 2, 0, 3, 4).reshape(o.shape))

    def _scores(self, q, k, t):
        g, m = self.geo, self.mesh
        j = (m.i - t) % g.P_r
        G = q.shape[2] // k.shape[2]
        kk = k.double().repeat_interleave(G, dim=2)
        s = torch.einsum("bqhd,bkhd->bhqk", q.double(), kk) * self.scale
        if g.causal:
            pq, pk = _positions(m.i, g.P_u, g.P_r, g.S), _positions(j, g.P_u, g.P_r, g.S)
            s = s.masked_fill(pk[None, None, None, :] > pq[None, None, :, None], -math.inf)
        return s, G

    def fwd_step(self, q, k, v, o_part, lse_part, t):
        s, G = self._scores(q, k, t)
        lse = torch.logsumexp(s, dim=-1)  # [B, H, Lq]
        p = torch.exp(s - lse[..., None]).nan_to_num(0.0)
        o = torch.einsum("bhqk,bkhd->bqhd", p, v.double().repeat_interleave(G, dim=2))
        o_part.copy_(o.reshape(o_part.shape))
        lse_part.copy_(lse.permute(0, 2, 1).reshape(lse_part.shape))

    def fwd_acc(self, q, k, v, o_run, lse_run, t):
        if t == 0:
            self.fwd_step(q, k, v, o_run, lse_run, t)
            return
        o_t, l_t = torch.empty_like(o_run), torch.empty_like(lse_run)
        self.fwd_step(q, k, v, o_t, l_t, t)
        self.merge(torch.stack([o_run, o_t]), torch.stack([lse_run, l_t]), 2, o_run, lse_run)

    def merge(self, o_parts, lse_parts, n, out, lse_out):
        lp = lse_parts[:n].double()
        m = lp.max(0).values
        msafe = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
        w = torch.exp(lp - msafe)
        tot = w.sum(0)
        lse = torch.where(tot > 0, msafe + torch.log(tot), torch.full_like(m, -math.inf))
        a = torch.where(tot[None] > 0, w / tot.clamp_min(1e-300)[None], torch.zeros_like(w))
        o = (a[..., None] * o_parts[:n].double()).sum(0)
        out.copy_(o.to(out.dtype))
        lse_out.copy_(lse.to(lse_out.dtype))

    def bwd_prepare(self, out, lse, dO):
        self.lse = lse.double().permute(0, 2, 1)                   # [B, H, Lq]
        self.delta = (dO.double() * out.double()).sum(-1).permute(0, 2, 1)

    def bwd_step(self, q, k, v, dO, dq_acc, dq_out, dk_acc, dv_acc, t):
        s, G = self._scores(q, k, t)
        p = torch.exp(s - self.lse[..., None]).nan_to_num(0.0)    # [B, H, Lq, Lk]
        vv = v.double().repeat_interleave(G, dim=2)
        dp = torch.einsum("bqhd,bkhd->bhqk", dO.double(), vv)
        ds = p * (dp - self.delta[..., None])
        kk = k.double().repeat_interleave(G, dim=2)
        dq_acc += torch.einsum("bhqk,bkhd->bqhd", ds, kk) * self.scale
        B, Lk, Hkv, D = k.shape
        dk = (torch.einsum("bhqk,bqhd->bkhd", ds, q.double()) * self.scale).view(B, Lk, Hkv, G, D).sum(3)
        dv = torch.einsum("bhqk,bqhd->bkhd", p, dO.double()).view(B, Lk, Hkv, G, D).sum(3)
        dk_acc += dk
        dv_acc += dv
        if dq_out is not None:
            dq_out.copy_(dq_acc)


def _worker(rank, world, port, P_u, P_r, causal, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from long_context_exact_tma_b200 import dist as udist
        from usp_inputs import normal_bf16
        B, S, Hq, Hkv, D = 1, 2 * world * 6, 4, 2, 8
        geo = udist.Geometry(B, S, Hq, Hkv, D, causal, P_u, P_r)
        mesh = udist.Mesh(P_u, P_r)
        g = {n: normal_bf16(700 + x, (B, S, h, D)).double() for x, (n, h) in
             enumerate((("q", Hq), ("k", Hkv), ("v", Hkv), ("do", Hq)))}
        local = {n: oracle.zigzag_shard(x, world)[rank].contiguous() for n, x in g.items()}
        ops = TorchOps(geo, mesh)
        out, saved = udist.usp_attention(local["q"], local["k"], local["v"], geo, mesh, ops)
        dq, dk, dv = udist.usp_attention_bwd(local["do"], saved, geo, mesh, ops)
        ref = oracle.attn_full(g["q"], g["k"], g["v"], g["do"], causal)
        want = {n: oracle.zigzag_shard(torch.tensor(ref[n]), world)[rank].numpy() for n in ("o", "dq", "dk", "dv")}
        got = {"o": out.numpy(), "dq": dq.numpy(), "dk": dk.numpy(), "dv": dv.numpy()}
        results[rank] = {n: float(np.abs(got[n] - want[n]).max()) for n in got}
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("P_u,P_r,causal", [(2, 1, True), (1, 2, True), (2, 2, True), (2, 2, False), (1, 4, True)])
def test_usp_mesh_schedule_on_gloo(P_u, P_r, causal):
    world = P_u * P_r
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), P_u, P_r, causal, results), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(results)
    assert sorted(res) == list(range(world))
    for rank, errs in res.items():
        # the partials and accumulators are fp32 buffers, as on the GPU: fp32 rounding only
        assert all(e < 1e-5 for e in errs.values()), (rank, errs)


def _worker_peer_lost(rank, world, port, P_u, P_r, results):
    """Rank 1 leaves between steps (before the step's first collective, none of
    its work in flight); rank 0 runs the step and must get an error from the
    process group within its timeout instead of waiting for ever."""
    import datetime
    import time
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    from long_context_exact_tma_b200 import dist as udist
    B, S, Hq, Hkv, D = 1, 2 * world * 6, 4, 2, 8
    geo = udist.Geometry(B, S, Hq, Hkv, D, True, P_u, P_r)
    mesh = udist.Mesh(P_u, P_r)
    if rank == 1:
        results[rank] = "left"
        os._exit(0)  # gone without a goodbye: no destroy_process_group
    T = S // world
    x = {n: torch.zeros((B, T, h, D), dtype=torch.float64) for n, h in (("q", Hq), ("k", Hkv), ("v", Hkv))}
    t0 = time.monotonic()
    try:
        udist.usp_attention(x["q"], x["k"], x["v"], geo, mesh, TorchOps(geo, mesh))
        results[rank] = ("no error", time.monotonic() - t0)
    except Exception as e:  # the process group's error for the lost peer
        results[rank] = ("error", time.monotonic() - t0, type(e).__name__)
    os._exit(0)


@pytest.mark.timeout(180)
@pytest.mark.parametrize("P_u,P_r", [(2, 1), (1, 2)])
def test_usp_mesh_lost_peer_raises_instead_of_hanging(P_u, P_r):
    """Failure detection on the host: a rank that leaves the mesh makes the
    surviving rank's next collective (the Ulysses all-to-all, or the ring's
    send/receive) end with an error within the process group's 5 s timeout."""
    world = P_u * P_r
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker_peer_lost, args=(world, _free_port(), P_u, P_r, results), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(results)
    assert res.get(1) == "left"
    status, elapsed = res[0][0], res[0][1]
    assert status == "error", res[0]
    assert elapsed < 60, res[0]

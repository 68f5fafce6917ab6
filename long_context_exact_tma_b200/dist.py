"""USP on a real multi-GPU mesh: one process per GPU, NCCL for the exchanges.

The method ("Boosting Spec Eagle: USP for Long-Context Training", "The
Solution"; DeepSpeed-Ulysses summary, "Wie DeepSpeed-Ulysses funktioniert"):
P = P_u x P_r ranks, rank r = i * P_u + u (ring index i, Ulysses index u),
holding the zigzag chunks r and 2P-1-r of the sequence ("Implementation
Details": load balancing). Per attention call:

  1. Ulysses all-to-all inside the group of the P_u ranks with the same i:
     every rank sends head group u' of its tokens to rank (i, u') and receives
     head group u of every group member's tokens (sequence -> heads);
  2. ring attention over the P_r ranks with the same u: at step t rank i
     attends the K/V block of ring rank j = (i - t) mod P_r while passing its
     current block on to ring rank i + 1; the per-step partials are merged by
     log-sum-exp;
  3. the inverse all-to-all of O (heads -> sequence).
The backward passes K/V around the ring again, the dK/dV of each block
travelling with it and arriving back at their owner after P_r hops.

Every step of the compute runs in libusp.so (usp_ulysses_pack,
usp_ring_fwd_step / usp_lse_merge, usp_ring_bwd_prepare / usp_ring_bwd_step);
the exchanges are torch.distributed collectives (NCCL on GPUs): an equal-split
all_to_all_single per group and batched isend/irecv to the ring neighbours,
with the next K/V block in flight while the current one is computed. The
`ops` object carries the compute so that the exchange schedule can be
exercised with another implementation of the same per-rank operations.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Geometry:
    """Global shape of the attention problem and the mesh."""
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    causal: bool
    P_u: int
    P_r: int

    @property
    def P(self) -> int:
        return self.P_u * self.P_r

    @property
    def T(self) -> int:  # tokens a rank holds before the all-to-all
        return self.S // self.P

    @property
    def L(self) -> int:  # tokens a rank holds after it (the whole ring rank's slice)
        return self.S // self.P_r


class Mesh:
    """The rank's place in the P_u x P_r mesh and its process groups. Every
    rank must construct it (torch.distributed.new_group is collective)."""

    def __init__(self, P_u: int, P_r: int, rank: int | None = None, world: int | None = None):
        self.rank = dist.get_rank() if rank is None else rank
        world = dist.get_world_size() if world is None else world
        if world != P_u * P_r:
            raise ValueError(f"world size {world} != P_u * P_r = {P_u * P_r}")
        self.P_u, self.P_r = P_u, P_r
        self.i, self.u = divmod(self.rank, P_u)
        self.ulysses_group = None
        for i in range(P_r):  # every rank creates every group, in the same order
            ranks = [i * P_u + u for u in range(P_u)]
            grp = dist.new_group(ranks) if P_u > 1 else None
            if i == self.i:
                self.ulysses_group = grp
        self.ring_next = ((self.i + 1) % P_r) * P_u + self.u
        self.ring_prev = ((self.i - 1) % P_r) * P_u + self.u


class CudaOps:
    """The per-rank compute in libusp.so kernels."""

    def __init__(self, geo: Geometry, mesh: Mesh, stream=None):
        from . import binding as B_
        self.B_ = B_
        self.geo, self.mesh, self.stream = geo, mesh, stream
        g = geo
        self.ws_f = torch.zeros(B_.usp_ring_workspace_size(g.B, g.S, g.Hq, g.Hkv, g.D, g.causal, g.P_u, g.P_r, 0),
                                dtype=torch.uint8, device="cuda")
        self.ws_b = torch.zeros(B_.usp_ring_workspace_size(g.B, g.S, g.Hq, g.Hkv, g.D, g.causal, g.P_u, g.P_r, 1),
                                dtype=torch.uint8, device="cuda")

    def _dt(self, t):
        return self.B_.USP_BF16 if t.dtype == torch.bfloat16 else self.B_.USP_F32

    def pack(self, map_, xs, outs, T):
        self.B_.usp_ulysses_pack(map_, [(x, o, H, x.shape[-1], self._dt(x)) for x, o, H in xs_outs(xs, outs)],
                                 self.geo.B, T, self.geo.P_u, self.stream)

    def fwd_step(self, q, k, v, o_part, lse_part, t):
        g, m = self.geo, self.mesh
        self.B_.usp_ring_fwd_step(q, k, v, o_part, lse_part, g.B, g.S, g.Hq, g.Hkv, g.D, g.causal, g.P_u, g.P_r, m.i,
                                  m.u, t, self.ws_f, self.ws_f.numel(), self.stream)

    def merge(self, o_parts, lse_parts, n, out, lse_out):
        """n partials o_parts [n, rows, D], lse_parts [n, rows] -> out (fp32 or bf16), lse_out."""
        rows, D = o_parts.shape[1], o_parts.shape[2]
        self.B_.usp_lse_merge(o_parts, lse_parts, n, rows, D, out, self._dt(out), lse_out, self.stream)

    def bwd_prepare(self, out, lse, dO):
        g = self.geo
        self.B_.usp_ring_bwd_prepare(out, lse, dO, g.B, g.S, g.Hq, g.Hkv, g.D, g.causal, g.P_u, g.P_r, self.ws_b,
                                     self.ws_b.numel(), self.stream)

    def bwd_step(self, q, k, v, dO, dq_acc, dq_out, dk_acc, dv_acc, t):
        g, m = self.geo, self.mesh
        self.B_.usp_ring_bwd_step(q, k, v, dO, dq_acc, dq_out, dk_acc, dv_acc, g.B, g.S, g.Hq, g.Hkv, g.D, g.causal,
                                  g.P_u, g.P_r, m.i, m.u, t, self.ws_b, self.ws_b.numel(), self.stream)

    def check(self):
        for ws in (self.ws_f, self.ws_b):
            rc, site = self.B_.usp_workspace_status(ws, self.stream)
            if rc != self.B_.USP_OK:
                raise self.B_.UspError(rc, f"device wait timed out (site {site:#x})")


def xs_outs(xs, outs):
    return [(x, o, h) for (x, h), o in zip(xs, outs)]


def _exchange(sends, recvs, to_rank, from_rank):
    """Send every tensor of `sends` to `to_rank` and receive `recvs` from
    `from_rank`, all in one batch (so that neighbours in a ring never wait on
    each other's order); returns the requests."""
    ops = [dist.P2POp(dist.isend, s, to_rank) for s in sends] + [dist.P2POp(dist.irecv, r, from_rank) for r in recvs]
    return dist.batch_isend_irecv(ops)


def seq2head(xs, geo: Geometry, mesh: Mesh, ops):
    """Ulysses all-to-all (sequence -> heads) of the rank-local tensors xs
    ([B, T, H_x, D_x] each): returns [B, L, H_x / P_u, D_x] each."""
    G, T = geo.P_u, geo.T
    sends = [torch.empty((G, geo.B, T, x.shape[2] // G, x.shape[3]), dtype=x.dtype, device=x.device) for x in xs]
    ops.pack(4, [(x, x.shape[2]) for x in xs], sends, T)  # USP_MAP_PACK_HEADS
    recvs = [torch.empty_like(s) for s in sends]
    for s, r in zip(sends, recvs):
        if G > 1:
            dist.all_to_all_single(r, s, group=mesh.ulysses_group)
        else:
            r.copy_(s)
    outs = [torch.empty((geo.B, G * T, r.shape[3], r.shape[4]), dtype=r.dtype, device=r.device) for r in recvs]
    ops.pack(5, [(r, r.shape[3] * G) for r in recvs], outs, T)  # USP_MAP_UNPACK_TOKENS
    return outs


def head2seq(xs, geo: Geometry, mesh: Mesh, ops):
    """The inverse all-to-all (heads -> sequence) of head-sharded tensors xs
    ([B, L, H_x / P_u, D_x] each): returns [B, T, H_x, D_x] each."""
    G, T = geo.P_u, geo.T
    sends = [torch.empty((G, geo.B, T, x.shape[2], x.shape[3]), dtype=x.dtype, device=x.device) for x in xs]
    ops.pack(6, [(x, x.shape[2] * G) for x in xs], sends, T)  # USP_MAP_PACK_TOKENS
    recvs = [torch.empty_like(s) for s in sends]
    for s, r in zip(sends, recvs):
        if G > 1:
            dist.all_to_all_single(r, s, group=mesh.ulysses_group)
        else:
            r.copy_(s)
    outs = [torch.empty((geo.B, T, r.shape[3] * G, r.shape[4]), dtype=r.dtype, device=r.device) for r in recvs]
    ops.pack(7, [(r, r.shape[3] * G) for r in recvs], outs, T)  # USP_MAP_UNPACK_HEADS
    return outs


def ring_attn_fwd(q, k, v, geo: Geometry, mesh: Mesh, ops):
    """Ring attention of this rank's head-sharded q [B, L, Hq/P_u, D] over the
    K/V blocks of its ring (k, v: its own block). Returns (O bf16 like q, LSE
    fp32 [B, L, Hq/P_u])."""
    rows = q.shape[0] * q.shape[1] * q.shape[2]
    D = q.shape[3]
    dev = q.device
    # slot 0: running merge of the steps done; slot 1: the current step's partial
    o_parts = torch.empty((2, rows, D), dtype=torch.float32, device=dev)
    l_parts = torch.empty((2, rows), dtype=torch.float32, device=dev)
    # the caller's k, v are only ever sent; blocks are received into two buffers of our own
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(geo.P_r - 1, 2))]
    cur = (k, v)
    for t in range(geo.P_r):
        nxt = bufs[t % 2] if t < geo.P_r - 1 else None
        reqs = _exchange(cur, nxt, mesh.ring_next, mesh.ring_prev) if nxt is not None else []
        slot = 0 if t == 0 else 1
        ops.fwd_step(q, cur[0], cur[1], o_parts[slot], l_parts[slot], t)
        if t > 0:
            ops.merge(o_parts, l_parts, 2, o_parts[0], l_parts[0])
        for r in reqs:
            r.wait()
        if nxt is not None:
            cur = nxt
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    ops.merge(o_parts[:1], l_parts[:1], 1, out.view(rows, D), lse.view(rows))
    return out, lse


def ring_attn_bwd(q, k, v, out, lse, dO, geo: Geometry, mesh: Mesh, ops):
    """Backward of ring_attn_fwd on this rank: returns (dQ bf16, dK fp32, dV fp32)
    of its own query rows and its own K/V block."""
    ops.bwd_prepare(out, lse, dO)
    dq_acc = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    dq = torch.empty_like(q)
    grads = (torch.zeros(k.shape, dtype=torch.float32, device=k.device),
             torch.zeros(v.shape, dtype=torch.float32, device=v.device))
    g_in = (torch.empty_like(grads[0]), torch.empty_like(grads[1])) if geo.P_r > 1 else None
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(geo.P_r - 1, 2))]
    cur = (k, v)
    for t in range(geo.P_r):
        # the next K/V block travels while this one is computed
        nxt = bufs[t % 2] if t < geo.P_r - 1 else None
        reqs = _exchange(cur, nxt, mesh.ring_next, mesh.ring_prev) if nxt is not None else []
        last = t == geo.P_r - 1
        ops.bwd_step(q, cur[0], cur[1], dO, dq_acc, dq if last else None, grads[0], grads[1], t)
        for r in reqs:
            r.wait()
        if geo.P_r > 1:
            # the block's gradients follow it (after the last step: home to its owner)
            for r in _exchange(grads, g_in, mesh.ring_next, mesh.ring_prev):
                r.wait()
            grads, g_in = g_in, grads
        if nxt is not None:
            cur = nxt
    return dq, grads[0], grads[1]


def usp_attention(q, k, v, geo: Geometry, mesh: Mesh, ops=None):
    """The whole USP forward of this rank: rank-local q [B, T, Hq, D], k/v
    [B, T, Hkv, D] (zigzag chunks r and 2P-1-r) -> rank-local O [B, T, Hq, D]
    plus the head-sharded tensors the backward needs."""
    ops = CudaOps(geo, mesh) if ops is None else ops
    qh, kh, vh = seq2head([q, k, v], geo, mesh, ops)
    out_h, lse_h = ring_attn_fwd(qh, kh, vh, geo, mesh, ops)
    (out,) = head2seq([out_h], geo, mesh, ops)
    return out, (qh, kh, vh, out_h, lse_h)


def usp_attention_bwd(dout, saved, geo: Geometry, mesh: Mesh, ops=None):
    """Backward of usp_attention: rank-local dO [B, T, Hq, D] -> rank-local
    (dQ bf16 [B, T, Hq, D], dK, dV fp32 [B, T, Hkv, D])."""
    ops = CudaOps(geo, mesh) if ops is None else ops
    qh, kh, vh, out_h, lse_h = saved
    (doh,) = seq2head([dout], geo, mesh, ops)
    dqh, dkh, dvh = ring_attn_bwd(qh, kh, vh, out_h, lse_h, doh, geo, mesh, ops)
    return tuple(head2seq([dqh, dkh, dvh], geo, mesh, ops))

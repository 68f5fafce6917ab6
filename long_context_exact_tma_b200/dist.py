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
usp_ring_fwd_accumulate / usp_lse_merge, usp_ring_bwd_prepare / usp_ring_bwd_step);
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

    def fwd_acc(self, q, k, v, o_run, lse_run, t):
        """Step t folded into the running fp32 result (written at t = 0)."""
        g, m = self.geo, self.mesh
        self.B_.usp_ring_fwd_accumulate(q, k, v, o_run, lse_run, g.B, g.S, g.Hq, g.Hkv, g.D, g.causal, g.P_u, g.P_r,
                                        m.i, m.u, t, self.ws_f, self.ws_f.numel(), self.stream)

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
    # the running fp32 result: step 0 writes it, every later step is folded into it
    o_run = torch.empty((1, rows, D), dtype=torch.float32, device=dev)
    l_run = torch.empty((1, rows), dtype=torch.float32, device=dev)
    # the caller's k, v are only ever sent; blocks are received into two buffers of our own
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(geo.P_r - 1, 2))]
    cur = (k, v)
    for t in range(geo.P_r):
        nxt = bufs[t % 2] if t < geo.P_r - 1 else None
        reqs = _exchange(cur, nxt, mesh.ring_next, mesh.ring_prev) if nxt is not None else []
        ops.fwd_acc(q, cur[0], cur[1], o_run[0], l_run[0], t)
        for r in reqs:
            r.wait()
        if nxt is not None:
            cur = nxt
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    ops.merge(o_run, l_run, 1, out.view(rows, D), lse.view(rows))
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


# ---------------------------------------------------------------- LongNet's distributed layout
#
# LongNet slides, "LONGNET as a Distributed Trainer": the sequence is split
# into M contiguous slices of T = S / M tokens, one per rank. A dilated pair
# (w, r) whose segments fit a slice (w <= T) is computed locally. A longer
# segment spans G = w / T ranks: for each head offset o every rank packs its
# kept K/V rows (positions = o mod r, the kv heads of the query heads o, o + r,
# ...: 1/r of its rows), the G ranks all-gather them, and each rank's kept
# queries attend all the segment's kept rows. In the backward the all-gather's
# transpose, a reduce-scatter, brings every rank's contribution to the
# gathered rows' dK/dV back to the rank that holds those rows.


class TorchComm:
    """The collectives of the LongNet schedule over torch.distributed groups
    (NCCL on GPUs; gloo lacks the tensor forms, so there the same sums are
    taken by all_gather / all_reduce)."""

    def all_gather(self, recv, send, group):
        """recv [G, *send.shape] <- every group member's send, in group-rank order."""
        if dist.get_backend(group) == "nccl":
            dist.all_gather_into_tensor(recv.view(-1), send.reshape(-1), group=group)
        else:
            dist.all_gather(list(recv.unbind(0)), send, group=group)

    def reduce_scatter(self, recv, send, group):
        """recv <- sum over the group of send[this member's group rank]."""
        if dist.get_backend(group) == "nccl":
            dist.reduce_scatter_tensor(recv.reshape(-1), send.reshape(-1), op=dist.ReduceOp.SUM, group=group)
        else:
            buf = send.clone()
            dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
            recv.copy_(buf[dist.get_rank(group)])


class LongNetMesh:
    """Rank d of M holds positions [d T, (d + 1) T). For every gathered segment
    length w (w > T) the M / G groups of G = w / T consecutive ranks; every
    rank must construct this (torch.distributed.new_group is collective)."""

    def __init__(self, S: int, pairs, rank: int | None = None, world: int | None = None, make_groups: bool = True):
        self.rank = dist.get_rank() if rank is None else rank
        self.M = dist.get_world_size() if world is None else world
        if S % self.M != 0:
            raise ValueError(f"S={S} is not a multiple of the world size {self.M}")
        self.T = S // self.M
        self.groups = {}
        for w, r in pairs:
            if w <= self.T:
                if self.T % w != 0:
                    raise ValueError(f"segment {w} does not divide the slice {self.T}")
                continue
            if w % self.T != 0 or S % w != 0:
                raise ValueError(f"segment {w} is not a multiple of the slice {self.T} or does not divide S")
            G = w // self.T
            if G in self.groups:
                continue
            mine = None
            for s in range(self.M // G):  # every rank creates every group, in the same order
                ranks = list(range(s * G, (s + 1) * G))
                grp = dist.new_group(ranks) if make_groups else ranks
                if self.rank in ranks:
                    mine = grp
            self.groups[G] = mine

    def seg_rank(self, w: int) -> int:
        return self.rank % (w // self.T)


def longnet_rows(T, w, r, o, g):
    """(lp0, k_lo, n_rows, n_kept): rank g's kept rows of offset o in a segment
    of w = G T tokens (the plain arithmetic of usp_longnet_rows)."""
    a = g * T
    p0 = a + (o - a) % r
    n_rows = (a + T - p0 + r - 1) // r if p0 < a + T else 0
    return p0 - a, (p0 - o) // r, n_rows, (w - o + r - 1) // r


def _n_sel(Hq, r, o):
    return (Hq - o + r - 1) // r


def _gather_kept(k, v, w, r, o, Hq, lm: LongNetMesh, ops, comm):
    """The kept K/V rows of offset o of the whole segment on every rank of it:
    kc, vc [B, n_kept, n_sel, D] (head j = the kv head of query head o + j r)."""
    B, T, Hkv, D = k.shape
    Gq = Hq // Hkv
    G = w // T
    g = lm.seg_rank(w)
    ns = _n_sel(Hq, r, o)
    shares = [longnet_rows(T, w, r, o, x) for x in range(G)]
    n_max = max(s[2] for s in shares)
    n_kept = shares[0][3]
    lp0, _, n_rows, _ = shares[g]
    send = torch.empty((2, B, n_max, ns, D), dtype=k.dtype, device=k.device)
    jobs = [dict(src=x, dst=send[c], dtype=ops.BF16, n_b=B, n_k=n_rows, n_j=ns, D=D,
                 s_b=T * Hkv * D, s_k=Hkv * D, s_h=D, s_k0=lp0, s_kstep=r, s_h0=o, s_hstep=r, s_hdiv=Gq,
                 d_b=n_max * ns * D, d_k=ns * D, d_h=D) for c, x in enumerate((k, v))]
    ops.rows_copy(jobs)
    recv = torch.empty((G,) + tuple(send.shape), dtype=k.dtype, device=k.device)
    comm.all_gather(recv, send, lm.groups[G])
    kc = torch.empty((B, n_kept, ns, D), dtype=k.dtype, device=k.device)
    vc = torch.empty_like(kc)
    jobs = []
    for x, (_, k_lo, nr, _) in enumerate(shares):
        for c, dst in enumerate((kc, vc)):
            jobs.append(dict(src=recv[x, c], dst=dst, dtype=ops.BF16, n_b=B, n_k=nr, n_j=ns, D=D,
                             s_b=n_max * ns * D, s_k=ns * D, s_h=D, d_b=n_kept * ns * D, d_k=ns * D, d_h=D,
                             d_k0=k_lo))
    for x in range(0, len(jobs), 16):
        ops.rows_copy(jobs[x:x + 16])
    return kc, vc, shares, n_max


def longnet_attn_fwd(q, k, v, pairs, causal, lm: LongNetMesh, ops, comm=None):
    """LongNet dilated attention of this rank's slice q [B, T, Hq, D], k, v
    [B, T, Hkv, D]: returns (O bf16 [B, T, Hq, D], LSE fp32 [B, T, Hq]), equal to
    rows [d T, (d + 1) T) of dilated attention over the whole sequence."""
    comm = TorchComm() if comm is None else comm
    Hq = q.shape[2]
    ops.fwd_begin()
    for w, r in pairs:
        if w <= lm.T:
            ops.fwd_local(q, k, v, causal, w, r)
            continue
        # the offsets write disjoint heads: ops may run their cross attentions side by side
        for o in range(min(r, Hq)):
            kc, vc, _, _ = _gather_kept(k, v, w, r, o, Hq, lm, ops, comm)
            ops.fwd_cross(q, kc, vc, causal, w, r, o, lm.seg_rank(w))
        ops.cross_join()
    return ops.fwd_end()


def longnet_attn_bwd(q, k, v, out, lse, dO, pairs, causal, lm: LongNetMesh, ops, comm=None):
    """Backward of longnet_attn_fwd on this rank: (dQ bf16, dK fp32, dV fp32) of
    its own slice. Gathered pairs gather the kept K/V rows again, compute this
    rank's queries' share of their gradients and reduce-scatter them home."""
    comm = TorchComm() if comm is None else comm
    B, T, Hkv, D = k.shape
    Hq = q.shape[2]
    Gq = Hq // Hkv
    dK = torch.empty((B, T, Hkv, D), dtype=torch.float32, device=k.device)
    dV = torch.empty_like(dK)
    ops.bwd_begin(out, lse, dO, dK, dV)
    for w, r in pairs:
        if w <= T:
            ops.bwd_local(q, k, v, dO, lse, dK, dV, causal, w, r)
            continue
        G = w // T
        # every offset's cross backward first (ops may run them side by side: disjoint
        # heads, their own dkc / dvc), then their gradients home
        pending = []
        for o in range(min(r, Hq)):
            kc, vc, shares, n_max = _gather_kept(k, v, w, r, o, Hq, lm, ops, comm)
            dkc = torch.empty(kc.shape, dtype=torch.float32, device=k.device)
            dvc = torch.empty_like(dkc)
            ops.bwd_cross(q, kc, vc, dO, lse, dkc, dvc, causal, w, r, o, lm.seg_rank(w))
            pending.append((o, shares, n_max, dkc, dvc))
        ops.cross_join()
        for o, shares, n_max, dkc, dvc in pending:
            ns = dkc.shape[2]
            n_kept = dkc.shape[1]
            send = torch.empty((G, 2, B, n_max, ns, D), dtype=torch.float32, device=k.device)
            jobs = []
            for x, (_, k_lo, nr, _) in enumerate(shares):
                for c, src in enumerate((dkc, dvc)):
                    jobs.append(dict(src=src, dst=send[x, c], dtype=ops.F32, n_b=B, n_k=nr, n_j=ns, D=D,
                                     s_b=n_kept * ns * D, s_k=ns * D, s_h=D, s_k0=k_lo,
                                     d_b=n_max * ns * D, d_k=ns * D, d_h=D))
            for x in range(0, len(jobs), 16):
                ops.rows_copy(jobs[x:x + 16])
            recv = torch.empty((2, B, n_max, ns, D), dtype=torch.float32, device=k.device)
            comm.reduce_scatter(recv, send, lm.groups[G])
            lp0, _, nr, _ = shares[lm.seg_rank(w)]
            ops.rows_copy([dict(src=recv[c], dst=dst, dtype=ops.F32, add=1, n_b=B, n_k=nr, n_j=ns, D=D,
                                s_b=n_max * ns * D, s_k=ns * D, s_h=D,
                                d_b=T * Hkv * D, d_k=Hkv * D, d_h=D, d_k0=lp0, d_kstep=r, d_h0=o, d_hstep=r,
                                d_hdiv=Gq) for c, dst in enumerate((dK, dV))])
    dq = ops.bwd_end()
    return dq, dK, dV


class CudaLongNetOps:
    """The per-rank LongNet compute in libusp.so kernels. The cross attentions of
    one gathered pair's head offsets run on side streams (offset o on stream
    o mod min(16, offsets): the library's row-table slot of a cross backward is o
    mod 16); cross_join makes the main stream wait for them."""

    N_SIDE = 16

    def __init__(self, B, T, Hq, Hkv, D, pairs, stream=None, device="cuda"):
        from . import binding as B_
        self.B_ = B_
        self.BF16, self.F32 = B_.USP_BF16, B_.USP_F32
        self.shape = (B, T, Hq, Hkv, D)
        # (a raw cudaStream_t handle is wrapped, so that events can be recorded on it)
        self.stream = torch.cuda.ExternalStream(stream, device=device) if isinstance(stream, int) else stream
        self._side = None
        self._used = []
        self.ws_f = torch.zeros(B_.usp_longnet_workspace_size(B, T, Hq, D, pairs, 0), dtype=torch.uint8,
                                device=device)
        self.ws_b = torch.zeros(B_.usp_longnet_workspace_size(B, T, Hq, D, pairs, 1), dtype=torch.uint8,
                                device=device)
        self.device = device

    def rows_copy(self, jobs):
        self.B_.usp_rows_copy(jobs, self.stream)

    def fwd_begin(self):
        B, T, Hq, Hkv, D = self.shape
        self.B_.usp_longnet_fwd_begin(B, T, Hq, D, self.ws_f, self.ws_f.numel(), self.stream)

    def fwd_local(self, q, k, v, causal, w, r):
        B, T, Hq, Hkv, D = self.shape
        self.B_.usp_longnet_fwd_local(q, k, v, B, T, Hq, Hkv, D, causal, w, r, self.ws_f, self.ws_f.numel(),
                                      self.stream)

    def _main(self):
        return self.stream if self.stream is not None else torch.cuda.current_stream(self.device)

    def _side_for(self, o, r, tensors):
        """The side stream of offset o, after everything issued so far on the main
        stream; the given tensors are kept from reuse until its work is done."""
        if self._side is None:
            self._side = [torch.cuda.Stream(device=self.device) for _ in range(self.N_SIDE)]
        s = self._side[o % min(self.N_SIDE, r, self.shape[2])]
        ev = torch.cuda.Event()
        ev.record(self._main())
        s.wait_event(ev)
        for t in tensors:
            t.record_stream(s)
        if s not in self._used:
            self._used.append(s)
        return s

    def cross_join(self):
        main = self._main()
        for s in self._used:
            ev = torch.cuda.Event()
            ev.record(s)
            main.wait_event(ev)
        self._used = []

    def fwd_cross(self, q, kc, vc, causal, w, r, o, g):
        B, T, Hq, Hkv, D = self.shape
        s = self._side_for(o, r, (q, kc, vc))
        self.B_.usp_longnet_fwd_cross(q, kc, vc, B, T, Hq, Hkv, D, causal, w, r, o, g, self.ws_f, self.ws_f.numel(),
                                      s)

    def fwd_end(self):
        B, T, Hq, Hkv, D = self.shape
        out = torch.empty((B, T, Hq, D), dtype=torch.bfloat16, device=self.device)
        lse = torch.empty((B, T, Hq), dtype=torch.float32, device=self.device)
        self.B_.usp_longnet_fwd_end(out, lse, B, T, Hq, D, self.ws_f, self.ws_f.numel(), self.stream)
        return out, lse

    def bwd_begin(self, out, lse, dO, dK, dV):
        B, T, Hq, Hkv, D = self.shape
        self.B_.usp_longnet_bwd_begin(out, lse, dO, dK, dV, B, T, Hq, Hkv, D, self.ws_b, self.ws_b.numel(),
                                      self.stream)

    def bwd_local(self, q, k, v, dO, lse, dK, dV, causal, w, r):
        B, T, Hq, Hkv, D = self.shape
        self.B_.usp_longnet_bwd_local(q, k, v, dO, lse, dK, dV, B, T, Hq, Hkv, D, causal, w, r, self.ws_b,
                                      self.ws_b.numel(), self.stream)

    def bwd_cross(self, q, kc, vc, dO, lse, dkc, dvc, causal, w, r, o, g):
        B, T, Hq, Hkv, D = self.shape
        s = self._side_for(o, r, (q, kc, vc, dO, lse, dkc, dvc))
        self.B_.usp_longnet_bwd_cross(q, kc, vc, dO, lse, dkc, dvc, B, T, Hq, Hkv, D, causal, w, r, o, g, self.ws_b,
                                      self.ws_b.numel(), s)

    def bwd_end(self):
        B, T, Hq, Hkv, D = self.shape
        dq = torch.empty((B, T, Hq, D), dtype=torch.bfloat16, device=self.device)
        self.B_.usp_longnet_bwd_end(dq, B, T, Hq, D, self.ws_b, self.ws_b.numel(), self.stream)
        return dq

    def check(self):
        for ws in (self.ws_f, self.ws_b):
            rc, site = self.B_.usp_workspace_status(ws, self.stream)
            if rc != self.B_.USP_OK:
                raise self.B_.UspError(rc, f"device wait timed out (site {site:#x})")

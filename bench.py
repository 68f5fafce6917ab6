"""Benchmark of the USP attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

One step = one pass of the whole per-rank hot path over one batch, with the
inputs already sharded the way the ranks hold them (zigzag, rank-major):
  seq->head all-to-all of Q, K, V  ->  attention forward (ring steps merged
  in-kernel)  ->  head->seq of O  ->  seq->head of dO  ->  attention backward
  (preprocess, blockwise dQ/dK/dV)  ->  head->seq of dQ, dK, dV.
Every step runs in libusp.so kernels through the C ABI. The metric is the
algorithmic attention FLOPs of forward + backward (fwd = 4*B*Hq*S^2*D, x1/2
when causal; bwd = 2.5 x fwd) per second of step time, for the whole job.

Default workload: the S=16384 causal configuration (B=1, H=32, D=128, ring of
8 zigzag chunks), forward and backward. --config picks another workload.
With --gpus N (under torchrun) every rank runs its own independent batch
(weak scaling; no collective on the data path), timing is the max over ranks.
--impl reference times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from usp_inputs import WORKLOADS, workload  # noqa: E402

METRIC = "attention TFLOP/s fwd+bwd at S=16K-256K; % of bf16 dense tensor peak"
UNIT = "TFLOP/s"
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the
# dK/dV kernel on causal_fwd_s16k_ring8, from an ncu capture of that kernel.
# Reported only while the kernel's sources hash to what was captured (else the
# figure is stale: null).
DKDV_TRAFFIC = {"workload": "causal_fwd_s16k_ring8", "bytes": 781505280,
                "sources_sha256": "32597b7fde5007a9c6a2ae01b8c7791ba3409860dcd136afc193b6d95c6a9540"}
DKDV_SOURCES = ("usp_attn_bwd.cu", "usp_attn_common.cuh", "usp_ptx.cuh", "usp_internal.h")


def dkdv_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in DKDV_SOURCES:
        with open(os.path.join(ROOT, "long_context_exact_tma_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def dkdv_traffic(workload_name: str):
    rec = DKDV_TRAFFIC
    if rec["bytes"] is None or workload_name != rec["workload"]:
        return None
    return rec["bytes"] if dkdv_sources_sha256() == rec["sources_sha256"] else None



def flops_fwd(w) -> float:
    return 4.0 * w["B"] * w["Hq"] * w["S"] * w["S"] * w["D"] * (0.5 if w["causal"] else 1.0)


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured"
    return 1590.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        return summarize_clock_lines(self.lines)


def summarize_clock_lines(lines):
    """Median SM clock, max clock and the throttle reasons seen in nvidia-smi CSV lines."""
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 7:
            continue
        try:
            sm.append(float(parts[0]))
            mx.append(float(parts[1]))
        except ValueError:
            continue
        for n, v in zip(names, parts[3:7]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "samples": len(sm)}


def setup_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Largest value over the ranks (timing only; the data path has no collective)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------- our implementation
class Step:
    """Buffers and the launch sequence of one step of the hot path on one GPU."""

    def __init__(self, w, dev, seed_offset=0):
        from long_context_exact_tma_b200 import api
        from long_context_exact_tma_b200 import binding as B_
        self.api, self.B_ = api, B_
        self.w = w
        B, S, Hq, Hkv, D = w["B"], w["S"], w["Hq"], w["Hkv"], w["D"]
        P_u, P_r = w["P_u"], w["P_r"]
        P = P_u * P_r
        spec = dict(w)
        spec["seed"] = w["seed"] + seed_offset
        t = workload(spec, device=dev, which=("q", "k", "v", "do"))
        # inputs as the ranks hold them: zigzag-sharded, rank-major
        self.rm = {n: api.zigzag_shard(t[n], P_u, P_r) for n in ("q", "k", "v", "do")}
        del t
        L = S // P_r
        bf = torch.bfloat16
        self.hs = {"q": torch.empty((P_r, P_u, B, L, Hq // P_u, D), dtype=bf, device=dev),
                   "k": torch.empty((P_r, P_u, B, L, Hkv // P_u, D), dtype=bf, device=dev),
                   "v": torch.empty((P_r, P_u, B, L, Hkv // P_u, D), dtype=bf, device=dev),
                   "do": torch.empty((P_r, P_u, B, L, Hq // P_u, D), dtype=bf, device=dev)}
        self.out = torch.empty_like(self.hs["q"])
        self.lse = torch.empty(self.hs["q"].shape[:-1], dtype=torch.float32, device=dev)
        # gradients in the inputs' type (bf16, accumulated in fp32 on chip)
        self.dq = torch.empty_like(self.hs["q"])
        self.dk = torch.empty_like(self.hs["k"])
        self.dv = torch.empty_like(self.hs["v"])
        self.o_rm = torch.empty((P, B, S // P, Hq, D), dtype=bf, device=dev)
        self.dq_rm = torch.empty_like(self.o_rm)
        self.dk_rm = torch.empty((P, B, S // P, Hkv, D), dtype=bf, device=dev)
        self.dv_rm = torch.empty_like(self.dk_rm)
        self.ws_f = api.workspace(B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, w["causal"], P_u, P_r, 0, 0), dev)
        self.ws_b = api.workspace(B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, w["causal"], P_u, P_r, 0, 1), dev)
        # the permutes of dO and O run on a second stream, overlapping the attention kernels
        self.side = torch.cuda.Stream(device=dev)
        self.e_start, self.e_do, self.e_fwd, self.e_o = (torch.cuda.Event() for _ in range(4))

    def run(self, ev=None):
        """One step; ev = (start, end) event pairs per timed call, or None."""
        api, w = self.api, self.w
        P_u, P_r, causal = w["P_u"], w["P_r"], w["causal"]
        st = torch.cuda.current_stream()
        side = self.side
        # Ulysses all-to-all of dO on the side stream while Q, K, V are permuted and
        # the forward runs (it only waits for the previous step's use of hs["do"])
        self.e_start.record(st)
        side.wait_event(self.e_start)
        with torch.cuda.stream(side):
            api.seq2head(self.rm["do"], P_u, P_r, out=self.hs["do"])
            self.e_do.record(side)
        # the Ulysses all-to-all of Q, K and V in one launch
        api.seq2head_many([self.rm[n] for n in ("q", "k", "v")], P_u, P_r,
                          outs=[self.hs[n] for n in ("q", "k", "v")])
        if ev:
            ev["fwd"][0].record(st)
        api.attn_fwd(self.hs["q"], self.hs["k"], self.hs["v"], causal, P_u, P_r, ws=self.ws_f, out=self.out,
                     lse=self.lse)
        if ev:
            ev["fwd"][1].record(st)
        # O back to the sequence layout on the side stream while the backward runs
        self.e_fwd.record(st)
        side.wait_event(self.e_fwd)
        with torch.cuda.stream(side):
            api.head2seq(self.out, P_u, P_r, out=self.o_rm)
            self.e_o.record(side)
        st.wait_event(self.e_do)
        # backward = prepare + key-major dK/dV kernel + query-major dQ kernel (what
        # usp_attn_bwd runs), called phase by phase so the dK/dV kernel is timed alone
        geo = (w["B"], w["S"], w["Hq"], w["Hkv"], w["D"], causal, P_u, P_r)
        B_, ws_b = self.B_, self.ws_b
        if ev:
            ev["bwd"][0].record(st)
        B_.usp_attn_bwd_prepare(self.out, self.lse, self.hs["do"], *geo, ws_b, ws_b.numel(), st)
        if ev:
            ev["dkdv"][0].record(st)
        B_.usp_attn_bwd_dkdv_bf16(self.hs["q"], self.hs["k"], self.hs["v"], self.hs["do"], self.dk, self.dv, *geo,
                                  ws_b, ws_b.numel(), st)
        if ev:
            ev["dkdv"][1].record(st)
        B_.usp_attn_bwd_dq(self.hs["q"], self.hs["k"], self.hs["v"], self.hs["do"], self.dq, *geo,
                           ws_b, ws_b.numel(), st)
        if ev:
            ev["bwd"][1].record(st)
        # the regather of dQ, dK and dV in one launch
        api.head2seq_many([self.dq, self.dk, self.dv], P_u, P_r, outs=[self.dq_rm, self.dk_rm, self.dv_rm])
        st.wait_event(self.e_o)  # the step ends with O's permute done too

    def check_status(self):
        for ws in (self.ws_f, self.ws_b):
            rc, site = self.B_.usp_workspace_status(ws)
            if rc != 0:
                raise RuntimeError(f"device wait timed out (site {site:#x})")

    def host_io(self):
        """Pinned host buffers for the end-to-end measurement."""
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)  # noqa: E731
        self.h_in = {n: pin(self.rm[n]) for n in self.rm}
        for n in self.rm:
            self.h_in[n].copy_(self.rm[n])
        self.h_out = [pin(self.o_rm), pin(self.dq_rm), pin(self.dk_rm), pin(self.dv_rm)]
        h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        d2h = sum(t.numel() * t.element_size() for t in self.h_out)
        return h2d, d2h

    def copy_in(self):
        for n in self.rm:
            self.rm[n].copy_(self.h_in[n], non_blocking=True)

    def copy_out(self):
        for h, d in zip(self.h_out, (self.o_rm, self.dq_rm, self.dk_rm, self.dv_rm)):
            h.copy_(d, non_blocking=True)


class E2EPipeline:
    """End-to-end steps through the C ABI with host buffers on both sides. Two
    buffer sets alternate; each step's host-to-device copy (one stream), its
    kernels (a second stream) and the device-to-host copy of its results (a
    third) are ordered by events, so step i+1's inputs cross PCIe while step i
    computes and step i-1's results come back: every step still moves all of its
    own bytes inside the timed region."""

    def __init__(self, steps):
        self.steps = steps
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream() for _ in range(3))
        self.ev_in = [torch.cuda.Event() for _ in steps]
        self.ev_comp = [torch.cuda.Event() for _ in steps]
        self.ev_out = [torch.cuda.Event() for _ in steps]

    def run(self, n):
        nb = len(self.steps)
        for i in range(n):
            b = i % nb
            st = self.steps[b]
            with torch.cuda.stream(self.s_in):
                if i >= nb:
                    self.s_in.wait_event(self.ev_comp[b])  # the step that last used these inputs is done
                st.copy_in()
                self.ev_in[b].record()
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(self.ev_in[b])
                if i >= nb:
                    self.s_comp.wait_event(self.ev_out[b])  # its previous results have been read back
                st.run()
                self.ev_comp[b].record()
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_comp[b])
                st.copy_out()
                self.ev_out[b].record()


def cpu_baseline_sample(w, seconds=10.0, seed=0):
    """Time the fp64 oracle (forward + dQ rows) on a bounded sample of the workload.

    Returns (tflops, n_rows, elapsed, threads). Each sampled query row is credited
    with the algorithmic FLOPs the oracle performs for it: 8*D per visible key
    (QK^T and PV of the forward, dP and dQ of the backward).
    """
    import numpy as np

    import oracle
    t = workload(dict(w), device="cuda", which=("q", "k", "v", "do"))
    tc = {n: t[n].cpu() for n in ("q", "k", "v", "do")}
    del t
    rng = np.random.default_rng(seed)
    B, S, Hq, D = w["B"], w["S"], w["Hq"], w["D"]

    def rows_of(n):
        return [(int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(S))) for _ in range(n)]

    def vis(rows):
        return sum((i + 1) if w["causal"] else S for _, _, i in rows)

    probe = rows_of(32)
    t0 = time.perf_counter()
    oracle.attn_dq_rows(tc["q"], tc["k"], tc["v"], tc["do"], w["causal"], probe)
    per_row = max((time.perf_counter() - t0) / len(probe), 1e-6)
    n = int(min(max(32, seconds / per_row), 200000))
    rows = rows_of(n)
    t0 = time.perf_counter()
    oracle.attn_dq_rows(tc["q"], tc["k"], tc["v"], tc["do"], w["causal"], rows)
    el = time.perf_counter() - t0
    fl = 8.0 * D * vis(rows)
    return fl / el / 1e12, n, el, oracle.max_threads()


def _time_ms(fn, reps=5):
    """Mean device time of fn() over `reps` back-to-back calls (CUDA events on the
    current stream, one untimed call first)."""
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def permute_bandwidth(step):
    """GB/s of the step's seq->head all-to-all of Q, K and V (one launch), timed
    alone (inside the step it shares HBM with the side stream's permutes): read +
    write of every element once."""
    api, w = step.api, step.w
    names = ("q", "k", "v")
    ms = _time_ms(lambda: api.seq2head_many([step.rm[n] for n in names], w["P_u"], w["P_r"],
                                            outs=[step.hs[n] for n in names]))
    nbytes = 2 * sum(step.rm[n].numel() * step.rm[n].element_size() for n in names)
    return nbytes / (ms / 1e3) / 1e9, nbytes


def merge_bandwidth(step):
    """GB/s of usp_lse_merge on the partials the stepwise forward really leaves in
    its workspace: the running merge of ring steps 0..P_r-2 and step P_r-1's
    partial (fp32 O [rows, D] + LSE [rows] each), merged into O bf16 + LSE, the
    last step of the streamed ring merge. Read 2*(4D+4), write 2D+4 bytes a row."""
    api, B_, w = step.api, step.B_, step.w
    B, S, Hq, Hkv, D, P_u, P_r = (w[k] for k in ("B", "S", "Hq", "Hkv", "D", "P_u", "P_r"))
    need = B_.usp_attn_workspace_size(B, S, Hq, Hkv, D, w["causal"], P_u, P_r, B_.USP_MODE_STEPWISE, 0)
    ws = api.workspace(need, step.out.device)
    api.attn_fwd(step.hs["q"], step.hs["k"], step.hs["v"], w["causal"], P_u, P_r, mode=B_.USP_MODE_STEPWISE, ws=ws,
                 check_status=True)
    rows = B * S * Hq
    body = ws[256:]
    o_parts = body[: 2 * rows * D * 4].view(torch.float32).view(2, rows, D)
    l_parts = body[2 * rows * D * 4:].view(torch.float32).view(2, rows)
    out = torch.empty((rows, D), dtype=torch.bfloat16, device=ws.device)
    lse = torch.empty(rows, dtype=torch.float32, device=ws.device)
    ms = _time_ms(lambda: B_.usp_lse_merge(o_parts, l_parts, 2, rows, D, out, B_.USP_BF16, lse))
    nbytes = 2 * rows * (4 * D + 4) + rows * (2 * D + 4)
    del ws
    return nbytes / (ms / 1e3) / 1e9


def per_workload(dev, peak_tf, peak_hbm):
    """Event-timed figures on the workloads the targets are stated for: the causal
    GQA S=128K USP 4x2 forward and its permutes (seq->head of Q, K, V in one launch;
    head->seq of O), and the causal B=2 S=32K ring-4 backward. Inputs are seeded
    N(0,1) of each shape, already resident; 3 timed calls after one untimed."""
    from long_context_exact_tma_b200 import api
    from long_context_exact_tma_b200 import binding as B_
    res = {}
    for cfg, kind in ((3, "fwd"), (4, "bwd")):
        w = dict(WORKLOADS[cfg])
        P_u, P_r, causal = w["P_u"], w["P_r"], w["causal"]
        t = workload(w, device=dev, which=("q", "k", "v", "do") if kind == "bwd" else ("q", "k", "v"))
        rm = {n: api.zigzag_shard(t[n], P_u, P_r) for n in t if n != "spec"}
        del t
        names = ("q", "k", "v")
        hs = api.seq2head_many([rm[n] for n in names], P_u, P_r)
        hs = dict(zip(names, hs))
        f_fwd = flops_fwd(w)
        rec = {"workload": w["name"]}
        if kind == "fwd":
            ms = _time_ms(lambda: api.seq2head_many([rm[n] for n in names], P_u, P_r,
                                                    outs=[hs[n] for n in names]), reps=3)
            nb = 2 * sum(rm[n].numel() * rm[n].element_size() for n in names)
            rec["seq2head_qkv"] = {"GB/s": round(nb / (ms / 1e3) / 1e9, 1),
                                   "frac_of_hbm": round(nb / (ms / 1e3) / 1e9 / peak_hbm, 4), "bytes": nb}
            ws = api.workspace(256, dev)
            out, lse = api.attn_fwd(hs["q"], hs["k"], hs["v"], causal, P_u, P_r, ws=ws)
            ms = _time_ms(lambda: api.attn_fwd(hs["q"], hs["k"], hs["v"], causal, P_u, P_r, ws=ws, out=out, lse=lse),
                          reps=3)
            api.check_workspace(ws)
            tf = f_fwd / (ms / 1e3) / 1e12
            rec["fwd"] = {"TFLOP/s": round(tf, 1), "frac_of_peak": round(tf / peak_tf, 4), "ms": round(ms, 3)}
            o_rm = torch.empty((P_u * P_r,) + tuple(rm["q"].shape[1:]), dtype=torch.bfloat16, device=dev)
            ms = _time_ms(lambda: api.head2seq(out, P_u, P_r, out=o_rm), reps=3)
            nb = 2 * out.numel() * out.element_size()
            rec["head2seq_o"] = {"GB/s": round(nb / (ms / 1e3) / 1e9, 1),
                                 "frac_of_hbm": round(nb / (ms / 1e3) / 1e9 / peak_hbm, 4), "bytes": nb}
            del out, lse, o_rm
        else:
            do = api.seq2head(rm["do"], P_u, P_r)
            out, lse = api.attn_fwd(hs["q"], hs["k"], hs["v"], causal, P_u, P_r)
            geo = (w["B"], w["S"], w["Hq"], w["Hkv"], w["D"], causal, P_u, P_r)
            ws = api.workspace(B_.usp_attn_workspace_size(*geo, 0, 1), dev)
            dq, dk, dv = api.attn_bwd(hs["q"], hs["k"], hs["v"], out, lse, do, causal, P_u, P_r, ws=ws)
            ms = _time_ms(lambda: api.attn_bwd(hs["q"], hs["k"], hs["v"], out, lse, do, causal, P_u, P_r, ws=ws,
                                               dq=dq, dk=dk, dv=dv), reps=3)
            api.check_workspace(ws)
            tf = 2.5 * f_fwd / (ms / 1e3) / 1e12
            rec["bwd"] = {"TFLOP/s": round(tf, 1), "frac_of_peak": round(tf / peak_tf, 4), "ms": round(ms, 3),
                          "convention": "2.5 x forward FLOPs (5 GEMMs per visible 128x128 pair)"}
            del do, out, lse, dq, dk, dv
        res[f"cfg{cfg}"] = rec
        del rm, hs
        torch.cuda.empty_cache()
    res.update(variants_per_workload(dev, peak_tf))
    res.update(rank_per_workload(dev, peak_tf))
    return res


def _time_pair(fwd, bwd, reps=3):
    ms_f = _time_ms(fwd, reps)
    ms_b = _time_ms(bwd, reps)
    return ms_f, ms_b


def variants_per_workload(dev, peak_tf):
    """Event-timed forward and backward of the attention variants on workloads
    of the pages' shapes: LongNet dilated attention with its segment/dilation
    schedule (w = 2048..32768, r = 1, 2, 4, 6, 12) on a 32K sequence, and a
    block-sparse (half the 128 x 128 blocks, seeded) causal attention on the
    S=16K ring-8 workload. FLOPs are the algorithmic ones of the visible
    (query, key) pairs: 4*D per pair forward, 2.5x that backward."""
    from long_context_exact_tma_b200 import api
    import numpy as np
    from usp_inputs import normal_bf16
    res = {}
    # LongNet dilated attention
    B, S, H, D = 1, 32768, 16, 128
    pairs = [(2048, 1), (4096, 2), (8192, 4), (16384, 6), (32768, 12)]
    q, k, v, do = (normal_bf16(900 + x, (B, S, H, D), device=dev) for x in range(4))
    vis = 0
    for w, r in pairs:
        for h in range(H):
            kept = (w - h % r + r - 1) // r
            vis += (S // w) * kept * (kept + 1) // 2
    fl = 4.0 * D * B * vis
    o, l = api.dilated_attn_fwd(q, k, v, True, pairs)
    ms_f, ms_b = _time_pair(lambda: api.dilated_attn_fwd(q, k, v, True, pairs),
                            lambda: api.dilated_attn_bwd(q, k, v, o, l, do, True, pairs))
    res["dilated_longnet_s32k"] = {
        "shape": "B=1 S=32768 H=16 D=128 causal, (w, r) = (2048,1) (4096,2) (8192,4) (16384,6) (32768,12)",
        "fwd": {"TFLOP/s": round(fl / ms_f / 1e9, 1), "frac_of_peak": round(fl / ms_f / 1e9 / peak_tf, 4),
                "ms": round(ms_f, 3)},
        "bwd": {"TFLOP/s": round(2.5 * fl / ms_b / 1e9, 1), "frac_of_peak": round(2.5 * fl / ms_b / 1e9 / peak_tf, 4),
                "ms": round(ms_b, 3)}}
    del q, k, v, do, o, l
    # block-sparse causal attention, S=16K ring 8
    w = dict(WORKLOADS[2])
    P_u, P_r = w["P_u"], w["P_r"]
    t = workload(w, device=dev, which=("q", "k", "v", "do"))
    qh, kh, vh, doh = (api.to_head_sharded(t[n], P_u, P_r) for n in ("q", "k", "v", "do"))
    del t
    nb = w["S"] // 128
    rng = np.random.default_rng(17)
    bm = (rng.random((w["B"], w["Hq"], nb, nb)) < 0.5).astype(np.uint8)
    causal_blocks = np.tril(np.ones((nb, nb), np.int64), -1) * 128 * 128 + np.eye(nb, dtype=np.int64) * (128 * 129 // 2)
    fl = 4.0 * w["D"] * float((bm.astype(np.int64) * causal_blocks).sum())
    bmd = torch.tensor(bm, device=dev)
    o, l = api.attn_fwd_masked(qh, kh, vh, True, P_u, P_r, block_mask=bmd)
    ms_f, ms_b = _time_pair(lambda: api.attn_fwd_masked(qh, kh, vh, True, P_u, P_r, block_mask=bmd),
                            lambda: api.attn_bwd_masked(qh, kh, vh, o, l, doh, True, P_u, P_r, block_mask=bmd))
    res["block_sparse_s16k_ring8"] = {
        "shape": "the S=16K ring-8 workload with a seeded half-dense 128x128 block mask, causal",
        "fwd": {"TFLOP/s": round(fl / ms_f / 1e9, 1), "frac_of_peak": round(fl / ms_f / 1e9 / peak_tf, 4),
                "ms": round(ms_f, 3)},
        "bwd": {"TFLOP/s": round(2.5 * fl / ms_b / 1e9, 1), "frac_of_peak": round(2.5 * fl / ms_b / 1e9 / peak_tf, 4),
                "ms": round(ms_b, 3)}}
    del qh, kh, vh, doh, o, l, bmd
    torch.cuda.empty_cache()
    return res


def rank_per_workload(dev, peak_tf):
    """Event-timed per-rank compute of the two multi-GPU layouts, on one GPU
    (the collectives between the calls are not part of it):
      - one rank of a real USP mesh, rank (0, 0) of the S=16K ring-8 and of the
        S=128K USP 4x2 workloads: its ring steps (usp_ring_fwd_accumulate: each
        step's partial folded into a running one in the kernel) and the backward
        steps (usp_ring_bwd_prepare + usp_ring_bwd_step) against resident K/V
        blocks;
      - rank 0 of LongNet's distributed layout over 4 ranks on the S=32K
        dilated schedule: its local pairs and, for the gathered pairs, the cross
        attention of its kept rows against the segment's kept K/V rows (gathered
        beforehand by usp_rows_copy from the whole sequence, as the all-gather
        would deliver them), forward and backward.
    FLOPs are those of the rank's visible (query, key) pairs."""
    from long_context_exact_tma_b200 import binding as B_
    from long_context_exact_tma_b200 import dist as udist
    from usp_inputs import normal_bf16
    res = {}
    # -- one rank of the USP mesh: ring 8 at S=16K (2048 rows a rank) and USP 4x2 at S=128K (64K rows)
    for cfg, key in ((2, "usp_rank_s16k_ring8"), (3, "usp_rank_s128k_usp4x2")):
        w = dict(WORKLOADS[cfg])
        B, S, Hq, Hkv, D, P_u, P_r = w["B"], w["S"], w["Hq"], w["Hkv"], w["D"], w["P_u"], w["P_r"]
        causal, L = w["causal"], w["S"] // w["P_r"]
        P, c = P_u * P_r, S // (2 * P_u * P_r)
        Hl, Hkl = Hq // P_u, Hkv // P_u
        q = normal_bf16(950, (B, L, Hl, D), device=dev)
        do = normal_bf16(951, (B, L, Hl, D), device=dev)
        ks = [normal_bf16(960 + j, (B, L, Hkl, D), device=dev) for j in range(P_r)]
        vs = [normal_bf16(980 + j, (B, L, Hkl, D), device=dev) for j in range(P_r)]
        # rank (i=0, u=0) holds, after the all-to-all, the zigzag chunks of ranks 0 .. P_u-1
        pos0 = [x for rr in range(P_u) for ch in (rr, 2 * P - 1 - rr) for x in range(ch * c, (ch + 1) * c)]
        vis = sum(p + 1 for p in pos0) if causal else len(pos0) * S
        fl = 4.0 * D * B * Hl * vis
        rows = B * L * Hl
        wsf = torch.zeros(B_.usp_ring_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, 0), dtype=torch.uint8,
                          device=dev)
        wsb = torch.zeros(B_.usp_ring_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, 1), dtype=torch.uint8,
                          device=dev)
        o_run = torch.empty((1, rows, D), dtype=torch.float32, device=dev)
        l_run = torch.empty((1, rows), dtype=torch.float32, device=dev)
        out = torch.empty_like(q)
        lse = torch.empty((B, L, Hl), dtype=torch.float32, device=dev)

        def ring_fwd():  # each step folded into the running partial in the kernel's epilogue
            for t in range(P_r):
                j = (0 - t) % P_r
                B_.usp_ring_fwd_accumulate(q, ks[j], vs[j], o_run[0], l_run[0], B, S, Hq, Hkv, D, causal, P_u, P_r,
                                           0, 0, t, wsf, wsf.numel())
            B_.usp_lse_merge(o_run, l_run, 1, rows, D, out, B_.USP_BF16, lse)

        ring_fwd()
        dq_acc = torch.zeros((B, L, Hl, D), dtype=torch.float32, device=dev)
        dq = torch.empty_like(q)
        dk = torch.zeros((B, L, Hkl, D), dtype=torch.float32, device=dev)
        dv = torch.zeros_like(dk)

        def ring_bwd():
            B_.usp_ring_bwd_prepare(out, lse, do, B, S, Hq, Hkv, D, causal, P_u, P_r, wsb, wsb.numel())
            for t in range(P_r):
                j = (0 - t) % P_r
                B_.usp_ring_bwd_step(q, ks[j], vs[j], do, dq_acc, dq if t == P_r - 1 else None, dk, dv, B, S, Hq,
                                     Hkv, D, causal, P_u, P_r, 0, 0, t, wsb, wsb.numel())

        ms_f, ms_b = _time_pair(ring_fwd, ring_bwd, reps=10 if cfg == 2 else 2)
        for ws in (wsf, wsb):
            rc, site = B_.usp_workspace_status(ws)
            if rc != B_.USP_OK:
                raise B_.UspError(rc, f"device wait timed out (site {site:#x})")
        res[key] = {
            "shape": f"rank (0, 0) of the {w['name']} mesh: its {P_r} ring steps against resident K/V blocks "
                     f"({L} rows, {Hl} heads; no NCCL)",
            "fwd": {"TFLOP/s": round(fl / ms_f / 1e9, 1), "frac_of_peak": round(fl / ms_f / 1e9 / peak_tf, 4),
                    "ms": round(ms_f, 3)},
            "bwd": {"TFLOP/s": round(2.5 * fl / ms_b / 1e9, 1),
                    "frac_of_peak": round(2.5 * fl / ms_b / 1e9 / peak_tf, 4), "ms": round(ms_b, 3)}}
        del q, do, ks, vs, o_run, l_run, out, lse, dq_acc, dq, dk, dv, wsf, wsb
        torch.cuda.empty_cache()
    # -- rank 0 of LongNet's distributed layout, 4 ranks, S=32K
    B, S, H, D, M = 1, 32768, 16, 128, 4
    T = S // M
    pairs = [(2048, 1), (4096, 2), (8192, 4), (16384, 6), (32768, 12)]
    qg, kg, vg, dog = (normal_bf16(900 + x, (B, S, H, D), device=dev) for x in range(4))
    q, k, v, do = (x[:, :T].contiguous() for x in (qg, kg, vg, dog))
    ops = udist.CudaLongNetOps(B, T, H, H, D, pairs, device=dev)
    gathered = {}
    vis = 0
    for w_, r in pairs:
        for h in range(H):
            o = h % r
            if w_ <= T:  # every segment of the slice, causal among its kept rows
                kept = (w_ - o + r - 1) // r
                vis += (T // w_) * kept * (kept + 1) // 2
            else:  # rank 0 holds the first kept rows of its segment
                _, k_lo, n_rows, _ = udist.longnet_rows(T, w_, r, o, 0)
                vis += sum(k_lo + x + 1 for x in range(n_rows))
        if w_ <= T:
            continue
        for o in range(min(r, H)):
            ns = (H - o + r - 1) // r
            n_kept = (w_ - o + r - 1) // r
            kc = torch.empty((B, n_kept, ns, D), dtype=torch.bfloat16, device=dev)
            vc = torch.empty_like(kc)
            # the segment's kept rows of the kv heads of query heads o, o + r, ..., in kept order
            B_.usp_rows_copy([dict(src=x, dst=y, dtype=B_.USP_BF16, n_b=B, n_k=n_kept, n_j=ns, D=D, s_b=S * H * D,
                                   s_k=H * D, s_h=D, s_k0=o, s_kstep=r, s_h0=o, s_hstep=r, d_b=n_kept * ns * D,
                                   d_k=ns * D, d_h=D) for x, y in ((kg, kc), (vg, vc))])
            gathered[(w_, r, o)] = (kc, vc, torch.empty(kc.shape, dtype=torch.float32, device=dev),
                                    torch.empty(kc.shape, dtype=torch.float32, device=dev))
    fl = 4.0 * D * B * vis
    state = {}

    def ln_fwd():
        ops.fwd_begin()
        for w_, r in pairs:
            if w_ <= T:
                ops.fwd_local(q, k, v, True, w_, r)
            else:
                for o in range(min(r, H)):
                    kc, vc, _, _ = gathered[(w_, r, o)]
                    ops.fwd_cross(q, kc, vc, True, w_, r, o, 0)
                ops.cross_join()
        state["out"], state["lse"] = ops.fwd_end()

    ln_fwd()
    dK = torch.empty((B, T, H, D), dtype=torch.float32, device=dev)
    dV = torch.empty_like(dK)

    def ln_bwd():
        ops.bwd_begin(state["out"], state["lse"], do, dK, dV)
        for w_, r in pairs:
            if w_ <= T:
                ops.bwd_local(q, k, v, do, state["lse"], dK, dV, True, w_, r)
            else:
                for o in range(min(r, H)):
                    kc, vc, dkc, dvc = gathered[(w_, r, o)]
                    ops.bwd_cross(q, kc, vc, do, state["lse"], dkc, dvc, True, w_, r, o, 0)
                ops.cross_join()
        ops.bwd_end()

    ms_f, ms_b = _time_pair(ln_fwd, ln_bwd, reps=5)
    ops.check()
    res["longnet_rank_s32k_4ranks"] = {
        "shape": "rank 0 of 4 (T=8192) on the S=32K dilated schedule H=16 D=128 causal; gathered pairs "
                 "(16384,6) (32768,12) from pre-gathered kept K/V rows (no NCCL)",
        "fwd": {"TFLOP/s": round(fl / ms_f / 1e9, 1), "frac_of_peak": round(fl / ms_f / 1e9 / peak_tf, 4),
                "ms": round(ms_f, 3)},
        "bwd": {"TFLOP/s": round(2.5 * fl / ms_b / 1e9, 1), "frac_of_peak": round(2.5 * fl / ms_b / 1e9 / peak_tf, 4),
                "ms": round(ms_b, 3)}}
    del qg, kg, vg, dog, q, k, v, do, gathered, dK, dV, state, ops
    torch.cuda.empty_cache()
    return res


def l2_note(step, dev):
    """Whether every input of the step is larger than L2 (then no flush is needed
    between timed iterations)."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    sizes = {n: t.numel() * t.element_size() for n, t in step.rm.items()}
    big = all(v > l2 for v in sizes.values())
    txt = ", ".join(f"{n} {v / 1e6:.0f} MB" for n, v in sizes.items())
    return (f"inputs larger than L2 ({txt}; L2 {l2 / 1e6:.0f} MB)" if big else
            f"NOT all inputs larger than L2 ({txt}; L2 {l2 / 1e6:.0f} MB)")


def bench_ours(args, w, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    step = Step(w, dev, seed_offset=1000 * rank)
    peak_tf, peak_hbm, peak_src = read_peaks()
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    step.check_status()
    ev = {k: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)] for k in ("fwd", "bwd", "dkdv")}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    n_launch0 = step.B_.usp_launch_count()
    with ClockSampler(local) as clk:
        start.record()
        for s in range(args.steps):
            step.run({k: ev[k][s] for k in ev})
        end.record()
        torch.cuda.synchronize()
    gpu_launches = step.B_.usp_launch_count() - n_launch0
    barrier(world)
    step.check_status()
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, world)
    f_fwd = flops_fwd(w)
    f_step = 3.5 * f_fwd
    value = world * args.steps * f_step / (ms / 1e3) / 1e12
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["fwd"])
    bwd_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["bwd"])
    dkdv_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["dkdv"])
    # end to end: host buffers in, host buffers out, through the same C ABI calls,
    # with the copies of neighbouring steps overlapping the kernels
    e2e = h2d = d2h = None
    if not args.no_e2e:
        h2d, d2h = step.host_io()
        step2 = Step(w, dev, seed_offset=1000 * rank)
        step2.host_io()
        pipe = E2EPipeline([step, step2])
        pipe.run(2)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        e0.record(pipe.s_in)
        pipe.run(args.steps)
        e1.record(pipe.s_out)
        torch.cuda.synchronize()
        for st_ in (step, step2):
            st_.check_status()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = world * args.steps * f_step / (e2e_ms / 1e3) / 1e12
    if rank != 0:
        return None
    merge_gbs = merge_bandwidth(step)
    perm_gbs, perm_bytes = permute_bandwidth(step)
    per_wl = None if args.no_per_workload else per_workload(dev, peak_tf, peak_hbm)
    bwd_tf = 2.5 * f_fwd / (bwd_ms / 1e3) / 1e12
    # dominant kernel: the key-major dK/dV kernel, whose algorithmic work is its four
    # GEMMs per (key tile, query tile) pair (S^T, dP^T, dV, dK) = 2 x the forward FLOPs
    dkdv_tf = 2.0 * f_fwd / (dkdv_ms / 1e3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 + Box-Muller N(0,1), rounded to bf16)",
        "config": {"workload": w["name"], "B": w["B"], "S": w["S"], "Hq": w["Hq"], "Hkv": w["Hkv"],
                   "D": w["D"], "causal": bool(w["causal"]), "P_ulysses": w["P_u"], "P_ring": w["P_r"],
                   "global_batch": w["B"] * world, "seq_len": w["S"],
                   "parallelism": f"{world} independent replicas x (USP {w['P_u']}x{w['P_r']} virtual ranks)",
                   "l2": l2_note(step, dev)},
        "grad_dtype": "bf16 (dQ, dK, dV; fp32 accumulation on chip)",
        "pct_of_peak": round(100.0 * value / world / peak_tf, 2),
        "fwd_tflops": round(f_fwd / (fwd_ms / 1e3) / 1e12, 2),
        # the Ulysses seq->head all-to-all of Q, K, V (one launch): read + write of every element once
        "permute": {"kernel": "layout_gather_kernel (seq2head of Q, K, V in one launch, timed alone)",
                    "GB/s": round(perm_gbs, 1), "bytes": perm_bytes,
                    "frac_of_hbm": round(perm_gbs / peak_hbm, 4), "peak_source": f"{peak_src} hbm_gbs"},
        # the last step of the streamed ring merge, on the stepwise forward's own partials
        "merge": {"kernel": "lse_merge_kernel (running fp32 merge + last ring step's partial -> bf16 O + LSE)",
                  "GB/s": round(merge_gbs, 1), "frac_of_hbm": round(merge_gbs / peak_hbm, 4),
                  "peak_source": f"{peak_src} hbm_gbs"},
        "exp_count_fwd": int(flops_fwd(w) / (4 * w["D"])),  # B*Hq*S^2 (/2 causal); the backward recomputes them
        "bwd_tflops": round(bwd_tf, 2),
        "roofline": {"bound": "tensor", "kernel": "attn_bwd_kernel (key-major dK/dV; usp_attn_bwd_dkdv_bf16 call)",
                     "achieved": round(dkdv_tf, 2), "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": round(dkdv_tf / peak_tf, 4), "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "launch_ms": round(dkdv_ms, 4), "traffic": dkdv_traffic(w["name"])},
        "e2e": ({"value": round(e2e, 2), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                 "overlap": "copies of neighbouring steps overlap the kernels (3 streams, 2 buffer sets)"}
                if e2e is not None else None),
        "gpu_launches": gpu_launches,
        "per_workload": per_wl,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        tf, n, el, thr = cpu_baseline_sample(w, seconds=args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(tf, 6), "unit": UNIT, "cores": thr, "kind": "oracle",
                                "sample": f"fp64 oracle forward + dQ on {n} seeded query rows of {w['name']} "
                                          f"({el:.1f} s), credited 8*D FLOPs per visible key"}
    return line


def bench_reference(args, w, world, rank):
    """The oracle as the reference arm: each step a bounded sample, timed on the host cores."""
    if rank != 0:
        return None
    samples = []
    for _ in range(args.warmup):
        cpu_baseline_sample(w, seconds=args.ref_seconds, seed=7)
    tot_fl, tot_s, rows, thr = 0.0, 0.0, 0, 1
    for s in range(args.steps):
        tf, n, el, thr = cpu_baseline_sample(w, seconds=args.ref_seconds, seed=100 + s)
        samples.append(tf)
        tot_fl += tf * 1e12 * el
        tot_s += el
        rows += n
    value = tot_fl / tot_s / 1e12
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w["name"], "B": w["B"], "S": w["S"], "Hq": w["Hq"], "Hkv": w["Hkv"],
                   "D": w["D"], "causal": bool(w["causal"]), "P_ulysses": w["P_u"], "P_ring": w["P_r"],
                   "global_batch": w["B"], "seq_len": w["S"]},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": f"{rows} seeded query rows over {args.steps} steps (forward + dQ rows)"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--config", type=int, default=2, help="workload number (1-5), default the S=16K one")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the event-timed S=128K forward/permute and S=32K backward figures")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end host-buffer run (its pinned buffers are 2 x the step's IO)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: warmup raised to the minimum of 3", file=sys.stderr)
        args.warmup = 3
    w = dict(WORKLOADS[args.config])
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; other ranks have nothing to do
        if int(os.environ.get("RANK", "0")) != 0:
            return
        line = bench_reference(args, w, int(os.environ.get("WORLD_SIZE", "1")), 0)
        print(json.dumps(line), flush=True)
        return
    world, rank, local = setup_dist(args)
    try:
        line = bench_ours(args, w, world, rank, local)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

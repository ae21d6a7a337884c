#!/usr/bin/env python
"""Benchmark of the SA / STCA hot path on B200.

A step is one pass of the whole hot path over one batch: sa_forward and
sa_backward over 64 ragged users (mean 85K events, k=1024, d=128, bf16), then
STCA on the produced sketches and on each user's last 10K events against 256
candidates per user, then the linear fusion.  The headline metric is SA
history tokens per second (k=1024, d=128); STCA candidates per second and the
per-phase rates are reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU, NCCL) every rank runs its own
batch (weak scaling) and the weight gradients are all-reduced, the one
exchange step of data-parallel SA training.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

from sketch_attention_b200.dist import allreduce_weight_grads

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SA history-tokens/s (k=1024,d=128) + % of roofline; STCA candidates/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SMS, FP32_LANES = 148, 128


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


# --------------------------------------------------------------------------
# clocks during the timed region
class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled every 10 ms by a
    thread reading NVML during the timed region (read-only queries); the summary
    covers the samples taken between entry and exit.  Falls back to nvidia-smi's
    query loop when NVML is unavailable."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.max_mhz = None
        self.handle = None
        self.proc = None
        self.path = os.path.join("/tmp", f"sa_bench_clocks_{os.getpid()}.csv")

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            bus = torch.cuda.get_device_properties(self.dev).pci_bus_id
            pci = "%04x:%02x:%02x.0" % (torch.cuda.get_device_properties(self.dev).pci_domain_id, bus,
                                        torch.cuda.get_device_properties(self.dev).pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(pci.encode())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def _loop(self):
        nv, h = self.nv, self.handle
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                self.samples.append((time.time(), sm, pw, rs))
            except Exception:
                pass
            self.stop.wait(0.01)

    def __enter__(self):
        import threading
        try:
            self.nv, self.handle = self._nvml_handle()
            self.max_mhz = self.nv.nvmlDeviceGetMaxClockInfo(self.handle, self.nv.NVML_CLOCK_SM)
            self.stop = threading.Event()
            self.th = threading.Thread(target=self._loop, daemon=True)
            self.th.start()
            deadline = time.time() + 2.0
            while not self.samples and time.time() < deadline:
                time.sleep(0.005)
        except Exception:
            self.handle = None
            self._smi_start()
        self.t0 = time.time()
        return self

    def __exit__(self, *exc):
        self.t1 = time.time()
        if self.handle is not None:
            time.sleep(0.02)                        # one more sample after the region
            self.stop.set()
            self.th.join(timeout=2)
        elif self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    # -- fallback: nvidia-smi's query loop
    def _smi_start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
            deadline = time.time() + 5.0
            while time.time() < deadline and os.path.getsize(self.path) == 0:
                time.sleep(0.02)
        except Exception:
            self.proc = None

    @staticmethod
    def _epoch(ts):
        import datetime
        try:
            return datetime.datetime.strptime(ts, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def summary(self):
        if self.handle is not None:
            inside = [r for r in self.samples if self.t0 <= r[0] <= self.t1]
            rows = inside or self.samples
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
            reasons = sorted({name for r in rows for bit, name in self.REASONS.items() if r[3] & bit})
            return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": float(self.max_mhz),
                    "sm_mhz_min": min(r[1] for r in rows), "power_w_max": max(r[2] for r in rows),
                    "samples": len(self.samples), "samples_in_region": len(inside), "reasons": reasons,
                    "source": "NVML, every 10 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10 and parts[2].replace(".", "").isdigit():
                    rows.append(parts)
        inside = [r for r in rows if (lambda e: e is not None and self.t0 <= e <= self.t1)(self._epoch(r[0]))]
        if inside:
            rows = inside
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][3]),
                "power_w_max": max(float(r[4]) for r in rows if r[4].replace(".", "").isdigit()),
                "samples": len(rows), "samples_in_region": len(inside), "reasons": reasons,
                "source": "nvidia-smi -lms 50"}


# --------------------------------------------------------------------------
# workloads on the device
def _dev_bf16(bits, device):
    return torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)


def _f32(a, device):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


# the end-to-end step copies and computes in this many user groups, overlapped
E2E_GROUPS = 4


class TrainStepRunner:
    """Device buffers and the step of the end-to-end training workload."""

    def __init__(self, w, device, world):
        import sketch_attention_b200 as sab
        self.sab, self.w, self.dev, self.world = sab, w, device, world
        sa = w.sa
        self.B, self.k, self.d = sa.B, sa.k, sa.d
        self.off = sa.offsets
        self.X = _dev_bf16(sa.X, device)
        self.offd = torch.from_numpy(self.off).to(device)
        self.P, self.WQ, self.WK, self.WV = (_f32(a, device) for a in (sa.P, sa.W_Q, sa.W_K, sa.W_V))
        self.dS = _f32(sa.dS, device)
        self.q = _dev_bf16(w.q, device)
        self.cand = w.cand_offsets
        self.candd = torch.from_numpy(self.cand).to(device)
        self.rb, self.re = w.recent_begin, w.recent_end
        self.rbd, self.red = torch.from_numpy(self.rb).to(device), torch.from_numpy(self.re).to(device)
        self.sb = np.arange(self.B, dtype=np.int64) * self.k
        self.se = self.sb + self.k
        self.sbd, self.sed = torch.from_numpy(self.sb).to(device), torch.from_numpy(self.se).to(device)
        lay = lambda L: dict(W_Q=_f32(L.W_Q, device), W_K=_f32(L.W_K, device),
                             W_V=_f32(L.W_V, device), W_O=_f32(L.W_O, device))
        self.layers_r = [lay(L) for L in w.layers_r]
        self.layers_u = [lay(L) for L in w.layers_u]
        self.WF, self.bF = _f32(w.W_F, device), _f32(w.b_F, device)
        B, k, d, C = self.B, self.k, self.d, int(self.cand[-1])
        n = sa.n_total
        e = lambda *s, dt=torch.float32: torch.empty(*s, device=device, dtype=dt)
        self.fo = {"S": e(B, k, d), "mass": e(B, k), "H": e(B, k, d),
                   "S_bf16": e(B, k, d, dt=torch.bfloat16), "lse": e(n)}
        self.go = {"dX": e(n, d, dt=torch.bfloat16), "dP": e(k, d), "dW_Q": e(d, d), "dW_K": e(d, d), "dW_V": e(d, d)}
        self.zr, self.zu, self.z = e(C, d), e(C, d), e(C, d)
        sab_ws = lambda nbytes: torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
        self.ws_f = sab_ws(sab.sa_forward_workspace(B, n, k, d, sab.SA_BF16))
        self.ws_b = sab_ws(sab.sa_backward_workspace(B, n, k, d, sab.SA_BF16))
        self.ws_s = sab_ws(sab.stca_forward_workspace(B, C, d, w.heads, w.d_h, sab.SA_BF16))
        self.tokens = n
        self.cands = C
        self.phase_events = None

    def step(self, phases=None):
        sab, w = self.sab, self.w
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if phases is not None else None
        if ev: ev[0].record()
        fwd = sab.sa_forward(self.X, self.off, self.P, self.WQ, self.WK, self.WV, w.sa.eps,
                             offsets_dev=self.offd, out=self.fo, workspace=self.ws_f)
        if ev: ev[1].record()
        g = sab.sa_backward(self.X, self.off, self.P, self.WQ, self.WK, self.WV, w.sa.eps,
                            fwd["H"], fwd["mass"], self.dS, None, fwd["lse"],
                            offsets_dev=self.offd, out=self.go, workspace=self.ws_b)
        if self.world > 1:
            allreduce_weight_grads(g)
        if ev: ev[2].record()
        sab.stca_forward(self.q, self.cand, self.X, self.rb, self.re, self.layers_r, w.heads, w.d_h,
                         cand_offsets_dev=self.candd, kv_begin_dev=self.rbd, kv_end_dev=self.red,
                         out=self.zr, workspace=self.ws_s)
        sk = fwd["S_bf16"].view(self.B * self.k, self.d)
        sab.stca_forward(self.q, self.cand, sk, self.sb, self.se, self.layers_u, w.heads, w.d_h,
                         cand_offsets_dev=self.candd, kv_begin_dev=self.sbd, kv_end_dev=self.sed,
                         out=self.zu, workspace=self.ws_s)
        sab.stca_fuse(self.zr, self.zu, self.WF, self.bF, out=self.z)
        if ev:
            ev[3].record()
            phases.append(ev)
        return self.z, g

    def make_pipelined_e2e(self, groups: int, events: bool = False):
        """The end-to-end step through the public API with host buffers, in user
        groups: group g+1's rows of X, q and dS cross PCIe (a side stream) while
        group g computes; every group's calls are the public ones (the backward
        of groups after the first adds into the weight gradients), and each
        group's result is read back as soon as it is ready.  With ``events`` the
        host ships each event's item id and action type (5 bytes) instead of its
        row, and the rows are built on the device before the group's forward from
        the resident bf16 embedding tables and fusion weights, with the
        action-side SwiGLU fusion of eq. (20) (sa_gather_events_fused).
        Returns (step, h2d bytes, d2h bytes)."""
        from sketch_attention_b200.dist import shard_users
        sab, w, dev = self.sab, self.w, self.dev
        if events:
            hI = torch.from_numpy(w.sa.item_ids).pin_memory()
            hA = torch.from_numpy(w.sa.action_ids).pin_memory()
            dI, dA = torch.empty_like(hI, device=dev), torch.empty_like(hA, device=dev)
            item_t = torch.from_numpy(w.item_table.view(np.int16)).to(dev).view(torch.bfloat16)
            act_t = torch.from_numpy(w.action_table.view(np.int16)).to(dev).view(torch.bfloat16)
            from sa_inputs import event_ffn_weights, rng_for
            fW1, fW3, fW2 = (_f32(a, dev) for a in event_ffn_weights(rng_for(5009), self.d))
            f_ws = torch.empty(sab.sa_gather_events_fused_workspace(act_t.shape[0], self.d, 2 * self.d),
                               dtype=torch.uint8, device=dev)
        else:
            hX = torch.empty(self.X.shape, dtype=torch.bfloat16, pin_memory=True)
            hX.copy_(self.X)
        hq = torch.empty(self.q.shape, dtype=torch.bfloat16, pin_memory=True)
        hq.copy_(self.q)
        hdS = torch.empty(self.dS.shape, dtype=torch.float32, pin_memory=True)
        hdS.copy_(self.dS)
        hz = torch.empty(self.z.shape, dtype=torch.float32, pin_memory=True)
        hg = {n: torch.empty(self.go[n].shape, dtype=torch.float32, pin_memory=True)
              for n in ("dP", "dW_Q", "dW_K", "dW_V")}
        off, cand = self.off, self.cand
        plan = []
        for gi in range(groups):
            u0, u1 = shard_users(self.B, gi, groups)
            if u1 <= u0:
                continue
            lo, hi = int(off[u0]), int(off[u1])
            c0, c1 = int(cand[u0]), int(cand[u1])
            og = (off[u0:u1 + 1] - off[u0]).astype(np.int64)
            cg = (cand[u0:u1 + 1] - cand[u0]).astype(np.int64)
            rb, re = self.rb[u0:u1] - lo, self.re[u0:u1] - lo
            sb = np.arange(u1 - u0, dtype=np.int64) * self.k
            plan.append(dict(u0=u0, u1=u1, lo=lo, hi=hi, c0=c0, c1=c1, off=og, cand=cg, rb=rb, re=re,
                             sb=sb, se=sb + self.k,
                             offd=torch.from_numpy(og).to(dev), candd=torch.from_numpy(cg).to(dev),
                             rbd=torch.from_numpy(rb).to(dev), red=torch.from_numpy(re).to(dev),
                             sbd=torch.from_numpy(sb).to(dev), sed=torch.from_numpy(sb + self.k).to(dev),
                             lse=torch.empty(max(hi - lo, 1), device=dev),
                             ev=torch.cuda.Event()))
        copy_stream = torch.cuda.Stream(device=dev)
        fo, go = self.fo, self.go

        def step():
            main = torch.cuda.current_stream()
            copy_stream.wait_stream(main)          # the previous step's reads of these buffers are done
            with torch.cuda.stream(copy_stream):
                for g in plan:
                    if events:
                        dI[g["lo"]:g["hi"]].copy_(hI[g["lo"]:g["hi"]], non_blocking=True)
                        dA[g["lo"]:g["hi"]].copy_(hA[g["lo"]:g["hi"]], non_blocking=True)
                    else:
                        self.X[g["lo"]:g["hi"]].copy_(hX[g["lo"]:g["hi"]], non_blocking=True)
                    self.q[g["c0"]:g["c1"]].copy_(hq[g["c0"]:g["c1"]], non_blocking=True)
                    self.dS[g["u0"]:g["u1"]].copy_(hdS[g["u0"]:g["u1"]], non_blocking=True)
                    g["ev"].record(copy_stream)
            for i, g in enumerate(plan):
                main.wait_event(g["ev"])
                u0, u1, lo, hi, c0, c1 = g["u0"], g["u1"], g["lo"], g["hi"], g["c0"], g["c1"]
                Xg = self.X[lo:hi]
                if events:
                    sab.sa_gather_events_fused(item_t, act_t, dI[lo:hi], dA[lo:hi], fW1, fW3, fW2, out=Xg,
                                               workspace=f_ws)
                f = sab.sa_forward(Xg, g["off"], self.P, self.WQ, self.WK, self.WV, w.sa.eps,
                                   offsets_dev=g["offd"], workspace=self.ws_f,
                                   out={"S": fo["S"][u0:u1], "mass": fo["mass"][u0:u1],
                                        "H": fo["H"][u0:u1], "S_bf16": fo["S_bf16"][u0:u1],
                                        "lse": g["lse"]})
                sab.sa_backward(Xg, g["off"], self.P, self.WQ, self.WK, self.WV, w.sa.eps, f["H"],
                                f["mass"], self.dS[u0:u1], None, f["lse"], offsets_dev=g["offd"],
                                workspace=self.ws_b, accumulate=i > 0,
                                out={"dX": go["dX"][lo:hi], "dP": go["dP"], "dW_Q": go["dW_Q"],
                                     "dW_K": go["dW_K"], "dW_V": go["dW_V"]})
                qg = self.q[c0:c1]
                sab.stca_forward(qg, g["cand"], Xg, g["rb"], g["re"], self.layers_r, w.heads, w.d_h,
                                 cand_offsets_dev=g["candd"], kv_begin_dev=g["rbd"], kv_end_dev=g["red"],
                                 out=self.zr[c0:c1], workspace=self.ws_s)
                sk = f["S_bf16"].view((u1 - u0) * self.k, self.d)
                sab.stca_forward(qg, g["cand"], sk, g["sb"], g["se"], self.layers_u, w.heads, w.d_h,
                                 cand_offsets_dev=g["candd"], kv_begin_dev=g["sbd"], kv_end_dev=g["sed"],
                                 out=self.zu[c0:c1], workspace=self.ws_s)
                sab.stca_fuse(self.zr[c0:c1], self.zu[c0:c1], self.WF, self.bF, out=self.z[c0:c1])
                hz[c0:c1].copy_(self.z[c0:c1], non_blocking=True)
            if self.world > 1:
                allreduce_weight_grads(go)
            for n in hg:
                hg[n].copy_(go[n], non_blocking=True)

        rows_bytes = (hI.numel() * 4 + hA.numel()) if events else hX.numel() * 2
        h2d = rows_bytes + hq.numel() * 2 + hdS.numel() * 4
        return step, h2d, self.results_nbytes()

    def results_nbytes(self):
        return self.z.numel() * 4 + sum(self.go[n].numel() * 4 for n in ("dP", "dW_Q", "dW_K", "dW_V"))


# Per-kernel algorithmic work (flops) per launch, for the roofline of the
# dominant kernel.  tokens = history tokens of the call.
KERNEL_SOURCES = {
    "sa_lse_tc_kernel": "sa_tc.cu", "sa_agg_tc_kernel": "sa_tc.cu", "sa_bwd_dx_tc_kernel": "sa_bwd_tc.cu",
    "sa_bwd_e_tc_kernel": "sa_bwd_tc.cu", "stca_attn_tc_kernel": "stca_tc.cu",
}


def source_digest(kernel):
    import hashlib
    src = KERNEL_SOURCES.get(kernel)
    if not src:
        return None
    path = os.path.join(ROOT, "sketch_attention_b200", "csrc", src)
    with open(path, "rb") as f:
        text = f.read()
    # the device code only: host-side launch code after the marker does not change a kernel's traffic
    cut = text.find(b"==== host side")
    return hashlib.sha256(text if cut < 0 else text[:cut]).hexdigest()[:16]


def measured_traffic(kernel, units):
    """DRAM bytes of one launch of `kernel` over `units` tokens, scaled from the
    committed ncu record (profiles/dram_traffic.txt: kernel, bytes per token,
    source digest); None when there is no record or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split("#", 1)[0].split()
            if len(parts) >= 3 and parts[0] == kernel:
                if parts[2] != source_digest(kernel):
                    return None
                return float(parts[1]) * units
    return None


def kernel_model(name, w):
    k, d = w.sa.k, w.sa.d
    n = w.sa.n_total
    if name == "sa_lse_tc_kernel":
        # the logits of every token against all k prototypes
        return "tensor", 2.0 * k * d * n
    if name == "sa_agg_tc_kernel":
        # H = A X with its mass (its recomputed logits are not counted)
        return "tensor", 2.0 * k * d * n
    if name == "sa_lse_kernel":
        return "alu", 2.0 * k * d * n
    if name == "sa_agg_kernel":
        return "alu", 2.0 * k * d * n
    if name == "sa_bwd_token_kernel":
        return "alu", 8.0 * k * d * n
    if name == "sa_bwd_E_kernel":
        return "alu", 2.0 * k * d * n
    if name == "sa_bwd_dx_tc_kernel":
        # logits, dH.x and dX = A dH + dZ P' for every token (its V = A P' term and
        # the bf16 residual of dH are extra work of this formulation, not counted)
        return "tensor", 8.0 * k * d * n
    if name == "sa_bwd_e_tc_kernel":
        # E = dZ^T X (its recomputed logits and dH.x are not counted)
        return "tensor", 2.0 * k * d * n
    if name.startswith("stca_attn"):
        # one launch: one layer of one branch; the two branches differ in L
        C = int(w.cand_offsets[-1])
        L_avg = 0.5 * (float(np.mean(w.recent_end - w.recent_begin)) + k)
        return ("tensor" if "tc" in name else "alu"), 4.0 * L_avg * d * C * w.heads
    return None, None


def run_ours(args, rank, world, device):
    import sketch_attention_b200 as sab
    from sketch_attention_b200 import build as _b
    if rank == 0 or not os.path.exists(_b.LIB):
        _b.build()
    if world > 1:
        torch.distributed.barrier()
    sab.load()
    from sa_inputs import TRAIN_STEP_WORKLOAD, train_step_workload
    t0 = time.time()
    w = train_step_workload(users=args.users)
    gen_s = time.time() - t0
    R = TrainStepRunner(w, device, world)
    peaks, peaks_src = load_peaks()

    for _ in range(args.warmup):
        R.step()
    torch.cuda.synchronize()
    phases = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sab.profile(True)
    launches0 = sab.launch_count()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        start.record()
        for _ in range(args.steps):
            R.step(phases)
        end.record()
        torch.cuda.synchronize()
    launches = sab.launch_count() - launches0
    prof = sab.profile_read()
    sab.profile(False)
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end) / args.steps
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms = float(t.item())
    ph = np.array([[a.elapsed_time(b) for a, b in zip(e[:-1], e[1:])] for e in phases])
    ph_ms = ph.mean(axis=0) if len(ph) else np.zeros(3)

    # ---- end to end through the public API with host buffers
    def time_e2e(events):
        e2e_step, h2d, d2h = R.make_pipelined_e2e(E2E_GROUPS, events=events)
        torch.cuda.synchronize()
        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sab.profile(True)
        s2.record()
        for _ in range(args.steps):
            e2e_step()
        e2.record()
        torch.cuda.synchronize()
        eprof = sab.profile_read()
        sab.profile(False)
        e2e_ms = s2.elapsed_time(e2) / args.steps
        t = torch.tensor([e2e_ms], device=device, dtype=torch.float64)
        if world > 1:
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
        # the device time of building the event rows (the separate gather pass), per step
        rows_ms = sum(v[0] for n, v in eprof.items()
                      if n in ("events_ffn_tc_kernel", "action_bias_kernel", "ffn_weights_f16_kernel",
                               "gather_events_kernel")) / args.steps
        return {"value": world * R.tokens / (e2e_ms / 1e3), "unit": "history-tokens/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "user_groups": E2E_GROUPS, "event_rows_kernels_ms_per_step": rows_ms}

    configs = None if args.no_configs else config_records(args, device, peaks, peaks_src)

    e2e = e2e_rows = None
    if not args.no_e2e:
        # the events as the pages define the history, (item id, action type) pairs shipped
        # from the host (5 bytes each); the bf16 embedding tables and the fusion FFN are
        # resident parameters and the rows x = e + FFN([e; a]) (eq. (20)) are built on the
        # device before each group's forward
        e2e = time_e2e(True)
        e2e["inputs"] = ("item ids (int32) + action types (uint8) per event, q, dS; embedding tables and "
                         "the eq. (20) fusion weights resident; rows built by sa_gather_events_fused")
        # the same step shipping each event's 256-byte row instead (no fusion)
        e2e_rows = time_e2e(False)
        e2e_rows["inputs"] = "bf16 event rows, q, dS"

    # ---- roofline of the dominant kernel
    roof = None
    modeled = {n: v for n, v in prof.items() if kernel_model(n, w)[0] is not None}
    if modeled:
        # the dominant kernel among those with an algorithmic-work model
        dom = max(modeled.items(), key=lambda kv: kv[1][0])
        name, (tot_ms, cnt) = dom
        bound, flops = kernel_model(name, w)
        if bound is not None:
            avg_s = tot_ms / cnt / 1e3
            achieved = flops / avg_s / 1e12
            if bound == "tensor":
                # the burst figure: the step is tens of ms and the timed region well under a
                # second, not the seconds-long loop the sustained figure was taken over (the
                # fraction against that one is reported beside it)
                peak = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
                peak_sus = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
                peak_note = f"bf16 dense, burst ({peaks_src})"
            else:
                mhz = peaks.get("sm_max_mhz", 1965.0)
                peak = SMS * FP32_LANES * 2 * mhz * 1e6 / 1e12
                peak_note = f"fp32 FMA: {SMS} SMs x {FP32_LANES} lanes x 2 x {mhz:.0f} MHz"
            roof = {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak,
                    "unit": "TFLOP/s", "frac": achieved / peak,
                    "traffic": measured_traffic(name, w.sa.n_total),
                    "peak_source": peak_note, "avg_launch_ms": tot_ms / cnt,
                    "launches": cnt, "share_of_step": tot_ms / (ms * args.steps)}
            if bound == "tensor":
                roof["frac_of_sustained_peak"] = achieved / peak_sus
                roof["sustained_peak"] = peak_sus
    kernels = {n: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
               for n, v in sorted(prof.items(), key=lambda kv: -kv[1][0])}

    tokens = R.tokens
    value = world * tokens / (ms / 1e3)
    line = {
        "metric": METRIC, "value": value, "unit": "history-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded item+action events (Zipf(1.1) ids over 1M items), lognormal lengths",
        "config": {"workload": TRAIN_STEP_WORKLOAD, "users_per_gpu": R.B,
                   "history_tokens_per_gpu": tokens, "k": R.k, "d": R.d,
                   "stca_candidates_per_gpu": R.cands, "parallelism": f"dp{world}",
                   "l2": "inputs larger than L2 (X is %.2f GB per GPU)" % (R.X.numel() * 2 / 1e9)},
        "phases": {"sa_forward_ms": float(ph_ms[0]), "sa_backward_ms": float(ph_ms[1]),
                   "stca_fuse_ms": float(ph_ms[2]),
                   "sa_forward_tokens_per_s": tokens / (ph_ms[0] / 1e3) if ph_ms[0] else None,
                   "sa_backward_tokens_per_s": tokens / (ph_ms[1] / 1e3) if ph_ms[1] else None,
                   "stca_candidates_per_s": R.cands / (ph_ms[2] / 1e3) if ph_ms[2] else None},
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": int(launches),
        "e2e": e2e,
        "e2e_rows": e2e_rows,
        "configs": configs,
        "clocks": clk.summary(),
        "input_generation_s": gen_s,
    }
    from sketch_attention_b200 import flops as flop_model
    hl = flop_model.headline(100_000)
    line["analytic_context"] = {
        "train_flop_reduction_vs_direct_stca": round(hl["train_ratio"], 2),
        "infer_flop_reduction_vs_direct_stca": round(hl["infer_ratio"], 2),
        "note": "the pages' GEMM-FLOP ratios at 100K events (Sec. 5.4, eqs. 28-34), recomputed by "
                "sketch_attention_b200.flops; analytic context, not a hardware target"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, 30_000)
    return line



# --------------------------------------------------------------------------
# the other workloads of the metric, each timed in the same run as the step
def _time_loop(sab, step, steps, warmup, device, flush=None):
    """Device time per call of `step`.  Without `flush`: `steps` calls back to back
    between two events (inputs larger than L2).  With `flush`: each call between its
    own pair of events and the L2 flushed (a write larger than L2) between calls,
    outside the timed pairs; the median.  Returns (ms, per-kernel profile, clocks)."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    sab.profile(True)
    with ClockSampler(device.index or 0) as clk:
        if flush is None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(steps):
                step()
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / steps
        else:
            pairs = []
            for _ in range(steps):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                step()
                b.record()
                pairs.append((a, b))
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in pairs)
    prof = sab.profile_read()
    sab.profile(False)
    return ms, prof, clk.summary()


def _sa_forward_step(sab, p, device):
    X = _dev_bf16(p.X, device) if p.dtype == "bf16" else _f32(p.X, device)
    offd = torch.from_numpy(p.offsets).to(device)
    P, WQ, WK, WV = (_f32(a, device) for a in (p.P, p.W_Q, p.W_K, p.W_V))
    out = {"S": torch.empty(p.B, p.k, p.d, device=device), "mass": torch.empty(p.B, p.k, device=device),
           "lse": torch.empty(max(p.n_total, 1), device=device)}
    ws = torch.empty(max(sab.sa_forward_workspace(p.B, p.n_total, p.k, p.d,
                                                  sab.SA_BF16 if p.dtype == "bf16" else sab.SA_F32), 1),
                     dtype=torch.uint8, device=device)
    return lambda: sab.sa_forward(X, p.offsets, P, WQ, WK, WV, p.eps, offsets_dev=offd, out=out, workspace=ws)


def config_records(args, device, peaks, peaks_src):
    """SA forward at the configurations the metric names (32 users x 100K events at
    k=1024, the tensor/exponential roofline case; 8 ragged users at k=512; the small
    fp32 case) and STCA at 16 users x 512 candidates, each timed on the device in
    this run with its clocks sampled inside its own region."""
    import sketch_attention_b200 as sab
    from sa_inputs import sa_workload, stca_workload
    pk = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    pk_sus = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)   # 256 MB > L2
    flush = lambda: flush_buf.fill_(1)
    rate_mix, rate_mufu = sab.measure_exp2_rate(1), sab.measure_exp2_rate(0)
    recs = {}

    # -- SA forward, 32 x 100K, k=1024: the two forward kernels against the tensor and
    #    exponential co-rooflines (4kd flop and 2k exponentials per token credited)
    p = sa_workload(3)
    step = _sa_forward_step(sab, p, device)
    ms, prof, clk = _time_loop(sab, step, 200, 5, device)
    kern = {n: v[0] / 200 for n, v in prof.items()}
    fwd_ms = kern.get("sa_lse_tc_kernel", 0.0) + kern.get("sa_agg_tc_kernel", 0.0)
    tf = 4.0 * p.k * p.d * p.n_total / (fwd_ms / 1e3) / 1e12 if fwd_ms else None
    ex = 2.0 * p.k * p.n_total / (fwd_ms / 1e3) if fwd_ms else None
    tf_call = 4.0 * p.k * p.d * p.n_total / (ms / 1e3) / 1e12
    recs["sa_fwd_32x100K_k1024"] = {
        "workload": p.name, "value": p.n_total / (ms / 1e3), "unit": "history-tokens/s",
        "ms_per_call": ms, "forward_kernels_ms": fwd_ms,
        "tensor": {"achieved": tf, "peak": pk, "unit": "TFLOP/s", "frac": tf / pk if tf else None,
                   "frac_of_sustained_peak": tf / pk_sus if tf else None,
                   "achieved_whole_call": tf_call, "frac_whole_call": tf_call / pk,
                   "peak_source": f"bf16 dense, burst ({peaks_src}); 4kd flop per token credited "
                                  "(the logits and H = A X, 2kd each)"},
        "exp": {"achieved": ex, "peak": rate_mix, "unit": "exp2/s", "frac": ex / rate_mix if ex else None,
                "peak_source": "measured on this GPU in this run (sa_measure_exp2_rate, the kernels' "
                               "mix of MUFU ex2 and the FMA-pipe cubic, one pair in eight); 2k exponentials per token "
                               "(k in each of the two kernels)", "mufu_only_rate": rate_mufu},
        "kernels_ms": kern, "clocks": clk, "l2": "inputs larger than L2 (X is 0.82 GB)"}
    del step, p
    torch.cuda.empty_cache()

    # -- SA forward, 8 ragged users (U[20K, 100K]), k=512
    p = sa_workload(2)
    step = _sa_forward_step(sab, p, device)
    ms, prof, clk = _time_loop(sab, step, 100, 5, device, flush)
    tf = 4.0 * p.k * p.d * p.n_total / (ms / 1e3) / 1e12
    recs["sa_fwd_8users_k512"] = {
        "workload": p.name, "value": p.n_total / (ms / 1e3), "unit": "history-tokens/s",
        "ms_per_call": ms, "tensor": {"achieved": tf, "peak": pk, "unit": "TFLOP/s", "frac": tf / pk,
                                      "peak_source": f"bf16 dense, burst ({peaks_src}); whole call"},
        "clocks": clk, "l2": "flushed between calls (256 MB write, outside the timed pairs)"}
    del step, p

    # -- SA forward, fp32, n=4096, d=64, k=64 (launch/latency bound)
    p = sa_workload(1)
    step = _sa_forward_step(sab, p, device)
    ms, prof, clk = _time_loop(sab, step, 100, 5, device, flush)
    mhz = peaks.get("sm_max_mhz", 1965.0)
    fma_peak = SMS * FP32_LANES * 2 * mhz * 1e6 / 1e12
    tf = 4.0 * p.k * p.d * p.n_total / (ms / 1e3) / 1e12
    recs["sa_fwd_fp32_4096_k64"] = {
        "workload": p.name, "value": p.n_total / (ms / 1e3), "unit": "history-tokens/s",
        "ms_per_call": ms, "alu": {"achieved": tf, "peak": fma_peak, "unit": "TFLOP/s", "frac": tf / fma_peak,
                                   "peak_source": f"fp32 FMA: {SMS} SMs x {FP32_LANES} lanes x 2 x {mhz:.0f} MHz"},
        "launches_per_call": sum(v[1] for v in prof.values()) / 100,
        "clocks": clk, "l2": "flushed between calls (256 MB write, outside the timed pairs)"}
    del step, p

    # -- STCA, 16 users x 512 candidates, both branches and the fusion
    w = stca_workload()
    q, kvr, kvs = (_dev_bf16(a, device) for a in (w.recent.q, w.recent.kv, w.sketch.kv))
    lay = lambda L: dict(W_Q=_f32(L.W_Q, device), W_K=_f32(L.W_K, device), W_V=_f32(L.W_V, device),
                         W_O=_f32(L.W_O, device))
    lr, lu = [lay(L) for L in w.layers_r], [lay(L) for L in w.layers_u]
    WF, bF = _f32(w.W_F, device), _f32(w.b_F, device)
    C = int(w.recent.cand_offsets[-1])
    zr, zu, z = (torch.empty(C, 128, device=device) for _ in range(3))
    dv = lambda a: torch.from_numpy(np.asarray(a, np.int64)).to(device)
    cd, rbd, red, sbd, sed = (dv(a) for a in (w.recent.cand_offsets, w.recent.kv_begin, w.recent.kv_end,
                                              w.sketch.kv_begin, w.sketch.kv_end))
    B = len(w.recent.cand_offsets) - 1
    ws = torch.empty(sab.stca_forward_workspace(B, C, 128, w.heads, w.d_h, sab.SA_BF16),
                     dtype=torch.uint8, device=device)

    def stca_step():
        sab.stca_forward(q, w.recent.cand_offsets, kvr, w.recent.kv_begin, w.recent.kv_end, lr, w.heads,
                         w.d_h, cand_offsets_dev=cd, kv_begin_dev=rbd, kv_end_dev=red, out=zr, workspace=ws)
        sab.stca_forward(q, w.sketch.cand_offsets, kvs, w.sketch.kv_begin, w.sketch.kv_end, lu, w.heads,
                         w.d_h, cand_offsets_dev=cd, kv_begin_dev=sbd, kv_end_dev=sed, out=zu, workspace=ws)
        sab.stca_fuse(zr, zu, WF, bF, out=z)
    ms, prof, clk = _time_loop(sab, stca_step, 100, 5, device, flush)
    L_sum = float(np.sum((w.recent.kv_end - w.recent.kv_begin) * np.diff(w.recent.cand_offsets)) +
                  np.sum((w.sketch.kv_end - w.sketch.kv_begin) * np.diff(w.sketch.cand_offsets)))
    attn_flops = 4.0 * L_sum * 128 * w.heads * len(w.layers_r)     # eq. (25)'s length term, both branches
    a_ms = prof.get("stca_attn_tc_kernel", (0.0, 1))[0] / 100
    tf_a = attn_flops / (a_ms / 1e3) / 1e12 if a_ms else None
    tf = attn_flops / (ms / 1e3) / 1e12
    recs["stca_16users_512cand"] = {
        "workload": w.name, "value": C / (ms / 1e3),
        "unit": "candidates/s", "ms_per_call": ms,
        "tensor": {"achieved": tf, "peak": pk, "unit": "TFLOP/s", "frac": tf / pk,
                   "attention_kernel_achieved": tf_a, "attention_kernel_frac": tf_a / pk if tf_a else None,
                   "peak_source": f"bf16 dense, burst ({peaks_src}); 4 L D flop per (candidate, head, "
                                  "layer), both branches"},
        "kernels_ms": {n: v[0] / 100 for n, v in sorted(prof.items(), key=lambda kv: -kv[1][0])},
        "clocks": clk, "l2": "flushed between calls (256 MB write, outside the timed pairs)"}
    del flush_buf
    torch.cuda.empty_cache()
    return recs

# --------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
def _oracle_sample(w, n_tokens=None, users=(0,)):
    """One bounded sample of the step: for each listed user, its forward and
    backward (its first n_tokens events) plus STCA of its 256 candidates on both
    branches and the fusion, all by the fp64 oracle.  Returns (events, seconds)."""
    import oracle
    from sa_inputs import bf16_to_f64
    sa = w.sa
    events, secs = 0, 0.0
    for u in users:
        lo, hi = int(sa.offsets[u]), int(sa.offsets[u + 1])
        if n_tokens is not None:
            hi = min(hi, lo + n_tokens)
        X = sa.x_f64(lo, hi)
        t0 = time.perf_counter()
        S, m, H = oracle.sa_forward(X, [0, hi - lo], sa.P, sa.W_Q, sa.W_K, sa.W_V, sa.eps)
        oracle.sa_backward(X, [0, hi - lo], sa.P, sa.W_Q, sa.W_K, sa.W_V, sa.eps, sa.dS[u:u + 1])
        c0, c1 = int(w.cand_offsets[u]), int(w.cand_offsets[u + 1])
        q = bf16_to_f64(w.q[c0:c1])
        rb = max(lo, hi - 10_000)
        zr = oracle.stca_branch(q, [0, c1 - c0], X, [rb - lo], [hi - lo], w.layers_r, w.heads, w.d_h)
        zu = oracle.stca_branch(q, [0, c1 - c0], S[0], [0], [sa.k], w.layers_u, w.heads, w.d_h)
        oracle.stca_fuse(zr, zu, w.W_F, w.b_F)
        secs += time.perf_counter() - t0
        events += hi - lo
    return events, secs


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, n_tokens=None, n_users=10):
    users = tuple(range(min(n_users, w.sa.B)))
    n, secs = _oracle_sample(w, n_tokens, users)
    return {"value": n / secs, "unit": "history-tokens/s", "cores": _cores(), "kind": "oracle",
            "sample": f"users 0-{users[-1]}, the first {n_tokens} events of each ({n} events): "
                      f"forward+backward, STCA on each user's 256 candidates (both branches), "
                      f"fusion; fp64 numpy, {secs:.1f} s"}


def run_reference(args):
    from sa_inputs import TRAIN_STEP_WORKLOAD, train_step_workload
    w = train_step_workload(users=1)
    for _ in range(args.warmup):
        _oracle_sample(w, 20_000)
    times, n = [], 0
    for _ in range(args.steps):
        n, s = _oracle_sample(w, 20_000)
        times.append(s)
    ms = 1e3 * float(np.mean(times))
    value = n / (ms / 1e3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "history-tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same generator as the GPU arm)",
        "config": {"workload": TRAIN_STEP_WORKLOAD, "sample": "user 0, first 20000 events"},
        "cpu_baseline": {"value": value, "unit": "history-tokens/s", "cores": _cores(),
                         "kind": "oracle",
                         "sample": "per step: user 0's first 20000 events forward+backward, STCA "
                                   "on its 256 candidates (both branches), fusion"},
        "e2e": {"value": value, "unit": "history-tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_component(args, rank, world, device):
    """SA forward alone (32 users x 100K, k=1024) or STCA alone (16 users x 512
    candidates): for profiling the two tensor-core kernels in isolation."""
    import sketch_attention_b200 as sab
    from sketch_attention_b200 import build as _b
    if rank == 0 or not os.path.exists(_b.LIB):
        _b.build()
    sab.load()
    from sa_inputs import STCA_WORKLOAD_4, sa_workload, stca_workload

    def stca_label(w):
        # the STCA workload's name with its actual user count (--users)
        return STCA_WORKLOAD_4.replace("B=16", f"B={len(w.recent.cand_offsets) - 1}")
    peaks, peaks_src = load_peaks()
    extra = []          # (kernel, flops per launch) of other tensor-core kernels to report
    if args.workload == "sa_fwd":
        p = sa_workload(3, users=args.users)
        X = _dev_bf16(p.X, device)
        offd = torch.from_numpy(p.offsets).to(device)
        P, WQ, WK, WV = (_f32(a, device) for a in (p.P, p.W_Q, p.W_K, p.W_V))
        out = {"S": torch.empty(p.B, p.k, p.d, device=device),
               "mass": torch.empty(p.B, p.k, device=device),
               "lse": torch.empty(p.n_total, device=device)}
        ws = torch.empty(sab.sa_forward_workspace(p.B, p.n_total, p.k, p.d, sab.SA_BF16),
                         dtype=torch.uint8, device=device)
        step = lambda: sab.sa_forward(X, p.offsets, P, WQ, WK, WV, p.eps, offsets_dev=offd, out=out,
                                      workspace=ws)
        units, unit, name = p.n_total, "history-tokens/s", p.name
        kname, flops = "sa_agg_tc_kernel", 2.0 * p.k * p.d * p.n_total
        fwd_k = p.k
    elif args.workload == "tokenwise":
        p = sa_workload(5, users=args.users)
        X = _dev_bf16(p.X, device)
        offd = torch.from_numpy(p.offsets).to(device)
        P, WQ, WK, WV = (_f32(a, device) for a in (p.P, p.W_Q, p.W_K, p.W_V))
        out = {"S": torch.empty(p.B, p.k, p.d, device=device),
               "mass": torch.empty(p.B, p.k, device=device)}
        ws = torch.empty(sab.sa_forward_tokenwise_workspace(p.B, p.n_total, p.k, p.d, sab.SA_BF16),
                         dtype=torch.uint8, device=device)
        step = lambda: sab.sa_forward_tokenwise(X, p.offsets, P, WQ, WK, WV, p.eps, offsets_dev=offd,
                                                out=out, workspace=ws)
        units, unit = p.n_total, "history-tokens/s"
        name = (f"token-wise normalisation variant, {p.B} users x mean "
                f"{p.n_total // max(p.B, 1)} events, k={p.k}, d={p.d}, bf16")
        # the attention of the k prototypes over the user's events: S = Q K^T and A V, 4kd per event
        kname, flops = "stca_attn_tc_kernel", 4.0 * p.k * p.d * p.n_total
    elif args.workload == "refine":
        from sa_inputs import refine_layers, rng_for
        p = sa_workload(5, users=args.users)
        X = _dev_bf16(p.X, device)
        offd = torch.from_numpy(p.offsets).to(device)
        P0 = _f32(p.P, device)
        layers = [{k: (_f32(v, device) if v is not None else None) for k, v in L.items()}
                  for L in refine_layers(rng_for(5005), 2, p.d)]
        out = torch.empty(p.B, p.k, p.d, device=device)
        ws = torch.empty(sab.sa_refine_workspace(p.B, p.n_total, p.k, p.d, sab.SA_BF16),
                         dtype=torch.uint8, device=device)
        step = lambda: sab.sa_refine_forward(X, p.offsets, P0, layers, 1e-5, offsets_dev=offd,
                                             out=out, workspace=ws)
        units, unit = p.n_total, "history-tokens/s"
        name = (f"stacked SA refinement, 2 iterations (per-user prototypes in the second), "
                f"{p.B} users x mean {p.n_total // max(p.B, 1)} events, k={p.k}, d={p.d}, bf16")
        # per launch of the dominant kernel: H = A X with its mass (2kd flop per token)
        kname, flops = "sa_agg_tc_kernel", 2.0 * p.k * p.d * p.n_total
    elif args.workload == "refine_bwd":
        from sa_inputs import refine_layers, rng_for
        p = sa_workload(5, users=args.users)
        X = _dev_bf16(p.X, device)
        offd = torch.from_numpy(p.offsets).to(device)
        P0 = _f32(p.P, device)
        n_iter = 2
        layers = [{k: (_f32(v, device) if v is not None else None) for k, v in L.items()}
                  for L in refine_layers(rng_for(5005), n_iter, p.d)]
        gen = torch.Generator(device="cpu").manual_seed(5009)
        dsk = torch.randn(p.B, p.k, p.d, generator=gen).to(device)
        ws = torch.empty(sab.sa_refine_backward_workspace(p.B, p.n_total, p.k, p.d, n_iter, sab.SA_BF16),
                         dtype=torch.uint8, device=device)
        rb_out = {"dX": torch.empty(p.n_total, p.d, device=device), "dP0": torch.empty(p.k, p.d, device=device)}
        step = lambda: sab.sa_refine_backward(X, p.offsets, P0, layers, dsk, 1e-5, offsets_dev=offd,
                                              out=rb_out, workspace=ws)
        units, unit = p.n_total, "history-tokens/s"
        name = (f"backward of the stacked SA refinement (forward recomputed), {n_iter} iterations, "
                f"{p.B} users x mean {p.n_total // max(p.B, 1)} events, k={p.k}, d={p.d}, bf16")
        # the dX kernel's credited 8kd flop per token and iteration, spread over its per-user launches
        kname, refine_dx_flops_step = "sa_bwd_dx_tc_kernel", 8.0 * p.k * p.d * p.n_total * n_iter
        extra_step = [("sa_bwd_e_tc_kernel", 2.0 * p.k * p.d * p.n_total * n_iter),
                      ("sa_agg_tc_kernel", 2.0 * p.k * p.d * p.n_total * n_iter)]
    elif args.workload == "stca_full":
        from sa_inputs import add_stca_ffns, rng_for
        w = stca_workload(users=args.users or 16)
        add_stca_ffns(rng_for(5006), w.layers_r, 128)
        add_stca_ffns(rng_for(5007), w.layers_u, 128)
        q, kvr, kvs = (_dev_bf16(a, device) for a in (w.recent.q, w.recent.kv, w.sketch.kv))
        ffn_keys = ("hist_W1", "hist_W3", "hist_W2", "q_W1", "q_W3", "q_W2")
        lay = lambda L: dict(W_Q=_f32(L.W_Q, device), W_K=_f32(L.W_K, device), W_V=_f32(L.W_V, device),
                             W_O=_f32(L.W_O, device), **{k: _f32(getattr(L, k), device) for k in ffn_keys})
        lr, lu = [lay(L) for L in w.layers_r], [lay(L) for L in w.layers_u]
        WF, bF = _f32(w.W_F, device), _f32(w.b_F, device)
        C = int(w.recent.cand_offsets[-1])
        zr, zu, z = (torch.empty(C, 128, device=device) for _ in range(3))
        rows_r = int((w.recent.kv_end - w.recent.kv_begin).sum())
        rows_s = int((w.sketch.kv_end - w.sketch.kv_begin).sum())
        B = len(w.recent.cand_offsets) - 1
        ws_r = torch.empty(sab.stca_forward_full_workspace(B, C, rows_r, 128, w.heads, w.d_h, sab.SA_BF16),
                           dtype=torch.uint8, device=device)
        ws_s = torch.empty(sab.stca_forward_full_workspace(B, C, rows_s, 128, w.heads, w.d_h, sab.SA_BF16),
                           dtype=torch.uint8, device=device)
        dv = lambda a: torch.from_numpy(np.asarray(a, np.int64)).to(device)
        cd, rbd, red, sbd, sed = (dv(a) for a in (w.recent.cand_offsets, w.recent.kv_begin, w.recent.kv_end,
                                                  w.sketch.kv_begin, w.sketch.kv_end))

        def step():
            sab.stca_forward_full(q, w.recent.cand_offsets, kvr, w.recent.kv_begin, w.recent.kv_end,
                                  lr, w.heads, w.d_h, cand_offsets_dev=cd, kv_begin_dev=rbd,
                                  kv_end_dev=red, out=zr, workspace=ws_r)
            sab.stca_forward_full(q, w.sketch.cand_offsets, kvs, w.sketch.kv_begin, w.sketch.kv_end,
                                  lu, w.heads, w.d_h, cand_offsets_dev=cd, kv_begin_dev=sbd,
                                  kv_end_dev=sed, out=zu, workspace=ws_s)
            sab.stca_fuse(zr, zu, WF, bF, out=z)
        units, unit = C, "candidates/s"
        name = ("full STCA layers (history-side SwiGLU FFN before and query-side after each attention), "
                + stca_label(w))
        L_avg = 0.5 * (float(np.mean(w.recent.kv_end - w.recent.kv_begin)) + 1024)
        kname, flops = "stca_attn_tc_kernel", 4.0 * L_avg * 128 * C * w.heads
        # the history FFN: 12 D^2 flop per key row (eq. (27) with inner width 2D), once per row;
        # per launch the mean of the two branches' row counts
        extra.append(("stca_hist_ffn_tc_kernel", 12.0 * 128 * 128 * 0.5 * (rows_r + rows_s)))
    elif args.workload == "stca_bwd":
        from sa_inputs import add_stca_ffns, rng_for
        w = stca_workload(users=args.users or 16)
        add_stca_ffns(rng_for(5006), w.layers_r, 128)
        add_stca_ffns(rng_for(5007), w.layers_u, 128)
        q, kvr, kvs = (_dev_bf16(a, device) for a in (w.recent.q, w.recent.kv, w.sketch.kv))
        wkeys = ("W_Q", "W_K", "W_V", "W_O", "hist_W1", "hist_W3", "hist_W2", "q_W1", "q_W3", "q_W2")
        lay = lambda L: {k: _f32(getattr(L, k), device) for k in wkeys}
        lr, lu = [lay(L) for L in w.layers_r], [lay(L) for L in w.layers_u]
        C = int(w.recent.cand_offsets[-1])
        gen = torch.Generator(device="cpu").manual_seed(5008)
        dzr, dzu = (torch.randn(C, 128, generator=gen).to(device) for _ in range(2))
        dv = lambda a: torch.from_numpy(np.asarray(a, np.int64)).to(device)
        cd, rbd, red, sbd, sed = (dv(a) for a in (w.recent.cand_offsets, w.recent.kv_begin, w.recent.kv_end,
                                                  w.sketch.kv_begin, w.sketch.kv_end))
        nlay = len(lr)
        ws_r = torch.empty(sab.stca_backward_full_workspace(w.recent.cand_offsets, w.recent.kv_begin,
                                                            w.recent.kv_end, 128, w.heads, w.d_h, nlay, sab.SA_BF16),
                           dtype=torch.uint8, device=device)
        ws_s = torch.empty(sab.stca_backward_full_workspace(w.sketch.cand_offsets, w.sketch.kv_begin,
                                                            w.sketch.kv_end, 128, w.heads, w.d_h, nlay, sab.SA_BF16),
                           dtype=torch.uint8, device=device)
        gr = sab.stca_backward_full(q, w.recent.cand_offsets, kvr, w.recent.kv_begin, w.recent.kv_end, lr, w.heads,
                                    w.d_h, dzr, cand_offsets_dev=cd, kv_begin_dev=rbd, kv_end_dev=red, workspace=ws_r)
        gs = sab.stca_backward_full(q, w.sketch.cand_offsets, kvs, w.sketch.kv_begin, w.sketch.kv_end, lu, w.heads,
                                    w.d_h, dzu, cand_offsets_dev=cd, kv_begin_dev=sbd, kv_end_dev=sed, workspace=ws_s)

        def step():
            sab.stca_backward_full(q, w.recent.cand_offsets, kvr, w.recent.kv_begin, w.recent.kv_end, lr, w.heads,
                                   w.d_h, dzr, cand_offsets_dev=cd, kv_begin_dev=rbd, kv_end_dev=red, out=gr,
                                   workspace=ws_r)
            sab.stca_backward_full(q, w.sketch.cand_offsets, kvs, w.sketch.kv_begin, w.sketch.kv_end, lu, w.heads,
                                   w.d_h, dzu, cand_offsets_dev=cd, kv_begin_dev=sbd, kv_end_dev=sed, out=gs,
                                   workspace=ws_s)
        units, unit = C, "candidates/s"
        name = ("backward of full STCA layers (both FFNs, both branches), " + stca_label(w))
        # the per-user attention GEMMs: S and Y in the recompute, S, dP, dU and the two dX
        # products in the backward, 14 R_u L_u D flop per user and layer (tensor cores, each
        # fp32 operand split into hi + lo bf16 parts: three MMA passes per algorithmic flop)
        rows_x_keys = sum(float(w.recent.cand_offsets[u + 1] - w.recent.cand_offsets[u]) * w.heads *
                          float(w.recent.kv_end[u] - w.recent.kv_begin[u]) +
                          float(w.sketch.cand_offsets[u + 1] - w.sketch.cand_offsets[u]) * w.heads *
                          float(w.sketch.kv_end[u] - w.sketch.kv_begin[u])
                          for u in range(len(w.recent.cand_offsets) - 1))
        kname, attn_flops_step = "tc_gemm:stca_bwd_attn", 14.0 * rows_x_keys * 128 * nlay
        # the FFN products (history FFN on every key row, query FFN on every candidate row, both
        # branches): 12 D^2 flop per row in the recompute and 32 D^2 in the backward, per layer
        ffn_rows = (float(np.sum(w.recent.kv_end - w.recent.kv_begin)) +
                    float(np.sum(w.sketch.kv_end - w.sketch.kv_begin)) + 2.0 * C)
        ffn_flops_step = 44.0 * 128 * 128 * ffn_rows * nlay
    else:
        w = stca_workload(users=args.users or 16)
        q, kvr, kvs = (_dev_bf16(a, device) for a in (w.recent.q, w.recent.kv, w.sketch.kv))
        lay = lambda L: dict(W_Q=_f32(L.W_Q, device), W_K=_f32(L.W_K, device),
                             W_V=_f32(L.W_V, device), W_O=_f32(L.W_O, device))
        lr, lu = [lay(L) for L in w.layers_r], [lay(L) for L in w.layers_u]
        WF, bF = _f32(w.W_F, device), _f32(w.b_F, device)
        C = int(w.recent.cand_offsets[-1])
        zr, zu, z = (torch.empty(C, 128, device=device) for _ in range(3))

        def step():
            sab.stca_forward(q, w.recent.cand_offsets, kvr, w.recent.kv_begin, w.recent.kv_end,
                             lr, w.heads, w.d_h, out=zr)
            sab.stca_forward(q, w.sketch.cand_offsets, kvs, w.sketch.kv_begin, w.sketch.kv_end,
                             lu, w.heads, w.d_h, out=zu)
            sab.stca_fuse(zr, zu, WF, bF, out=z)
        units, unit, name = C, "candidates/s", stca_label(w)
        L_avg = 0.5 * (float(np.mean(w.recent.kv_end - w.recent.kv_begin)) + 1024)
        kname, flops = "stca_attn_tc_kernel", 4.0 * L_avg * 128 * C * w.heads
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sab.profile(True)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index or 0) as clk:
        start.record()
        for _ in range(args.steps):
            step()
        end.record()
        torch.cuda.synchronize()
    prof = sab.profile_read()
    sab.profile(False)
    ms = start.elapsed_time(end) / args.steps
    if args.workload == "refine_bwd":
        # per-user launches: flops per launch = the step's credited total over its launches
        per_launch = lambda kn, fl: fl / max(prof.get(kn, (0, 1))[1] / args.steps, 1)
        flops = per_launch(kname, refine_dx_flops_step)
        extra.extend((kn, per_launch(kn, fl)) for kn, fl in extra_step)
    if args.workload == "stca_bwd":
        # flops per launch of the dominant (tensor-core GEMM) call site: the step's total over its launches
        flops = attn_flops_step / max(prof.get(kname, (0, 1))[1] / args.steps, 1)
        extra.append(("tc_gemm:stca_bwd_ffn",
                      ffn_flops_step / max(prof.get("tc_gemm:stca_bwd_ffn", (0, 1))[1] / args.steps, 1)))

    def roof_of(kn, fl):
        if kn not in prof:
            return None
        tot, cnt = prof[kn]
        ach = fl / (tot / cnt / 1e3) / 1e12
        if args.workload == "stca_bwd":
            pk = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
            return {"kernel": kn, "bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s",
                    "frac": ach / pk, "traffic": None,
                    "peak_source": f"bf16 dense, sustained ({peaks_src}): timed inside a long step; "
                                   "algorithmic flops, while the hi/lo operand split issues three MMA "
                                   "passes for each, so this scheme tops out at a third of the peak",
                    "avg_launch_ms": tot / cnt}
        pk = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
        return {"kernel": kn, "bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s",
                "frac": ach / pk, "traffic": None,
                "peak_source": f"bf16 dense, burst ({peaks_src}): the kernel is timed alone",
                "avg_launch_ms": tot / cnt}
    roof = roof_of(kname, flops)
    extra_roofs = {kn: roof_of(kn, fl) for kn, fl in extra}
    line = {"metric": unit, "value": world * units / (ms / 1e3), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16x3" if args.workload == "stca_bwd" else "bf16",
            "data": "synthetic", "config": {"workload": name},
            "roofline": roof,
            "kernels": {n: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
                        for n, v in sorted(prof.items(), key=lambda kv: -kv[1][0])},
            "clocks": clk.summary()}
    if extra_roofs:
        line["other_rooflines"] = extra_roofs
    if args.workload == "sa_fwd" and "sa_lse_tc_kernel" in prof and "sa_agg_tc_kernel" in prof:
        # the forward as a whole (its two kernels): 4kd flop and 2k exponentials per token
        # credited, against the burst bf16 peak and the measured exponential rate of the
        # kernels' MUFU / FMA mix
        fwd_s = (prof["sa_lse_tc_kernel"][0] + prof["sa_agg_tc_kernel"][0]) / args.steps / 1e3
        rate_mix, rate_mufu = sab.measure_exp2_rate(1), sab.measure_exp2_rate(0)
        pk = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
        tf = 4.0 * fwd_k * 128 * units / fwd_s / 1e12
        ex = 2.0 * fwd_k * units / fwd_s
        line["forward_rooflines"] = {
            "kernels_ms": fwd_s * 1e3,
            "tensor": {"achieved": tf, "peak": pk, "unit": "TFLOP/s", "frac": tf / pk,
                       "peak_source": f"bf16 dense, burst ({peaks_src})"},
            "exp": {"achieved": ex, "peak": rate_mix, "unit": "exp2/s", "frac": ex / rate_mix,
                    "peak_source": "measured on this GPU in this run (sa_measure_exp2_rate, the kernels' "
                                   "mix: 7/8 MUFU ex2, 1/8 FMA cubic)", "mufu_only_rate": rate_mufu}}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration records (SA forward at 32 x 100K, 8 users and the "
                         "small fp32 case; STCA at 16 users x 512 candidates)")
    ap.add_argument("--workload", choices=["train", "sa_fwd", "stca", "stca_full", "stca_bwd", "refine", "refine_bwd",
                                           "tokenwise"],
                    default="train",
                    help="train: the full step (default, the headline); sa_fwd: SA forward over "
                         "32 users x 100K (k=1024); stca: STCA of 16 users x 512 candidates; "
                         "stca_full: the same with full layers (history- and query-side FFNs); "
                         "stca_bwd: the backward of those full layers; "
                         "refine: stacked SA refinement, 2 iterations, on the train step's users; "
                         "tokenwise: the token-wise normalisation variant on the train step's users")
    ap.add_argument("--users", type=int, default=None, help="shrink the batch (profiling)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=device)
    try:
        if args.workload == "train":
            line = run_ours(args, rank, world, device)
        else:
            line = run_component(args, rank, world, device)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Throughput of the TTT-KV fast-weight layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step = one call of the layer over the whole synthetic sequence (state
re-initialised from W0, then the chunk loop: read, key pass, gradients,
update, row normalisation).  Default workload: the 32K-token causal LaCT
language layer (B=2, H=4, d=128, dh=256, chunk 2048, GD).  With N > 1 (one
process per GPU under torchrun) every rank runs its own replica on
rank-seeded inputs: weak scaling, no data-path collective; the step time is
the max over ranks.

The line also carries `secondary` (the 32K-token linear layer, HBM-bound,
with its own roofline) and `extra` (the view-synthesis LaCT shapes: one
196K-token chunk with GD, and ~1M tokens in 64K chunks with Muon), timed
over a few host-launched steps each.

`--impl reference` times the CPU oracle (float64 numpy) on the host cores, a
bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TTT layer tokens/s at N=32K; achieved TFLOP/s vs B200 BF16 tensor peak"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def traffic_table():
    p = os.path.join(ROOT, "profiles", "traffic.json")
    return json.load(open(p)) if os.path.exists(p) else {}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid, self.proc, self.path = uuid, None, None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            if self.uuid and self.uuid not in f[1]:
                continue
            rows.append(f)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------- workloads
class LaCTBench:
    def __init__(self, name, device, seed):
        import torch
        import learned_linear_attention_b200 as T
        from ttt_synth import WORKLOADS, make_workload
        self.T, self.torch = T, torch
        self.name, self.w = name, dict(WORKLOADS[name])
        w = self.w
        self.x = make_workload(name, seed=seed)
        x = self.x
        self.B, self.H, self.N, self.d, self.dh = w["B"], w["H"], w["N"], w["d"], w["dh"]
        self.Nq = x.q.values.shape[2]
        self.causal = w["order"] == "causal"
        self.opt = w.get("opt", "gd")
        self.update_mask = w.get("update_mask", 7)
        self.normalize_rows = w.get("normalize_rows", True)
        self.window = w.get("window", 0)   # > 0: the full layer, memory + window attention
        self.desc = T.make_lact_desc(self.B, self.H, self.N, self.d, self.dh, w["chunk"],
                                     N_q=self.Nq, order=w["order"], opt=self.opt,
                                     beta=w.get("beta", 0.9), ns_steps=w.get("ns_steps", 5),
                                     out_dtype="bf16", update_mask=self.update_mask,
                                     normalize_rows=self.normalize_rows)
        tok = lambda tt: torch.from_numpy(tt.bits.view("int16")).view(torch.bfloat16)  # noqa
        self.h_q, self.h_k, self.h_v = tok(x.q), tok(x.k), tok(x.v)
        self.h_lr = torch.from_numpy(x.lr)
        self.q, self.k, self.v = (t.to(device) for t in (self.h_q, self.h_k, self.h_v))
        self.lr = self.h_lr.to(device)
        self.W = [torch.from_numpy(a).to(device) for a in (x.W1, x.W3, x.W2)]
        self.state = T.alloc_lact_state(self.desc, device)
        self.ws = T.alloc_workspace(T.lact_workspace_bytes(self.desc), device)
        self.out = torch.empty(self.B, self.H, self.Nq, self.d, dtype=torch.bfloat16,
                               device=device)
        self.device = device

    # units
    def tokens_per_step(self):
        return self.B * (self.N if self.causal else self.N + self.Nq)

    def flops_per_step(self):
        BH, d, dh = self.B * self.H, self.d, self.dh
        if self.update_mask == 4:   # W2 only: phi(k) 4 d dh, its gradient 2, phi(q) 4, read 2
            return 6 * d * dh * self.N * BH + 6 * d * dh * self.Nq * BH
        f = 12 * d * dh * self.N * BH + 6 * d * dh * self.Nq * BH
        if self.opt == "muon":
            r, c = min(d, dh), max(d, dh)
            nch = -(-self.N // self.w["chunk"])
            f += nch * self.w.get("ns_steps", 5) * 3 * BH * (4 * r * r * c + 2 * r ** 3)
        return f + self.window_flops()

    def window_flops(self):
        # q.k and p v for every (query, key) pair inside the causal window
        if not self.window:
            return 0
        W, N = self.window, self.N
        pairs = N * W - W * (W - 1) // 2 if N >= W else N * (N + 1) // 2
        return 4 * self.d * pairs * self.B * self.H

    def kernel_flops_per_step(self):
        """Algorithmic FLOPs per step of each kernel kind (per token-head:
        key forward 4 d dh, dG 2 d dh, three gradient products 6 d dh, query
        forward 4 d dh, read 2 d dh)."""
        BH, d, dh, N, Nq = self.B * self.H, self.d, self.dh, self.N, self.Nq
        kp = (6 * N + 4 * Nq) * d * dh * BH
        kg = (12 * N + (4 * Nq if self.causal else 0)) * d * dh * BH
        read = 2 * d * dh * Nq * BH
        return {"lact_keypass": kp, "gemm_grad": 6 * d * dh * N * BH,
                "gemm_read": read, "lact_keygrad": kg,
                # the causal chunk loop in one launch: key/gradient work and read
                "lact_loop": kg + (read if self.causal else 0),
                "window_attention": self.window_flops()}

    def resident_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.q, self.k, self.v, self.lr,
                                                          self.out))

    def step(self, stream):
        T = self.T
        T.lact_state_init(self.desc, *self.W, 0, self.state, stream)
        if self.window:
            T.lact_layer_fwd(self.desc, self.window, 0.0, self.q, self.k, self.v, self.lr,
                             self.state, self.out, self.ws, stream=stream)
        else:
            T.lact_chunk_fwd(self.desc, self.q, self.k, self.v, self.lr, self.state, self.out,
                             self.ws, stream=stream)

    def setup_e2e(self, step_fn=None):
        self.e2e_step = step_fn or self.step
        torch = self.torch
        self.p_q, self.p_k, self.p_v = (t.pin_memory() for t in (self.h_q, self.h_k, self.h_v))
        self.p_lr = self.h_lr.pin_memory()
        self.p_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in (self.p_q, self.p_k, self.p_v,
                                                               self.p_lr))
        self.d2h = self.p_out.numel() * self.p_out.element_size()

    def step_e2e(self, stream):
        self.q.copy_(self.p_q, non_blocking=True)
        self.k.copy_(self.p_k, non_blocking=True)
        self.v.copy_(self.p_v, non_blocking=True)
        self.lr.copy_(self.p_lr, non_blocking=True)
        self.e2e_step(stream)
        self.p_out.copy_(self.out, non_blocking=True)

    def config(self):
        w = self.w
        cfg = {"workload": self.name, "B": self.B, "H": self.H, "N_in": self.N,
               "N_q": self.Nq, "d": self.d, "dh": self.dh, "chunk": w["chunk"],
               "order": w["order"], "optimizer": self.opt, "out_dtype": "bf16",
               "state_dtype": "f32"}
        if self.update_mask != 7 or not self.normalize_rows:
            cfg["update_mask"] = self.update_mask
            cfg["normalize_rows"] = self.normalize_rows
        if self.window:
            cfg["window"] = self.window
            cfg["layer"] = "memory + causal sliding-window attention, summed"
        return cfg

    def oracle_sample(self, n_chunks):
        """Oracle on one (b,h) stream and the first n_chunks chunks."""
        import numpy as np
        from oracle import lact_forward
        from oracle.lact import lact_init_state
        x, C = self.x, self.w["chunk"]
        n = min(self.N, n_chunks * C)
        sl = lambda a: a[:1, :1, :n]  # noqa: E731
        q = sl(x.q.values) if self.causal else x.q.values[:1, :1]
        st = lact_init_state(x.W1[:1], x.W3[:1], x.W2[:1], 1, self.opt)
        t0 = time.perf_counter()
        lact_forward(q, sl(x.k.values), sl(x.v.values), sl(x.lr), st, chunk=C,
                     order=self.w["order"], opt=self.opt, update_mask=self.update_mask,
                     normalize_rows=self.normalize_rows)
        if self.window:
            from oracle import sliding_window_attention
            sliding_window_attention(q, sl(x.k.values), sl(x.v.values), self.window)
        dt = time.perf_counter() - t0
        # tokens of the metric: every token counts once across all H heads
        toks = (n if self.causal else n + (self.Nq if n >= self.N else 0)) / self.H
        return toks, dt, f"1 of {self.B*self.H} (b,h) streams, first {n} input tokens" + \
            ("" if self.causal or n < self.N else f" + {self.Nq} queries")


class LinearBench:
    def __init__(self, name, device, seed):
        import torch
        import learned_linear_attention_b200 as T
        from ttt_synth import WORKLOADS, make_workload
        self.T, self.torch, self.name, self.w = T, torch, name, dict(WORKLOADS[name])
        w = self.w
        self.x = make_workload(name, seed=seed)
        x = self.x
        self.B, self.H, self.N, self.dk, self.dv = w["B"], w["H"], w["N"], w["dk"], w["dv"]
        self.bf16 = w["dtype"] == "bf16"
        self.desc = T.make_linear_desc(self.B, self.H, self.N, self.dk, self.dv, w["chunk"],
                                       in_dtype=w["dtype"], out_dtype="bf16")
        if self.bf16:
            tok = lambda tt: torch.from_numpy(tt.bits.view("int16")).view(torch.bfloat16)  # noqa
        else:
            tok = lambda tt: torch.from_numpy(tt.values)  # noqa
        self.h_q, self.h_k, self.h_v = tok(x.q), tok(x.k), tok(x.v)
        self.h_lr = torch.from_numpy(x.lr)
        self.q, self.k, self.v = (t.to(device) for t in (self.h_q, self.h_k, self.h_v))
        self.lr = self.h_lr.to(device)
        self.S = torch.zeros(self.B, self.H, self.dk, self.dv, device=device)
        self.out = torch.empty(self.B, self.H, self.N, self.dv, dtype=torch.bfloat16,
                               device=device)
        self.ws = T.alloc_workspace(T.ttt_linear_workspace_bytes(self.desc), device)

    def tokens_per_step(self):
        return self.B * self.N

    def flops_per_step(self):
        # dense-tile chunked form with 128-token tiles: QK^T, PV, QS, K^T V
        BH, N, d, Tt = self.B * self.H, self.N, self.dk, 128
        return BH * N * (2 * Tt * d + 2 * Tt * d + 2 * d * d + 2 * d * d)

    def bytes_per_step(self):
        BH, N = self.B * self.H, self.N
        el = 2 if self.bf16 else 4
        return BH * N * (2 * self.dk * el + self.dv * el + 4 + self.dv * 2) + \
            2 * BH * self.dk * self.dv * 4

    def step(self, stream):
        T = self.T
        T.ttt_linear_state_init(self.desc, None, self.S, stream)
        T.ttt_linear_fwd(self.desc, self.q, self.k, self.v, self.lr, self.S, self.out, self.ws,
                         stream=stream)

    def setup_e2e(self, step_fn=None):
        self.e2e_step = step_fn or self.step
        torch = self.torch
        self.p_q, self.p_k, self.p_v = (t.pin_memory() for t in (self.h_q, self.h_k, self.h_v))
        self.p_lr = self.h_lr.pin_memory()
        self.p_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in (self.p_q, self.p_k, self.p_v,
                                                               self.p_lr))
        self.d2h = self.p_out.numel() * self.p_out.element_size()

    def step_e2e(self, stream):
        self.q.copy_(self.p_q, non_blocking=True)
        self.k.copy_(self.p_k, non_blocking=True)
        self.v.copy_(self.p_v, non_blocking=True)
        self.lr.copy_(self.p_lr, non_blocking=True)
        self.e2e_step(stream)
        self.p_out.copy_(self.out, non_blocking=True)

    def resident_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.q, self.k, self.v, self.lr,
                                                          self.out))

    def config(self):
        return {"workload": self.name, "B": self.B, "H": self.H, "N": self.N, "dk": self.dk,
                "dv": self.dv, "chunk": self.w["chunk"], "in_dtype": self.w["dtype"],
                "out_dtype": "bf16", "state_dtype": "f32"}


class LinearBwdBench(LinearBench):
    """Backward pass of the linear layer: gradients of q, k, v, lr and S0
    from seeded upstream gradients dout and dS_end; float32 gradients."""

    def __init__(self, name, device, seed):
        super().__init__(name, device, seed)
        torch, T = self.torch, self.T
        from ttt_synth import make_linear_grads
        g = make_linear_grads(self.x, cfg=self.w["cfg"], seed=seed)
        if self.bf16:
            self.dout = torch.from_numpy(g.dout.bits.view("int16")).view(torch.bfloat16).to(device)
        else:
            self.dout = torch.from_numpy(g.dout.values).to(device)
        self.dS_end = torch.from_numpy(g.dS_end).to(device)
        B, H, N, dk, dv = self.B, self.H, self.N, self.dk, self.dv
        self.grads = [torch.empty(s, device=device) for s in
                      ((B, H, N, dk), (B, H, N, dk), (B, H, N, dv), (B, H, N), (B, H, dk, dv))]
        self.out = self.grads[0]   # dq: the result read back in the end-to-end timing
        self.h_dout = self.dout.cpu()
        self.ws = T.alloc_workspace(T.ttt_linear_bwd_workspace_bytes(self.desc), device)

    def setup_e2e(self, step_fn=None):
        super().setup_e2e(step_fn)
        self.p_dout = self.h_dout.pin_memory()
        self.h2d += self.p_dout.numel() * self.p_dout.element_size()

    def step_e2e(self, stream):
        self.dout.copy_(self.p_dout, non_blocking=True)
        super().step_e2e(stream)

    def flops_per_step(self):
        return 4 * super().flops_per_step()

    def bytes_per_step(self):
        # read q, k, v, dout, lr; write dq, dk, dv, dlr (float32) and dS0
        BH, N, dk, dv = self.B * self.H, self.N, self.dk, self.dv
        el = 2 if self.bf16 else 4
        return BH * N * ((2 * dk + 2 * dv) * el + 4 + (2 * dk + dv) * 4 + 4) + \
            2 * BH * dk * dv * 4

    def step(self, stream):
        self.T.ttt_linear_bwd(self.desc, self.q, self.k, self.v, self.lr, None, self.dout,
                              self.dS_end, *self.grads, self.ws, stream=stream)

    def resident_bytes(self):
        return sum(t.numel() * t.element_size() for t in
                   [self.q, self.k, self.v, self.lr, self.dout] + self.grads)

    def config(self):
        c = super().config()
        c["pass"] = "backward"
        c["out_dtype"] = "f32"
        return c


class LaCTBwdBench(LaCTBench):
    """Backward pass of the LaCT layer (lact_chunk_bwd): gradients of q, k,
    v, lr and the start weights from seeded upstream gradients dout and
    dW_end.  Algorithmic work per token-head: 30 d dh for the chunk
    gradient's vector-Jacobian product and 16 d dh for the read's (the
    forward replay that keeps each chunk's start weights is not counted)."""

    def __init__(self, name, device, seed):
        super().__init__(name, device, seed)
        torch, T = self.torch, self.T
        from ttt_synth import make_lact_grads
        g = make_lact_grads(self.x, cfg=self.w["cfg"], seed=seed)
        B, H, N, d, dh = self.B, self.H, self.N, self.d, self.dh
        self.dout = torch.from_numpy(g.dout.bits.view("int16")).view(torch.bfloat16).to(device)
        self.dW_end = torch.from_numpy(
            __import__("numpy").concatenate([w.ravel() for w in g.dW_end])).to(device)
        self.state0 = T.alloc_lact_state(self.desc, device)
        T.lact_state_init(self.desc, *self.W, 0, self.state0)
        self.grads = [torch.empty(B, H, N, d, device=device), torch.empty(B, H, N, d, device=device),
                      torch.empty(B, H, N, d, device=device), torch.empty(B, H, N, device=device),
                      torch.empty(3 * B * H * d * dh, device=device)]
        self.ws = T.alloc_workspace(T.lact_bwd_workspace_bytes(self.desc), device)
        self.h_dout = self.dout.cpu()
        self.out = self.grads[0]   # dq: the result read back in the end-to-end timing

    def setup_e2e(self, step_fn=None):
        super().setup_e2e(step_fn)
        self.p_dout = self.h_dout.pin_memory()
        self.h2d += self.p_dout.numel() * self.p_dout.element_size()

    def step_e2e(self, stream):
        self.dout.copy_(self.p_dout, non_blocking=True)
        super().step_e2e(stream)

    def flops_per_step(self):
        return 46 * self.d * self.dh * self.N * self.B * self.H

    def kernel_flops_per_step(self):
        """Per token-head, causal order: the fused forward products of the
        key step ([h1|h3], [r1|r3], [vw2|vr2]: 12 d dh) and of the read step
        ([hq1|hq3], dgq: 6 d dh); the grouped chunk products (dk 8 d dh, d_dy
        4, dq 4, the three weight gradients 12).  The forward replay's
        key/gradient work: 12 d dh per key token."""
        BH, d, dh, N, Nq = self.B * self.H, self.d, self.dh, self.N, self.Nq
        # the forward replay: per-chunk key/gradient kernels, or the chunk
        # loop without queries (12 d dh per key token either way)
        f = {"lact_keygrad": 12 * d * dh * N * BH, "lact_loop": 12 * d * dh * N * BH}
        if self.causal:
            f.update({"lact_bwd_fwd": 18 * d * dh * N * BH, "lact_bwd_gemm": 28 * d * dh * N * BH})
        else:
            f.update({"lact_bwd_fwd": (12 * N + 6 * Nq) * d * dh * BH,
                      "lact_bwd_gemm": 18 * d * dh * N * BH})
        return f

    def step(self, stream):
        self.T.lact_chunk_bwd(self.desc, self.q, self.k, self.v, self.lr, self.state0, self.dout,
                              self.dW_end, *self.grads, self.ws, stream=stream)

    def resident_bytes(self):
        return sum(t.numel() * t.element_size() for t in
                   [self.q, self.k, self.v, self.lr, self.dout] + self.grads)

    def config(self):
        c = super().config()
        c["pass"] = "backward"
        return c


def capture_graph(bench, stream):
    """Capture one step (state init + layer call) in a CUDA graph; replaying
    it removes host launch overhead from the timed region."""
    import torch
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        bench.step(torch.cuda.current_stream())
    torch.cuda.synchronize()
    return g


def make_bench(name, device, seed):
    from ttt_synth import WORKLOADS
    w = WORKLOADS[name]
    if w["kind"] == "linear":
        return (LinearBwdBench if w.get("backward") else LinearBench)(name, device, seed)
    return (LaCTBwdBench if w.get("backward") else LaCTBench)(name, device, seed)


# --------------------------------------------------------------------------- timing
def max_over_ranks(ms, dist):
    """The job's time: the slowest rank's (NCCL on the GPU, gloo on the host)."""
    if dist is None:
        return ms
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, units_per_step_per_rank, step_ms):
    """Whole-job throughput under weak scaling: every rank processes its own
    replica, and the step takes the slowest rank's time."""
    return world * units_per_step_per_rank / (step_ms * 1e-3)


def timed(bench, steps, stream, fn=None, dist=None):
    import torch
    fn = fn or bench.step
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), dist)


def profile_kernels(bench, steps, stream):
    import torch
    T = bench.T
    torch.cuda.synchronize()
    T.ttt_profile_begin()
    for _ in range(steps):
        bench.step(stream)
    torch.cuda.synchronize()
    return T.ttt_profile_end()


def roofline_for(bench, prof, steps, pk, pk_kind):
    """Roofline of the dominant kernel: for the LaCT layer the kernel doing the
    most algorithmic work (the fused key/gradient kernel, on the critical
    path; the read runs beside it on a helper stream), for the linear layer
    the kernel taking the most time."""
    total = sum(v["total_ms"] for v in prof.values())
    name, rec = max(prof.items(), key=lambda kv: kv[1]["total_ms"])
    if not isinstance(bench, LinearBench):
        kfs = bench.kernel_flops_per_step()
        cands = [k for k in prof if k in kfs]
        if cands:
            name = max(cands, key=lambda k: kfs[k])
            rec = prof[name]
    per_launch_ms = rec["total_ms"] / rec["launches"]
    launches_per_step = rec["launches"] / steps
    tr = traffic_table().get(name, {}).get(bench.name)
    if isinstance(bench, LinearBench):
        algo = bench.bytes_per_step() / launches_per_step
        achieved = algo / (per_launch_ms * 1e-3) / 1e9
        peak = pk["hbm_gbs"]
        return {"kernel": name, "bound": "hbm", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": pk_kind,
                "algorithmic_per_launch": algo, "launch_ms": per_launch_ms,
                "time_share": rec["total_ms"] / total, "traffic": tr}
    kf = bench.kernel_flops_per_step().get(name)
    if kf is None:
        return {"kernel": name, "bound": None, "note": "dominant kernel has no flop model",
                "time_share": rec["total_ms"] / total}
    algo = kf / launches_per_step
    achieved = algo / (per_launch_ms * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    return {"kernel": name, "bound": "tensor", "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": pk_kind,
            "algorithmic_per_launch": algo, "launch_ms": per_launch_ms,
            "time_share": rec["total_ms"] / total, "traffic": tr}


def cpu_baseline(bench, budget_s=12.0):
    if isinstance(bench, LinearBench):
        import numpy as np
        from oracle import ttt_linear_recurrent
        x = bench.x
        n, t_all, toks = 2048, 0.0, 0.0
        while t_all < budget_s:
            sl = lambda a: a[:1, :, :n]  # noqa: E731
            t0 = time.perf_counter()
            ttt_linear_recurrent(sl(x.q.values), sl(x.k.values), sl(x.v.values), sl(x.lr))
            t_all += time.perf_counter() - t0
            toks += n
        sample = f"batch entry 0 (all {bench.H} heads), first {n} tokens, repeated"
        del np
    else:
        toks, t_all, chunks = 0.0, 0.0, 1
        while t_all < budget_s:
            tk, dt, sample = bench.oracle_sample(chunks)
            toks += tk
            t_all += dt
            chunks = min(chunks * 2, 1 << 20)
        sample += " (repeated, growing)"
    return {"value": toks / t_all, "unit": "tokens/s", "cores": os.cpu_count(),
            "kind": "oracle", "sample": sample, "seconds": t_all}


def parallelism(world):
    return "replicas" if world == 1 else f"dp{world} (independent replicas)"


def l2_note(resident):
    return (f"inputs larger than L2: {resident / 2**20:.0f} MiB touched per step vs "
            f"{L2_BYTES / 2**20:.0f} MiB L2; no flush")


def per_config_summary(name, value, step_ms, tflops, peak, secondary, extra):
    """One compact entry per workload timed in this run: tokens/s, ms per
    step, TFLOP/s and its fraction of the bf16 peak, and for the HBM-bound
    linear layers GB/s and its fraction of the HBM peak."""
    r = lambda x, n=4: None if x is None else float(f"{x:.{n}g}")  # noqa: E731
    out = {name: {"tok_s": r(value), "ms": r(step_ms), "tflops": r(tflops),
                  "frac_bf16": r(tflops / peak, 3)}}
    if secondary:
        rf = secondary["roofline"]
        out[secondary["config"]["workload"]] = {
            "tok_s": r(secondary["value"]), "ms": r(secondary["ms_per_step"]),
            "gbs": r(rf.get("achieved")), "frac_hbm": r(rf.get("frac"), 3),
            "kernel": rf.get("kernel")}
    for k, e in (extra or {}).items():
        d = {"tok_s": r(e["value"]), "ms": r(e["ms_per_step"]), "tflops": r(e["tflops"]),
             "frac_bf16": r(e["frac_bf16_peak"], 3)}
        if e.get("hbm"):
            d["gbs"], d["frac_hbm"] = r(e["hbm"]["gbs"]), r(e["hbm"]["frac"], 3)
        out[k] = d
    return out


# --------------------------------------------------------------------------- arms
def run_reference(args):
    """CPU oracle on the host cores: each step is a bounded sample."""
    from ttt_synth import WORKLOADS
    import torch  # noqa: F401  (device not used)
    name = args.workload
    bench = make_bench_cpu(name)
    step_times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        toks, dt, sample = bench.oracle_sample(1)
        if i >= args.warmup:
            step_times.append((toks, time.perf_counter() - t0))
    toks = sum(t for t, _ in step_times)
    secs = sum(s for _, s in step_times)
    val = toks / secs
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {**bench.config(), "parallelism": parallelism(args.gpus),
                       "l2": l2_note(bench.resident_bytes())},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": os.cpu_count(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class _CPUOnlyLaCT(LaCTBench):
    def __init__(self, name):  # noqa: super init needs a device; only oracle bits here
        from ttt_synth import WORKLOADS, make_workload
        self.name, self.w = name, dict(WORKLOADS[name])
        w = self.w
        self.x = make_workload(name)
        self.B, self.H, self.N, self.d, self.dh = w["B"], w["H"], w["N"], w["d"], w["dh"]
        self.Nq = self.x.q.values.shape[2]
        self.causal = w["order"] == "causal"
        self.opt = w.get("opt", "gd")
        self.update_mask = w.get("update_mask", 7)
        self.normalize_rows = w.get("normalize_rows", True)
        self.window = w.get("window", 0)

    def resident_bytes(self):
        """Bytes the GPU arm keeps resident for this workload (same tensors:
        bf16 q, k, v and out, fp32 lr)."""
        BH = self.B * self.H
        return BH * (self.Nq * self.d * 2 * 2 + self.N * (2 * self.d * 2 + 4))


class _CPUOnlyLinear:
    """Oracle side of a linear workload (forward, or backward when the
    workload says so): no device needed."""

    def __init__(self, name):
        from ttt_synth import WORKLOADS, make_linear_grads, make_workload
        self.name, self.w = name, dict(WORKLOADS[name])
        self.x = make_workload(name)
        self.g = make_linear_grads(self.x, cfg=self.w["cfg"]) if self.w.get("backward") else None
        w = self.w
        self.B, self.H, self.N, self.dk, self.dv = w["B"], w["H"], w["N"], w["dk"], w["dv"]

    def config(self):
        """The same workload description as the GPU arm's."""
        c = LinearBench.config(self)
        if self.g is not None:
            c["pass"], c["out_dtype"] = "backward", "f32"
        return c

    def resident_bytes(self):
        """Bytes the GPU arm keeps resident for this workload (same tensors)."""
        el = 2 if self.w["dtype"] == "bf16" else 4
        tok = self.B * self.H * self.N
        if self.g is None:   # q, k, v, lr, bf16 out
            return tok * ((2 * self.dk + self.dv) * el + 4 + 2 * self.dv)
        return tok * ((2 * self.dk + 2 * self.dv) * el + 4 + (2 * self.dk + self.dv) * 4 + 4) + \
            self.B * self.H * self.dk * self.dv * 4

    def oracle_sample(self, n_blocks):
        """Batch entry 0, all heads, the first 512 * n_blocks tokens."""
        from oracle import ttt_linear_backward, ttt_linear_recurrent
        x, w = self.x, self.w
        n = min(w["N"], 512 * n_blocks)
        sl = lambda a: a[:1, :, :n]  # noqa: E731
        t0 = time.perf_counter()
        if self.g is None:
            ttt_linear_recurrent(sl(x.q.values), sl(x.k.values), sl(x.v.values), sl(x.lr))
        else:
            ttt_linear_backward(sl(x.q.values), sl(x.k.values), sl(x.v.values), sl(x.lr),
                                sl(self.g.dout.values), None, self.g.dS_end[:1])
        dt = time.perf_counter() - t0
        what = "backward" if self.g is not None else "forward"
        return n, dt, f"{what}: batch entry 0 (all {w['H']} heads), first {n} tokens"


def make_bench_cpu(name):
    from ttt_synth import WORKLOADS
    if WORKLOADS[name]["kind"] == "linear":
        return _CPUOnlyLinear(name)
    return _CPUOnlyLaCT(name)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="lact_causal_n32k")
    ap.add_argument("--secondary", default="ttt_linear_bf16_n32k")
    ap.add_argument("--extra", default="lact_bidir_196k,lact_bidir_muon_1m,lact_w2only_causal_n32k,"
                    "ttt_linear_bwd_bf16_n32k,lact_layer_causal_n32k,lact_bwd_causal_n32k",
                    help="further workloads timed once each (comma list, or none)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel from the host instead of replaying a CUDA graph")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist_mod
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import learned_linear_attention_b200 as T
    T.load()
    pk, pk_kind = peaks()

    bench = make_bench(args.workload, device, seed=rank)
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        bench.step(stream)
    torch.cuda.synchronize()
    step_fn = bench.step
    if not args.no_graph:
        graph = capture_graph(bench, stream)
        step_fn = lambda s: graph.replay()  # noqa: E731
        for _ in range(args.warmup):
            step_fn(stream)
        torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(device)
    uuid = str(getattr(props, "uuid", "") or "")
    sampler = ClockSampler(uuid)
    sampler.start()
    ms = timed(bench, args.steps, stream, fn=step_fn, dist=dist)
    clocks = sampler.stop()

    prof = profile_kernels(bench, args.steps, stream)
    launches = sum(v["launches"] for v in prof.values())
    roof = roofline_for(bench, prof, args.steps, pk, pk_kind)
    total_ms = sum(v["total_ms"] for v in prof.values())
    kernels = {k: {"launches_per_step": v["launches"] / args.steps,
                   "ms_per_step": v["total_ms"] / args.steps,
                   "share": v["total_ms"] / total_ms} for k, v in prof.items()}

    # end to end through the public API with host buffers
    e2e = None
    if hasattr(bench, "setup_e2e"):
        bench.setup_e2e(step_fn)
        for _ in range(2):
            bench.step_e2e(stream)
        ems = timed(bench, args.steps, stream, fn=bench.step_e2e, dist=dist)
        e2e = {"value": job_value(world, bench.tokens_per_step(), ems / args.steps),
               "unit": "tokens/s", "h2d_bytes_per_step": bench.h2d,
               "d2h_bytes_per_step": bench.d2h, "ms_per_step": ems / args.steps}

    step_ms = ms / args.steps
    value = job_value(world, bench.tokens_per_step(), step_ms)
    tflops = bench.flops_per_step() / (step_ms * 1e-3) / 1e12

    secondary = None
    if args.secondary and args.secondary not in ("none", args.workload):
        sb = make_bench(args.secondary, device, seed=rank)
        for _ in range(args.warmup):
            sb.step(stream)
        sfn = sb.step
        if not args.no_graph:
            sgraph = capture_graph(sb, stream)
            sfn = lambda s: sgraph.replay()  # noqa: E731
            sfn(stream)
        sms = timed(sb, args.steps, stream, fn=sfn, dist=dist) / args.steps
        sprof = profile_kernels(sb, args.steps, stream)
        secondary = {"config": sb.config(),
                     "value": job_value(world, sb.tokens_per_step(), sms),
                     "unit": "tokens/s", "ms_per_step": sms,
                     "roofline": roofline_for(sb, sprof, args.steps, pk, pk_kind)}
        del sb

    # the other LaCT shapes (view-synthesis sets, Muon): a few eager steps each
    extra = {}
    for name in ([] if args.extra in ("", "none") else args.extra.split(",")):
        if name == args.workload:
            continue
        eb = make_bench(name, device, seed=rank)
        for _ in range(2):
            eb.step(stream)
        # one step replayed as a CUDA graph, like the headline (host launches
        # with --no-graph, or where a capture is refused)
        efn, elaunch, eg = eb.step, "host launches", None
        if not args.no_graph:
            try:
                eg = capture_graph(eb, stream)
                efn, elaunch = (lambda s, g=eg: g.replay()), "CUDA graph replay of one step"
                efn(stream)
                torch.cuda.synchronize()
            except RuntimeError:
                efn, elaunch = eb.step, "host launches (graph capture refused)"
        probe = timed(eb, 1, stream, fn=efn, dist=dist)
        esteps = 10 if probe < 5.0 else 3
        ems = timed(eb, esteps, stream, fn=efn, dist=dist) / esteps
        eprof = profile_kernels(eb, 1, stream)
        etot = sum(v["total_ms"] for v in eprof.values()) or 1.0
        etf = eb.flops_per_step() / (ems * 1e-3) / 1e12
        ecfg = eb.config()
        ecfg["launch"] = elaunch
        extra[name] = {"config": ecfg, "value": job_value(world, eb.tokens_per_step(), ems),
                       "unit": "tokens/s", "ms_per_step": ems, "steps": esteps, "tflops": etf,
                       "frac_bf16_peak": etf / pk["bf16_tflops"],
                       "hbm": ({"algorithmic_bytes": eb.bytes_per_step(),
                                "gbs": eb.bytes_per_step() / (ems * 1e-3) / 1e9,
                                "frac": eb.bytes_per_step() / (ems * 1e-3) / 1e9 / pk["hbm_gbs"]}
                               if isinstance(eb, LinearBench) else None),
                       "kernels": {k: {"launches_per_step": v["launches"],
                                       "share": v["total_ms"] / etot}
                                   for k, v in sorted(eprof.items(), key=lambda kv: -kv[1]["total_ms"])}}
        efn = eg = None   # the graph's memory goes with the workload
        del eb
        torch.cuda.empty_cache()

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(bench)
        cfg = bench.config()
        cfg["parallelism"] = parallelism(world)
        cfg["l2"] = l2_note(bench.resident_bytes())
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic", "config": cfg,
                "tflops": tflops, "frac_bf16_peak": tflops / pk["bf16_tflops"],
                "peak_source": pk_kind, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clocks, "kernels": kernels,
                "launch": "host launches" if args.no_graph else "CUDA graph replay of one step",
                "secondary": secondary, "extra": extra or None}
        # last, so that a record keeping only the end of the line still holds
        # every workload's figures
        line["per_config"] = per_config_summary(args.workload, value, step_ms, tflops,
                                                pk["bf16_tflops"], secondary, extra)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

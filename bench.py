#!/usr/bin/env python
"""Benchmark of the routed-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl flux|reference]

One step is one pass of the routed prefill hot path over the 36-layer
Qwen3-4B-shaped workload (B 1, T 65536, Hq 32, Hkv 8, d 128; every layer has its
own bf16 N(0,1) Q/K/V resident in HBM, with 16 planted needles per kv head):
  flux_route (hidden 65536 x 2560, MLP 5120 -> 512 -> 36; the biases put 18 layers
  on each side with a wide margin) -> flux_build_streaming_mask +
  flux_build_block_index (block 128, sink 1, window 16) -> 36 flux_attn_prefill
  launches, each reading its layer's routing bit on the device.
value = TFLOP/s over the computed (query, key) pairs of all 36 layers (4 d FLOPs
per pair per query head) / step time.  "roofline" is the FA layer's prefill kernel
in that step; "roofline_sa_prefill" the SA layer's; "roofline_decode" the decode
kernel of an FA layer in the decode half of the metric.

The decode half of the metric (KV GB/s) is timed in the same run on the 36-layer
Qwen3-4B-shaped decode workload (batch 16, KV 131072 + step, 18 FA / 18 SA layers,
64 steps; every layer appends the new token's K/V -- the full cache of an FA layer,
the compact sink + window ring of an SA layer -- and decodes) and reported under
"decode", with one SA ring layer timed alone with and without an L2 flush.  On one
GPU the line also carries, each timed in a few seconds: "layer_pair_T32768" (one FA
and one SA layer of the Qwen3-4B shape at T 32768 with the 2-layer router),
"soft_prefill", "dynamic_sa" (flux_select_blocks on that layer's Q/K, the CSR build
and SA prefill over the selected mask) and "llama_3_1_8b" (the 32-layer prefill
step at T 131072 measured as one step per SA fraction 0/25/50/75/100 % and per
window 8/16/32 blocks; the 32-layer decode step at B 4, S 131072); --no-extended
skips them.

Every input is seeded and synthetic; every timed input (29 GB of Q/K/V for the
prefill step, 17 GB of KV for decode) is larger than the 126 MB L2, so no flush is
needed.  Multi-GPU: the units are independent (no exchange), so each rank runs its
own replica of the step (weak scaling) and rank 0 reports the max time.

--impl reference times the oracle (plain fp64 C, OpenMP) on the host cores on a
bounded sample of the same workload, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HQ, HKV, D = 32, 8, 128
HD, H1 = 2560, 512
BLOCK, SINK, WIN = 128, 1, 16
T_STEP, L_STEP = 65536, 36                 # the routed prefill step
T_PAIR = 32768                              # the single-layer pair (extra)
DEC_B, DEC_S, DEC_LAYERS, DEC_STEPS = 16, 131072, 36, 64
E2E_BUFFERS = 8                             # layers' inputs/outputs in flight in the e2e step
# Dense bf16 tensor and HBM figures of the B200 specification, beside the measured peaks.
SPEC_TFLOPS, SPEC_HBM_GBS = 2250.0, 8000.0


def causal_pairs_fa(T):
    return T * (T + 1) // 2


def pairs_sa(T, block, sink, W):
    """(query, key) pairs visible under the sink + window mask (diagonal tiles causal)."""
    nb = (T + block - 1) // block
    total = 0
    for i in range(nb):
        q0, q1 = i * block, min(T, (i + 1) * block)
        for j in range(i + 1):
            if not (j < sink or j >= i - W + 1):
                continue
            k0, k1 = j * block, min(T, (j + 1) * block)
            if j < i:
                total += (q1 - q0) * (k1 - k0)
            else:
                n = q1 - q0
                total += n * (n + 1) // 2
    return total


def sa_decode_tokens(s, block, sink, W):
    n_sink = min(sink * block, s)
    nbs = -(-s // block)
    win_start = max(n_sink, max(0, nbs - W) * block)
    return n_sink + (s - win_start)


def recorded_traffic(key):
    """DRAM bytes per launch (read + write) of a kernel from its ncu capture, recorded in
    profiles/dram_traffic.json together with a SHA-256 of the code it was built from
    (comments and whitespace removed); None when there is no record or that code has
    changed since the capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(key)
    if not rec:
        return None
    from sparse_attention_flux_b200.record_traffic import sources_sha256
    if sources_sha256(rec["sources"]) != rec["sources_sha256"]:
        return None
    return int(rec["bytes_per_launch"])


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(1.0)  # let nvidia-smi start sampling before the timed region
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except Exception:
                self.proc.kill()

    def summary(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if not self.path or not os.path.exists(self.path):
            return out
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return out
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        out.update(sm_mhz=statistics.median(sm) if sm else None,
                   sm_max_mhz=max(mx) if mx else None, reasons=sorted(reasons),
                   samples=len(rows))
        return out


# --------------------------------------------------------------------------- ranks

def dist_barrier(world: int) -> None:
    """Barrier across ranks (no-op for one process)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of a per-rank time over all ranks (the timing the contract asks for)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float, scale: float = 1e12) -> float:
    """Aggregate throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms * 1e-3) / scale


def roofline_entry(achieved, peaks, peak_src, bound, kernel, traffic, algorithmic, per,
                   long_step=False):
    """A roofline object: achieved against the measured peak and against the
    specification's nominal peak.  For the tensor pipe the measured peak is cuBLAS's
    sustained figure (a seconds-long loop under the power cap) for a kernel timed inside
    a long step (long_step), else its burst figure; the other one is reported beside it.
    algorithmic: the kernel's algorithmic FLOPs or bytes per launch."""
    if bound == "tensor":
        burst = peaks.get("bf16_tflops", peaks.get("bf16_tflops_sustained"))
        sus = peaks.get("bf16_tflops_sustained", burst)
        peak = sus if long_step else burst
        spec, unit = SPEC_TFLOPS, "TFLOP/s"
        src = f"{peak_src} bf16_tflops{'_sustained' if long_step else ''} " \
              f"({'sustained: timed inside a seconds-long step' if long_step else 'burst'})"
    else:
        peak = peaks["hbm_gbs"]
        spec, unit = SPEC_HBM_GBS, "GB/s"
        src = f"{peak_src} hbm_gbs (copy)"
    out = {"bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
           "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kernel,
           "peak_source": src, "algorithmic_per_launch": algorithmic, "per": per,
           "frac_of_spec": round(achieved / spec, 4), "spec_peak": spec}
    if bound == "tensor":
        if long_step:
            out["frac_of_burst"] = round(achieved / burst, 4)
        else:
            out["frac_of_sustained"] = round(achieved / sus, 4)
    return out


# --------------------------------------------------------------------------- flux arm

def _events(torch, n):
    return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(n)]


class LayerStack:
    """L attention layers of one model at prompt length T (B 1, Hq 32, Hkv 8, d 128),
    every layer with its own Q/K/V resident in HBM (bf16 N(0,1) drawn on the device,
    16 planted needles per kv head when asked), and one output buffer that every layer
    writes in turn (the next op of a model reads it before the next layer runs)."""

    def __init__(self, ctx, dev, T, L, cfg, salt0=0, needles=True):
        import torch
        from sparse_attention_flux_b200 import synth
        self.ctx, self.dev, self.T, self.L = ctx, dev, T, L
        self.q, self.k, self.v = [], [], []
        for l in range(L):
            q = synth.torch_normal_bf16((1, T, HQ, D), synth.seed_for(cfg, l, salt0 + 1), dev)
            k = synth.torch_normal_bf16((1, T, HKV, D), synth.seed_for(cfg, l, salt0 + 2), dev)
            v = synth.torch_normal_bf16((1, T, HKV, D), synth.seed_for(cfg, l, salt0 + 3), dev)
            if needles:
                synth.plant_needles_torch(q, k, synth.seed_for(cfg, l, salt0))
            self.q.append(q)
            self.k.append(k)
            self.v.append(v)
        self.o = torch.empty_like(self.q[0])
        self.nb = (T + BLOCK - 1) // BLOCK
        self.scale = 1.0 / math.sqrt(D)

    def flops(self, mode_h, W=WIN):
        f_fa = 4.0 * D * causal_pairs_fa(self.T) * HQ
        f_sa = 4.0 * D * pairs_sa(self.T, BLOCK, SINK, W) * HQ
        return sum(f_fa if m else f_sa for m in mode_h), f_fa, f_sa

    def layers(self, mode, row_ptr, col, evs=None):
        """Every layer's prefill launch, each reading its bit mode[l] on the device;
        CUDA events around each launch when given."""
        c = self.ctx
        for l in range(self.L):
            if evs is not None:
                evs[l][0].record()
            c.attn_prefill(self.q[l], self.k[l], self.v[l], self.o, self.scale, layer_mode=mode,
                           layer=l, row_ptr=row_ptr, col=col, block=BLOCK)
            if evs is not None:
                evs[l][1].record()


class RoutedPrefill:
    """The routed prefill step: the 36-layer Qwen3-4B-shaped workload at T 65536.
    Router on hidden 65536 x 2560 (MLP 5120 -> 512 -> 36; b2 = +4 on 18 layers and -4
    on the other 18, chosen by a seeded permutation, so 18 layers go to each mode with
    |z| >= 1.4) -> streaming mask -> CSR -> 36 prefill launches reading their bits."""

    def __init__(self, ctx, dev, rank):
        import torch
        from sparse_attention_flux_b200 import synth
        self.ctx, self.dev = ctx, dev
        self.stack = LayerStack(ctx, dev, T_STEP, L_STEP, 2, salt0=10 * rank)
        h, W1, b1, W2, b2 = synth.router_inputs(T_STEP, HD, H1, L_STEP, synth.seed_for(2) + rank,
                                                coin_bias=4.0, n_positive=L_STEP // 2)
        self.hidden_h = synth.torch_from_bits(h).pin_memory()
        self.hidden = self.hidden_h.to(dev)
        self.W1, self.b1, self.W2, self.b2 = (torch.from_numpy(x).to(dev) for x in (W1, b1, W2, b2))
        self.mode = torch.zeros(L_STEP, dtype=torch.uint8, device=dev)
        nb = self.stack.nb
        self.nb = nb
        self.mask = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
        self.row_ptr = torch.empty(nb + 1, dtype=torch.int32, device=dev)
        self.col = torch.empty(nb * (SINK + WIN), dtype=torch.int32, device=dev)
        self.launches = 2 + 1 + 3 + L_STEP   # router (pool, MLP), mask, CSR (3), 36 layers
        self.step()
        ctx.check()
        self.mode_h = self.mode.cpu().numpy()
        self.flops, self.flops_fa, self.flops_sa = self.stack.flops(self.mode_h)

    def head(self, hidden=None, stream=None):
        c = self.ctx
        c.route(self.hidden if hidden is None else hidden, self.W1, self.b1, self.W2, self.b2, 0.5,
                self.mode, stream=stream)
        c.build_streaming_mask(self.nb, self.nb, SINK, WIN, self.mask, stream=stream)
        c.build_block_index(self.mask, self.row_ptr, self.col, stream=stream)

    def step(self, evs=None):
        self.head()
        self.stack.layers(self.mode, self.row_ptr, self.col, evs)

    # ---- end to end: host buffers in and out
    def e2e_setup(self):
        import torch
        st = self.stack
        # One layer's inputs in pinned host memory, sent for every layer: every byte
        # of every layer's Q/K/V crosses PCIe each step (the values do not change the
        # work).  Two pinned output buffers take the layers' outputs in turn.
        self.qkv_h = [x.cpu().pin_memory() for x in (st.q[0], st.k[0], st.v[0])]
        self.o_h = [torch.empty(st.o.shape, dtype=st.o.dtype).pin_memory() for _ in range(2)]
        # Device buffers for E2E_BUFFERS layers in flight: uploads run ahead while an FA
        # layer computes (an FA layer takes about twice a layer's upload, an SA layer a
        # tenth of it).
        self.ins = [[torch.empty_like(x) for x in (st.q[0], st.k[0], st.v[0])]
                    for _ in range(E2E_BUFFERS)]
        self.outs = [torch.empty_like(st.o) for _ in range(E2E_BUFFERS)]
        self.hid_d = torch.empty_like(self.hidden)

    @property
    def h2d_bytes(self):
        return self.hidden_h.numel() * 2 + L_STEP * sum(x.numel() * 2 for x in self.qkv_h)

    @property
    def d2h_bytes(self):
        return L_STEP * self.o_h[0].numel() * 2

    def e2e_pipelined(self, steps):
        """The step from pinned host memory through the public API, pipelined per layer
        over three streams: layer n's prefill overlaps the host->device copies of the
        next layers' Q/K/V (up to E2E_BUFFERS - 1 ahead) and the device->host copies of
        earlier layers' outputs; each step first uploads the router's hidden states.
        Returns ms per step, from an event before the first copy to one after the last
        copy back."""
        import torch
        dev, c, st = self.dev, self.ctx, self.stack
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev = lambda: torch.cuda.Event(enable_timing=False)
        nbuf = E2E_BUFFERS
        h2d, cmp, d2h = ([ev() for _ in range(nbuf)] for _ in range(3))
        hid_done, head_done = ev(), ev()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(s_in)
        n = 0
        for k in range(steps):
            with torch.cuda.stream(s_in):
                if k:
                    s_in.wait_event(head_done)
                self.hid_d.copy_(self.hidden_h, non_blocking=True)
                hid_done.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(hid_done)
                self.head(self.hid_d, stream=s_cmp)
                head_done.record(s_cmp)
            for l in range(L_STEP):
                b = n % nbuf
                with torch.cuda.stream(s_in):
                    if n >= nbuf:
                        s_in.wait_event(cmp[b])
                    for dst, x in zip(self.ins[b], self.qkv_h):
                        dst.copy_(x, non_blocking=True)
                    h2d[b].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(h2d[b])
                    if n >= nbuf:
                        s_cmp.wait_event(d2h[b])
                    q, kk, v = self.ins[b]
                    c.attn_prefill(q, kk, v, self.outs[b], st.scale, layer_mode=self.mode,
                                   layer=l, row_ptr=self.row_ptr, col=self.col, block=BLOCK,
                                   stream=s_cmp)
                    cmp[b].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(cmp[b])
                    self.o_h[n % 2].copy_(self.outs[b], non_blocking=True)
                    d2h[b].record(s_out)
                n += 1
        s_out.wait_stream(s_in)
        s_out.wait_stream(s_cmp)
        t1.record(s_out)
        t1.synchronize()
        return t0.elapsed_time(t1) / steps

    def copy_floor_ms(self, reps=2):
        """ms for one step's host<->device traffic alone: every upload on one stream and
        every download on another, concurrently (no compute) -- the floor of the
        pipelined e2e step on this machine's PCIe link."""
        import torch
        s_in, s_out = torch.cuda.Stream(self.dev), torch.cuda.Stream(self.dev)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        s_out.wait_stream(s_in)
        for _ in range(reps):
            with torch.cuda.stream(s_in):
                self.hid_d.copy_(self.hidden_h, non_blocking=True)
                for l in range(L_STEP):
                    for dst, x in zip(self.ins[l % E2E_BUFFERS], self.qkv_h):
                        dst.copy_(x, non_blocking=True)
            with torch.cuda.stream(s_out):
                for l in range(L_STEP):
                    self.o_h[l % 2].copy_(self.outs[l % E2E_BUFFERS], non_blocking=True)
        s_in.wait_stream(s_out)
        b.record(s_in)
        b.synchronize()
        return a.elapsed_time(b) / reps

    def release(self):
        for name in ("stack", "ins", "outs", "hid_d", "qkv_h", "o_h", "hidden", "hidden_h"):
            if hasattr(self, name):
                delattr(self, name)


class LayerPair:
    """One FA and one SA layer of the Qwen3-4B shape at T 32768 (B 1, needles), routed
    by a 2-logit router on hidden 32768 x 2560 (layer 0 FA, layer 1 SA)."""

    def __init__(self, ctx, seed, dev):
        import torch
        from sparse_attention_flux_b200 import synth
        self.ctx, self.dev = ctx, dev
        T = T_PAIR
        q, k, v = synth.attention_inputs(1, T, HQ, HKV, D, seed)
        self.needles = synth.plant_needles_np(q, k, seed)
        self.q, self.k, self.v = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
        hidden, W1, b1, W2, b2 = synth.router_inputs(T, HD, H1, 2, seed + 50)
        b2[:] = np.array([4.0, -4.0], np.float32)   # layer 0 -> FA, layer 1 -> SA
        self.hidden = synth.torch_from_bits(hidden).to(dev)
        self.W1, self.b1, self.W2, self.b2 = (torch.from_numpy(x).to(dev) for x in (W1, b1, W2, b2))
        self.mode = torch.zeros(2, dtype=torch.uint8, device=dev)
        self.nb = T // BLOCK
        self.mask = torch.empty((self.nb, self.nb), dtype=torch.uint8, device=dev)
        self.row_ptr = torch.empty(self.nb + 1, dtype=torch.int32, device=dev)
        self.col = torch.empty(self.nb * (SINK + WIN), dtype=torch.int32, device=dev)
        self.o = [torch.empty_like(self.q) for _ in range(2)]
        self.flops_fa = 4.0 * D * causal_pairs_fa(T) * HQ
        self.flops_sa = 4.0 * D * pairs_sa(T, BLOCK, SINK, WIN) * HQ
        self.flops = self.flops_fa + self.flops_sa
        self.scale = 1.0 / math.sqrt(D)

    def step(self, events=None):
        c = self.ctx
        c.route(self.hidden, self.W1, self.b1, self.W2, self.b2, 0.5, self.mode)
        c.build_streaming_mask(self.nb, self.nb, SINK, WIN, self.mask)
        c.build_block_index(self.mask, self.row_ptr, self.col)
        for layer in (0, 1):
            if events:
                events[layer][0].record()
            c.attn_prefill(self.q, self.k, self.v, self.o[layer], self.scale, layer_mode=self.mode,
                           layer=layer, row_ptr=self.row_ptr, col=self.col, block=BLOCK)
            if events:
                events[layer][1].record()

    def measure(self, steps=5):
        import torch
        for _ in range(2):
            self.step()
        evs = [_events(torch, 2) for _ in range(steps)]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for e in evs:
            self.step(e)
        b.record()
        b.synchronize()
        self.ctx.check()
        ms = a.elapsed_time(b) / steps
        fa = statistics.mean(e[0][0].elapsed_time(e[0][1]) for e in evs)
        sa = statistics.mean(e[1][0].elapsed_time(e[1][1]) for e in evs)
        return {"workload": "qwen3-4b-layer-pair: B 1, T 32768, Hq 32, Hkv 8, d 128, needles; "
                            "router 32768x2560 -> MLP 5120-512-2 (layer 0 FA, layer 1 SA); "
                            "SA block 128, sink 1, window 16",
                "ms_per_step": round(ms, 4),
                "TFLOP/s": round(self.flops / (ms * 1e-3) / 1e12, 1),
                "fa_layer": {"ms": round(fa, 4),
                             "TFLOP/s": round(self.flops_fa / (fa * 1e-3) / 1e12, 1)},
                "sa_layer": {"ms": round(sa, 4),
                             "TFLOP/s": round(self.flops_sa / (sa * 1e-3) / 1e12, 1)},
                "timed_steps": steps}


class DecodeWorkload:
    """36 layers, batch 16, KV 131072 + step.  Per layer and step the new token's K/V is
    appended (flux_kv_write: the full cache of an FA layer, the compact ring of an SA
    layer) and then decoded: FA layers read the whole cache, SA layers their ring of
    sink + 16 blocks (the minimal KV the pages say SA layers keep)."""

    def __init__(self, ctx, seed, dev, steps):
        import torch
        from sparse_attention_flux_b200 import synth
        self.ctx, self.dev, self.steps = ctx, dev, steps
        self.S_max = DEC_S + steps
        shape = (DEC_B, self.S_max, HKV, D)
        # 18 FA layers alias onto 2 physical caches (each 8.6 GB, far above L2).
        self.fa_caches = [(synth.torch_normal_bf16(shape, seed + 10 * i + 1, dev),
                           synth.torch_normal_bf16(shape, seed + 10 * i + 2, dev)) for i in range(2)]
        self.mode = torch.from_numpy(synth.layer_mode_choice(DEC_LAYERS, DEC_LAYERS // 2, seed)).to(dev)
        self.mode_h = self.mode.cpu().numpy()
        ring = (DEC_B, (SINK + WIN) * BLOCK, HKV, D)
        self.rings = {l: (synth.torch_normal_bf16(ring, seed + 1000 + 2 * l, dev),
                          synth.torch_normal_bf16(ring, seed + 1001 + 2 * l, dev))
                      for l in range(DEC_LAYERS) if not self.mode_h[l]}
        self.q = synth.torch_normal_bf16((DEC_B, HQ, D), seed + 99, dev)
        self.new_k = synth.torch_normal_bf16((DEC_B, 1, HKV, D), seed + 97, dev)
        self.new_v = synth.torch_normal_bf16((DEC_B, 1, HKV, D), seed + 98, dev)
        self.o = torch.empty_like(self.q)
        self.seqlens = [torch.full((DEC_B,), DEC_S + s + 1, dtype=torch.int32, device=dev)
                        for s in range(steps)]
        self.scale = 1.0 / math.sqrt(D)
        kv_row = HKV * D * 2 * 2
        self.bytes_fa = sum(DEC_B * (DEC_S + s + 1) * kv_row for s in range(steps)) / steps
        self.bytes_sa = sum(DEC_B * sa_decode_tokens(DEC_S + s + 1, BLOCK, SINK, WIN) * kv_row
                            for s in range(steps)) / steps
        n_fa = int(self.mode_h.sum())
        self.bytes_per_step = n_fa * self.bytes_fa + (DEC_LAYERS - n_fa) * self.bytes_sa
        self.launches = DEC_LAYERS   # one fused append + decode per layer
        self.kv_gb = (2 * 2 * DEC_B * self.S_max * HKV * D * 2 +
                      len(self.rings) * 2 * DEC_B * (SINK + WIN) * BLOCK * HKV * D * 2) / 1e9

    def granularity(self, steps):
        """ms per 36-layer decode step, layer-level vs head-level routing at the same SA
        fraction (one half): layer level routes 18 whole layers to SA; head level routes a
        seeded half of each layer's query heads to SA, so a GQA group containing any FA
        head streams the full history (no appends; full caches for every layer)."""
        import torch
        from sparse_attention_flux_b200 import synth
        rng = synth.rng(4242)
        heads = [torch.from_numpy((rng.permutation(HQ) < HQ // 2).astype(np.uint8)).to(self.dev)
                 for _ in range(DEC_LAYERS)]
        sl = self.seqlens[0]
        out = {}
        for level in ("layer", "head"):
            def one():
                for layer in range(DEC_LAYERS):
                    kc, vc = self.fa_caches[layer % 2]
                    if level == "layer":
                        self.ctx.attn_decode(self.q, kc, vc, sl, self.o, self.scale,
                                             layer_mode=self.mode, layer=layer, sink_blocks=SINK,
                                             window_blocks=WIN, block=BLOCK)
                    else:
                        self.ctx.attn_decode_heads(self.q, kc, vc, sl, self.o, self.scale,
                                                   heads[layer], SINK, WIN, BLOCK)
            one()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(steps):
                one()
            b.record()
            b.synchronize()
            out[level + "_ms_per_step"] = round(a.elapsed_time(b) / steps, 4)
        frac_groups_all_sa = float(np.mean([(h.cpu().numpy().reshape(HKV, HQ // HKV) == 0).all(1).mean()
                                            for h in heads]))
        out["head_over_layer"] = round(out["head_ms_per_step"] / out["layer_ms_per_step"], 3)
        out["groups_fully_sa_at_head_level"] = round(frac_groups_all_sa, 3)
        out["sa_fraction"] = 0.5
        return out

    def sa_layer(self, reps):
        """One SA layer's decode over its compact ring (B 16, the last step's length), timed
        launch by launch with CUDA events around each eager launch: back to back (ring
        partly L2-resident: 143 MB of K+V against a 126 MB L2) and with a 256 MB write
        between launches (cold L2); and 40 launches replayed from a CUDA graph (the
        GPU-side cost per layer, without the host's per-call submission)."""
        import torch
        layer = min(self.rings)
        kr, vr = self.rings[layer]
        sl = self.seqlens[-1]
        s = DEC_S + self.steps
        byts = DEC_B * sa_decode_tokens(s, BLOCK, SINK, WIN) * HKV * D * 2 * 2
        fn = lambda: self.ctx.attn_decode_sa_compact(self.q, kr, vr, sl, self.o, self.scale,
                                                     SINK, WIN, BLOCK)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=self.dev)
        out = {}
        for name, flushed in (("unflushed", False), ("flushed", True)):
            evs = _events(torch, reps)
            fn()
            for i, (a, b) in enumerate(evs):
                if flushed:
                    flush.fill_(i & 0xFF)
                a.record()
                fn()
                b.record()
            torch.cuda.synchronize()
            us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3
            out[name] = {"us": round(us, 2), "GB/s": round(byts / (us * 1e-6) / 1e9, 1)}
        # Back to back from a CUDA graph of 40 launches: the GPU-side cost of a layer
        # with no host submission in it (each launch's dispatch overlaps the previous
        # one's tail: programmatic dependent launch).
        n_graph = 40
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(self.dev)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=cs):
            for _ in range(n_graph):
                fn()
        torch.cuda.current_stream().wait_stream(cs)
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) / n_graph * 1e3)
        us = statistics.median(ts)
        out["graph_back_to_back"] = {"us": round(us, 2), "GB/s": round(byts / (us * 1e-6) / 1e9, 1),
                                     "launches": n_graph}
        out["kv_bytes"] = byts
        del g, flush
        return out

    def capture(self):
        """One 36-layer decode step (72 launches) captured as a CUDA graph; per step the
        device seqlens are updated and the graph replayed."""
        import torch
        self.sl_cur = torch.empty(DEC_B, dtype=torch.int32, device=self.dev)
        self.sl_cur.copy_(self.seqlens[0])
        self.graph = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(self.dev)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(self.graph, stream=cs):
            self.step(0, sl=self.sl_cur)
        torch.cuda.current_stream().wait_stream(cs)

    def replay(self, s):
        self.sl_cur.copy_(self.seqlens[s], non_blocking=True)
        self.graph.replay()

    def step(self, s, fa_events=None, sl=None, fused=True):
        """One 36-layer decode step.  fused: flux_attn_decode_append (the step's token is
        written into the layer's cache by the decode launch itself: 36 launches); else
        flux_kv_write then the decode (72 launches)."""
        c = self.ctx
        fa_i = 0
        sl = self.seqlens[s] if sl is None else sl
        for layer in range(DEC_LAYERS):
            if self.mode_h[layer]:
                kc, vc = self.fa_caches[fa_i % 2]
                fa_i += 1
                timed = fa_events is not None and fa_i == 1
                if timed:
                    fa_events[0].record()
                if fused:
                    c.attn_decode_append(self.q, self.new_k, self.new_v, kc, vc, sl, self.o,
                                         self.scale, layer_mode=self.mode, layer=layer,
                                         sink_blocks=SINK, window_blocks=WIN, block=BLOCK)
                else:
                    c.kv_write(self.new_k, self.new_v, sl, kc, vc)
                    c.attn_decode(self.q, kc, vc, sl, self.o, self.scale, layer_mode=self.mode,
                                  layer=layer, sink_blocks=SINK, window_blocks=WIN, block=BLOCK)
                if timed:
                    fa_events[1].record()
            else:
                kr, vr = self.rings[layer]
                if fused:
                    c.attn_decode_append(self.q, self.new_k, self.new_v, kr, vr, sl, self.o,
                                         self.scale, sink_blocks=SINK, window_blocks=WIN,
                                         block=BLOCK, compact=True)
                else:
                    c.kv_write(self.new_k, self.new_v, sl, kr, vr, SINK, WIN, BLOCK)
                    c.attn_decode_sa_compact(self.q, kr, vr, sl, self.o, self.scale, SINK, WIN,
                                             BLOCK)


def dynamic_sa(ctx, wl, dev, reps=5):
    """Dynamic SA block selection on the bench layer's own Q and K (flux_select_blocks:
    strided antidiagonal block scores, stride 8, then the fewest blocks after the sink
    and the diagonal whose score mass reaches tau 0.9), the CSR build and SA prefill
    over the selected mask; the share of causal blocks kept; and how many of the
    planted needles' key blocks the selected mask keeps for the needle rows, against
    the streaming (sink + window) mask."""
    import torch
    nb, S, tau = wl.nb, 8, 0.9
    mask = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
    rp = torch.empty(nb + 1, dtype=torch.int32, device=dev)
    col = torch.empty(nb * nb, dtype=torch.int32, device=dev)
    o = torch.empty_like(wl.q)
    lm = torch.zeros(1, dtype=torch.uint8, device=dev)
    sel = lambda: ctx.select_blocks(wl.q, wl.k, mask, wl.scale, tau, SINK, stride=S)
    idx = lambda: ctx.build_block_index(mask, rp, col)
    att = lambda: ctx.attn_prefill(wl.q, wl.k, wl.v, o, wl.scale, layer_mode=lm, row_ptr=rp,
                                   col=col, block=BLOCK)
    for f in (sel, idx, att):
        f()
    ctx.check()

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        b.synchronize()
        return a.elapsed_time(b) / reps
    sel_ms, idx_ms, att_ms = timed(sel), timed(idx), timed(att)
    ctx.check()
    m = mask.cpu().numpy().astype(np.int64)
    stream_mask = wl.mask.cpu().numpy()
    kept = int(m.sum())
    pairs = (kept - int(np.trace(m))) * BLOCK * BLOCK + nb * BLOCK * (BLOCK + 1) // 2
    flops_sa = 4.0 * D * pairs * HQ
    nr = T_PAIR // S
    flops_sel = 2.0 * S * D * (nr * (nr + 1) / 2) * HQ
    hit_dyn = hit_st = total = 0
    for (_h, r, pos) in wl.needles:
        i = r // BLOCK
        for j in sorted(set(int(p) // BLOCK for p in pos)):
            total += 1
            hit_dyn += int(m[i, j])
            hit_st += int(stream_mask[i, j])
    return {
        "how": "flux_select_blocks on the layer's Q/K (stride 8, tau 0.9, sink 1, block 128) -> "
               "flux_build_block_index -> SA prefill over the selected mask; scores are a "
               "reading of the strided-antidiagonal selector the pages name (parity unpinned "
               "against the pages)",
        "select_ms": round(sel_ms, 4),
        "select_TFLOP/s": round(flops_sel / (sel_ms * 1e-3) / 1e12, 1),
        "csr_ms": round(idx_ms, 4),
        "sa_prefill_ms": round(att_ms, 4),
        "sa_prefill_TFLOP/s": round(flops_sa / (att_ms * 1e-3) / 1e12, 1),
        "kept_blocks": kept, "causal_blocks": nb * (nb + 1) // 2,
        "kept_fraction": round(kept / (nb * (nb + 1) / 2), 4),
        "needle_key_blocks_kept": {"selected_mask": hit_dyn, "streaming_mask": hit_st,
                                   "of": total},
    }


def llama_sweep(ctx, dev, rank, hbm_gbs):
    """Llama-3.1-8B shapes (32 layers, Hq 32, Hkv 8, d 128), no router (fixed modes from
    a seeded layer choice).

    prefill, B 1, T 131072, every layer with its own Q/K/V (48 GB resident): the whole
    32-layer step (mask + CSR + 32 launches reading their bits on the device) measured
    once per SA fraction 0/25/50/75/100 % at W 16 and at 50 % for W 8 and 32, after one
    warm-up step; per-layer CUDA events give the FA and SA layer rates inside it.
    decode, B 4, S 131072: the whole 32-layer step, replayed from a CUDA graph (and launched
    eagerly, for comparison), at SA fractions 0/25/50/75/100 % (W 16) and at 50 % for W 8
    and 32; every layer has its own full cache (2.15 GB; 69 GB in all), so no layer's
    window is left in L2 by another's."""
    import torch
    from sparse_attention_flux_b200 import synth
    L, T3, B4, S4 = 32, 131072, 4, 131072
    scale = 1.0 / math.sqrt(D)
    out = {"workload": "llama-3.1-8b: 32 layers, Hq 32, Hkv 8, d 128; prefill B 1 T 131072 "
                       "(per-layer Q/K/V resident); decode B 4 S 131072; sink 1, W in {8, 16, 32} "
                       "blocks of 128"}
    # ---- prefill
    st = LayerStack(ctx, dev, T3, L, 4, salt0=10 * rank, needles=False)
    nb = st.nb
    mask = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
    row_ptr = torch.empty(nb + 1, dtype=torch.int32, device=dev)
    col = torch.empty(nb * (SINK + 32), dtype=torch.int32, device=dev)

    def step(mode_t, W, evs=None):
        ctx.build_streaming_mask(nb, nb, SINK, W, mask)
        ctx.build_block_index(mask, row_ptr, col)
        st.layers(mode_t, row_ptr, col, evs)

    pre = {}
    warmed = False
    for pct, W in [(0, 16), (25, 16), (50, 16), (75, 16), (100, 16), (50, 8), (50, 32)]:
        n_sa = L * pct // 100
        mode_h = synth.layer_mode_choice(L, L - n_sa, synth.seed_for(4) + pct)
        mode_t = torch.from_numpy(mode_h).to(dev)
        if not warmed:
            step(mode_t, W)
            warmed = True
        evs = _events(torch, L)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step(mode_t, W, evs)
        b.record()
        b.synchronize()
        ctx.check()
        ms = a.elapsed_time(b)
        flops, f_fa, f_sa = st.flops(mode_h, W)
        per = [x.elapsed_time(y) for x, y in evs]
        fa_ms = [per[l] for l in range(L) if mode_h[l]]
        sa_ms = [per[l] for l in range(L) if not mode_h[l]]
        ent = {"ms_per_step": round(ms, 2), "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1)}
        if fa_ms:
            ent["fa_layer_TFLOP/s"] = round(f_fa / (statistics.mean(fa_ms) * 1e-3) / 1e12, 1)
        if sa_ms:
            ent["sa_layer_ms"] = round(statistics.mean(sa_ms), 3)
            ent["sa_layer_TFLOP/s"] = round(f_sa / (statistics.mean(sa_ms) * 1e-3) / 1e12, 1)
        pre[f"sa{pct}%_W{W}"] = ent
    pre["how"] = ("one measured 32-layer step per entry (mask + CSR + 32 prefill launches), "
                  "CUDA events around the step and around each layer's launch")
    out["prefill"] = pre
    del st
    torch.cuda.empty_cache()
    # ---- decode
    shape = (B4, S4, HKV, D)
    caches = [(synth.torch_normal_bf16(shape, synth.seed_for(4, l, 4) + rank, dev),
               synth.torch_normal_bf16(shape, synth.seed_for(4, l, 5) + rank, dev)) for l in range(L)]
    qd = synth.torch_normal_bf16((B4, HQ, D), synth.seed_for(4, 0, 6) + rank, dev)
    od = torch.empty_like(qd)
    sl = torch.full((B4,), S4, dtype=torch.int32, device=dev)
    kv_row = HKV * D * 2 * 2

    def dec_step(mode_t, W):
        for layer in range(L):
            kc, vc = caches[layer]
            ctx.attn_decode(qd, kc, vc, sl, od, scale, layer_mode=mode_t, layer=layer,
                            sink_blocks=SINK, window_blocks=W, block=BLOCK)

    def timed(fn, n):
        fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        b.synchronize()
        return a.elapsed_time(b) / n

    def graph_timed(fn, n):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=cs):
            fn()
        torch.cuda.current_stream().wait_stream(cs)
        ms = timed(g.replay, n)
        del g
        return ms

    dec = {}
    for pct, W in [(0, 16), (25, 16), (50, 16), (75, 16), (100, 16), (50, 8), (50, 32)]:
        n_sa = L * pct // 100
        mode_t = torch.from_numpy(synth.layer_mode_choice(L, L - n_sa, synth.seed_for(4) + pct)).to(dev)
        eager_ms = timed(lambda: dec_step(mode_t, W), 5)
        ms = graph_timed(lambda: dec_step(mode_t, W), 5)
        byts = B4 * ((L - n_sa) * S4 + n_sa * sa_decode_tokens(S4, BLOCK, SINK, W)) * kv_row
        dec[f"sa{pct}%_W{W}"] = {"ms_per_step": round(ms, 3),
                                 "GB/s": round(byts / (ms * 1e-3) / 1e9, 1),
                                 "frac_of_hbm": round(byts / (ms * 1e-3) / 1e9 / hbm_gbs, 4),
                                 "eager_ms_per_step": round(eager_ms, 3)}
    dec["how"] = ("the 32-layer step (one decode launch per layer, each reading its routing bit "
                  "on the device) captured once as a CUDA graph and replayed 5 times; "
                  "eager_ms_per_step launches the same step from the host")
    ctx.check()
    out["decode"] = dec
    del caches
    torch.cuda.empty_cache()
    return out


def run_flux(args, rank, world, dev_index):
    import torch
    from sparse_attention_flux_b200 import synth
    from sparse_attention_flux_b200.flux import Context

    torch.cuda.set_device(dev_index)
    dev = torch.device("cuda", dev_index)
    peaks, peak_src = load_peaks()
    ctx = Context(dev_index, 512 << 20)
    wl = RoutedPrefill(ctx, dev, rank)

    barrier = lambda: dist_barrier(world)
    ranks_max = lambda x: max_over_ranks(x, world, dev)

    for _ in range(args.warmup):
        wl.step()
    ctx.check()
    # Per-layer CUDA events on the launching (current) stream, read after the loop so
    # that no host synchronisation sits inside the timed region.
    new_ev = lambda: torch.cuda.Event(enable_timing=True)
    evs = [_events(torch, L_STEP) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev_index) as clk:
        start, stop = new_ev(), new_ev()
        start.record()
        for k in range(args.steps):
            wl.step(evs[k])
        stop.record()
        torch.cuda.synchronize()
    barrier()
    total_ms = start.elapsed_time(stop)
    ctx.check()
    clocks = clk.summary()
    if not np.array_equal(wl.mode.cpu().numpy(), wl.mode_h):
        raise RuntimeError("routing changed between steps")
    fa_l = [l for l in range(L_STEP) if wl.mode_h[l]]
    sa_l = [l for l in range(L_STEP) if not wl.mode_h[l]]
    per = [[a.elapsed_time(b) for a, b in e] for e in evs]
    fa_avg = statistics.mean(p[l] for p in per for l in fa_l)
    sa_avg = statistics.mean(p[l] for p in per for l in sa_l)
    layers_ms = statistics.mean(sum(p) for p in per)
    total_ms = ranks_max(total_ms)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(wl.flops, world, ms_per_step)
    fa_tflops = wl.flops_fa / (fa_avg * 1e-3) / 1e12
    sa_tflops = wl.flops_sa / (sa_avg * 1e-3) / 1e12
    fa_bytes = 2 * (2 * T_STEP * HQ * D + 2 * T_STEP * HKV * D)    # Q, O + K, V (bf16)

    # router latency on the step's router (hidden 65536 x 2560, MLP 5120 -> 512 -> 36):
    # 20 back-to-back calls launched eagerly (host submission included) and replayed
    # from a CUDA graph (the GPU-side time)
    def time_router():
        fn = lambda: ctx.route(wl.hidden, wl.W1, wl.b1, wl.W2, wl.b2, 0.5, wl.mode)
        fn()
        a_, b_ = new_ev(), new_ev()
        a_.record()
        for _ in range(20):
            fn()
        b_.record()
        b_.synchronize()
        eager = a_.elapsed_time(b_) / 20 * 1e3
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=cs):
            for _ in range(20):
                fn()
        torch.cuda.current_stream().wait_stream(cs)
        g.replay()
        ts = []
        for _ in range(5):
            a_.record()
            g.replay()
            b_.record()
            b_.synchronize()
            ts.append(a_.elapsed_time(b_) / 20 * 1e3)
        del g
        return statistics.median(ts), eager
    router_us, router_eager_us = time_router()

    # e2e: host buffers in and out through the same public API, copies inside the timed
    # region, pipelined per layer over three streams.
    wl.e2e_setup()
    e2e_steps = args.steps
    wl.e2e_pipelined(1)
    barrier()
    e2e_ms = ranks_max(wl.e2e_pipelined(e2e_steps))
    ctx.check()
    e2e_value = whole_job_rate(wl.flops, world, e2e_ms)
    copy_floor = wl.copy_floor_ms()
    h2d_bytes, d2h_bytes = wl.h2d_bytes, wl.d2h_bytes
    launches = wl.launches * args.steps
    step_line = {"fa_layers": len(fa_l), "sa_layers": len(sa_l),
                 "fa_layer": {"ms": round(fa_avg, 3), "TFLOP/s": round(fa_tflops, 1)},
                 "sa_layer": {"ms": round(sa_avg, 4), "TFLOP/s": round(sa_tflops, 1)},
                 "router_mask_csr_ms": round(ms_per_step - layers_ms, 4),
                 "router_us": round(router_us, 2),
                 "router_eager_us": round(router_eager_us, 2),
                 "router_how": "36-layer router; router_us: 20 calls replayed from a CUDA graph "
                               "(GPU-side); router_eager_us: the same calls launched from the host",
                 "router_context": "pages: 0.20 ms per layer for their router (hardware not stated)",
                 "resident_qkv_gb": round(sum(x.numel() * 2 for x in wl.stack.q + wl.stack.k +
                                              wl.stack.v) / 1e9, 2),
                 "flops_per_step": wl.flops}
    wl.release()
    del wl
    torch.cuda.empty_cache()

    extra = {}
    # ---- the single-layer pair at T 32768, the soft blend and dynamic SA on it
    if not args.no_extended and world == 1:
        pair = LayerPair(ctx, synth.seed_for(1), dev)
        extra["layer_pair_T32768"] = pair.measure()
        score = torch.tensor([0.3], dtype=torch.float32, device=dev)
        soft = lambda: ctx.attn_prefill_soft(pair.q, pair.k, pair.v, pair.o[0], pair.scale, score,
                                             0, pair.row_ptr, pair.col, BLOCK)
        soft()
        s0, s1 = new_ev(), new_ev()
        s0.record()
        for _ in range(3):
            soft()
        s1.record()
        s1.synchronize()
        soft_ms = s0.elapsed_time(s1) / 3
        extra["soft_prefill"] = {
            "ms": round(soft_ms, 4), "TFLOP/s": round(pair.flops / (soft_ms * 1e-3) / 1e12, 1),
            "note": "flux_attn_prefill_soft on the T 32768 layer, r = 0.3: FA + SA passes, "
                    "blended in the SA epilogue"}
        extra["dynamic_sa"] = dynamic_sa(ctx, pair, dev)
        del pair
        torch.cuda.empty_cache()

    # ---- decode half of the metric
    dec = roof_dec = None
    if not args.no_decode:
        dw = DecodeWorkload(ctx, synth.seed_for(3) + 1000 * rank, dev, args.decode_steps)
        for s in range(min(3, dw.steps)):
            dw.step(s)
        ctx.check()
        # eager steps: per-kernel events for the first FA layer (and the eager step time)
        fevs = [(new_ev(), new_ev()) for _ in range(dw.steps)]
        torch.cuda.synchronize()
        e0, e1 = new_ev(), new_ev()
        e0.record()
        for s in range(dw.steps):
            dw.step(s, fevs[s])
        e1.record()
        e1.synchronize()
        fa_dec_ms = [a_.elapsed_time(b_) for a_, b_ in fevs]
        eager_ms = e0.elapsed_time(e1) / dw.steps
        n_sep = min(8, dw.steps)
        e0.record()
        for s in range(n_sep):
            dw.step(s, fused=False)
        e1.record()
        e1.synchronize()
        separate_ms = e0.elapsed_time(e1) / n_sep
        ctx.check()
        # timed: the same steps replayed from a CUDA graph
        dw.capture()
        dw.replay(0)
        barrier()
        torch.cuda.synchronize()
        d0, d1 = new_ev(), new_ev()
        d0.record()
        for s in range(dw.steps):
            dw.replay(s)
        d1.record()
        d1.synchronize()
        ctx.check()
        dec_ms = ranks_max(d0.elapsed_time(d1) / dw.steps)
        dec_gbs = whole_job_rate(dw.bytes_per_step, world, dec_ms, 1e9)
        fa_dec_avg = statistics.mean(fa_dec_ms)
        fa_dec_gbs = dw.bytes_fa / (fa_dec_avg * 1e-3) / 1e9
        roof_dec = roofline_entry(fa_dec_gbs, peaks, peak_src, "hbm",
                                  "decode_kernel<128> (FA layer, incl. its append)",
                                  recorded_traffic("decode_fa_B16_S131072"), dw.bytes_fa,
                                  "K+V bytes of every cached token, B 16 x (131072 + step) tokens")
        dec = {
            "workload": "qwen3-4b-36L-routed-decode: B 16, KV 131072+step, 18 FA (full cache) / "
                        f"18 SA (ring of sink 1 + 16 blocks), fused append + decode per layer, "
                        f"{dw.steps} steps",
            "kv_resident_gb": round(dw.kv_gb, 2),
            "value": round(dec_gbs, 1), "unit": "GB/s (KV bytes that must be read)",
            "ms_per_step": round(dec_ms, 4), "gpu_launches_per_step": dw.launches,
            "launch": "CUDA graph of one 36-layer step (36 fused append + decode launches), "
                      "seqlens updated per replay",
            "eager_ms_per_step": round(eager_ms, 4),
            "separate_append_eager_ms_per_step": round(separate_ms, 4),
            "frac_of_hbm": round(dec_gbs / peaks["hbm_gbs"], 4),
            "frac_of_spec": round(dec_gbs / SPEC_HBM_GBS, 4),
            "fa_layer": {"GB/s": round(fa_dec_gbs, 1), "ms": round(fa_dec_avg, 4),
                         "frac": round(fa_dec_gbs / peaks["hbm_gbs"], 4)},
        }
        dec["routing_granularity"] = dw.granularity(8)
        dec["sa_layer"] = dw.sa_layer(10)
        ctx.check()
        del dw.graph
        del dw
    torch.cuda.empty_cache()
    if not args.no_extended and world == 1:
        extra["llama_3_1_8b"] = llama_sweep(ctx, dev, rank, peaks["hbm_gbs"])
    ctx.close()

    line = {
        "metric": METRIC,
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(world),
        "roofline": roofline_entry(fa_tflops, peaks, peak_src, "tensor",
                                   "prefill_kernel<128> (FA layer of the routed step)",
                                   recorded_traffic("prefill_fa_T65536"), wl_flops_fa(),
                                   "4 d FLOPs per causal (query, key) pair per query head; "
                                   f"algorithmic bytes {fa_bytes} (Q, K, V read once, O written)",
                                   long_step=True),
        "roofline_sa_prefill": roofline_entry(sa_tflops, peaks, peak_src, "tensor",
                                              "prefill_kernel<128> (SA layer of the routed step)",
                                              recorded_traffic("prefill_sa_T65536"),
                                              wl_flops_sa(),
                                              "4 d FLOPs per computed (query, key) pair per "
                                              "query head (sink 1 + window 16 blocks of 128)",
                                              long_step=True),
        "roofline_decode": roof_dec,
        "prefill_step": step_line,
        "decode": dec,
        **extra,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                "how": "pinned host -> device copy of the router's hidden states and of every "
                       "layer's Q/K/V, the router + index + 36 layers, device -> host copy of "
                       "every layer's output, every step; layer n's prefill overlaps the "
                       "uploads of up to 7 later layers and the downloads of earlier ones on "
                       "separate streams (8 layers' buffers in flight); timed over K steps "
                       "from the first upload to the last download",
                "steps": e2e_steps,
                "copy_floor_ms_per_step": round(copy_floor, 4),
                "copy_floor_note": "the step's uploads and downloads alone, concurrently on two "
                                   "streams, on this machine: the PCIe floor of the e2e step"},
        "gpu_launches": launches,
        "clocks": clocks,
        "context": "pages: up to 2.8x prefill / 2.0x decode speedup vs FA baseline, hardware not "
                   "stated on the pages",
    }
    return line


def wl_flops_fa():
    return 4.0 * D * causal_pairs_fa(T_STEP) * HQ


def wl_flops_sa():
    return 4.0 * D * pairs_sa(T_STEP, BLOCK, SINK, WIN) * HQ


METRIC = "routed-attn prefill TFLOP/s & decode KV GB/s at 1 B200; % of roofline"


def bench_config(world: int) -> dict:
    """The workload both arms (this library and the oracle) report."""
    return {"workload": "qwen3-4b-36L-routed-prefill: B 1, T 65536, Hq 32, Hkv 8, d 128, 36 "
                        "layers each with its own Q/K/V (needles planted); router 65536x2560 -> "
                        "MLP 5120-512-36 (18 FA / 18 SA); SA block 128, sink 1, window 16",
            "l2": "inputs larger than L2 (29 GB of per-layer Q/K/V for prefill, 17 GB of decode "
                  "KV); no flush",
            "parallelism": f"replicas x{world} (no exchange)"}


class OracleSample:
    """The oracle, as it stands, on bounded samples of one layer of the routed prefill
    step (T 65536, needles): uniformly drawn query rows, FA rows for half of a sample's
    time, then SA rows.  FLOPs are counted like the GPU's (4 d per visible pair)."""

    def __init__(self, T=T_STEP):
        import oracle
        from sparse_attention_flux_b200 import synth
        self.oracle, self.T = oracle, T
        seed = synth.seed_for(2)
        self.q, self.k, self.v = synth.attention_inputs(1, T, HQ, HKV, D, seed)
        synth.plant_needles_np(self.q, self.k, seed)
        self.scale = 1.0 / math.sqrt(D)
        nb = T // BLOCK
        self.mask = oracle.streaming_mask(nb, nb, SINK, WIN)
        self.r = synth.rng(seed + 9)

    def run(self, seconds):
        """One bounded sample: (visible pairs, seconds taken, rows)."""
        pairs, used, n_rows = 0, 0.0, 0
        T = self.T
        for sparse in (False, True):
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < seconds / 2:
                rows = np.stack([np.zeros(64, np.int32),
                                 self.r.integers(0, HQ, 64).astype(np.int32),
                                 self.r.integers(0, T, 64).astype(np.int32)], 1)
                self.oracle.attn_prefill(self.q, self.k, self.v, self.scale,
                                         block_mask=self.mask if sparse else None, block=BLOCK,
                                         rows=rows)
                for t in rows[:, 2]:
                    if sparse:
                        i = t // BLOCK
                        pairs += sum(min(BLOCK, t + 1 - j * BLOCK) for j in range(i + 1)
                                     if (j < SINK or j >= i - WIN + 1))
                    else:
                        pairs += t + 1
                n_rows += 64
            used += time.perf_counter() - t0
        return pairs, used, n_rows


def cpu_baseline(seconds_budget=15.0, threads=None, sampler=None):
    """The oracle on one bounded sample of the prefill step's workload (all host cores,
    or `threads` of them)."""
    sampler = sampler or OracleSample()
    oracle = sampler.oracle
    if threads is not None:
        all_threads = oracle.num_threads()
        oracle.set_num_threads(threads)
    pairs, used, n_rows = sampler.run(seconds_budget)
    cores = oracle.num_threads()
    if threads is not None:
        oracle.set_num_threads(all_threads)
    return {"value": 4.0 * D * pairs / used / 1e12, "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{n_rows} uniformly sampled query rows (half of the time FA rows, half SA "
                      f"rows) of one T=65536 layer of the routed step, {used:.1f} s; FLOPs "
                      f"counted like the GPU's (4 d per visible pair)"}


def cpu_baseline_decode(threads=None):
    """The oracle on one sequence of the 36-layer decode workload (KV 131072 + 1 tokens,
    Hq 32, Hkv 8, d 128): one FA-layer decode and one SA-layer decode (sink 1 + 16 blocks),
    extrapolated to the step (16 sequences x (18 FA + 18 SA layers)); GB/s over the KV
    bytes that must be read, like the GPU's figure."""
    import oracle
    from sparse_attention_flux_b200 import synth
    s = DEC_S + 1
    q, kc, vc = synth.decode_inputs(1, s, HQ, HKV, D, synth.seed_for(3))
    sl = np.array([s], np.int32)
    scale = 1.0 / math.sqrt(D)
    if threads is not None:
        all_threads = oracle.num_threads()
        oracle.set_num_threads(threads)
    cores = oracle.num_threads()
    t0 = time.perf_counter()
    oracle.attn_decode(q, kc, vc, sl, scale, 1, SINK, WIN, BLOCK)
    t_fa = time.perf_counter() - t0
    t0 = time.perf_counter()
    reps = 20
    for _ in range(reps):
        oracle.attn_decode(q, kc, vc, sl, scale, 0, SINK, WIN, BLOCK)
    t_sa = (time.perf_counter() - t0) / reps
    if threads is not None:
        oracle.set_num_threads(all_threads)
    kv_row = HKV * D * 2 * 2
    step_s = DEC_B * (DEC_LAYERS // 2) * (t_fa + t_sa)
    step_bytes = DEC_B * (DEC_LAYERS // 2) * (s + sa_decode_tokens(s, BLOCK, SINK, WIN)) * kv_row
    return {"value": step_bytes / step_s / 1e9, "unit": "GB/s (KV bytes that must be read)",
            "cores": cores, "kind": "oracle",
            "ms_per_step_extrapolated": round(step_s * 1e3, 1),
            "sample": f"one sequence at KV {s}: FA-layer decode {t_fa * 1e3:.1f} ms, SA-layer "
                      f"decode {t_sa * 1e3:.2f} ms (mean of {reps}); step time extrapolated to "
                      f"16 sequences x 18 FA + 18 SA layers"}


def run_reference(args, world):
    """The reference arm: the oracle on the host cores, W untimed and K timed steps,
    each step a bounded sample of the bench's workload (sized so that the whole run
    takes about 150 s), value = FLOPs of all timed steps / their time."""
    sampler = OracleSample()                     # inputs prepared before timing, as on the GPU
    per_step = max(0.5, min(4.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        sampler.run(per_step)
    pairs = rows = 0
    used = 0.0
    for _ in range(args.steps):
        p, u, n = sampler.run(per_step)
        pairs, used, rows = pairs + p, used + u, rows + n
    value = 4.0 * D * pairs / used / 1e12
    sample = (f"{args.steps} steps of {per_step:.2f} s each ({args.warmup} more untimed): "
              f"{rows} uniformly sampled query rows of one T=65536 layer of the routed step "
              f"(half of each step FA rows, half SA rows); FLOPs counted like the GPU's (4 d per "
              f"visible pair)")
    return {"metric": METRIC,
            "impl": "reference", "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": used / max(1, args.steps) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s",
                             "cores": sampler.oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["flux", "reference"], default="flux")
    ap.add_argument("--decode-steps", type=int, default=DEC_STEPS)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extended", action="store_true",
                    help="skip the T 32768 layer pair, soft blend, dynamic SA and Llama-3.1-8B runs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args, world)))
        return

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    line = run_flux(args, rank, world, local)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            sampler = OracleSample()
            line["cpu_baseline"] = cpu_baseline(args.cpu_seconds, sampler=sampler)
            one = cpu_baseline(4.0, threads=1, sampler=sampler)
            line["cpu_baseline"]["single_thread"] = {"value": one["value"], "cores": 1,
                                                     "sample": one["sample"]}
            del sampler
            if line.get("decode"):
                dcb = cpu_baseline_decode()
                dcb["single_thread"] = cpu_baseline_decode(threads=1)
                line["decode"]["cpu_baseline"] = dcb
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the gated delta-rule hot path on B200.

One step = one gdn_chunk_fwd over the Gated DeltaNet prefill workload
(B=8, H=16, T=8192, dk=dv=128, bf16 q/k/v, fp32 gate/beta/state/output, chunk 64),
which runs every prefill row of the path (gate prefix, K-Gram, UT solve, W/U,
state correction, output, state pass).  The line also carries the decode
workload (256 x 32 heads, 1000 in-place steps, and 4-token calls) and, unless
--quick, the linear attention, per-channel (KDA), Gated DeltaProduct and
long-context segmented (1 x 8 heads x 65536 tokens, 16 segments) prefills.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]

Prints ONE JSON line on rank 0.  Under torchrun (N > 1) every rank runs its own
full batch (weak scaling, no collective on the data path); timing uses a
barrier plus device synchronisation on both sides and the max over ranks.
The reference arm (--impl reference) times the float64 CPU oracle on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, iter_decode_blocks, make_decode_state, make_prefill_inputs  # noqa: E402

HEADLINE = "gdn_prefill_bf16"
METRIC = "gated-delta prefill tokens/s + % roofline; decode state-update HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# Algorithmic work (bytes: each input read once, each output written once)
# ---------------------------------------------------------------------------

def measured_traffic(workload):
    """DRAM bytes of one launch from the committed ncu capture, or None when the
    kernel source has changed since that capture (the figure would be stale)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        rec = json.load(open(path))[workload]
        src = open(os.path.join(ROOT, rec["source"]), "rb").read()
    except (OSError, KeyError, ValueError):
        return None
    if hashlib.sha256(src).hexdigest() != rec["source_sha256"]:
        return None
    return rec["dram_bytes_read"] + rec["dram_bytes_write"]


def prefill_bytes(w, out_bytes=None):
    """Algorithmic bytes of one prefill launch: q, k, v, g, beta read once, o
    written once, S0 read and S_T written once per head.  By default o is
    counted in the input dtype (o as the pages' layer returns it); ``out_bytes=4``
    counts the fp32 o this benchmark actually writes."""
    in_b = 2 if w.dtype == "bf16" else 4
    if out_bytes is None:
        out_bytes = in_b
    per_tok = (2 * w.dk + w.dv) * in_b + w.dv * out_bytes
    if w.gate == "scalar":
        per_tok += 4
    elif w.gate == "channel":
        per_tok += 4 * w.dk
    if w.update == "delta":
        per_tok += 4
    state = w.dv * w.dk * 4 * ((1 if w.s0_std > 0 else 0) + 1)
    return w.n_heads * (w.T * per_tok + state)


def prefill_flops(w, C=64):
    d = w.dk
    per = (10 * C * d + 6 * d * d) if w.update == "delta" else (4 * C * d + 4 * d * d)
    return w.n_heads * w.T * per


def decode_bytes_per_step(w, out_bytes=4):
    in_b = 2 if w.dtype == "bf16" else 4
    per_head = 2 * w.dv * w.dk * 4 + (2 * w.dk + w.dv) * in_b + w.dv * out_bytes + 4
    if w.update == "delta":
        per_head += 4
    if w.gate == "channel":
        per_head += 4 * (w.dk - 1)
    return w.n_heads * per_head


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [s for s in sm if mx and s > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def to_dev(x, dtype, torch):
    if x is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda().to(dtype).contiguous()


def time_prefill(w, x, steps, warmup, torch, gdn, dist=None, nseg=1):
    """Device-timed steps of gdn_chunk_fwd over the whole batch (of
    gdn_chunk_fwd_segmented with ``nseg`` > 1 segments per sequence, workspace
    allocated once outside the timed region); returns ms/step (max over ranks)."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q, k, v = to_dev(x["q"], dt, torch), to_dev(x["k"], dt, torch), to_dev(x["v"], dt, torch)
    g, beta, S0 = to_dev(x["g"], torch.float32, torch), to_dev(x["beta"], torch.float32, torch), \
        to_dev(x["S0"], torch.float32, torch)
    o = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device="cuda")
    ST = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device="cuda")
    ws = None
    if nseg > 1:
        ws = torch.empty(gdn.segmented_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, nseg), dtype=torch.uint8,
                         device="cuda")

    def step():
        if nseg > 1:
            gdn.chunk_fwd_segmented(q, k, v, g, beta, S0, update=w.update, gate=w.gate, nseg=nseg, o=o, S_T=ST,
                                    workspace=ws)
        else:
            gdn.chunk_fwd(q, k, v, g, beta, S0, update=w.update, gate=w.gate, o=o, S_T=ST)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if gdn.device_status() != 0:
        raise RuntimeError("device status after warm-up: %d" % gdn.device_status())
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dist, "cuda")
    del q, k, v, g, beta, S0, o, ST, ws
    return ms


def time_product(w, nh, steps, warmup, torch, gdn):
    """Device-timed gdn_product_fwd (Gated DeltaProduct, nh substeps per token)
    over workload ``w``'s shape; returns ms/step."""
    from synth import make_product_inputs

    x = make_product_inputs(w, nh)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    t = {k: (None if v is None else to_dev(v, dt if k in ("q", "k", "v") else torch.float32, torch))
         for k, v in x.items()}
    o = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device="cuda")
    ST = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device="cuda")

    def step():
        gdn.product_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], gate=w.gate, o=o, S_T=ST)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(torch.cuda.current_stream())
    for _ in range(steps):
        step()
    e1.record(torch.cuda.current_stream())
    torch.cuda.synchronize()
    if gdn.device_status() != 0:
        raise RuntimeError("device status after product prefill")
    return e0.elapsed_time(e1) / steps


def product_bytes(w, nh, out_bytes=None):
    in_b = 2 if w.dtype == "bf16" else 4
    if out_bytes is None:
        out_bytes = in_b
    per_tok = w.dk * in_b + nh * (w.dk + w.dv) * in_b + w.dv * out_bytes + 4 + 4 * nh
    state = w.dv * w.dk * 4 * ((1 if w.s0_std > 0 else 0) + 1)
    return w.n_heads * (w.T * per_tok + state)


E2E_SLICES = 8


def time_prefill_e2e(w, x, steps, warmup, torch, gdn):
    """Same metric through the public API with pinned host buffers: every step
    is one gdn_chunk_fwd_host call, which copies the inputs host->device, runs
    the prefill and copies o and S_T back, in E2E_SLICES head slices so that
    the two copy directions and the kernels overlap (device workspace allocated
    once, outside the timed region)."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def pin(a, dtype):
        if a is None:
            return None
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dtype).pin_memory()

    hq, hk, hv = pin(x["q"], dt), pin(x["k"], dt), pin(x["v"], dt)
    hg, hb, hS = pin(x["g"], torch.float32), pin(x["beta"], torch.float32), pin(x["S0"], torch.float32)
    ho = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32).pin_memory()
    hST = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hg, hb, hS) if t is not None)
    d2h = ho.numel() * 4 + hST.numel() * 4

    ws = torch.empty(gdn.host_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, w.update, w.gate,
                                              gdn.BF16 if dt == torch.bfloat16 else gdn.F32, gdn.F32, E2E_SLICES),
                     dtype=torch.uint8, device="cuda")

    def step():
        gdn.chunk_fwd_host(hq, hk, hv, hg, hb, hS, update=w.update, gate=w.gate, n_slices=E2E_SLICES, o=ho,
                           S_T=hST, workspace=ws)

    for _ in range(max(1, min(warmup, 2))):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, h2d, d2h


def time_decode(w, n_steps, torch, gdn, warmup=3):
    """Device time of ``n_steps`` consecutive in-place decode steps (inputs of
    every step resident in HBM before timing); returns ms/step."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    S = to_dev(make_decode_state(w), torch.float32, torch)
    dev_in = []
    for _, blk in iter_decode_blocks(w, n_steps):
        dev_in += [{k: to_dev(v, dt if k in ("q", "k", "v") else torch.float32, torch) for k, v in s.items()}
                   for s in blk]
    o = torch.empty((w.B, w.H, 1, w.dv), dtype=torch.float32, device="cuda")

    def run(s):
        gdn.decode_step(s["q"], s["k"], s["v"], s["g"], s["beta"], S, update=w.update, gate=w.gate, o=o)

    for i in range(warmup):
        run(dev_in[i % len(dev_in)])
    S.copy_(to_dev(make_decode_state(w), torch.float32, torch))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in dev_in:
        run(s)
    e1.record(stream)
    torch.cuda.synchronize()
    if gdn.device_status() != 0:
        raise RuntimeError("device status after decode")
    del dev_in, S
    return e0.elapsed_time(e1) / n_steps


def time_decode_multi(w, T, n_calls, torch, gdn, warmup=3):
    """Device time of ``n_calls`` in-place decode calls of ``T`` tokens each (the
    state is read and written once per call); returns ms/call."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    S = to_dev(make_decode_state(w), torch.float32, torch)
    flat = []
    for _, blk in iter_decode_blocks(w, n_calls * T):
        flat += blk
    dev_in = []
    for c in range(n_calls):
        grp = flat[c * T:(c + 1) * T]
        dev_in.append({k: (None if grp[0][k] is None else
                           to_dev(np.concatenate([s[k] for s in grp], axis=2),
                                  dt if k in ("q", "k", "v") else torch.float32, torch)) for k in grp[0]})
    o = torch.empty((w.B, w.H, T, w.dv), dtype=torch.float32, device="cuda")

    def run(s):
        gdn.decode_step(s["q"], s["k"], s["v"], s["g"], s["beta"], S, update=w.update, gate=w.gate, o=o)

    for i in range(warmup):
        run(dev_in[i % len(dev_in)])
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in dev_in:
        run(s)
    e1.record(stream)
    torch.cuda.synchronize()
    if gdn.device_status() != 0:
        raise RuntimeError("device status after multi-token decode")
    del dev_in, S
    return e0.elapsed_time(e1) / n_calls


# The prefill -> decode serving loop: a prompt of SERVE_PROMPT tokens per
# sequence is prefilled (gdn_chunk_fwd writes S_T into the decode state
# buffer), then SERVE_DECODE tokens are generated one at a time in place
# (gdn_decode_step), the forward(x, state) -> (o, state) hand-off of the pages.
SERVE_B, SERVE_H, SERVE_PROMPT, SERVE_DECODE = 32, 32, 1024, 128


def serving_workloads(B=SERVE_B):
    wp = WORKLOADS["gdn_prefill_bf16"].with_(B=B, H=SERVE_H, T=SERVE_PROMPT, name="serve_prompt")
    wd = WORKLOADS["decode_gdn_bf16"].with_(B=B, H=SERVE_H, name="serve_decode")
    return wp, wd


def time_serving_loop(reps, torch, gdn, warmup=1, B=SERVE_B, graph=False):
    """Device time of one serving loop (prefill of the prompt into the state,
    then SERVE_DECODE single-token steps on it); returns (ms per loop, ms of
    the prefill, ms per decode step).  With ``graph`` the decode steps are
    captured once in a CUDA graph and replayed (the prefill runs eagerly)."""
    wp, wd = serving_workloads(B)
    x = make_prefill_inputs(wp)
    dt = torch.bfloat16
    q, k, v = (to_dev(x[n], dt, torch) for n in ("q", "k", "v"))
    g, beta, S0 = (to_dev(x[n], torch.float32, torch) for n in ("g", "beta", "S0"))
    del x
    steps = []
    for _, blk in iter_decode_blocks(wd, SERVE_DECODE):
        steps += [{n: to_dev(a, dt if n in ("q", "k", "v") else torch.float32, torch) for n, a in st.items()}
                  for st in blk]
    S = torch.empty((wp.B, wp.H, wp.dv, wp.dk), dtype=torch.float32, device="cuda")
    o_pf = torch.empty((wp.B, wp.H, wp.T, wp.dv), dtype=torch.float32, device="cuda")
    o_dec = torch.empty((wd.B, wd.H, 1, wd.dv), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]

    def decode_all():
        for st in steps:
            gdn.decode_step(st["q"], st["k"], st["v"], st["g"], st["beta"], S, update=wd.update, gate=wd.gate,
                            o=o_dec)

    cg = None
    if graph:
        decode_all()  # warm (first-use attribute setup happens outside the capture)
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg, stream=side):
            decode_all()
        torch.cuda.synchronize()

    def loop(timed):
        if timed:
            ev[0].record(stream)
        gdn.chunk_fwd(q, k, v, g, beta, S0, update=wp.update, gate=wp.gate, o=o_pf, S_T=S)
        if timed:
            ev[1].record(stream)
        if cg is not None:
            cg.replay()
        else:
            decode_all()
        if timed:
            ev[2].record(stream)

    for _ in range(warmup):
        loop(False)
    torch.cuda.synchronize()
    tot, pf = [], []
    for _ in range(reps):
        loop(True)
        torch.cuda.synchronize()
        tot.append(ev[0].elapsed_time(ev[2]))
        pf.append(ev[0].elapsed_time(ev[1]))
    if gdn.device_status() != 0:
        raise RuntimeError("device status after the serving loop")
    ms, ms_pf = sorted(tot)[len(tot) // 2], sorted(pf)[len(pf) // 2]
    return ms, ms_pf, (ms - ms_pf) / SERVE_DECODE


def time_backward(w, steps, torch, gdn, warmup=1, saved=False, tc=False):
    """Device time of gdn_chunk_bwd (gradients of the prefill) on workload ``w``
    with random upstream gradients of o and S_T; returns ms per call (``tc``:
    with GDN_ALGO_TC, the tensor-core forward's states and the chunkwise
    backward in one call).  With ``saved``: a training step's forward
    gdn_chunk_fwd_states and then gdn_chunk_bwd_states (``tc``:
    gdn_chunk_bwd_tc, the chunkwise tensor-core backward) from its chunk
    states; returns (ms of the forward, ms of the backward) per step."""
    x = make_prefill_inputs(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q, k, v = to_dev(x["q"], dt, torch), to_dev(x["k"], dt, torch), to_dev(x["v"], dt, torch)
    g, beta, S0 = (to_dev(x[n], torch.float32, torch) for n in ("g", "beta", "S0"))
    del x
    gen = torch.Generator(device="cuda").manual_seed(w.seed)
    dO = torch.randn((w.B, w.H, w.T, w.dv), device="cuda", generator=gen)
    dST = torch.randn((w.B, w.H, w.dv, w.dk), device="cuda", generator=gen)
    algo = "tc" if tc and not saved else "auto"
    ws = torch.empty(gdn.bwd_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, w.update, w.gate, algo=algo),
                     dtype=torch.uint8, device="cuda")
    if saved:
        states = ws.view(torch.float32).view(w.B, w.H, (w.T + 63) // 64, w.dv, w.dk)
        o = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device="cuda")
        ST = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device="cuda")
        stream = torch.cuda.current_stream()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        wtc = None
        if tc:
            wtc = torch.empty(gdn.bwd_tc_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, w.update, w.gate),
                              dtype=torch.uint8, device="cuda")
        fw, bw = [], []
        for it in range(warmup + steps):
            ev[0].record(stream)
            gdn.chunk_fwd(q, k, v, g, beta, S0, update=w.update, gate=w.gate, o=o, S_T=ST, states=states)
            ev[1].record(stream)
            if tc:
                gdn.chunk_bwd(q, k, v, g, beta, None, dO, dST, update=w.update, gate=w.gate, states=states,
                              algo="tc", workspace=wtc)
            else:
                gdn.chunk_bwd(q, k, v, g, beta, None, dO, dST, update=w.update, gate=w.gate, states=states)
            ev[2].record(stream)
            torch.cuda.synchronize()
            if it >= warmup:
                fw.append(ev[0].elapsed_time(ev[1]))
                bw.append(ev[1].elapsed_time(ev[2]))
        if gdn.device_status() != 0:
            raise RuntimeError("device status after the saved-state training step")
        return sum(fw) / len(fw), sum(bw) / len(bw)

    def step():
        gdn.chunk_bwd(q, k, v, g, beta, S0, dO, dST, update=w.update, gate=w.gate, workspace=ws,
                      algo="tc" if tc else "token")

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(torch.cuda.current_stream())
    for _ in range(steps):
        step()
    e1.record(torch.cuda.current_stream())
    torch.cuda.synchronize()
    if gdn.device_status() != 0:
        raise RuntimeError("device status after the backward pass")
    return e0.elapsed_time(e1) / steps


def backward_tc_flops(w):
    """Dense MACs x 2 of gdn_chunk_bwd_tc per launch, per chunk of C = 64 tokens
    and head (d = dk = dv): prep (q k^T, k k^T, W = T Mk, A W: 4 C^2 d; the solve
    C^3 / 3), chain (dS Kc^T, X W, dO^T Q~: 3 C d^2), local (W S^T, k dSn^T,
    Z dSn, dO S, dZ S: 5 C d^2; T Mv, A^T dO, dO Z^T, dZ v^T, T^T dZ: 5 C^2 d;
    dW k^T, T^T dW, E k, E^T k, F^T q, F k: 6 C^2 d; dT T^T, T^T Y: 2 C^3)."""
    C, d = 64, w.dk
    nch = (w.T + C - 1) // C
    macs = 4 * C * C * d + C ** 3 / 3 + 3 * C * d * d + 5 * C * d * d + 11 * C * C * d + 2 * C ** 3
    return 2 * macs * nch * w.n_heads


def backward_flops(w):
    """fp32 arithmetic of gdn_chunk_bwd per launch: four forward token steps per
    token (the forward pass, the chunk recompute, the sub-block recompute and the
    S_t of the backward step; 4 dv dk each) and the backward step (dq, dO q^T, du,
    dk, dS', the gate term, the decay: 15 dv dk)."""
    return w.n_heads * w.T * (4 * 4 + 15) * w.dv * w.dk


def max_over_ranks(value, dist, device):
    """Max of a per-rank float over all ranks (timing only; not on the data path)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([float(value)], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_baseline(w, budget_s=15.0):
    """The oracle, as it stands, on a bounded sample of the workload: whole
    sequences of a few heads, sized to roughly ``budget_s`` of CPU time."""
    import oracle

    oracle.build()
    threads = oracle.num_threads()
    probe_T = min(w.T, 1024)
    xs = make_prefill_inputs(w.with_(T=probe_T), heads=[(0, 0)])
    t0 = time.perf_counter()
    oracle.gdn_forward(w.update, w.gate, xs["q"], xs["k"], xs["v"], g=xs["g"], beta=xs["beta"], S0=xs["S0"])
    per_tok = (time.perf_counter() - t0) / probe_T
    # as many whole heads as fit the budget on this host's cores (all of them when
    # the whole workload does)
    n_heads = max(1, min(w.n_heads, int(budget_s * threads / max(per_tok * w.T, 1e-9))))
    heads = [(i // w.H, i % w.H) for i in range(n_heads)]
    xs = make_prefill_inputs(w, heads=heads)
    t0 = time.perf_counter()
    oracle.gdn_forward(w.update, w.gate, xs["q"], xs["k"], xs["v"], g=xs["g"], beta=xs["beta"], S0=xs["S0"])
    dt = time.perf_counter() - t0
    token_heads = n_heads * w.T
    return {"value": token_heads / dt / w.H, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": "%d of %d heads, full T=%d (%d token-heads), float64 C recurrence, %.1f s"
                      % (n_heads, w.n_heads, w.T, token_heads, dt)}


def bench_config(w, world):
    """The workload description both arms print (same keys, same values)."""
    nbytes = prefill_bytes(w, out_bytes=4)
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv, "update": w.update,
            "gate": w.gate, "chunk": w.chunk, "global_batch": w.B * world, "seq_len": w.T,
            "parallelism": "replicas x%d (batch per GPU fixed)" % world,
            "l2": "inputs and outputs (%.2f GB) larger than the 126 MB L2, no flush" % (nbytes / 1e9)}


def roofline(w, ms, peaks, peak_kind):
    """HBM roofline of one prefill launch.  ``frac`` counts the algorithmic bytes
    with o in the input dtype (bf16 here); the kernel writes o in fp32, and
    ``fp32_output`` gives the same figures with those bytes counted."""
    nbytes = prefill_bytes(w)
    nbytes32 = prefill_bytes(w, out_bytes=4)
    flops = prefill_flops(w)
    s = ms * 1e-3
    achieved = nbytes / s / 1e9
    t_roof = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    t_roof32 = max(nbytes32 / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic(w.name), "peak_source": peak_kind,
            "algorithmic_bytes_per_launch": nbytes, "bytes_note": "o counted in the input dtype (bf16)",
            "flops_per_launch": flops, "achieved_tflops": flops / s / 1e12,
            "tensor_frac": flops / s / 1e12 / peaks["bf16_tflops"],
            "roofline_us": t_roof * 1e6, "frac_of_roofline_time": t_roof / s,
            "fp32_output": {"bytes_per_launch": nbytes32, "achieved": nbytes32 / s / 1e9,
                            "frac": nbytes32 / s / 1e9 / peaks["hbm_gbs"], "roofline_us": t_roof32 * 1e6,
                            "note": "o counted as the fp32 tensor the kernel writes"}}


def run_ours(args):
    import torch

    import gated_delta_rule_97_b200 as gdn

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    else:
        torch.cuda.set_device(0)
    gdn.load()
    gdn.device_status(clear=True)
    peaks, peak_kind = load_peaks()

    if args.only == "decode":
        wd = WORKLOADS["decode_gdn_bf16"]
        n_dec = wd.steps if not args.quick else 100
        ms_d = time_decode(wd, n_dec, torch, gdn)
        if rank == 0:
            print(json.dumps({"only": "decode", "ms_per_step": ms_d}), flush=True)
        return
    if args.only == "serving":
        out = {"only": "serving"}
        for B in (SERVE_B, 1):
            for graph in (False, True):
                ms_sv, ms_pf, ms_dec = time_serving_loop(3, torch, gdn, B=B, graph=graph)
                out["B%d_%s" % (B, "graph" if graph else "eager")] = {
                    "ms_per_loop": ms_sv, "ms_prefill": ms_pf, "ms_per_decode_step": ms_dec}
        if rank == 0:
            print(json.dumps(out), flush=True)
        return
    if args.only == "decode_multi":
        wd = WORKLOADS["decode_gdn_bf16"]
        ms_m = time_decode_multi(wd, 4, 25 if args.quick else 100, torch, gdn)
        if rank == 0:
            print(json.dumps({"only": "decode_multi", "tokens_per_call": 4, "ms_per_call": ms_m}), flush=True)
        return
    w = WORKLOADS[args.workload]
    if args.only in ("prefill", "backward"):
        # profiling aids: the workload's distributions on an optionally smaller shape
        w = w.with_(B=args.batch or w.B, H=args.heads or w.H, T=args.seq_len or w.T)
    if args.only == "backward":
        ms = time_backward(w, args.steps, torch, gdn, warmup=args.warmup)
        msf_s, msb_s = time_backward(w, args.steps, torch, gdn, warmup=1, saved=True)
        msf_t, msb_t = time_backward(w, args.steps, torch, gdn, warmup=1, saved=True, tc=True)
        ms_one = time_backward(w, args.steps, torch, gdn, warmup=1, tc=True)
        if rank == 0:
            print(json.dumps({"only": "backward", "workload": w.name, "B": w.B, "H": w.H, "T": w.T,
                              "ms_per_call": ms, "saved_states": {"ms_forward": msf_s, "ms_backward": msb_s},
                              "tensor_core": {"ms_forward": msf_t, "ms_backward": msb_t, "ms_one_call": ms_one}}),
                  flush=True)
        return
    x = make_prefill_inputs(w)
    if args.only == "prefill":
        ms = time_prefill(w, x, args.steps, args.warmup, torch, gdn, dist)
        if rank == 0:
            print(json.dumps({"only": "prefill", "workload": w.name, "ms_per_step": ms}), flush=True)
        return
    with ClockSampler(local) as clk:
        ms = time_prefill(w, x, args.steps, args.warmup, torch, gdn, dist)
    clocks = clk.summary()
    tokens = w.B * w.T
    value = world * tokens / (ms * 1e-3)
    result = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
              "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
              "vs_baseline": None, "dtype": "bf16 in / fp32 state, accumulation, output", "data": "synthetic",
              "config": bench_config(w, world),
              "token_heads_per_s": world * w.n_heads * w.T / (ms * 1e-3),
              "roofline": roofline(w, ms, peaks, peak_kind),
              "gpu_launches": args.steps, "clocks": clocks}

    ms_e2e, h2d, d2h = time_prefill_e2e(w, x, max(2, min(args.steps, 5)), args.warmup, torch, gdn)
    result["e2e"] = {"value": tokens / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                     "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                     "api": "gdn_chunk_fwd_host, %d head slices, pinned host buffers" % E2E_SLICES}
    del x

    wd = WORKLOADS["decode_gdn_bf16"]
    n_dec = wd.steps if not args.quick else 100
    ms_d = max_over_ranks(time_decode(wd, n_dec, torch, gdn), dist, "cuda")
    dbytes = decode_bytes_per_step(wd)
    result["decode"] = {"workload": wd.name, "steps": n_dec, "ms_per_step": ms_d,
                        "value": dbytes / (ms_d * 1e-3) / 1e9, "unit": "GB/s",
                        "frac": dbytes / (ms_d * 1e-3) / 1e9 / peaks["hbm_gbs"],
                        "bytes_per_step": dbytes, "tokens_per_s": wd.n_heads / wd.H * world / (ms_d * 1e-3)}
    result["gpu_launches"] += n_dec
    # T = 4 tokens per call through the same entry point (state read / written once per call)
    T_mt, n_mt = 4, (25 if args.quick else 100)
    ms_mt = max_over_ranks(time_decode_multi(wd, T_mt, n_mt, torch, gdn), dist, "cuda")
    in_b = 2 if wd.dtype == "bf16" else 4
    per_tok = wd.n_heads * ((2 * wd.dk + wd.dv) * in_b + 4 * wd.dv + 8)
    mt_bytes = wd.n_heads * wd.dv * wd.dk * 4 * 2 + T_mt * per_tok
    result["decode"]["multi_token"] = {"tokens_per_call": T_mt, "calls": n_mt, "ms_per_call": ms_mt,
                                       "value": mt_bytes / (ms_mt * 1e-3) / 1e9, "unit": "GB/s",
                                       "frac": mt_bytes / (ms_mt * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                       "bytes_per_call": mt_bytes,
                                       "tokens_per_s": wd.B * T_mt * world / (ms_mt * 1e-3)}
    result["gpu_launches"] += n_mt

    if not args.quick:
        others = {}
        for name in ("linear_attn_bf16", "kda_prefill_bf16"):
            wo = WORKLOADS[name]
            xo = make_prefill_inputs(wo)
            mso = time_prefill(wo, xo, max(3, args.steps // 2), args.warmup, torch, gdn, dist)
            result["gpu_launches"] += max(3, args.steps // 2)
            del xo
            rf = roofline(wo, mso, peaks, peak_kind)
            others[name] = {"kernel": "chunk_la (additive, 128-token chunks)" if wo.update == "additive"
                            else "chunk_tc2 (pipelined, 64-token chunks)",
                            "ms_per_step": mso, "tokens_per_s": wo.B * wo.T * world / (mso * 1e-3),
                            "achieved_gbs": rf["achieved"], "roofline_us": rf["roofline_us"],
                            "frac_of_roofline_time": rf["frac_of_roofline_time"],
                            "frac_fp32_output": rf["fp32_output"]["frac"]}
        # Gated DeltaProduct with the pages' 3 substeps per token, on the GDN workload's
        # heads and 2731 tokens (8193 virtual steps, about the GDN workload's length)
        wp, nh = WORKLOADS["gdn_prefill_bf16"].with_(T=2731, name="gdp_prefill_bf16"), 3
        msp = max_over_ranks(time_product(wp, nh, max(3, args.steps // 2), args.warmup, torch, gdn), dist, "cuda")
        nb = product_bytes(wp, nh)
        fl = prefill_flops(wp.with_(T=wp.T * nh))
        tr = max(nb / (peaks["hbm_gbs"] * 1e9), fl / (peaks["bf16_tflops"] * 1e12))
        others["gdp_prefill_bf16"] = {"substeps": nh, "B": wp.B, "H": wp.H, "T": wp.T, "ms_per_step": msp,
                                      "tokens_per_s": wp.B * wp.T * world / (msp * 1e-3),
                                      "achieved_gbs": nb / (msp * 1e-3) / 1e9, "roofline_us": tr * 1e6,
                                      "frac_of_roofline_time": tr / (msp * 1e-3)}
        result["gpu_launches"] += max(3, args.steps // 2)
        # Long context, few heads: 8 heads of 65536 tokens occupy 8 of the 148 SMs in
        # gdn_chunk_fwd; gdn_chunk_fwd_segmented runs 16 segments per sequence in
        # parallel (4 launches per call: zero-state pass, transition pass,
        # composition, output pass)
        wl, nseg = WORKLOADS["gdn_prefill_bf16"].with_(B=1, H=8, T=65536, name="gdn_long_bf16"), 16
        xl = make_prefill_inputs(wl)
        ns = max(3, args.steps // 2)
        ms1 = time_prefill(wl, xl, ns, args.warmup, torch, gdn, dist)
        msn = time_prefill(wl, xl, ns, args.warmup, torch, gdn, dist, nseg=nseg)
        del xl
        result["gpu_launches"] += ns * (1 + 4)
        nb = prefill_bytes(wl)
        others["gdn_long_bf16"] = {"B": wl.B, "H": wl.H, "T": wl.T, "nseg": nseg,
                                   "ms_per_step_unsegmented": ms1, "ms_per_step": msn,
                                   "tokens_per_s": wl.B * wl.T * world / (msn * 1e-3),
                                   "speedup_vs_unsegmented": ms1 / msn,
                                   "achieved_gbs": nb / (msn * 1e-3) / 1e9,
                                   "frac_of_roofline_time": nb / (peaks["hbm_gbs"] * 1e9) / (msn * 1e-3)}
        result["prefill_workloads"] = others
        # the prefill -> decode serving loop (second workload), eager and with the
        # decode steps replayed from one CUDA graph, at 32 and at 1 sequence
        sv = {"H": SERVE_H, "prompt_tokens": SERVE_PROMPT, "decode_tokens": SERVE_DECODE,
              "note": "gdn_chunk_fwd writes S_T into the decode state, then gdn_decode_step runs in place; "
                      "graph: the decode steps captured once in a CUDA graph and replayed"}
        for B in (SERVE_B, 1):
            for graph in (False, True):
                ms_sv, ms_pf, ms_dec = time_serving_loop(3, torch, gdn, B=B, graph=graph)
                ms_sv = max_over_ranks(ms_sv, dist, "cuda")
                result["gpu_launches"] += 3 * (1 + SERVE_DECODE)
                sv["B%d_%s" % (B, "graph" if graph else "eager")] = {
                    "ms_per_loop": ms_sv, "ms_prefill": ms_pf, "ms_per_decode_step": ms_dec,
                    "tokens_per_s": B * (SERVE_PROMPT + SERVE_DECODE) * world / (ms_sv * 1e-3),
                    "decode_tokens_per_s": B * world / (ms_dec * 1e-3)}
        result["serving_loop"] = sv
        # training backward (gdn_chunk_bwd) on the GDN workload
        nb_steps = 2
        msb = max_over_ranks(time_backward(w, nb_steps, torch, gdn), dist, "cuda")
        result["gpu_launches"] += nb_steps * 5  # four output zeroings and the kernel per call
        fl = backward_flops(w)
        fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12  # FP32 lanes x FMA x max SM clock
        result["backward"] = {"workload": w.name, "ms_per_call": msb,
                              "tokens_per_s": w.B * w.T * world / (msb * 1e-3),
                              "flops_per_call": fl, "achieved_tflops": fl / (msb * 1e-3) / 1e12,
                              "bound": "alu", "fp32_peak_tflops": fp32_peak,
                              "frac": fl / (msb * 1e-3) / 1e12 / fp32_peak}
        # the same gradients from the chunk states a training forward saved
        msf_s, msb_s = time_backward(w, nb_steps, torch, gdn, saved=True)
        msf_s, msb_s = max_over_ranks(msf_s, dist, "cuda"), max_over_ranks(msb_s, dist, "cuda")
        result["gpu_launches"] += (nb_steps + 1) * 6
        result["backward"]["from_saved_states"] = {
            "ms_forward_with_states": msf_s, "ms_backward": msb_s,
            "note": "gdn_chunk_fwd_states (tensor-core forward writing the chunk-entry states), then "
                    "gdn_chunk_bwd_states (no forward pass of its own)"}
        # the chunkwise tensor-core backward from the same saved states
        msf_t, msb_t = time_backward(w, nb_steps, torch, gdn, saved=True, tc=True)
        msf_t, msb_t = max_over_ranks(msf_t, dist, "cuda"), max_over_ranks(msb_t, dist, "cuda")
        result["gpu_launches"] += (nb_steps + 1) * 4  # the forward kernel, then prep, chain, local
        fl_tc = backward_tc_flops(w)
        tf32_peak = peaks["bf16_tflops"] / 2.0
        result["backward"]["tensor_core"] = {
            "ms_forward_with_states": msf_t, "ms_backward": msb_t,
            "tokens_per_s": w.B * w.T * world / (msb_t * 1e-3),
            "flops_per_call": fl_tc, "achieved_tflops": fl_tc / (msb_t * 1e-3) / 1e12,
            "bound": "tensor", "tf32_peak_tflops": tf32_peak,
            "frac": fl_tc / (msb_t * 1e-3) / 1e12 / tf32_peak,
            "note": "gdn_chunk_bwd_tc: prep, state-gradient chain and local kernels on tf32 warp MMAs; "
                    "peak = measured bf16 dense x 1/2 (the nominal tf32 : bf16 ratio)"}
        # gdn_chunk_bwd with GDN_ALGO_TC: the states from its own tensor-core forward, one call
        ms_one = max_over_ranks(time_backward(w, nb_steps, torch, gdn, tc=True), dist, "cuda")
        result["gpu_launches"] += (nb_steps + 1) * 4
        result["backward"]["tensor_core"]["ms_one_call"] = ms_one

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_reference(args):
    """The oracle as the reference arm: float64 CPU recurrence on a bounded
    sample per step (one whole head sequence per step), on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    oracle.build()
    w = WORKLOADS[args.workload]
    threads = oracle.num_threads()
    heads = [(i // w.H, i % w.H) for i in range(threads)]
    xs = make_prefill_inputs(w, heads=heads)
    run = lambda: oracle.gdn_forward(w.update, w.gate, xs["q"], xs["k"], xs["v"], g=xs["g"], beta=xs["beta"],
                                     S0=xs["S0"])
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    value = len(heads) * w.T / dt / w.H
    sample = "%d of %d heads per step, full T=%d, float64 C oracle" % (len(heads), w.n_heads, w.T)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
        flush=True)


def relaunch(n_procs):
    """``--gpus N`` (N > 1) started as a single process: start N ranks of this
    script on one node with torch.distributed.run (rendezvous on 127.0.0.1) and
    return the launcher's exit status."""
    import socket

    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=%d" % n_procs,
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def launch_check(args):
    """The rank protocol alone, on CPU (gloo): every rank joins, takes the same
    barrier and max-over-ranks steps as a timed run, and rank 0 prints the line's
    rank-dependent keys.  No GPU work; a test of the launcher."""
    import datetime

    import torch.distributed as tdist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        tdist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        dist = tdist
        dist.barrier()
    ms = max_over_ranks(1.0 + rank, dist, "cpu")
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"launch_check": True, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": ms}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=[k for k, w in WORKLOADS.items() if w.steps == 0])
    ap.add_argument("--quick", action="store_true", help="skip the extra prefill workloads; 100 decode steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="with --only prefill/backward: override B")
    ap.add_argument("--heads", type=int, default=0, help="with --only prefill/backward: override H")
    ap.add_argument("--seq-len", type=int, default=0, help="with --only prefill/backward: override T")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "decode_multi", "backward", "serving"], default="all",
                    help="profiling aid: run one part only (its line is not a benchmark result)")
    ap.add_argument("--launch-check", action="store_true",
                    help="test aid: run only the rank protocol on CPU (gloo), no GPU work")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        sys.exit(relaunch(args.gpus))
    if env_world is not None and int(env_world) != args.gpus:
        ap.error("--gpus %d but WORLD_SIZE=%s" % (args.gpus, env_world))
    if args.launch_check:
        launch_check(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

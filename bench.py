#!/usr/bin/env python
"""Decode throughput of windowed INT8 GDN decode on B200, with its comparators.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one window of the workload for every one of L rotated layer-states:
W decode launches per layer (one token for all 64 x 32 (sequence, head) units
per launch) followed by one window flush per layer.  The L layer-states (4 by
default, ~540 MB together) are visited round-robin like the layers of a model,
so no layer's state is still in the 126 MB L2 when it is read again; L2 is not
flushed.  value = decode tokens/s per layer = batch x W x L / step time.

Also reported: the FP32-state and naive per-token INT8 decode kernels on the
same inputs, the roofline of the dominant kernel (windowed decode, algorithmic
bytes / event-timed duration vs the measured HBM copy bandwidth), an
end-to-end number through the public API with host buffers, the oracle on the
host cores, and the SM clocks sampled during the timed region.

Under torchrun each rank runs its own batch of sequences (independent units,
no collective on the data path); rank 0 prints the JSON line with the
whole-job value, timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from recurrent_state_quantization_lq_b200 import inputs, ranks  # noqa: E402

METRIC = "decode tokens/s per layer & achieved HBM GB/s vs 8 TB/s roofline (INT8 vs FP32 state)"
UNIT = "tokens/s per layer"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------ byte accounting

def decode_window_bytes(d: int, in_b: int, kda: bool, ncr: int, ncc: int, n_buf: int) -> int:
    """Algorithmic HBM bytes one (sequence, head) unit moves in one windowed
    decode step with n_buf tokens buffered."""
    cis = ((ncr + ncc + 3) // 4) * 4
    fixed = d * d + 4 * d + 4 * d            # INT8 tile, row scales, smoothing factors
    fixed += 3 * in_b * d + 4                # q, k, v, beta
    fixed += 4 * cis + 4 * d * (ncr + ncc)   # compensators
    fixed += 4 * d + 4 * d                   # o written, delta_t appended
    if kda:
        fixed += 4 * d + 8 * d + 8 * d       # g read, G read + written
        fixed += 4 * d                       # kappa_t appended
        per_entry = 4 * d + 4 * d            # delta_j, kappa_j
    else:
        fixed += 4 + 8 + 8 + 4               # g read, G read + written, exp(-G_t) appended
        fixed += in_b * d                    # k_t appended
        per_entry = 4 * d + in_b * d + 4     # delta_j, k_j, exp(-G_j)
    return fixed + per_entry * n_buf


def flush_bytes(d: int, in_b: int, kda: bool, ncr: int, ncc: int, n_buf: int) -> int:
    """Algorithmic bytes of one unit's window flush (read the window-start state
    and the buffer, write the new state)."""
    cis = ((ncr + ncc + 3) // 4) * 4
    state = d * d + 8 * d + 4 * cis + 4 * d * (ncr + ncc)
    gd = d if kda else 1
    entry = 4 * d + (4 * d if kda else in_b * d + 4)
    return 2 * state + 2 * 8 * gd + entry * n_buf


def fp32_bytes(d: int, in_b: int, kda: bool) -> int:
    return 8 * d * d + 3 * in_b * d + 4 + (4 * d if kda else 4) + 4 * d


def naive_bytes(d: int, in_b: int, kda: bool) -> int:
    return 2 * (d * d + 4 * d) + 3 * in_b * d + 4 + (4 * d if kda else 4) + 4 * d


# --------------------------------------------------------------- environment

def profiled_traffic(workload: str, kernel: str) -> tuple[int | None, str]:
    """DRAM bytes (read + write) per launch from the committed ncu summary of
    `kernel` on `workload`, or None when there is none or when a kernel source
    it names has changed since the capture (its sha256 no longer matches)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None, "no ncu capture of this workload"
    srcs = re.findall(r"^kernel-source: (\S+) sha256 ([0-9a-f]{64})$", text, re.M)
    m = re.search(r"^traffic_bytes_per_launch: (\d+)$", text, re.M)
    if not srcs or not m:
        return None, "capture has no traffic figure"
    for rel, digest in srcs:
        with open(os.path.join(ROOT, "recurrent_state_quantization_lq_b200", rel), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != digest:
                return None, f"kernel changed since the capture ({rel})"
    return int(m.group(1)), f"ncu dram__bytes_read.sum + dram__bytes_write.sum, profiles/{kernel}_{workload}.md"


def measured_hbm_gbs() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        try:
            p = torch.cuda.get_device_properties(device_index)
            self.gpu = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            self.gpu = str(device_index)
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# -------------------------------------------------------------- distributed

def dist_setup(n_gpus: int):
    rank, world, local = ranks.env_ranks()
    if world > 1:
        torch.cuda.set_device(local)
        ranks.init("nccl", torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    ranks.barrier(world)


def max_over_ranks(x: float, world: int) -> float:
    return ranks.max_over_ranks(x, world, device=torch.device("cuda", torch.cuda.current_device()))


# ------------------------------------------------------------ the CPU oracle

def oracle_sample(wl: inputs.Workload, n_units: int, n_tokens: int, n_threads: int, seed: int) -> tuple[float, int]:
    """Time the oracle's windowed decode on a sample of units; returns
    (seconds, threads used)."""
    import numpy as np

    import oracle
    d = wl.d_k
    gate = oracle.GATE_CHANNEL if wl.per_channel_gate else oracle.GATE_SCALAR
    p = oracle.Params(d, d, window=wl.window, n_comp_rows=wl.n_comp_rows, n_comp_cols=wl.n_comp_cols,
                      gate=gate, mode=oracle.MODE_WINDOW)
    tb = inputs.tokens(seed, 0, n_tokens, 1, n_units, d, d, wl.per_channel_gate, wl.dtype)

    def heads(x):
        return x.reshape(n_tokens, n_units, *x.shape[3:]).transpose(0, 1).double().numpy()

    S0 = 0.1 * torch.randn(n_units, d, d, generator=torch.Generator().manual_seed(seed)).double().numpy()
    args = (heads(tb.q), heads(tb.k), heads(tb.v), heads(tb.g), heads(tb.beta))
    used = oracle.max_threads(n_threads)
    t0 = time.perf_counter()
    oracle.run(p, S0, *args, snapshots=False, n_threads=n_threads)
    return time.perf_counter() - t0, used


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ our arm

class LayerStack:
    """L independent layer-states of one workload, their token inputs and
    CUDA graphs of each window (decode launches, then flushes)."""

    def __init__(self, wl, n_layers, mode, device, seed, tokens_per_layer, prefill_states=None, ragged=False):
        from recurrent_state_quantization_lq_b200 import lq
        gate = "channel" if wl.per_channel_gate else "scalar"
        self.wl, self.mode, self.L = wl, mode, n_layers
        self.states = [lq.DecodeState(wl.batch, wl.heads, wl.d_k, window=wl.window,
                                      n_comp_rows=wl.n_comp_rows, n_comp_cols=wl.n_comp_cols, gate=gate,
                                      mode=mode, in_dtype=wl.dtype, ragged=ragged, device=device)
                       for _ in range(n_layers)]
        self.tok = [inputs.tokens_on_device(seed * 100 + l, tokens_per_layer, wl.batch, wl.heads, wl.d_k,
                                            wl.d_v, wl.per_channel_gate, wl.dtype, device)
                    for l in range(n_layers)]
        self.out = torch.empty(n_layers, wl.batch, wl.heads, wl.d_v, dtype=torch.float32, device=device)
        for l, st in enumerate(self.states):
            st.prefill(prefill_states[l] if prefill_states is not None else None)
        self.T = tokens_per_layer
        # the states and tokens were made on the current stream; the graphs run on another
        torch.cuda.synchronize()

    def decode(self, l, t, active=None):
        tb = self.tok[l]
        self.states[l].decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t], out=self.out[l], active=active)

    def capture(self, window_index, stream):
        """Two graphs for one window: W x L decode launches, then L flushes."""
        W = self.wl.window
        gd, gf = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd, stream=stream):
            for i in range(W):
                t = (window_index * W + i) % self.T
                for l in range(self.L):
                    self.decode(l, t)
        with torch.cuda.graph(gf, stream=stream):
            for st in self.states:
                st.flush()
        return gd, gf


def fp32_prefill(wl, n_layers, device, seed):
    """Per layer: the FP32 recurrence over the workload's prefill tokens from
    zero (one lq_prefill_tokens launch on an FP32-state handle)."""
    from recurrent_state_quantization_lq_b200 import lq
    gate = "channel" if wl.per_channel_gate else "scalar"
    S = []
    for l in range(n_layers):
        st = lq.DecodeState(wl.batch, wl.heads, wl.d_k, gate=gate, mode="fp32", in_dtype=wl.dtype, device=device)
        tb = inputs.tokens_on_device(seed * 100 + 50 + l, wl.prefill_tokens, wl.batch, wl.heads, wl.d_k, wl.d_v,
                                     wl.per_channel_gate, wl.dtype, device)
        st.prefill_tokens(tb.q, tb.k, tb.v, tb.g, tb.beta)
        S.append(st.read("state_f32", device=st.device))
        del st, tb
    torch.cuda.synchronize()
    return S


def run_e2e(win, wl, dev, L: int, W: int, K: int, args, world: int) -> dict:
    """The step through the public binding with the inputs in pinned host
    memory: every step copies each token's q, k, v, g, beta (all layers, one
    packed buffer per token position) to the device, decodes that token
    through the L layers (a CUDA graph of the binding's calls per token
    position; the window's last token also flushes every layer) and copies
    the token's outputs back.  Copies in, compute and copies out run on three
    streams over a 4-deep ring of device buffers, so token t's outputs
    travel while token t + 1 computes and token t + 2 arrives."""
    R = 4
    assert W % R == 0 or W < R
    Ke = max(2, min(K, args.e2e_steps))
    B, H, d = wl.batch, wl.heads, wl.d_k
    parts = [(l, name) for l in range(L) for name in ("q", "k", "v", "g", "beta")]
    src = {(l, n): getattr(win.tok[l], n)[:W] for l, n in parts}
    sizes = [src[p][0].numel() * src[p].element_size() for p in parts]
    offs = [0]
    for z in sizes:
        offs.append(offs[-1] + (z + 255) // 256 * 256)
    tok_bytes = offs[-1]
    host_in = torch.empty(W, tok_bytes, dtype=torch.uint8).pin_memory()
    for i in range(W):
        for p, o, z in zip(parts, offs, sizes):
            host_in[i, o:o + z].copy_(src[p][i].contiguous().view(torch.uint8).reshape(-1).cpu())
    out_bytes = L * B * H * d * 4
    host_out = torch.empty(W, out_bytes, dtype=torch.uint8).pin_memory()
    dev_in = torch.empty(R, tok_bytes, dtype=torch.uint8, device=dev)
    dev_out = torch.empty(R, L, B, H, d, dtype=torch.float32, device=dev)

    def view(r, p):
        l, n = p
        j = parts.index(p)
        t = src[p]
        return dev_in[r, offs[j]:offs[j] + sizes[j]].view(t.dtype).view(t.shape[1:])

    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    graphs = []
    torch.cuda.synchronize()
    for i in range(W):
        r = i % R
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s_comp):
            for l in range(L):
                win.states[l].decode_step(view(r, (l, "q")), view(r, (l, "k")), view(r, (l, "v")),
                                          view(r, (l, "g")), view(r, (l, "beta")), out=dev_out[r, l])
            if i == W - 1:
                for st in win.states:
                    st.flush()
        graphs.append(g)
    ev = {k: [torch.cuda.Event() for _ in range(R)] for k in ("in", "comp", "out")}

    def step():
        for i in range(W):
            r = i % R
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev["comp"][r])          # the slot's previous inputs are consumed
                dev_in[r].copy_(host_in[i], non_blocking=True)
                ev["in"][r].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev["in"][r])
                s_comp.wait_event(ev["out"][r])         # the slot's previous outputs are on the host
                graphs[i].replay()
                ev["comp"][r].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["comp"][r])
                host_out[i].copy_(dev_out[r].view(torch.uint8).reshape(-1), non_blocking=True)
                ev["out"][r].record(s_out)

    for e in ev.values():
        for x in e:
            x.record(s_out)
    step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_comp.wait_event(e0)
    s_out.wait_event(e0)
    for _ in range(Ke):
        step()
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / Ke
    del graphs
    return {"value": ranks.whole_job_rate(B * W * L, world, ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": W * sum(sizes), "d2h_bytes_per_step": W * out_bytes,
            "path": "DecodeState.decode_step/flush (C ABI) per token through all layers, in CUDA graphs; "
                    "pinned host inputs copied in and outputs copied out every token on separate streams"}


def bench_config(wl, layers: int, world: int) -> dict:
    """The `config` of the bench line, the same for both arms."""
    d, W = wl.d_k, wl.window
    return {"workload": wl.name, "batch_per_gpu": wl.batch, "global_batch": wl.batch * world,
            "heads": wl.heads, "d_k": d, "d_v": d, "window": W, "n_comp": wl.n_comp_rows + wl.n_comp_cols,
            "gate": "per-key-channel (KDA)" if wl.per_channel_gate else "scalar (GDN)",
            "state": "int8 + fp32 buffer",
            "inputs": "bf16 q/k/v, fp32 g/beta" if wl.dtype == torch.bfloat16 else "fp32",
            "layers_rotated": layers,
            "step": f"one window per layer: {W} decode launches + 1 flush, x{layers} layers",
            "l2": f"not flushed; {layers} layer-states rotated, working set > L2",
            "parallelism": f"dp{world} (independent sequences per GPU, no collective)"}


def run_ours(args, rank, world, local):
    from recurrent_state_quantization_lq_b200 import lq
    dev = torch.device("cuda", local)
    wl = inputs.WORKLOADS[args.workload]
    L, W, K, WU = args.layers, wl.window, args.steps, args.warmup
    d, kda = wl.d_k, wl.per_channel_gate
    in_b = 2 if wl.dtype == torch.bfloat16 else 4
    ncr, ncc = wl.n_comp_rows, wl.n_comp_cols
    seed = ranks.shard_seed(wl.seed, rank)
    stream = torch.cuda.Stream(device=dev)
    n_windows = max(1, wl.decode_tokens // W)

    S0 = fp32_prefill(wl, L, dev, seed)
    win = LayerStack(wl, L, "window", dev, seed, wl.decode_tokens, S0)
    # warm-up launches outside capture (sets kernel attributes)
    with torch.cuda.stream(stream):
        for l in range(L):
            win.decode(l, 0)
            win.states[l].flush()
    torch.cuda.synchronize()
    graphs = []
    for wi in range(n_windows):
        graphs.append(win.capture(wi, stream))
    torch.cuda.synchronize()

    def run_steps(n, first, evs=None):
        with torch.cuda.stream(stream):
            for s in range(n):
                gd, gf = graphs[(first + s) % n_windows]
                if evs is not None:
                    evs[s][0].record(stream)
                gd.replay()
                if evs is not None:
                    evs[s][1].record(stream)
                gf.replay()
                if evs is not None:
                    evs[s][2].record(stream)

    run_steps(WU, 0)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        run_steps(K, WU, evs)
        end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_total = max_over_ranks(start.elapsed_time(end), world)
    ms_step = ms_total / K
    dec_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    fl_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    for st in win.states:
        assert st.device_status(stream) == lq.LQ_OK, lq.last_error()

    units = wl.batch * wl.heads
    # algorithmic bytes of all decode launches and flushes in the timed region
    dec_bytes = K * L * units * sum(decode_window_bytes(d, in_b, kda, ncr, ncc, n) for n in range(W))
    fl_bytes = K * L * units * flush_bytes(d, in_b, kda, ncr, ncc, W)
    n_dec = K * L * W
    dec_avg_us = dec_ms * 1e3 / n_dec
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_gbs()
    # weak scaling: the job's tokens are every rank's tokens over the slowest rank's time
    value = ranks.whole_job_rate(wl.batch * W * L * K, world, ms_total * 1e-3)

    # ---- comparators on the same workload (same inputs recipe, same rotation)
    comps = {}
    Kc = max(4, min(K, args.comparator_steps))
    for mode, nbytes in (("fp32", fp32_bytes(d, in_b, kda)), ("naive", naive_bytes(d, in_b, kda))):
        stk = LayerStack(wl, L, mode, dev, seed, W, S0)
        with torch.cuda.stream(stream):
            for l in range(L):
                stk.decode(l, 0)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(W):
                for l in range(L):
                    stk.decode(l, i)
        with torch.cuda.stream(stream):
            for _ in range(2):
                g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(Kc):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world) / Kc
        comps[mode] = {"value": ranks.whole_job_rate(wl.batch * W * L, world, ms * 1e-3), "ms_per_step": ms,
                       "hbm_gbs": units * nbytes * W * L / (ms * 1e-3) / 1e9,
                       "bytes_per_unit_token": nbytes}
        del g, stk
        torch.cuda.synchronize()

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(win, wl, dev, L, W, K, args, world)

    # ---- the oracle on the host cores (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = host_cores()
        n_units = min(units, 8 * threads)
        n_tok = args.cpu_tokens
        secs, used = oracle_sample(wl, n_units, n_tok, threads, seed)
        cpu = {"value": n_units * n_tok / wl.heads / secs, "unit": UNIT, "cores": used, "kind": "oracle",
               "sample": f"{n_units} (sequence, head) units x {n_tok} decode tokens of {wl.name} "
                         f"(windowed mode, W={W}, dense FP64 recurrence), {secs:.1f} s"}

    clocks = clk.summary()
    traffic, traffic_src = profiled_traffic(wl.name, "decode_window")
    roofline = {"bound": "hbm", "kernel": "decode_window_kernel", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": f"{peak_kind} HBM copy (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s", "traffic": traffic,
                "traffic_source": traffic_src,
                "frac_of_nominal_8TBs": achieved / NOMINAL_HBM_GBS,
                "avg_launch_us": dec_avg_us, "bytes_per_launch": dec_bytes / n_dec}
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": WU,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": bench_config(wl, L, world),
        "hbm_gbs": achieved,
        "decode_ms_per_step": dec_ms / K, "flush_ms_per_step": fl_ms / K,
        "flush_gbs": fl_bytes / (fl_ms * 1e-3) / 1e9,
        "fp32_state": comps["fp32"], "naive_int8": comps["naive"],
        "speedup_vs_fp32_state": value / comps["fp32"]["value"],
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": K * L * (W + 1), "clocks": clocks,
    }
    return res


# ------------------------------------------------------------ reference arm

def quality(wl, dev, n_tokens: int | None = None, smooth: int = 1) -> dict:
    """Windowed INT8, naive per-token INT8 and the FP32 state decode the same
    inputs from the same start state; the output error of each INT8 mode
    against the FP32 state, relative L2 per window and overall.

    Tokens are drawn per window on the device (seed = workload seed x 1000 +
    window index), so the run needs no more than one window of inputs."""
    from recurrent_state_quantization_lq_b200 import lq
    B, H, d, W = wl.batch, wl.heads, wl.d_k, wl.window
    T = n_tokens or wl.decode_tokens
    gate = "channel" if wl.per_channel_gate else "scalar"
    seed = wl.seed * 1000
    if wl.planted:
        S0 = inputs.planted_state(seed, B, H, d, d)[0].to(dev)
    elif wl.prefill_tokens:
        S0 = fp32_prefill(wl, 1, dev, seed)[0]
    else:
        S0 = None
    states = {m: lq.DecodeState(B, H, d, window=W, n_comp_rows=wl.n_comp_rows, n_comp_cols=wl.n_comp_cols,
                                gate=gate, mode=m, in_dtype=wl.dtype, device=dev,
                                smooth=smooth if m == "window" else 1)
              for m in ("window", "naive", "fp32")}
    for st in states.values():
        st.prefill(S0)
    out = {m: torch.empty(B, H, d, dtype=torch.float32, device=dev) for m in states}
    n_win = (T + W - 1) // W
    acc = torch.zeros(n_win, 3, dtype=torch.float64, device=dev)   # windowed, naive, reference energy
    for wi in range(n_win):
        n = min(W, T - wi * W)
        tb = inputs.tokens_on_device(seed + wi, n, B, H, d, d, wl.per_channel_gate, wl.dtype, dev)
        for i in range(n):
            for m, st in states.items():
                st.decode_step(tb.q[i], tb.k[i], tb.v[i], tb.g[i], tb.beta[i], out=out[m])
            ref = out["fp32"].double()
            acc[wi, 0] += (out["window"].double() - ref).square().sum()
            acc[wi, 1] += (out["naive"].double() - ref).square().sum()
            acc[wi, 2] += ref.square().sum()
        states["window"].flush()
    for st in states.values():
        if st.device_status() != lq.LQ_OK:
            raise RuntimeError(f"device error: {lq.last_error()}")
    a = acc.cpu()
    per = (a[:, :2] / a[:, 2:3]).sqrt()
    tot = (a[:, :2].sum(0) / a[:, 2].sum()).sqrt()
    return {"rel_l2_windowed_vs_fp32": float(tot[0]), "rel_l2_naive_vs_fp32": float(tot[1]),
            "naive_over_windowed": float(tot[1] / tot[0]) if tot[0] > 0 else None,
            "per_window": {"windowed": [float(x) for x in per[:, 0]], "naive": [float(x) for x in per[:, 1]]},
            "tokens": T, "units": B * H}


def sweep(dev, batches=(1, 8, 64, 256, 512), windows=(16, 32, 64, 128, 256), reps: int = 5) -> list[dict]:
    """Decode throughput of windowed INT8, naive per-token INT8 and the FP32
    state over a batch x window grid (32 heads, 128 x 128, n_c = 4).  Each
    point rotates enough layer-states to exceed L2 where the graph size
    allows (at most 8192 launches per captured window); start states are
    N(0, 0.3^2) (the state's values do not change the work)."""
    from recurrent_state_quantization_lq_b200 import lq
    L2 = 126 * 2 ** 20
    stream = torch.cuda.Stream(device=dev)
    rows = []
    for B in batches:
        for W in windows:
            wl = inputs.sweep_workload(B, W)
            d, units = wl.d_k, B * wl.heads
            for mode in ("window", "naive", "fp32"):
                if mode != "window" and W != windows[0]:
                    continue                      # the comparators do not depend on W
                per_state = lq.workspace_bytes(lq.make_config(B, wl.heads, d, window=W, n_comp_rows=2,
                                                              n_comp_cols=2, mode=mode, in_dtype=wl.dtype))
                L = max(2, min(-(-4 * L2 // per_state), 8192 // W, 256))
                S0 = [0.3 * torch.randn(B, wl.heads, d, d, device=dev) for _ in range(min(L, 4))]
                stk = LayerStack(wl, L, mode, dev, wl.seed, W, [S0[l % len(S0)] for l in range(L)])
                del S0
                with torch.cuda.stream(stream):
                    for l in range(L):
                        stk.decode(l, 0)
                        stk.states[l].flush()
                torch.cuda.synchronize()
                if mode == "window":
                    gd, gf = stk.capture(0, stream)
                else:                                   # no flush: one graph of decode launches
                    gd, gf = torch.cuda.CUDAGraph(), None
                    with torch.cuda.graph(gd, stream=stream):
                        for i in range(W):
                            for l in range(L):
                                stk.decode(l, i)
                graphs = [g for g in (gd, gf) if g is not None]
                with torch.cuda.stream(stream):
                    for g in graphs:
                        g.replay()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    for _ in range(reps):
                        for g in graphs:
                            g.replay()
                    e1.record(stream)
                torch.cuda.synchronize()
                for st in stk.states:
                    assert st.device_status(stream) == lq.LQ_OK, lq.last_error()
                ms = e0.elapsed_time(e1) / reps               # one window for every layer-state
                if mode == "window":
                    nb = sum(decode_window_bytes(d, 2, False, 2, 2, n) for n in range(W)) / W + \
                        flush_bytes(d, 2, False, 2, 2, W) / W
                elif mode == "naive":
                    nb = naive_bytes(d, 2, False)
                else:
                    nb = fp32_bytes(d, 2, False)
                rows.append({"batch": B, "window": W if mode == "window" else None, "mode": mode,
                             "tokens_per_s_per_layer": B * W * L / (ms * 1e-3),
                             "hbm_gbs": units * nb * W * L / (ms * 1e-3) / 1e9,
                             "bytes_per_unit_token": nb, "layers_rotated": L,
                             "l2": "working set > L2" if L * per_state > L2 else "working set fits in L2"})
                del gd, gf, graphs, stk
                torch.cuda.synchronize()
    return rows


def ragged_phases(dev, wl, L: int = 4, reps: int = 20) -> list[dict]:
    """Continuous batching: sequence b of every layer-state starts its window b mod W
    tokens in, so each step completes the windows of about B / W sequences.  A step
    is one decode of every sequence and one flush of the full windows, per layer.
    'serial' runs each layer's flush after its decode on one stream; 'overlap' runs
    it on a second stream, joined before that layer's next decode, so it overlaps
    the decodes of the later layers.  Beside them, on the same inputs: 'lockstep'
    (a shared-phase handle, one flush per window) and 'aligned' (a ragged handle
    used without masks, so all sequences stay in one phase, flushed every step)."""
    from recurrent_state_quantization_lq_b200 import lq
    W, B, d = wl.window, wl.batch, wl.d_k
    in_b = 2 if wl.dtype == torch.bfloat16 else 4
    ncr, ncc, kda = wl.n_comp_rows, wl.n_comp_cols, wl.per_channel_gate
    units = B * wl.heads
    stream, side = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    S0 = [0.3 * torch.randn(B, wl.heads, d, d, device=dev) for _ in range(L)]
    nb = sum(decode_window_bytes(d, in_b, kda, ncr, ncc, n) for n in range(W)) + flush_bytes(d, in_b, kda, ncr, ncc, W)
    rows = []
    for variant in ("lockstep", "aligned", "serial", "overlap"):
        rag = variant != "lockstep"
        stagger = variant in ("serial", "overlap")
        stk = LayerStack(wl, L, "window", dev, wl.seed, 2 * W, S0, ragged=rag)
        offset = torch.arange(B, device=dev) % W
        with torch.cuda.stream(stream):
            for l in range(L):                  # warm launches outside capture (kernel attributes)
                stk.decode(l, 0, active=torch.ones(B, dtype=torch.uint8, device=dev) if rag else None)
                stk.states[l].flush()
                if rag:
                    stk.states[l].flush_pending()
            if stagger:                         # sequence b holds b mod W tokens
                for i in range(W - 1):
                    act = (offset > i).to(torch.uint8)
                    for l in range(L):
                        stk.decode(l, W + i, active=act)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        evs = [torch.cuda.Event() for _ in range(L)]
        with torch.cuda.graph(g, stream=stream):
            for i in range(W):
                for l in range(L):
                    if variant == "overlap" and i > 0:
                        stream.wait_event(evs[l])
                    stk.decode(l, i)
                    if variant in ("serial", "aligned"):
                        stk.states[l].flush()
                    elif variant == "overlap":
                        side.wait_stream(stream)
                        with torch.cuda.stream(side):
                            stk.states[l].flush()
                            evs[l].record(side)
            if variant == "lockstep":
                for st in stk.states:
                    st.flush()
            elif variant == "overlap":
                stream.wait_stream(side)
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        for st in stk.states:
            assert st.device_status(stream) == lq.LQ_OK, lq.last_error()
        if rag:
            fills = torch.stack([st.fills() for st in stk.states]).view(L, B, wl.heads).to(offset.device)
            want = offset if stagger else torch.zeros_like(offset)
            assert bool((fills == want.view(1, B, 1)).all()), "phases drifted"
        ms = e0.elapsed_time(e1) / reps                   # W tokens of every sequence, every layer
        rows.append({"variant": variant, "workload": wl.name, "batch": B, "window": W, "layers_rotated": L,
                     "tokens_per_s_per_layer": B * W * L / (ms * 1e-3), "ms_per_window": ms,
                     "hbm_gbs": units * nb * L / (ms * 1e-3) / 1e9,
                     "launches_per_window": L * (W + (W if stagger else 1))})
        del g, stk
        torch.cuda.synchronize()
    return rows


FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12     # FP32 FMA lanes x 2 FLOP x max SM clock


def prefill_timing(dev, wl, T: int | None = None, reps: int = 5) -> list[dict]:
    """A prompt of T tokens for every sequence (default: the workload's prefill
    length) from a zero state to the encoded window-start state, with every
    prompt token's output: lq_prefill_tokens (register-resident FP32
    recurrence plus codec, one launch) against the route through the decode
    kernels (T FP32-state decode launches, then lq_prefill_state)."""
    from recurrent_state_quantization_lq_b200 import lq
    T = T or wl.prefill_tokens
    B, H, d = wl.batch, wl.heads, wl.d_k
    gate = "channel" if wl.per_channel_gate else "scalar"
    tb = inputs.tokens_on_device(wl.seed * 100 + 77, T, B, H, d, d, wl.per_channel_gate, wl.dtype, dev)
    out = torch.empty(T, B, H, d, device=dev)
    stream = torch.cuda.Stream(device=dev)
    win = lq.DecodeState(B, H, d, window=wl.window, n_comp_rows=wl.n_comp_rows, n_comp_cols=wl.n_comp_cols,
                         gate=gate, in_dtype=wl.dtype, device=dev)
    f32 = lq.DecodeState(B, H, d, gate=gate, mode="fp32", in_dtype=wl.dtype, device=dev)

    def fused():
        win.prefill_tokens(tb.q, tb.k, tb.v, tb.g, tb.beta, out=out)

    def token_loop():
        f32.prefill(None)
        for t in range(T):
            f32.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t], out=out[t])
        win.prefill(f32.view("state_f32"))               # the FP32 state in place (no copy, no sync)

    rows = []
    flop = (6 + (1 if wl.per_channel_gate else 0)) * d * d          # per token and head
    for name, fn in (("prefill_tokens", fused), ("decode_loop", token_loop)):
        with torch.cuda.stream(stream):
            fn()                                                    # warm (kernel attributes)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        assert win.device_status(stream) == lq.LQ_OK, lq.last_error()
        ms = e0.elapsed_time(e1) / reps
        tflops = B * H * T * flop / (ms * 1e-3) / 1e12
        rows.append({"path": name, "workload": wl.name, "batch": B, "heads": H, "d": d, "prompt_tokens": T,
                     "ms": ms, "prompt_tokens_per_s_per_layer": B * T / (ms * 1e-3),
                     "recurrence_tflops": tflops, "frac_of_fp32_simt_peak": tflops / FP32_SIMT_TFLOPS,
                     "launches": 1 if name == "prefill_tokens" else T + 1})
        del g
    rows.append({"path": "speedup", "value": rows[1]["ms"] / rows[0]["ms"]})
    return rows


def quality_study(dev, tokens: int = 1024) -> list[dict]:
    """Output error against the FP32 state over window sizes and compensator
    counts (16 sequences x 32 heads, 128 x 128), on the planted-outlier start
    state and on a state prefilled by the FP32 recurrence; smoothing off as an
    ablation at W = 64, n_c = 4."""
    rows = []
    points = [(W, nc, 1) for W in (16, 32, 64, 128, 256) for nc in (0, 2, 4, 8)] + [(64, 4, 0)]
    for planted in (True, False):
        for W, nc, smooth in points:
            wl = inputs.Workload(f"gdn_quality_b16_w{W}_nc{nc}", 16, 32, 128, 128, W, nc // 2, nc - nc // 2, False,
                                 0 if planted else 512, tokens, torch.bfloat16, 3, planted=planted)
            if not smooth:
                r = quality(wl, dev, smooth=0)
            else:
                r = quality(wl, dev)
            rows.append({"start": "planted outliers" if planted else "fp32 prefill", "window": W, "n_comp": nc,
                         "smooth": smooth, "rel_l2_windowed_vs_fp32": r["rel_l2_windowed_vs_fp32"],
                         "rel_l2_naive_vs_fp32": r["rel_l2_naive_vs_fp32"], "tokens": r["tokens"]})
    return rows


def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores: the reference arm."""
    if rank != 0:
        return None
    wl = inputs.WORKLOADS[args.workload]
    threads = host_cores()
    n_units = min(wl.units, 2 * threads)
    n_tok = 16
    for _ in range(args.warmup):
        oracle_sample(wl, n_units, n_tok, threads, 7)
    total, used = 0.0, 1
    for s in range(args.steps):
        secs, used = oracle_sample(wl, n_units, n_tok, threads, 11 + s)
        total += secs
    ms = total / args.steps * 1e3
    value = n_units * n_tok / wl.heads / (ms * 1e-3)
    sample = (f"{n_units} (sequence, head) units x {n_tok} decode tokens of {wl.name} per step "
              f"(windowed mode, dense FP64 recurrence)")
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": bench_config(wl, args.layers, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=240)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gdn_b64_h32_d128_w64", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--comparator-steps", type=int, default=40)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-tokens", type=int, default=768)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quality", nargs="?", const="gdn_outlier_b256_h32_d128_w64", default=None,
                    metavar="WORKLOAD", help="print the output errors of windowed and naive INT8 against the FP32 "
                    "state on WORKLOAD (default: the outlier-stress workload) instead of timing")
    ap.add_argument("--quality-tokens", type=int, default=None)
    ap.add_argument("--quality-study", action="store_true",
                    help="print one JSON line per (start state, W, n_c) point of the output-error study")
    ap.add_argument("--ragged", nargs="?", const="gdn_b64_h32_d128_w64", default=None, metavar="WORKLOAD",
                    help="print one JSON line per variant of the staggered-phase (continuous batching) timing")
    ap.add_argument("--prefill", nargs="?", const="gdn_b64_h32_d128_w64", default=None, metavar="WORKLOAD",
                    help="time the prompt prefill (lq_prefill_tokens against per-token decode launches)")
    ap.add_argument("--prefill-tokens", type=int, default=None)
    ap.add_argument("--sweep", action="store_true",
                    help="print one JSON line per point of the batch x window throughput sweep instead of timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.quality is not None:
        torch.cuda.set_device(0)
        wl = inputs.WORKLOADS[args.quality]
        res = quality(wl, torch.device("cuda", 0), args.quality_tokens)
        print(json.dumps({"mode": "quality", "workload": wl.name, "window": wl.window,
                          "n_comp": wl.n_comp_rows + wl.n_comp_cols, **res}), flush=True)
        return

    if args.quality_study:
        torch.cuda.set_device(0)
        for row in quality_study(torch.device("cuda", 0)):
            print(json.dumps({"mode": "quality_study", **row}), flush=True)
        return

    if args.prefill is not None:
        torch.cuda.set_device(0)
        for row in prefill_timing(torch.device("cuda", 0), inputs.WORKLOADS[args.prefill], args.prefill_tokens):
            print(json.dumps({"mode": "prefill", **row}), flush=True)
        return

    if args.ragged is not None:
        torch.cuda.set_device(0)
        for row in ragged_phases(torch.device("cuda", 0), inputs.WORKLOADS[args.ragged], args.layers):
            print(json.dumps({"mode": "ragged", **row}), flush=True)
        return

    if args.sweep:
        torch.cuda.set_device(0)
        for row in sweep(torch.device("cuda", 0)):
            print(json.dumps({"mode": "sweep", **row}), flush=True)
        return

    if args.impl == "reference":
        rank, world, _ = ranks.env_ranks()
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    rank, world, local = dist_setup(args.gpus)
    try:
        res = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

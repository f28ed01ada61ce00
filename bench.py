#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet-2 operator on B200.

One step = one gdn2_fwd_chunked call over the 1.3B-layer workload (B=1, H=16,
T=4096, dk=dv=128, bf16 inputs, fp32 decay and state, chunk 64).  `value` is in
tokens/s, a token being one position of one sequence with all 16 heads
(B*T tokens per call).  The same run also times the training-batch (B=8) and
long-context (T=65536) forwards, each against its own HBM roofline, and
gdn2_decode_step on the decode workload (B=256, H=16, d=128, fp32 state of
268 MB updated in place) with its HBM bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs N independent replicas (the operator is independent per
(batch, head); there is no exchange step), one process per GPU, launched by
torch.distributed.run.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import synth  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
METRIC = "tokens/s of GDN-2 fwd (H=16,dk=dv=128) + % roofline; decode HBM GB/s"
CASE = synth.LAYER_BF16
DEC = synth.DECODE_F32
N_INPUT_SETS = 4  # rotating input sets: 4 x 136 MB > 126 MB of L2

# dram__bytes_read.sum + dram__bytes_write.sum per call from an ncu capture of
# the current kernels (None once a kernel has changed since the capture), summed
# over the kernels of one call; the captures are summarised under profiles/.
NCU_TRAFFIC_BYTES = {"fwd": 118233344 + 57096704, "train": 939820032 + 695288576 + 742467328 + 117185280,
                     "long": 1880952832 + 1364458496, "decode": 281043456 + 212228864,
                     "decode_tokens_T16": 469875456 + 245164288,
                     "bwd": None}
EXTRA_CASES = ((synth.TRAIN_BF16, "train", 3, 10), (synth.LONG_BF16, "long", 3, 10))


def bench_config():
    """The `config` of the JSON line (the same for both arms)."""
    c = CASE
    return {"workload": c.name, "B": c.B, "T": c.T, "H": c.H, "dk": c.dk, "dv": c.dv, "chunk": 64,
            "inputs": "bf16 q,k,v,b,w; fp32 log_alpha; fp32 state",
            "l2": f"rotating {N_INPUT_SETS} device input sets (> 126 MB L2)"}


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def fwd_algorithmic_bytes(B, T, H, dk, dv, s_in, s_out, has_s0, has_st, layout=0):
    """Bytes a forward must move: inputs once, outputs once, states once.  With
    a gate layout (bit 1 erase, 2 write, 4 decay) that gate is one value per
    (token, head)."""
    b_ch = 1 if layout & 1 else dk
    w_ch = 1 if layout & 2 else dv
    a_ch = 1 if layout & 4 else dk
    per_head_token = (2 * dk + dv + b_ch + w_ch) * s_in + 4 * a_ch + dv * s_out
    state = B * H * dk * dv * 4
    return B * T * H * per_head_token + state * (int(has_s0) + int(has_st))


def decode_tokens_algorithmic_bytes(B, T, H, dk, dv, s_in=4, s_out=4):
    """T tokens on a resident state: the state read and written once, every token's inputs and outputs once."""
    return B * H * (2 * dk * dv * 4 + T * ((3 * dk + 2 * dv) * s_in + 4 * dk + dv * s_out))


def layer_algorithmic_bytes(B, T, H, dk, dv, s_in=2, s_out=2):
    """The fused layer: q, k, v, the erase/write/output-gate logits in the input dtype,
    the decay logits in fp32, y out, the final state."""
    per_head_token = (3 * dk + 3 * dv) * s_in + 4 * dk + dv * s_out
    return B * T * H * per_head_token + B * H * dk * dv * 4


def bwd_algorithmic_bytes(B, T, H, dk, dv, s_in=2):
    """The backward: the forward's inputs and dO once (input dtype, log_alpha fp32),
    the six gradients once (fp32), S0 / dS_T absent."""
    per_head_token = (3 * dk + 2 * dv + dv) * s_in + 4 * dk + 4 * (4 * dk + 2 * dv)
    return B * T * H * per_head_token


def decode_algorithmic_bytes(B, H, dk, dv, s_in=4, s_out=4):
    # state read + written once, q,k,b (dk) and v,w (dv) in the input dtype,
    # log_alpha fp32, o in the input dtype
    return B * H * (2 * dk * dv * 4 + (3 * dk + 2 * dv) * s_in + 4 * dk + dv * s_out)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        load = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def dist_setup(backend="nccl"):
    """One process per GPU (RANK / WORLD_SIZE / LOCAL_RANK from the launcher); the
    process group only carries the barrier and the max over ranks (replicas, no
    data exchange).  `backend` "gloo" runs the same logic on the host."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int, device: str = "cuda") -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_tokens_per_s(sample_T: int, heads: int, nthreads: int = 0):
    """Oracle (fp64, OpenMP over heads; nthreads 0 = every host core) on a bounded
    sample of the workload."""
    import oracle
    d = synth.draw_fwd(1, sample_T, heads, CASE.dk, CASE.dv, seed=CASE.seed, dtype=CASE.dtype,
                       log_alpha_range=CASE.log_alpha_range, gate_sigma=CASE.gate_sigma)
    args = [d[n] for n in ("q", "k", "v", "b", "w", "log_alpha")]
    orc = oracle.load()
    cores = nthreads if nthreads > 0 else orc.max_threads()
    t = time.perf_counter()
    orc.fwd(*args, S0=None, nthreads=nthreads)
    dt = time.perf_counter() - t
    return sample_T / dt, cores, dt


def run_reference(args, ws, rank):
    """The oracle timed as it stands; each step a bounded sample of the workload."""
    if rank != 0:
        return
    heads = CASE.H
    rate, cores, _ = cpu_oracle_tokens_per_s(256, heads)          # calibration
    per_step_s = 120.0 / (args.steps + args.warmup)                # whole run ~2 min
    T = int(max(64, min(CASE.T, per_step_s * rate)))
    vals = []
    for i in range(args.warmup + args.steps):
        v, cores, dt = cpu_oracle_tokens_per_s(T, heads)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    sample = (f"per step B=1 H={heads} T={T} d=128 of the B=1 H=16 T=4096 workload, fp64, "
              f"OpenMP over heads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": CASE.B * CASE.T / value * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """A few launches of one operator on the bench workload, for ncu (-s/-c pick one)."""
    import gated_delta_rule_118_b200 as g
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    names = ("q", "k", "v", "b", "w", "log_alpha")
    if args.profile in ("fwd", "fwd_train", "fwd_long"):
        c = {"fwd": CASE, "fwd_train": synth.TRAIN_BF16, "fwd_long": synth.LONG_BF16}[args.profile]
        d = synth.draw_fwd_device(c.B, c.T, c.H, c.dk, c.dv, seed=0, device=dev, dtype=c.dtype,
                                  log_alpha_range=c.log_alpha_range, gate_sigma=c.gate_sigma)
        for _ in range(args.warmup + args.steps):
            g.gdn2_fwd_chunked(*(d[n] for n in names), S0=None)
    elif args.profile == "bwd":
        c = CASE
        d = synth.draw_fwd_device(c.B, c.T, c.H, c.dk, c.dv, seed=0, device=dev, dtype=c.dtype,
                                  log_alpha_range=c.log_alpha_range, gate_sigma=c.gate_sigma)
        dO = torch.randn(c.B, c.T, c.H, c.dv, device=dev).to(c.dtype)
        for _ in range(args.warmup + args.steps):
            g.gdn2_bwd_chunked(*(d[n] for n in names), None, dO)
    else:
        dc = DEC
        S = 0.05 * torch.randn(dc.B, dc.H, dc.dk, dc.dv, device=dev)
        Tn = 16 if args.profile == "decode_tokens" else 1
        dd = synth.draw_fwd_device(dc.B, Tn, dc.H, dc.dk, dc.dv, seed=7000, device=dev, dtype=torch.float32)
        if Tn == 1:
            x = {n: dd[n][:, 0].contiguous() for n in names}
            for _ in range(args.warmup + args.steps):
                g.gdn2_decode_step(*(x[n] for n in names), S)
        else:
            for _ in range(args.warmup + args.steps):
                g.gdn2_decode_tokens(*(dd[n] for n in names), S)
    torch.cuda.synchronize()
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["fwd", "fwd_train", "fwd_long", "decode", "decode_tokens", "bwd"],
                    default=None,
                    help="run a few launches of one operator on the bench workload for an ncu "
                         "capture (no timing, no JSON line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, ws, rank)
        return

    import gated_delta_rule_118_b200 as g
    if args.profile:
        run_profile_case(args)
        return
    ws, rank, local = dist_setup()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    hbm_peak, peak_kind = peaks()

    # ---------------- chunked forward: device-resident inputs ----------------
    c = CASE
    sets = [synth.draw_fwd_device(c.B, c.T, c.H, c.dk, c.dv, seed=100 * rank + i, device=dev,
                                  dtype=c.dtype, log_alpha_range=c.log_alpha_range,
                                  gate_sigma=c.gate_sigma) for i in range(N_INPUT_SETS)]
    o = torch.empty(c.B, c.T, c.H, c.dv, dtype=c.dtype, device=dev)
    S_T = torch.empty(c.B, c.H, c.dk, c.dv, dtype=torch.float32, device=dev)
    names = ("q", "k", "v", "b", "w", "log_alpha")

    def step(i):
        d = sets[i % N_INPUT_SETS]
        g.gdn2_fwd_chunked(*(d[n] for n in names), S0=None, o=o, S_T=S_T, check=False)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error during warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    # soak so the clock sampler sees the GPU under load before the timed region
    soak_end = time.time() + 1.0
    i = 0
    while time.time() < soak_end:
        step(i); i += 1
        if i % 50 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    total_ms = max_over_ranks(t_all0.elapsed_time(t_all1), ws)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    mean_launch_ms = sum(launch_ms) / len(launch_ms)
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error during the timed region")

    tokens_per_step = c.B * c.T
    value = tokens_per_step * args.steps * ws / (total_ms / 1e3)
    alg_bytes = fwd_algorithmic_bytes(c.B, c.T, c.H, c.dk, c.dv, 2, 2, False, True)
    achieved = alg_bytes / (mean_launch_ms / 1e3) / 1e9

    # ---------------- end to end through the C ABI with host buffers ----------------
    host = {n: sets[0][n].cpu().pin_memory() for n in names}
    dev_in = {n: torch.empty_like(sets[0][n]) for n in names}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_host.numel() * o_host.element_size()
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        for n in names:
            dev_in[n].copy_(host[n], non_blocking=True)
        g.gdn2_fwd_chunked(*(dev_in[n] for n in names), S0=None, o=o, S_T=S_T, check=False)
        o_host.copy_(o, non_blocking=True)

    # Serial: each step's upload, call and download in turn on one stream.
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_serial_ms = max_over_ranks(e0.elapsed_time(e1), ws)

    # Pipelined, as a streaming caller runs it: two input and two output buffers;
    # step i's upload (on its own stream) and step i - 1's download (on another)
    # overlap step i - 1's call, the copy engines moving both directions at once.
    # Every step's copies stay inside the timed region.
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    din = [{n: torch.empty_like(sets[0][n]) for n in names} for _ in range(2)]
    dout = [torch.empty_like(o) for _ in range(2)]
    hout = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_pipelined(nsteps):
        for i in range(nsteps):
            bb = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[bb])  # the call of step i - 2 has read these inputs
                for n in names:
                    din[bb][n].copy_(host[n], non_blocking=True)
                ev_in[bb].record(s_in)
            stream.wait_event(ev_in[bb])
            if i >= 2:
                stream.wait_event(ev_out[bb])  # the download of step i - 2 has read this output
            g.gdn2_fwd_chunked(*(din[bb][n] for n in names), S0=None, o=dout[bb], S_T=S_T, check=False)
            ev_done[bb].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[bb])
                hout[bb].copy_(dout[bb], non_blocking=True)
                ev_out[bb].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    e2e_pipelined(2)
    torch.cuda.synchronize()
    barrier(ws)
    e0.record(stream)
    s_in.wait_stream(stream)
    e2e_pipelined(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), ws)
    e2e_value = tokens_per_step * e2e_steps * ws / (e2e_ms / 1e3)
    e2e_serial_value = tokens_per_step * e2e_steps * ws / (e2e_serial_ms / 1e3)
    del sets, host, dev_in, din, dout, hout

    # ---------------- the other bf16 workloads, each against its own roofline ----------------
    extra = {}
    for ce, key, warm, reps in EXTRA_CASES:
        d = synth.draw_fwd_device(ce.B, ce.T, ce.H, ce.dk, ce.dv, seed=300 + rank, device=dev, dtype=ce.dtype,
                                  log_alpha_range=ce.log_alpha_range, gate_sigma=ce.gate_sigma)
        s0 = (ce.s0_sigma * torch.randn(ce.B, ce.H, ce.dk, ce.dv, device=dev)) if ce.s0_sigma > 0 else None
        oe = torch.empty(ce.B, ce.T, ce.H, ce.dv, dtype=ce.dtype, device=dev)
        se = torch.empty(ce.B, ce.H, ce.dk, ce.dv, dtype=torch.float32, device=dev)
        for _ in range(warm):
            g.gdn2_fwd_chunked(*(d[n] for n in names), S0=s0, o=oe, S_T=se, check=False)
        torch.cuda.synchronize()
        barrier(ws)
        x0 = torch.cuda.Event(enable_timing=True); x1 = torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        for _ in range(reps):
            g.gdn2_fwd_chunked(*(d[n] for n in names), S0=s0, o=oe, S_T=se, check=False)
        x1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(x0.elapsed_time(x1), ws) / reps
        eb = fwd_algorithmic_bytes(ce.B, ce.T, ce.H, ce.dk, ce.dv, 2, 2, s0 is not None, True)
        gbs = eb / (ms / 1e3) / 1e9
        extra[key] = {"workload": ce.name, "us_per_call": ms * 1e3, "tokens_per_s": ce.B * ce.T * ws / (ms / 1e3),
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                                   "frac": gbs / hbm_peak, "traffic": NCU_TRAFFIC_BYTES[key],
                                   "algorithmic_bytes_per_call": eb},
                      "launches": g.gdn2_fwd_chunked_launches(ce.B, ce.T, ce.H, ce.dk, ce.dv, ce.dtype),
                      "calls": reps, "l2": "inputs > 126 MB L2"}
        del d, oe, se, s0
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error while timing the other workloads")

    # ---------------- gate-variant fast paths on the layer workload ----------------
    layouts = {}
    gen = torch.Generator(device=dev).manual_seed(401 + rank)
    lsets = []
    for i in range(N_INPUT_SETS):  # rotated, like the main measurement: more than L2 holds
        d = synth.draw_fwd_device(c.B, c.T, c.H, c.dk, c.dv, seed=400 + 10 * rank + i, device=dev, dtype=c.dtype,
                                  log_alpha_range=c.log_alpha_range, gate_sigma=c.gate_sigma)
        d["beta"] = torch.sigmoid(torch.randn(c.B, c.T, c.H, generator=gen, device=dev)).to(c.dtype)
        d["la_s"] = -torch.exp(torch.rand(c.B, c.T, c.H, generator=gen, device=dev) * 4.0 - 5.0)
        del d["b"], d["w"]
        lsets.append(d)
    for lname, lay, la_key in (("kda", 3, "log_alpha"), ("gdn", 7, "la_s")):
        def call(i):
            d = lsets[i % N_INPUT_SETS]
            g.gdn2_fwd_chunked(d["q"], d["k"], d["v"], d["beta"], d["beta"], d[la_key], S0=None, o=o, S_T=S_T,
                               check=False)
        for i in range(5):
            call(i)
        torch.cuda.synchronize()
        barrier(ws)
        x0 = torch.cuda.Event(enable_timing=True); x1 = torch.cuda.Event(enable_timing=True)
        reps = 100
        x0.record(stream)
        for i in range(reps):
            call(i)
        x1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(x0.elapsed_time(x1), ws) / reps
        eb = fwd_algorithmic_bytes(c.B, c.T, c.H, c.dk, c.dv, 2, 2, False, True, layout=lay)
        layouts[lname] = {"layout": lay, "us_per_call": ms * 1e3, "tokens_per_s": c.B * c.T * ws / (ms / 1e3),
                          "roofline": {"bound": "hbm", "achieved": eb / (ms / 1e3) / 1e9, "peak": hbm_peak,
                                       "unit": "GB/s", "frac": eb / (ms / 1e3) / 1e9 / hbm_peak,
                                       "algorithmic_bytes_per_call": eb},
                          "l2": f"rotating {N_INPUT_SETS} device input sets"}
    del lsets
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error while timing the gate layouts")

    # ---------------- the fused layer entry point on the layer workload ----------------
    lsets = [synth.draw_layer(c.B, c.T, c.H, c.dk, c.dv, seed=500 + 10 * rank + i, dtype=c.dtype)
             for i in range(N_INPUT_SETS)]
    lnames = ("q", "k", "v", "b_logit", "w_logit", "decay_logit", "g_logit", "norm_weight")
    lsets = [{n: d[n].to(dev) for n in lnames} for d in lsets]
    for i in range(5):
        g.gdn2_layer_fwd(*(lsets[i % N_INPUT_SETS][n] for n in lnames), 1e-6, y=o, S_T=S_T, check=False)
    torch.cuda.synchronize()
    barrier(ws)
    x0 = torch.cuda.Event(enable_timing=True); x1 = torch.cuda.Event(enable_timing=True)
    reps = 100
    x0.record(stream)
    for i in range(reps):
        g.gdn2_layer_fwd(*(lsets[i % N_INPUT_SETS][n] for n in lnames), 1e-6, y=o, S_T=S_T, check=False)
    x1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(x0.elapsed_time(x1), ws) / reps
    lb = layer_algorithmic_bytes(c.B, c.T, c.H, c.dk, c.dv)
    layer_line = {"workload": c.name + " (raw q, k and gate logits; RMS norm and output gate fused)",
                  "us_per_call": ms * 1e3, "tokens_per_s": c.B * c.T * ws / (ms / 1e3),
                  "roofline": {"bound": "hbm", "achieved": lb / (ms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                               "frac": lb / (ms / 1e3) / 1e9 / hbm_peak, "algorithmic_bytes_per_call": lb},
                  "vs_unfused": (mean_launch_ms * 1e3 + 0.0) / (ms * 1e3),
                  "l2": f"rotating {N_INPUT_SETS} device input sets"}
    del lsets
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error while timing the fused layer")

    # ---------------- backward on the layer workload ----------------
    bsets = [synth.draw_fwd_device(c.B, c.T, c.H, c.dk, c.dv, seed=600 + 10 * rank + i, device=dev, dtype=c.dtype,
                                   log_alpha_range=c.log_alpha_range, gate_sigma=c.gate_sigma) for i in range(2)]
    for i, d in enumerate(bsets):
        d["dO"] = torch.randn(c.B, c.T, c.H, c.dv, device=dev).to(c.dtype)
    for i in range(2):
        g.gdn2_bwd_chunked(*(bsets[i % 2][n] for n in names), None, bsets[i % 2]["dO"], check=False)
    torch.cuda.synchronize()
    barrier(ws)
    x0 = torch.cuda.Event(enable_timing=True); x1 = torch.cuda.Event(enable_timing=True)
    reps = 5
    x0.record(stream)
    for i in range(reps):
        g.gdn2_bwd_chunked(*(bsets[i % 2][n] for n in names), None, bsets[i % 2]["dO"], check=False)
    x1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(x0.elapsed_time(x1), ws) / reps
    bb = bwd_algorithmic_bytes(c.B, c.T, c.H, c.dk, c.dv)
    bwd_line = {"workload": c.name + " (gradients of q, k, v, b, w, log_alpha; fp32 outputs)",
                "us_per_call": ms * 1e3, "tokens_per_s": c.B * c.T * ws / (ms / 1e3),
                "roofline": {"bound": "hbm", "achieved": bb / (ms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                             "frac": bb / (ms / 1e3) / 1e9 / hbm_peak, "algorithmic_bytes_per_call": bb,
                             "traffic": NCU_TRAFFIC_BYTES["bwd"]},
                "launches": 3, "l2": "two input sets (> 126 MB of L2 between calls)"}
    del bsets
    # the training batch (one input set: 1.1 GB of inputs and dO, larger than L2)
    tc_ = synth.TRAIN_BF16
    tb = synth.draw_fwd_device(tc_.B, tc_.T, tc_.H, tc_.dk, tc_.dv, seed=650 + rank, device=dev, dtype=tc_.dtype,
                               log_alpha_range=tc_.log_alpha_range, gate_sigma=tc_.gate_sigma)
    tb["dO"] = torch.randn(tc_.B, tc_.T, tc_.H, tc_.dv, device=dev).to(tc_.dtype)
    g.gdn2_bwd_chunked(*(tb[n] for n in names), None, tb["dO"], check=False)
    torch.cuda.synchronize()
    barrier(ws)
    reps = 3
    x0.record(stream)
    for i in range(reps):
        g.gdn2_bwd_chunked(*(tb[n] for n in names), None, tb["dO"], check=False)
    x1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(x0.elapsed_time(x1), ws) / reps
    bb = bwd_algorithmic_bytes(tc_.B, tc_.T, tc_.H, tc_.dk, tc_.dv)
    bwd_line["train"] = {"workload": tc_.name, "us_per_call": ms * 1e3,
                         "tokens_per_s": tc_.B * tc_.T * ws / (ms / 1e3),
                         "roofline": {"bound": "hbm", "achieved": bb / (ms / 1e3) / 1e9, "peak": hbm_peak,
                                      "unit": "GB/s", "frac": bb / (ms / 1e3) / 1e9 / hbm_peak,
                                      "algorithmic_bytes_per_call": bb, "traffic": None}}
    del tb
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error while timing the backward")

    # ---------------- decode: fp32 state resident in HBM, in place ----------------
    dc = DEC
    S = 0.05 * torch.randn(dc.B, dc.H, dc.dk, dc.dv, device=dev)
    tok_sets = []
    for i in range(8):
        dd = synth.draw_fwd_device(dc.B, 1, dc.H, dc.dk, dc.dv, seed=7000 + i, device=dev,
                                   dtype=torch.float32)
        tok_sets.append({n: dd[n][:, 0].contiguous() for n in names})
    od = torch.empty(dc.B, dc.H, dc.dv, device=dev)
    for i in range(5):
        x = tok_sets[i % 8]
        g.gdn2_decode_step(*(x[n] for n in names), S, o=od, check=False)
    torch.cuda.synchronize()
    barrier(ws)
    d0 = torch.cuda.Event(enable_timing=True); d1 = torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for i in range(args.decode_steps):
        x = tok_sets[i % 8]
        g.gdn2_decode_step(*(x[n] for n in names), S, o=od, check=False)
    d1.record(stream)
    torch.cuda.synchronize()
    dec_ms = max_over_ranks(d0.elapsed_time(d1), ws) / args.decode_steps
    dec_bytes = decode_algorithmic_bytes(dc.B, dc.H, dc.dk, dc.dv)
    dec_gbs = dec_bytes / (dec_ms / 1e3) / 1e9
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error during decode timing")

    # ---------------- multi-token decode: T tokens per call on the resident state ----------------
    tok_calls = {}
    for Tn in (4, 16):
        dd = synth.draw_fwd_device(dc.B, Tn, dc.H, dc.dk, dc.dv, seed=7100 + Tn, device=dev, dtype=torch.float32)
        ot = torch.empty(dc.B, Tn, dc.H, dc.dv, device=dev)
        for _ in range(3):
            g.gdn2_decode_tokens(*(dd[n] for n in names), S, o=ot, check=False)
        torch.cuda.synchronize()
        barrier(ws)
        x0 = torch.cuda.Event(enable_timing=True); x1 = torch.cuda.Event(enable_timing=True)
        reps = 50
        x0.record(stream)
        for _ in range(reps):
            g.gdn2_decode_tokens(*(dd[n] for n in names), S, o=ot, check=False)
        x1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(x0.elapsed_time(x1), ws) / reps
        tb = decode_tokens_algorithmic_bytes(dc.B, Tn, dc.H, dc.dk, dc.dv)
        tok_calls[f"T{Tn}"] = {"T": Tn, "us_per_call": ms * 1e3, "tokens_per_s": dc.B * Tn * ws / (ms / 1e3),
                               "hbm_gbs": tb / (ms / 1e3) / 1e9, "frac": tb / (ms / 1e3) / 1e9 / hbm_peak,
                               "algorithmic_bytes_per_call": tb,
                               "traffic": NCU_TRAFFIC_BYTES.get(f"decode_tokens_T{Tn}"),
                               "vs_decode_steps": (Tn * dec_ms) / ms}
        del dd, ot
    if g.gdn2_check_device_error() != g.GDN2_OK:
        raise RuntimeError("device error during multi-token decode timing")

    # ---------------- CPU baseline (oracle) on rank 0, N = 1 ----------------
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, cores, dt = cpu_oracle_tokens_per_s(c.T, c.H)
        v1, _, dt1 = cpu_oracle_tokens_per_s(1024, c.H, nthreads=1)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"the whole workload (B=1 H=16 T=4096 d=128, 4,096 tokens of 16 heads), fp64, "
                         f"{dt:.1f} s",
               "single_core": {"value": v1, "unit": "tokens/s",
                               "sample": f"the first 1024 tokens of the workload, 16 heads, one thread, "
                                         f"{dt1:.1f} s"}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": bench_config(),
            "head_tokens_per_s": value * c.H,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": NCU_TRAFFIC_BYTES["fwd"],
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": alg_bytes,
                         "mean_launch_us": mean_launch_ms * 1e3,
                         "kernel": "gdn2_fwd_chunked (one persistent launch: prep, chain and output work)"},
            "decode": {"workload": dc.name, "us_per_step": dec_ms * 1e3, "hbm_gbs": dec_gbs,
                       "frac": dec_gbs / hbm_peak, "peak": hbm_peak,
                       "algorithmic_bytes_per_step": dec_bytes, "steps": args.decode_steps,
                       "traffic": NCU_TRAFFIC_BYTES["decode"],
                       "dram_gbs": NCU_TRAFFIC_BYTES["decode"] / (dec_ms / 1e3) / 1e9,
                       "l2": "state 268 MB > 126 MB L2, streamed every step (part of it stays in L2 "
                             "between steps: DRAM bytes per step below the algorithmic bytes)"},
            "workloads": extra,
            "gate_layouts": layouts,
            "layer_fused": layer_line,
            "backward": bwd_line,
            "decode_tokens": {"workload": "decode state B=256 H=16 d=128 fp32, T tokens per call",
                              "calls": tok_calls},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "copies": "pinned host buffers; uploads and downloads on their own streams, double-buffered "
                              "so that they overlap the neighbouring steps' calls",
                    "serial_value": e2e_serial_value},
            "gpu_launches": args.steps * g.gdn2_fwd_chunked_launches(c.B, c.T, c.H, c.dk, c.dv, c.dtype),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

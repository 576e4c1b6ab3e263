"""Benchmark of the Gated DeltaNet recurrence path on B200.

One step = one pass of the whole prefill path over one batch of synthetic
input: the front end (gdn_conv1d_silu: conv1d + SiLU + L2 norm) and the chunked
prefill (gdn_prefill) of one GDN layer, T = 8192 tokens, 16 key heads, 48 value
heads, d = 128, zero initial state.  The metric is tokens per second per layer.
Secondary lines are measured in the same run and attached under "extra": the
T = 262144 prefill (non-zero initial state), the 16-sequence varlen prefill
(lengths U[1024, 32768]), the gated output norm at T = 8192, the layer tail
(recurrence + gated norm, fused and in two passes), the backward pass at
T = 8192, and one decode step over 128 sequences x 48 layers with the 19.3 GB
float32 state updated in place (plain, with the front end fused, with a bf16
state, and with the gated norm fused); last, at N = 1 only, the backward pass
through the chunked form, the front end's backward and the gated norm's
backward at T = 8192 (an error there is recorded in its entry).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Timing: CUDA events on the launching stream around every step, L2 flushed
(a 256 MiB buffer written) before each timed step, W >= 3 untimed warm-up
steps, max over ranks.  With --gpus N > 1 (launched under torchrun) every rank
runs its own replica of the workload (weak scaling; the path has no exchange
step).  `--impl reference` times the fp64 CPU oracle on the host cores instead.
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

T_MAIN = 8192
E2E_BLOCKS = 6          # token ranges of the end-to-end call (448 tokens, then 1600 each, at T = 8192)
T_LONG = 262144
HQK, HV, D = 16, 48, 128
# algorithmic work per token per layer (chunked form, C = 64): 48 value heads x
# (3 x 2Cd + 3 x 2d^2) + 16 key heads x 2 x 2Cd
FLOP_PER_TOKEN = HV * (3 * 2 * 64 * D + 3 * 2 * D * D) + HQK * 2 * 2 * 64 * D
# bytes per token the prefill must move: q, k, v bf16 in; a, b f32 in; o f32 out
PREFILL_BYTES_PER_TOKEN = 2 * (2 * HQK * D + HV * D) + 4 * 2 * HV + 4 * HV * D
# front end: read (2Hqk + Hv) d bf16, write the same
FRONTEND_BYTES_PER_TOKEN = 2 * 2 * (2 * HQK + HV) * D
STATE_BYTES = HV * D * D * 4


def kernel_traffic(name):
    """DRAM bytes per launch of kernel `name` on the bench workload, from the
    committed ncu record profiles/ncu_traffic.json -- or None when there is no
    record or the kernel's source has changed since the counters were taken."""
    import hashlib
    rec_path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(rec_path):
        return None
    with open(rec_path) as f:
        rec = json.load(f).get(name)
    if not rec:
        return None
    src = os.path.join(ROOT, "gated_deltanet_recurrence_prefill_b200", "csrc", rec["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
            return None
    return int(rec["dram_bytes_per_launch"])


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class Clocks:
    """nvidia-smi sampled every 20 ms while the timed region runs (the timed
    region starts once the first sample has been written)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"gdn_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        # the timed region starts once the sampler is producing lines
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 5.0 and self.proc.poll() is None:
            try:
                if os.path.getsize(self.path) > 0:
                    break
            except OSError:
                pass
            time.sleep(0.02)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        loaded = [r[0] for r in rows if r[2] > 200.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------- GPU arm

def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _time_steps(step, warmup, steps, flush, streams_events, world=1):
    """Warm-up, then `steps` timed steps bracketed by a barrier and a device
    synchronize on both sides; returns per-step ms (CUDA events on the current
    stream) and per-kernel ms lists from streams_events()."""
    import torch
    for _ in range(warmup):
        step(None)
    torch.cuda.synchronize()
    _barrier(world)
    times = []
    per_kernel = {}
    for _ in range(steps):
        flush.zero_()
        ev = streams_events()
        step(ev)
        torch.cuda.synchronize()
        times.append(ev["start"].elapsed_time(ev["end"]))
        for name, (a, b) in ev.get("kernels", {}).items():
            per_kernel.setdefault(name, []).append(a.elapsed_time(b))
    _barrier(world)
    return times, per_kernel


def bench_main(args, world, rank, local):
    import numpy as np
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peaks = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    # ---- inputs of the 8K workload (seeded, synthetic), resident in HBM
    fe = synth.workload(1)
    g = fe.gates
    to16 = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    h_qkv = to16(fe.qkv).pin_memory()
    h_a = torch.from_numpy(g.a).pin_memory()
    h_b = torch.from_numpy(g.b).pin_memory()
    qkv = h_qkv.to(dev)
    conv_w = torch.from_numpy(fe.conv_w).to(dev)
    a = h_a.to(dev)
    b = h_b.to(dev)
    A_log = torch.from_numpy(g.A_log).to(dev)
    dt_bias = torch.from_numpy(g.dt_bias).to(dev)
    T = T_MAIN
    q = torch.empty(T, HQK, D, dtype=torch.bfloat16, device=dev)
    k = torch.empty_like(q)
    v = torch.empty(T, HV, D, dtype=torch.bfloat16, device=dev)
    o = torch.empty(T, HV, D, dtype=torch.float32, device=dev)
    fs = torch.empty(1, HV, D, D, dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(1, T, HQK, HV, D), dtype=torch.uint8, device=dev)

    def new_events():
        mk = lambda: torch.cuda.Event(enable_timing=True)
        e = {"start": mk(), "end": mk(), "kernels": {"conv1d_silu": (mk(), mk()),
                                                       "prefill": (mk(), mk())}}
        return e

    def step(ev):
        if ev:
            ev["start"].record()
            ev["kernels"]["conv1d_silu"][0].record()
        gdn.conv1d_silu(qkv, conv_w, HQK, HV, out=(q, k, v))
        if ev:
            ev["kernels"]["conv1d_silu"][1].record()
            ev["kernels"]["prefill"][0].record()
        gdn.prefill(q, k, v, a, b, A_log, dt_bias, o=o, final_state=fs, workspace=ws)
        if ev:
            ev["kernels"]["prefill"][1].record()
            ev["end"].record()

    torch.cuda.synchronize()
    with Clocks(local if "CUDA_VISIBLE_DEVICES" not in os.environ else _smi_index(local)) as clk:
        wall0 = time.perf_counter()
        times, per_kernel = _time_steps(step, args.warmup, args.steps, flush, new_events, world)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    clocks = clk.summary()
    ms = sum(times) / len(times)
    ms_max = _max_over_ranks(ms, world)
    launches_per_step = 2

    # ---- end to end through the public API with host buffers: gdn_layer_prefill_host
    # (pinned host inputs -> front end + prefill -> pinned host outputs, the
    # copies overlapped with the compute over E2E_BLOCKS token ranges)
    h_o = torch.empty(T, HV, D, dtype=torch.float32).pin_memory()
    h_fs = torch.empty(HV, D, D, dtype=torch.float32).pin_memory()
    e2e_ws = torch.empty(gdn.lib().gdn_layer_prefill_host_workspace_size(T, HQK, HV, D, E2E_BLOCKS),
                         dtype=torch.uint8, device=dev)
    copy_streams = (torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev))

    def e2e_step(ev):
        if ev:
            ev["start"].record()
        gdn.layer_prefill_host(h_qkv, h_a, h_b, conv_w, A_log, dt_bias, HQK, HV, h_o=h_o, h_final_state=h_fs,
                               n_blocks=E2E_BLOCKS, workspace=e2e_ws, copy_streams=copy_streams)
        if ev:
            ev["end"].record()

    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}
    e2e_times, _ = _time_steps(e2e_step, args.warmup, args.steps, flush, mk, world)
    e2e_ms = _max_over_ranks(sum(e2e_times) / len(e2e_times), world)
    h2d = h_qkv.numel() * 2 + h_a.numel() * 4 + h_b.numel() * 4
    d2h = h_o.numel() * 4 + h_fs.numel() * 4

    # ---- roofline of the dominant kernel
    kern_ms = {name: sum(v) / len(v) for name, v in per_kernel.items()}
    prefill_ms = kern_ms["prefill"]
    conv_ms = kern_ms["conv1d_silu"]
    if prefill_ms >= conv_ms:
        dom, dom_ms, dom_bytes = "prefill", prefill_ms, PREFILL_BYTES_PER_TOKEN * T
    else:
        dom, dom_ms, dom_bytes = "conv1d_silu", conv_ms, FRONTEND_BYTES_PER_TOKEN * T
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    roofline = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": kernel_traffic("prefill" if dom == "prefill" else "conv1d_silu"),
                "peak_source": peaks["source"], "bytes_per_launch": dom_bytes,
                "kernel_ms": round(dom_ms, 4)}
    prefill_tflops = FLOP_PER_TOKEN * T / (prefill_ms * 1e-3) / 1e12
    kernels = {
        "conv1d_silu": {"ms": round(conv_ms, 4),
                        "GB_s": round(FRONTEND_BYTES_PER_TOKEN * T / (conv_ms * 1e-3) / 1e9, 1)},
        "prefill": {"ms": round(prefill_ms, 4),
                    "GB_s": round(PREFILL_BYTES_PER_TOKEN * T / (prefill_ms * 1e-3) / 1e9, 1),
                    "TFLOP_s": round(prefill_tflops, 2),
                    "tensor_frac": round(prefill_tflops / peaks["bf16_tflops"], 4)},
    }

    extra = {}
    if not args.primary_only:
        extra["prefill_262k"] = bench_long_prefill(args, dev, flush, peaks, world)
        extra["prefill_varlen_16seq"] = bench_long_prefill(
            args, dev, flush, peaks, world, lengths=synth.varlen_lengths(3), seed=3)
        extra["prefill_262k_bf16o"] = bench_long_prefill(args, dev, flush, peaks, world, o_bf16=True)
        extra["gated_norm_T8192"] = bench_gated_norm(args, dev, flush, peaks, world)
        extra["layer_tail_T8192"] = bench_layer_tail(args, dev, flush, peaks, world)
        extra["backward_T8192"] = bench_backward(args, dev, flush, peaks, world)
        extra["decode_128seq_48layers"] = bench_decode(args, dev, peaks, world)
        extra["decode_fused_128seq_48layers"] = bench_decode_fused(args, dev, peaks, world)
        extra["decode_fused_bf16state_128seq_48layers"] = bench_decode_fused(args, dev, peaks, world, bf16_state=True)
        extra["decode_bf16state_128seq_48layers"] = bench_decode(args, dev, peaks, world, bf16_state=True)
        extra["decode_gated_128seq_48layers"] = bench_decode(args, dev, peaks, world, gated=True)
        if world == 1:
            # the chunked backward is the newest path: last, and an error is
            # recorded in its entry rather than ending the run
            try:
                extra["backward_chunked_T8192"] = bench_backward(args, dev, flush, peaks, world, chunked=True)
            except Exception as exc:     # noqa: BLE001
                extra["backward_chunked_T8192"] = {"error": str(exc)[:300]}
            try:
                extra["front_backward_T8192"] = bench_front_backward(args, dev, flush, peaks, world)
            except Exception as exc:     # noqa: BLE001
                extra["front_backward_T8192"] = {"error": str(exc)[:300]}
            try:
                extra["gated_norm_backward_T8192"] = bench_norm_backward(args, dev, flush, peaks, world)
            except Exception as exc:     # noqa: BLE001
                extra["gated_norm_backward_T8192"] = {"error": str(exc)[:300]}

    value = weak_scaling_rate(T, ms_max, world)
    line = {
        "metric": "GDN prefill tokens/s/layer (front end + chunked prefill, T=8192)",
        "value": round(value, 1), "unit": "tokens/s/layer", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded: N(0,1) bf16 q|k|v channels, conv w ~ N(0,0.25), gates per recipe)",
        "config": {"workload": "gdn_conv1d_silu + gdn_prefill, 1 layer, T=8192, N=1, Hqk=16, "
                               "Hv=48, d=128, zero S0, fp32 o and state",
                   "T": T, "n_seq": 1, "Hqk": HQK, "Hv": HV, "d": D, "chunk": 64,
                   "l2": "flushed before every timed step (256 MiB write)",
                   "parallelism": f"replicas x{world}"},
        "e2e": {"value": round(weak_scaling_rate(T, e2e_ms, world), 1), "unit": "tokens/s/layer",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": round(e2e_ms, 4),
                "api": f"gdn_layer_prefill_host, {E2E_BLOCKS} token ranges, upload / compute / download "
                       "on three streams"},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": roofline,
        "kernels": kernels,
        "clocks": clocks,
        "wall_s_timed_region": round(wall, 3),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    if extra:
        # the secondary lines go last, the long-context prefill at the very end,
        # so that a reader that keeps only the tail of the line still has them
        last = ["decode_bf16state_128seq_48layers", "decode_fused_128seq_48layers",
                "decode_128seq_48layers", "prefill_varlen_16seq", "prefill_262k_bf16o", "prefill_262k"]
        ordered = {k: v for k, v in extra.items() if k not in last}
        ordered.update({k: extra[k] for k in last if k in extra})
        line["extra"] = ordered
        line["summary"] = _summary(line)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _summary(line):
    """The headline numbers of the run in one small object (the JSON line's last key)."""
    ex = line.get("extra", {})
    out = {"prefill_T8192_ms": line["kernels"]["prefill"]["ms"],
           "prefill_T8192_hbm_frac": line["roofline"]["frac"]}
    lp = ex.get("prefill_262k")
    if isinstance(lp, dict) and "ms" in lp:
        out.update({"prefill_262k_ms": lp["ms"], "prefill_262k_tokens_per_s_layer": lp["tokens_per_s_layer"],
                    "prefill_262k_tensor_frac": lp["tensor_frac"], "prefill_262k_hbm_frac": lp["hbm_frac"]})
    lb = ex.get("prefill_262k_bf16o")
    if isinstance(lb, dict) and "ms" in lb:
        out.update({"prefill_262k_bf16o_ms": lb["ms"], "prefill_262k_bf16o_hbm_frac": lb["hbm_frac"]})
    vl = ex.get("prefill_varlen_16seq")
    if isinstance(vl, dict) and "ms" in vl:
        out.update({"prefill_varlen_ms": vl["ms"], "prefill_varlen_tensor_frac": vl["tensor_frac"],
                    "prefill_varlen_hbm_frac": vl["hbm_frac"],
                    "prefill_varlen_launches_per_step": vl["launches_per_step"]})
    for key, name in (("decode_128seq_48layers", "decode_fp32_state"),
                      ("decode_bf16state_128seq_48layers", "decode_bf16_state")):
        d = ex.get(key)
        if isinstance(d, dict) and "ms" in d:
            out.update({name + "_ms": d["ms"], name + "_hbm_frac": d["hbm_frac"]})
    return out


def _smi_index(local):
    """nvidia-smi --id for this rank's GPU (an index or a UUID)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in vis.split(",") if x.strip()]
    if local < len(ids):
        return ids[local]
    return local


def _max_over_ranks(x, world):
    """The largest of every rank's x (a collective: all ranks call it in the same
    order).  NCCL reduces a CUDA tensor, gloo a host one."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def weak_scaling_rate(units_per_rank, ms_per_step_max, world):
    """Whole-job rate of `world` replicas that each process `units_per_rank` per
    step, timed by the slowest rank (units per second)."""
    return world * units_per_rank / (ms_per_step_max * 1e-3)


def bench_long_prefill(args, dev, flush, peaks, world, lengths=None, seed=2, o_bf16=False):
    """One gdn_prefill launch over `lengths` (default: one sequence of T = 262144),
    per-sequence S0 ~ N(0, 0.02^2) (inputs drawn on the device).  o_bf16: the
    bf16-output variant gdn_prefill_bf16 (o is 2 bytes per element)."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    lengths = lengths or [T_LONG]
    N = len(lengths)
    T = sum(lengths)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)

    def unit(shape):
        x = torch.randn(*shape, generator=gen, device=dev)
        x = x / torch.sqrt((x * x).sum(-1, keepdim=True) + 1e-6)
        return x.to(torch.bfloat16)

    q = unit((T, HQK, D))
    k = unit((T, HQK, D))
    v = torch.randn(T, HV, D, generator=gen, device=dev).to(torch.bfloat16)
    a = torch.randn(T, HV, generator=gen, device=dev)
    b = torch.randn(T, HV, generator=gen, device=dev)
    A_log = torch.log(torch.empty(HV, device=dev).uniform_(1, 16, generator=gen))
    dt = torch.exp(torch.empty(HV, device=dev).uniform_(-6.907755, -2.302585, generator=gen))
    dt_bias = torch.log(torch.expm1(dt))
    s0 = 0.02 * torch.randn(N, HV, D, D, generator=gen, device=dev)
    o = torch.empty(T, HV, D, dtype=torch.bfloat16 if o_bf16 else torch.float32, device=dev)
    fs = torch.empty_like(s0)
    cu = None
    if N > 1:
        offs = [0]
        for n in lengths:
            offs.append(offs[-1] + n)
        cu = torch.tensor(offs, dtype=torch.int32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(N, T, HQK, HV, D), dtype=torch.uint8, device=dev)

    def step(ev):
        if ev:
            ev["start"].record()
        gdn.prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens=cu, initial_state=s0, o=o,
                    final_state=fs, workspace=ws)
        if ev:
            ev["end"].record()

    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}
    times, _ = _time_steps(step, max(3, args.warmup), max(3, min(args.steps, 10)), flush, mk, world)
    ms = _max_over_ranks(sum(times) / len(times), world)
    tflops = FLOP_PER_TOKEN * T / (ms * 1e-3) / 1e12
    bytes_per_token = PREFILL_BYTES_PER_TOKEN - (2 * HV * D if o_bf16 else 0)
    gbs = (bytes_per_token * T + 2 * N * STATE_BYTES) / (ms * 1e-3) / 1e9
    if N == 1:
        wl = f"gdn_prefill T={T} N=1 Hqk=16 Hv=48 d=128 S0~N(0,0.02^2)"
        if o_bf16:
            wl = wl.replace("gdn_prefill", "gdn_prefill_bf16 (bf16 o)")
    else:
        wl = (f"gdn_prefill varlen N={N} (lengths U[1024,32768], T={T}, longest {max(lengths)}) "
              f"Hqk=16 Hv=48 d=128 per-sequence S0~N(0,0.02^2)")
    out = {"workload": wl,
           "ms": round(ms, 4), "tokens_per_s_layer": round(weak_scaling_rate(T, ms, world), 1),
           "TFLOP_s": round(tflops, 2), "tensor_frac": round(tflops / peaks["bf16_tflops"], 4),
           "GB_s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
           # both roofs of the launch: algorithmic FLOPs (C = 64 chunked form) over
           # the measured dense bf16 peak, algorithmic bytes over the measured copy
           # bandwidth (the path is HBM-bound by arithmetic intensity)
           "roofline": {
               "tensor": {"achieved": round(tflops, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": round(tflops / peaks["bf16_tflops"], 4),
                          "flop_per_launch": int(FLOP_PER_TOKEN * T)},
               "hbm": {"achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": round(gbs / peaks["hbm_gbs"], 4),
                       "bytes_per_launch": int(bytes_per_token * T + 2 * N * STATE_BYTES)},
               "peak_source": peaks["source"]},
           # the producer/consumer kernel runs whole sequences (48 value heads, 144
           # CTAs) per cooperative launch when more units exist than fit at once
           "launches_per_step": N}
    del q, k, v, a, b, o
    torch.cuda.empty_cache()
    return out


def bench_gated_norm(args, dev, flush, peaks, world):
    """gdn_gated_norm over the T = 8192 output of one layer (48 heads): o
    float32 in, z bf16 in, y bf16 out, 1024 bytes per (token, head)."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T = T_MAIN
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    o = torch.randn(T, HV, D, generator=gen, device=dev)
    z = torch.randn(T, HV, D, generator=gen, device=dev).to(torch.bfloat16)
    w = torch.empty(D, device=dev).uniform_(0.5, 1.5, generator=gen)
    y = torch.empty(T, HV, D, dtype=torch.bfloat16, device=dev)

    def step(ev):
        if ev:
            ev["start"].record()
        gdn.gated_norm(o, z, w, y=y)
        if ev:
            ev["end"].record()

    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}
    times, _ = _time_steps(step, max(3, args.warmup), max(5, min(args.steps, 50)), flush, mk, world)
    ms = _max_over_ranks(sum(times) / len(times), world)
    bytes_step = T * HV * D * (4 + 2 + 2)
    gbs = bytes_step / (ms * 1e-3) / 1e9
    out = {"workload": f"gdn_gated_norm T={T} Hv=48 d=128 (o f32, z bf16 -> y bf16)",
           "ms": round(ms, 4), "GB_s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
           "bytes_per_step": int(bytes_step), "l2": "flushed before every timed step",
           "launches_per_step": 1}
    del o, z, y
    torch.cuda.empty_cache()
    return out


def bench_layer_tail(args, dev, flush, peaks, world):
    """The recurrence plus the gated output norm at T = 8192 (one sequence, zero
    S0): gdn_prefill_gated (norm fused, bf16 y only) against gdn_prefill followed
    by gdn_gated_norm (o written and read back)."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T = T_MAIN
    gen = torch.Generator(device=dev)
    gen.manual_seed(6)

    def unit(shape):
        x = torch.randn(*shape, generator=gen, device=dev)
        return (x / torch.sqrt((x * x).sum(-1, keepdim=True) + 1e-6)).to(torch.bfloat16)

    q, k = unit((T, HQK, D)), unit((T, HQK, D))
    v = torch.randn(T, HV, D, generator=gen, device=dev).to(torch.bfloat16)
    a = torch.randn(T, HV, generator=gen, device=dev)
    b = torch.randn(T, HV, generator=gen, device=dev)
    A_log = torch.log(torch.empty(HV, device=dev).uniform_(1, 16, generator=gen))
    dt = torch.exp(torch.empty(HV, device=dev).uniform_(-6.907755, -2.302585, generator=gen))
    dt_bias = torch.log(torch.expm1(dt))
    z = torch.randn(T, HV, D, generator=gen, device=dev).to(torch.bfloat16)
    w = torch.empty(D, device=dev).uniform_(0.5, 1.5, generator=gen)
    o = torch.empty(T, HV, D, device=dev)
    y = torch.empty(T, HV, D, dtype=torch.bfloat16, device=dev)
    fs = torch.empty(1, HV, D, D, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(1, T, HQK, HV, D), dtype=torch.uint8, device=dev)
    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}

    def fused(ev):
        if ev:
            ev["start"].record()
        gdn.prefill_gated(q, k, v, a, b, A_log, dt_bias, z, w, y=y, final_state=fs, workspace=ws)
        if ev:
            ev["end"].record()

    def unfused(ev):
        if ev:
            ev["start"].record()
        gdn.prefill(q, k, v, a, b, A_log, dt_bias, o=o, final_state=fs, workspace=ws)
        gdn.gated_norm(o, z, w, y=y)
        if ev:
            ev["end"].record()

    n = max(5, min(args.steps, 50))
    tf, _ = _time_steps(fused, max(3, args.warmup), n, flush, mk, world)
    tu, _ = _time_steps(unfused, max(3, args.warmup), n, flush, mk, world)
    ms_f = _max_over_ranks(sum(tf) / len(tf), world)
    ms_u = _max_over_ranks(sum(tu) / len(tu), world)
    # algorithmic bytes of the fused pass: q, k, v, a, b and z in, y out (o never stored)
    bytes_f = T * (2 * (2 * HQK * D + HV * D) + 4 * 2 * HV + 2 * HV * D + 2 * HV * D)
    out = {"workload": f"gdn_prefill_gated T={T} N=1 Hqk=16 Hv=48 d=128 zero S0, bf16 y (o not stored)",
           "fused_ms": round(ms_f, 4), "prefill_then_norm_ms": round(ms_u, 4),
           "tokens_per_s_layer": round(weak_scaling_rate(T, ms_f, world), 1),
           "GB_s": round(bytes_f / (ms_f * 1e-3) / 1e9, 1), "bytes_per_step": int(bytes_f),
           "launches_per_step": 1}
    del q, k, v, a, b, z, o, y
    torch.cuda.empty_cache()
    return out


def bench_backward(args, dev, flush, peaks, world, chunked=False):
    """gdn_prefill_backward (or, chunked, gdn_prefill_backward_chunked) at
    T = 8192 (one sequence, 16 / 48 heads, S0 and dL/dS_T given): all gradients
    of the recurrence."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T = T_MAIN
    gen = torch.Generator(device=dev)
    gen.manual_seed(8)

    def unit(shape):
        x = torch.randn(*shape, generator=gen, device=dev)
        return (x / torch.sqrt((x * x).sum(-1, keepdim=True) + 1e-6)).to(torch.bfloat16)

    q, k = unit((T, HQK, D)), unit((T, HQK, D))
    v = torch.randn(T, HV, D, generator=gen, device=dev).to(torch.bfloat16)
    a = torch.randn(T, HV, generator=gen, device=dev)
    b = torch.randn(T, HV, generator=gen, device=dev)
    A_log = torch.log(torch.empty(HV, device=dev).uniform_(1, 16, generator=gen))
    dt = torch.exp(torch.empty(HV, device=dev).uniform_(-6.907755, -2.302585, generator=gen))
    dt_bias = torch.log(torch.expm1(dt))
    s0 = 0.02 * torch.randn(1, HV, D, D, generator=gen, device=dev)
    d_o = torch.randn(T, HV, D, generator=gen, device=dev)
    d_fin = 0.1 * torch.randn(1, HV, D, D, generator=gen, device=dev)
    entry = "gdn_prefill_backward_chunked" if chunked else "gdn_prefill_backward"
    ws_bytes = getattr(gdn.lib(), entry + "_workspace_size")(1, T, HV, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    fn = gdn.prefill_backward_chunked if chunked else gdn.prefill_backward

    def step(ev):
        if ev:
            ev["start"].record()
        fn(q, k, v, a, b, A_log, dt_bias, d_o, d_final_state=d_fin, initial_state=s0, workspace=ws)
        if ev:
            ev["end"].record()

    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}
    times, _ = _time_steps(step, 3, 3, flush, mk, world)
    ms = _max_over_ranks(sum(times) / len(times), world)
    how = ("tensor cores (tcgen05): chunk-parallel preparation and gradient step, two state chains "
           "over chunks" if chunked else "CUDA cores, one CTA per value head, token by token")
    out = {"workload": f"{entry} T={T} N=1 Hqk=16 Hv=48 d=128, S0 and dL/dS_T given ({how})",
           "ms": round(ms, 3), "tokens_per_s_layer": round(weak_scaling_rate(T, ms, world), 1),
           "launches_per_step": 7 if chunked else 3}
    if chunked:
        # useful products per (chunk, value head), bf16 operands: preparation
        # 9.4 MFLOP, each chain 4.2 MFLOP, gradient step 25.2 MFLOP
        flop = (T // 64) * HV * (9.44e6 + 2 * 4.19e6 + 25.17e6)
        out["tensor_flop_per_step"] = flop
        out["roofline"] = {"bound": "latency (serial chains, per-chunk phases)",
                           "tensor_tflops": round(flop / (ms * 1e-3) / 1e12, 1),
                           "tensor_frac": round(flop / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}
    del q, k, v, d_o, ws
    torch.cuda.empty_cache()
    return out


def bench_front_backward(args, dev, flush, peaks, world):
    """gdn_conv1d_silu_backward at T = 8192 (one sequence, 16 / 48 heads, a
    conv history given): d qkv, d conv_w and d conv_state.  Algorithmic bytes
    per token: the bf16 input and the float32 dq, dk, dv read, the float32
    d qkv written (2 + 4 + 4 bytes per channel)."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T = T_MAIN
    ctot = (2 * HQK + HV) * D
    gen = torch.Generator(device=dev)
    gen.manual_seed(9)
    qkv = torch.randn(T, ctot, generator=gen, device=dev).to(torch.bfloat16)
    w = 0.5 * torch.randn(ctot, 4, generator=gen, device=dev)
    cs = torch.randn(1, ctot, 3, generator=gen, device=dev)
    dq = torch.randn(T, HQK, D, generator=gen, device=dev)
    dk = torch.randn(T, HQK, D, generator=gen, device=dev)
    dv = torch.randn(T, HV, D, generator=gen, device=dev)
    ws = torch.empty(gdn.lib().gdn_conv1d_silu_backward_workspace_size(T, HQK, HV, D), dtype=torch.uint8,
                     device=dev)

    def step(ev):
        if ev:
            ev["start"].record()
        gdn.conv1d_silu_backward(qkv, w, dq, dk, dv, HQK, HV, conv_state=cs, workspace=ws)
        if ev:
            ev["end"].record()

    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}
    times, _ = _time_steps(step, 3, 5, flush, mk, world)
    ms = _max_over_ranks(sum(times) / len(times), world)
    nbytes = T * ctot * (2 + 4 + 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    out = {"workload": f"gdn_conv1d_silu_backward T={T} N=1 Hqk=16 Hv=48 d=128, conv history given",
           "ms": round(ms, 4), "GB_s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
           "bytes_per_step": nbytes, "launches_per_step": 3}
    del qkv, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return out


def bench_norm_backward(args, dev, flush, peaks, world):
    """gdn_gated_norm_backward at T = 8192 x 48 heads, one layer: d o, d z and
    d norm_w.  Algorithmic bytes per (token, head): o, dy float32 and z bf16
    read, d o and d z float32 written (4 + 4 + 2 + 4 + 4 bytes per element)."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T = T_MAIN
    gen = torch.Generator(device=dev)
    gen.manual_seed(10)
    o = torch.randn(T, HV, D, generator=gen, device=dev)
    z = torch.randn(T, HV, D, generator=gen, device=dev).to(torch.bfloat16)
    w = 1.0 + 0.1 * torch.randn(1, D, generator=gen, device=dev)
    dy = torch.randn(T, HV, D, generator=gen, device=dev)
    ws = torch.empty(gdn.lib().gdn_gated_norm_backward_workspace_size(T, HV, D, 1), dtype=torch.uint8, device=dev)

    def step(ev):
        if ev:
            ev["start"].record()
        gdn.gated_norm_backward(o, z, w, dy, workspace=ws)
        if ev:
            ev["end"].record()

    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}
    times, _ = _time_steps(step, 3, 5, flush, mk, world)
    ms = _max_over_ranks(sum(times) / len(times), world)
    nbytes = T * HV * D * (4 + 4 + 2 + 4 + 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    out = {"workload": f"gdn_gated_norm_backward T={T} Hv=48 d=128, one layer",
           "ms": round(ms, 4), "GB_s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
           "bytes_per_step": nbytes, "launches_per_step": 3}
    del o, z, dy, ws
    torch.cuda.empty_cache()
    return out


def bench_decode(args, dev, peaks, world, bf16_state=False, gated=False):
    """One decode step for 128 sequences x 48 layers, 19.3 GB float32 state (or
    9.7 GB bf16 state) in place (inputs drawn on the device; the state is far
    larger than L2).  gated: the step with the gated output norm fused in
    (z in, bf16 y out instead of float32 o)."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    n_seq, L = 128, 48
    U = n_seq * L
    gen = torch.Generator(device=dev)
    gen.manual_seed(4)

    def unit(shape):
        x = torch.randn(*shape, generator=gen, device=dev)
        x = x / torch.sqrt((x * x).sum(-1, keepdim=True) + 1e-6)
        return x.to(torch.bfloat16)

    q = unit((U, HQK, D))
    k = unit((U, HQK, D))
    v = torch.randn(U, HV, D, generator=gen, device=dev).to(torch.bfloat16)
    a = torch.randn(U, HV, generator=gen, device=dev)
    b = torch.randn(U, HV, generator=gen, device=dev)
    A_log = torch.log(torch.empty(L, HV, device=dev).uniform_(1, 16, generator=gen))
    dt = torch.exp(torch.empty(L, HV, device=dev).uniform_(-6.907755, -2.302585, generator=gen))
    dt_bias = torch.log(torch.expm1(dt))
    state = torch.empty(U, HV, D, D, dtype=torch.bfloat16 if bf16_state else torch.float32, device=dev)
    for i in range(0, U, 512):
        state[i:i + 512].normal_(0.0, 0.02, generator=gen)
    o = torch.empty(U, HV, D, dtype=torch.float32, device=dev)
    if gated:
        z = torch.randn(U, HV, D, generator=gen, device=dev).to(torch.bfloat16)
        w = torch.empty(L, D, device=dev).uniform_(0.5, 1.5, generator=gen)
        y = torch.empty(U, HV, D, dtype=torch.bfloat16, device=dev)

    def step(ev):
        if ev:
            ev["start"].record()
        if gated:
            gdn.decode_step_gated(q, k, v, a, b, A_log, dt_bias, state, n_seq, L, z, w, y=y)
        else:
            gdn.decode_step(q, k, v, a, b, A_log, dt_bias, state, n_seq, L, o=o)
        if ev:
            ev["end"].record()

    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}
    dummy = torch.empty(1, device=dev)
    times, _ = _time_steps(step, max(3, args.warmup), max(5, args.steps), dummy, mk, world)
    ms = _max_over_ranks(sum(times) / len(times), world)
    state_bytes = STATE_BYTES // 2 if bf16_state else STATE_BYTES
    out_bytes = (2 + 2) * HV * D if gated else 4 * HV * D      # z in + y out, or o out
    bytes_step = 2 * U * state_bytes + U * (2 * 2 * HQK * D + 2 * HV * D + 2 * 4 * HV + out_bytes)
    gbs = bytes_step / (ms * 1e-3) / 1e9
    wl = ("gdn_decode_step_bf16 128 seq x 48 layers, bf16 state 9.66 GB in place" if bf16_state else
          "gdn_decode_step 128 seq x 48 layers, fp32 state 19.33 GB in place")
    if gated:
        wl = wl.replace("gdn_decode_step_bf16", "gdn_decode_step").replace(
            "gdn_decode_step", "gdn_decode_step_gated (output norm fused, bf16 y)", 1)
    out = {"workload": wl,
           "ms": round(ms, 4), "GB_s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
           "bytes_per_step": int(bytes_step), "l2": "state 19.3 GB >> L2, no flush needed",
           "launches_per_step": 1}
    del state, q, k, v, o
    if gated:
        del z, y
    torch.cuda.empty_cache()
    return out


def bench_decode_fused(args, dev, peaks, world, bf16_state=False):
    """One fused decode step (front end + recurrence) for 128 sequences x 48
    layers: 19.3 GB float32 state (or 9.7 GB bf16 state) and 0.75 GB of
    convolution history in place (inputs drawn on the device; far larger than L2)."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    n_seq, L = 128, 48
    U = n_seq * L
    ctot = (2 * HQK + HV) * D
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    qkv = torch.randn(U, ctot, generator=gen, device=dev).to(torch.bfloat16)
    conv_w = 0.5 * torch.randn(L, ctot, 4, generator=gen, device=dev)
    conv_state = torch.randn(U, ctot, 3, generator=gen, device=dev)
    a = torch.randn(U, HV, generator=gen, device=dev)
    b = torch.randn(U, HV, generator=gen, device=dev)
    A_log = torch.log(torch.empty(L, HV, device=dev).uniform_(1, 16, generator=gen))
    dt = torch.exp(torch.empty(L, HV, device=dev).uniform_(-6.907755, -2.302585, generator=gen))
    dt_bias = torch.log(torch.expm1(dt))
    state = torch.empty(U, HV, D, D, dtype=torch.bfloat16 if bf16_state else torch.float32, device=dev)
    for i in range(0, U, 512):
        state[i:i + 512].normal_(0.0, 0.02, generator=gen)
    slot = torch.randperm(n_seq, generator=gen, device=dev).to(torch.int32)
    o = torch.empty(U, HV, D, dtype=torch.float32, device=dev)

    def step(ev):
        if ev:
            ev["start"].record()
        gdn.decode_step_fused(qkv, conv_w, conv_state, a, b, A_log, dt_bias, state, n_seq, L, HQK, HV,
                              slot=slot, o=o)
        if ev:
            ev["end"].record()

    mk = lambda: {"start": torch.cuda.Event(enable_timing=True),
                  "end": torch.cuda.Event(enable_timing=True)}
    dummy = torch.empty(1, device=dev)
    times, _ = _time_steps(step, max(3, args.warmup), max(5, min(args.steps, 50)), dummy, mk, world)
    ms = _max_over_ranks(sum(times) / len(times), world)
    state_bytes = STATE_BYTES // 2 if bf16_state else STATE_BYTES
    bytes_step = (2 * U * state_bytes + 2 * U * ctot * 3 * 4 + U * ctot * 2 + L * ctot * 16
                  + U * HV * (2 * 4 + 4 * D))
    gbs = bytes_step / (ms * 1e-3) / 1e9
    wl = ("gdn_decode_step_fused_bf16 128 seq x 48 layers (front end fused), bf16 state 9.66 GB"
          if bf16_state else "gdn_decode_step_fused 128 seq x 48 layers (front end fused), fp32 state 19.33 GB")
    out = {"workload": wl + " + conv history 0.75 GB in place, shuffled slots",
           "ms": round(ms, 4), "GB_s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
           "bytes_per_step": int(bytes_step), "launches_per_step": 1}
    del state, conv_state, qkv, o
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------- CPU oracle

def cpu_baseline(seconds: float = 15.0, threads: int = 0, fe=None):
    """The fp64 oracle, as it stands, on the host cores: the 8K workload's front
    end plus recurrence on a sample of value heads, repeated until ~`seconds`.
    `fe` is the workload's input (synth.workload(1)), generated here if None."""
    import oracle
    import synth
    oracle.build()
    cores = oracle.max_threads(threads)
    if fe is None:
        fe = synth.workload(1)
    g = fe.gates
    t0 = time.perf_counter()
    q, k, v, _ = oracle.conv1d_silu(fe.qkv, fe.conv_w, None, HQK, HV, D, threads=threads)
    t_fe = time.perf_counter() - t0
    # recurrence on value-head groups of `cores` heads until the time budget is used
    heads_done = 0
    t_rec = 0.0
    h = 0
    # at least one group of heads, however long the front end took
    while heads_done < HV and (heads_done == 0 or (t_fe + t_rec) < seconds):
        h1 = min(HV, h + max(1, cores))
        t1 = time.perf_counter()
        oracle.prefill(q, k, v, g.a, g.b, g.A_log, g.dt_bias, heads=(h, h1), want_o=True,
                       threads=threads)
        t_rec += time.perf_counter() - t1
        heads_done += h1 - h
        h = h1
    per_layer_s = t_fe + t_rec * HV / heads_done
    return {"value": round(T_MAIN / per_layer_s, 2), "unit": "tokens/s/layer", "cores": cores,
            "kind": "oracle",
            "sample": f"front end on all T={T_MAIN} tokens x 80 heads ({t_fe:.2f} s) + recurrence "
                      f"on {heads_done}/48 value heads x {T_MAIN} tokens ({t_rec:.2f} s), "
                      f"scaled to 48 heads"}


def profile_case(args):
    """Runs one kernel a few times on a small case for an ncu capture (not a
    benchmark: nothing is timed or printed as a result).
      prefill8k   gdn_prefill, T=8192, 1 sequence, S0 != 0   (~0.5 GB resident)
      frontend8k  gdn_conv1d_silu, T=8192                      (~0.4 GB)
      decode16    gdn_decode_step, 16 sequences x 48 layers    (~2.4 GB of state)
      decode16bf  gdn_decode_step_bf16, the same units         (~1.2 GB of state)
      frontbw8k   gdn_conv1d_silu_backward, T=8192, history    (~1.3 GB)
      bwc2k       gdn_prefill_backward_chunked, T=2048          (~0.6 GB with its workspace)
    """
    import numpy as np
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    import synth
    dev = torch.device("cuda", 0)
    to16 = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)
    f32 = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev)
    if args.profile_case == "prefill8k":
        inp = synth.make_prefill([T_MAIN], 1, init_state=True)
        d = [to16(inp.q), to16(inp.k), to16(inp.v), f32(inp.a), f32(inp.b), f32(inp.A_log), f32(inp.dt_bias)]
        s0 = f32(inp.initial_state)
        for _ in range(args.warmup + args.steps):
            gdn.prefill(*d, initial_state=s0)
    elif args.profile_case == "frontend8k":
        fe = synth.workload(1)
        x, w = to16(fe.qkv), f32(fe.conv_w)
        for _ in range(args.warmup + args.steps):
            gdn.conv1d_silu(x, w, HQK, HV)
    elif args.profile_case == "decode16":
        inp = synth.make_decode(16, 48, 4)
        st = torch.empty(inp.U, HV, D, D, dtype=torch.float32, device=dev)
        st.normal_(0.0, 0.02)
        args_ = [to16(inp.q), to16(inp.k), to16(inp.v), f32(inp.a), f32(inp.b), f32(inp.A_log),
                 f32(inp.dt_bias), st, inp.n_seq, inp.layers]
        for _ in range(args.warmup + args.steps):
            gdn.decode_step(*args_)
    elif args.profile_case == "decode16bf":
        inp = synth.make_decode(16, 48, 4)
        st = torch.empty(inp.U, HV, D, D, dtype=torch.bfloat16, device=dev)
        st.normal_(0.0, 0.02)
        args_ = [to16(inp.q), to16(inp.k), to16(inp.v), f32(inp.a), f32(inp.b), f32(inp.A_log),
                 f32(inp.dt_bias), st, inp.n_seq, inp.layers]
        for _ in range(args.warmup + args.steps):
            gdn.decode_step(*args_)
    elif args.profile_case == "frontbw8k":
        fe = synth.workload(1)
        x, w = to16(fe.qkv), f32(fe.conv_w)
        cs = torch.randn(1, (2 * HQK + HV) * D, 3, device=dev)
        gen = torch.Generator(device=dev)
        gen.manual_seed(9)
        dq = torch.randn(T_MAIN, HQK, D, generator=gen, device=dev)
        dk = torch.randn(T_MAIN, HQK, D, generator=gen, device=dev)
        dv = torch.randn(T_MAIN, HV, D, generator=gen, device=dev)
        for _ in range(args.warmup + args.steps):
            gdn.conv1d_silu_backward(x, w, dq, dk, dv, HQK, HV, conv_state=cs)
    elif args.profile_case == "bwc2k":
        inp = synth.make_prefill([2048], 5, init_state=True)
        d = [to16(inp.q), to16(inp.k), to16(inp.v), f32(inp.a), f32(inp.b), f32(inp.A_log), f32(inp.dt_bias)]
        gen = torch.Generator(device=dev)
        gen.manual_seed(8)
        d_o = torch.randn(2048, HV, D, generator=gen, device=dev)
        d_fin = 0.1 * torch.randn(1, HV, D, D, generator=gen, device=dev)
        s0 = f32(inp.initial_state)
        for _ in range(args.warmup + args.steps):
            gdn.prefill_backward_chunked(*d, d_o, d_final_state=d_fin, initial_state=s0)
    torch.cuda.synchronize()
    print(f"profile case {args.profile_case}: ok")


def run_reference(args, world, rank):
    if rank != 0:
        return
    t0 = time.perf_counter()
    vals = []
    # each step is a bounded sample, sized so that the whole run stays within minutes
    per_step = max(1.0, min(args.cpu_seconds / 3, 150.0 / (args.steps + args.warmup)))
    import synth
    fe = synth.workload(1)
    for _ in range(args.warmup):
        cpu_baseline(seconds=per_step, fe=fe)
    for _ in range(args.steps):
        vals.append(cpu_baseline(seconds=per_step, fe=fe))
    value = statistics.median(v["value"] for v in vals)
    line = {"impl": "reference",
            "metric": "GDN prefill tokens/s/layer (front end + chunked prefill, T=8192)",
            "value": value, "unit": "tokens/s/layer", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(T_MAIN / value * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": "gdn_conv1d_silu + gdn_prefill, 1 layer, T=8192, N=1, Hqk=16, "
                                   "Hv=48, d=128, zero S0, fp32 o and state", "T": T_MAIN},
            "cpu_baseline": {"kind": "oracle", "cores": vals[-1]["cores"], "value": value,
                             "unit": "tokens/s/layer", "sample": vals[-1]["sample"]},
            "e2e": {"value": value, "unit": "tokens/s/layer", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t0, 2)}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["gdn", "reference"], default="gdn")
    ap.add_argument("--primary-only", action="store_true", help="skip the 262K and decode lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile-case", choices=["prefill8k", "frontend8k", "decode16", "decode16bf", "frontbw8k", "bwc2k"],
                    help="run one kernel on a small case for an ncu capture; no timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = _dist()
    if args.profile_case:
        profile_case(args)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    bench_main(args, world, rank, local)


if __name__ == "__main__":
    main()

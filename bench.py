"""Benchmark of the SWAT attention hot path on B200.

One step = one SWAT forward + backward of the 340M-shaped attention layer
(B=8 per GPU, H=16, d=64, N=4096, window 512, balanced ALiBi, RoPE 1e4,
bf16 I/O) through the C ABI. ``value`` is band TFLOP/s of the whole job
(forward 4*B*H*d*sum_i min(i+1, w), backward 2.5x that), device-timed with
CUDA events over exactly ``--steps`` steps, max over ranks. The ring-buffer
decode (batch 64, 32/8 heads, d 128, window 4096) is timed in the same run
and reported under ``decode``.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl swat|reference]

Multi-GPU: one process per GPU (torchrun); every rank processes its own
batch (independent units, no data-path collective): weak scaling.
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
sys.path.insert(0, ROOT)

METRIC = "SWA fwd/bwd TFLOP/s & % bf16 peak (N=4K, ω=512); decode tok/s & HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def band_pairs(N: int, window: int) -> int:
    """sum_i min(i+1, w): the number of (query, key) pairs of one (b, h)."""
    w = min(window, N)
    return w * (w + 1) // 2 + (N - w) * w


def fwd_flops(B, H, d, N, window):
    return 4.0 * B * H * d * band_pairs(N, window)


def bwd_traffic_per_call(B):
    """DRAM bytes (read + write) of one backward call (its dq and dk/dv
    kernels) at batch B, from the ncu captures summarised in profiles/ (batch
    4), scaled by B / 4: every unit of work (a 128-row tile of one head) moves
    the same bytes. None when the kernel source differs from the one captured
    (its sha256 is recorded in each summary) or a summary is missing."""
    import hashlib
    import re
    src = os.path.join(ROOT, "sliding_window_sigmoid_b200", "csrc", "bwd_tc.cuh")
    try:
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
        total = 0.0
        for role in ("dq", "dkdv"):
            with open(os.path.join(ROOT, "profiles", f"swat_bwd_tc_{role}_d64_sigmoid_B4.md")) as f:
                text = f.read()
            m = re.search(r"sha256 ([0-9a-f]{64})", text)
            if not m or m.group(1) != digest:
                return None
            for kind in ("read", "write"):
                b = re.search(r"\| dram__bytes_%s\.sum \| ([0-9.]+) Mbyte \|" % kind, text)
                if not b:
                    return None
                total += float(b.group(1)) * 1e6
        return total * B / 4.0
    except OSError:
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    """One process per GPU: NCCL over the GPUs; gloo when no GPU is present
    (the host-side logic is tested that way)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    if world > 1:
        import datetime
        import torch.distributed as dist
        if cuda:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif cuda:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time: every multi-GPU number is device-timed per
    rank and reduced with MAX."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of a rank's own batch (independent units: no data-path collective)."""
    return 100 * rank


def job_value(flops_per_rank_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: the units all ranks processed over the slowest rank's time."""
    return flops_per_rank_step * world * steps / (max_ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# CPU baseline (the oracle as it stands) — rank 0 at N = 1 only
# ---------------------------------------------------------------------------

_CPU_INPUTS = {}


def _cpu_inputs():
    """b=0 of the 340M-shaped layer's seeded inputs, as float32 arrays (cached)."""
    if not _CPU_INPUTS:
        import torch
        from sliding_window_sigmoid_b200 import inputs
        wl = inputs.SWAT_340M
        q, k, v, do = inputs.qkv(1, wl.N, wl.H, wl.Hkv, wl.d, seed=0, scale=wl.scale,
                                 dtype=torch.bfloat16, with_dout=True)
        _CPU_INPUTS.update(q=q.float().numpy(), k=k.float().numpy(), v=v.float().numpy(),
                           do=do.float().numpy(), slopes=wl.slope_tensor().numpy(), wl=wl)
    return _CPU_INPUTS


def cpu_baseline_sample(n_heads: int = 8):
    """Times the fp64 oracle's forward + backward on n_heads heads (b=0, all
    4096 rows each) of the 340M-shaped layer: a bounded sample of the workload."""
    import oracle
    c = _cpu_inputs()
    wl = c["wl"]
    f = lambda a: a[:, :, :n_heads].copy()
    q, k, v, do = f(c["q"]), f(c["k"]), f(c["v"]), f(c["do"])
    sl = c["slopes"][:n_heads].copy()
    t0 = time.perf_counter()
    oracle.swat_fwd(q, k, v, window=wl.window, slopes=sl, rope_base=wl.rope_base)
    oracle.swat_bwd(q, k, v, do, window=wl.window, slopes=sl, rope_base=wl.rope_base)
    dt = time.perf_counter() - t0
    flops = 3.5 * fwd_flops(1, n_heads, wl.d, wl.N, wl.window)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": dt,
            "sample": f"fp64 C oracle forward+backward of {n_heads} heads (b=0, all {wl.N} rows) "
                      f"of the B=8,H=16,d=64,N=4096,w=512 layer"}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from sliding_window_sigmoid_b200 import inputs
    wl = inputs.SWAT_340M
    n_heads = 1
    for _ in range(max(0, args.warmup)):
        cpu_baseline_sample(n_heads)   # untimed warm-up steps
    times, cb = [], None
    for _ in range(args.steps):
        cb = cpu_baseline_sample(n_heads)
        times.append(cb["seconds"])
    total = sum(times)
    flops = 3.5 * fwd_flops(1, n_heads, wl.d, wl.N, wl.window) * args.steps
    value = flops / total / 1e12
    cb = dict(cb)
    cb["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "swat_340m_layer fwd+bwd (oracle sample: 1 head of b=0)",
                       "B": 8, "H": 16, "d": 64, "N": 4096, "window": 512,
                       "inputs": "synthetic N(0,1)/8, seed 0"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_swat(args):
    import torch
    from sliding_window_sigmoid_b200 import binding, inputs

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local if world > 1 else 0)
    wl = inputs.SWAT_340M
    B, H, Hkv, N, d, w = args.batch or wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.window
    kw = dict(window=w, n_sink=0, mode=binding.MODE_SIGMOID, slopes=wl.slope_tensor(),
              rope_base=wl.rope_base)
    q, k, v, do = [t.to(dev) for t in inputs.qkv(B, N, H, Hkv, d, seed=rank_seed(rank), scale=wl.scale,
                                                  dtype=torch.bfloat16, with_dout=True)]
    slopes = kw["slopes"].to(dev)
    kw["slopes"] = slopes
    o = torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(16, binding.bwd_workspace_bytes(B, H, Hkv, N, d)), dtype=torch.uint8,
                     device=dev)
    fws = torch.empty(max(16, binding.fwd_workspace_bytes(B, H, Hkv, N, d)), dtype=torch.uint8,
                      device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        binding.attn_fwd(q, k, v, out=o, workspace=fws, **kw)
        binding.attn_bwd(q, k, v, o, None, do, dq=dq, dk=dk, dv=dv, workspace=ws, qk_rot=fws, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if binding.device_status() != 0:
        raise RuntimeError("device status word set during warm-up")

    # timed region: exactly K steps, events between the fwd and bwd calls too
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local if world > 1 else 0)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    n0 = binding.launch_count()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        evs[i][0].record(stream)
        binding.attn_fwd(q, k, v, out=o, workspace=fws, **kw)
        evs[i][1].record(stream)
        binding.attn_bwd(q, k, v, o, None, do, dq=dq, dk=dk, dv=dv, workspace=ws, qk_rot=fws, **kw)
        evs[i][2].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = binding.launch_count() - n0
    clocks = sampler.stop()
    ms = max_over_ranks(start.elapsed_time(end), world)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    fwd_ms = max_over_ranks(fwd_ms, world)
    bwd_ms = max_over_ranks(bwd_ms, world)
    ff = fwd_flops(B, H, d, N, w)
    bf = 2.5 * ff
    step_flops = ff + bf
    value = job_value(step_flops, world, args.steps, ms)
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    fwd_tf = ff / (fwd_ms * 1e-3) / 1e12
    bwd_tf = bf / (bwd_ms * 1e-3) / 1e12
    dom = ("swat_attn_bwd", bwd_ms, bf) if bwd_ms >= fwd_ms else ("swat_attn_fwd", fwd_ms, ff)
    achieved = dom[2] / (dom[1] * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": dom[0], "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": bwd_traffic_per_call(B) if dom[0] == "swat_attn_bwd" and d == 64 else None,
                "traffic_unit": "bytes per call (ncu DRAM read + write, batch-4 captures scaled to the batch)",
                "peak_source": f"{peak_src} bf16 burst",
                "fwd": {"tflops": fwd_tf, "frac": fwd_tf / peak, "ms": fwd_ms},
                "bwd": {"tflops": bwd_tf, "frac": bwd_tf / peak, "ms": bwd_ms}}

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = bench_e2e(args, world, stream, step_flops, q, k, v, do, o, dq, dk, dv, ws, fws, kw)

    # ---- ring-buffer decode (batch 64, 32/8 heads, d 128, window 4096) ----
    decode = {}
    if not args.no_decode:
        del q, k, v, do, o, dq, dk, dv, ws, fws
        torch.cuda.empty_cache()
        decode = bench_decode(args, dev, world, rank, peaks, peak_src)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_sample(8)
    _print_line(args, rank, world, value, ms, B, H, Hkv, d, N, w, wl, roofline, cpu, e2e, clocks,
                launches, fwd_tf, bwd_tf, decode)


def bench_e2e(args, world, stream, step_flops, q, k, v, do, o, dq, dk, dv, ws, fws, kw):
    """Same step through the public API with host buffers: every step copies
    Q, K, V, dO from pinned host memory and reads O, dQ, dK, dV back. Steps
    are pipelined over three streams (host-to-device copies, compute,
    device-to-host copies) with two device buffer sets, so the copies of
    neighbouring steps overlap each other and the compute, as a training
    loop that streams batches would run them."""
    import torch
    from sliding_window_sigmoid_b200 import binding
    dev = q.device
    hq, hk, hv, hdo = [t.cpu().pin_memory() for t in (q, k, v, do)]
    ho, hdq, hdk, hdv = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (o, dq, dk, dv)]
    ins = [tuple(torch.empty_like(t) for t in (q, k, v, do)) for _ in range(2)]
    outs = [(o, dq, dk, dv), tuple(torch.empty_like(t) for t in (o, dq, dk, dv))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_ready, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(n_steps):
        for t in range(n_steps):
            j = t % 2
            if t >= 2:
                s_in.wait_event(comp_done[j])          # inputs set j free again
            with torch.cuda.stream(s_in):
                for dst, src in zip(ins[j], (hq, hk, hv, hdo)):
                    dst.copy_(src, non_blocking=True)
                in_ready[j].record(s_in)
            stream.wait_event(in_ready[j])
            if t >= 2:
                stream.wait_event(out_done[j])         # outputs set j read back
            iq, ik, iv, ido = ins[j]
            oo, odq, odk, odv = outs[j]
            binding.attn_fwd(iq, ik, iv, out=oo, workspace=fws, stream=stream, **kw)
            binding.attn_bwd(iq, ik, iv, oo, None, ido, dq=odq, dk=odk, dv=odv, workspace=ws, qk_rot=fws,
                             stream=stream, **kw)
            comp_done[j].record(stream)
            s_out.wait_event(comp_done[j])
            with torch.cuda.stream(s_out):
                for dst, src in zip((ho, hdq, hdk, hdv), outs[j]):
                    dst.copy_(src, non_blocking=True)
                out_done[j].record(s_out)

    run(max(1, args.warmup))
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    run(args.steps)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    nbytes = lambda ts: sum(t.numel() * t.element_size() for t in ts)
    e2e = {"value": job_value(step_flops, world, args.steps, e2e_ms), "unit": "TFLOP/s",
           "h2d_bytes_per_step": nbytes((hq, hk, hv, hdo)),
           "d2h_bytes_per_step": nbytes((ho, hdq, hdk, hdv)),
           "pipelined": "h2d / compute / d2h streams, 2 buffer sets"}
    return e2e


def _print_line(args, rank, world, value, ms, B, H, Hkv, d, N, w, wl, roofline, cpu, e2e, clocks,
                launches, fwd_tf, bwd_tf, decode):
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": {"workload": "swat_340m_layer fwd+bwd", "B_per_gpu": B, "H": H, "Hkv": Hkv,
                           "d": d, "N": N, "window": w, "mode": "sigmoid", "slopes": "balanced 8+8",
                           "rope_base": wl.rope_base, "global_batch": B * world,
                           "parallelism": f"independent batches x{world}",
                           "l2": "inputs+outputs 536 MB > 126 MB L2, no flush"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
                "gpu_launches": launches, "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
                "decode": decode}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def bench_decode(args, dev, world, rank, peaks, peak_src):
    import torch
    from sliding_window_sigmoid_b200 import binding, inputs
    out = {}
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    for wl in (inputs.DECODE_SIGMOID, inputs.DECODE_SOFTMAX):
        B, H, Hkv, d, w, s = args.decode_batch or wl.B, wl.H, wl.Hkv, wl.d, wl.window, wl.n_sink
        cache = binding.RingCache(B, H, Hkv, d, w, s, mode=wl.mode, slopes=wl.slope_tensor(),
                                  rope_base=wl.rope_base, device=dev)
        g = torch.Generator(device=dev)
        g.manual_seed(501 + rank)
        kf = torch.randn(B, w, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
        vf = torch.randn(B, w, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
        if s > 0:
            cache.fill(kf[:, :s].contiguous(), vf[:, :s].contiguous(), 0)
        cache.fill(kf, vf, wl.start_pos - w)
        del kf, vf
        n_steps = args.decode_steps
        qs = torch.randn(n_steps, B, H, d, generator=g, device=dev).to(torch.bfloat16)
        ks = torch.randn(n_steps, B, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
        vs = torch.randn(n_steps, B, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
        pos = torch.arange(wl.start_pos, wl.start_pos + n_steps, device=dev,
                           dtype=torch.int64)[:, None].expand(n_steps, B).contiguous()
        o = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
        for t in range(min(3, n_steps)):
            cache.step(qs[t], ks[t], vs[t], pos[t], out=o)
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier(world)
        e0.record(stream)
        for t in range(n_steps):
            cache.step(qs[t], ks[t], vs[t], pos[t], out=o)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world) / n_steps
        ring_bytes = 2 * B * Hkv * w * d * 2
        tok_s = B * world / (ms * 1e-3)
        gbs = ring_bytes / (ms * 1e-3) / 1e9
        out[wl.name] = {"batch": B, "ms_per_step": ms, "tokens_per_s": tok_s, "hbm_gbs_ring": gbs,
                        "hbm_frac": gbs / hbm, "hbm_peak": hbm, "peak_source": peak_src,
                        "steps": n_steps, "ring_bytes_per_step": ring_bytes}
        del cache, qs, ks, vs, pos, o
        torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="swat", choices=["swat", "reference"])
    ap.add_argument("--decode-steps", type=int, default=100)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences per GPU of the fwd+bwd layer (default: the workload's 8; "
                         "smaller only for profiling captures)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="decode sequences (default: the workload's 64; smaller only for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_swat(args)


if __name__ == "__main__":
    main()

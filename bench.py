"""Benchmark of the W8A8 CausalConv3d layer on B200.

One step = the whole per-call path of one layer: activation absmax + INT8
quantisation, then the implicit-GEMM convolution with its fused epilogue
(weights are quantised and packed once, before timing, as a model load
would).  Default workload: the decoder top-stage layer for a 1024x1024 image
(Cin = Cout = 384, 128x128 latent, T = 1, 1% outliers at +-8).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]

Rank 0 prints one JSON line.  With N > 1 (torchrun) every rank decodes its
own independently seeded layer (weak scaling, no collective on the data
path); the value is the ops of all ranks over the slowest rank's time.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W8A8 CausalConv3d TOPS (per layer: act absmax+quant + conv)"
UNIT = "TOPS"
DATASHEET_INT8_TOPS = 4500.0          # B200 dense INT8, NVIDIA datasheet
INT8_PER_BF16 = 2.0                    # nominal dense INT8 : BF16 ratio (4.5 / 2.25 PFLOP/s)
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decoder_top_384_128x128")
    ap.add_argument("--layer", type=int, default=0, help="layer index inside the workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def conv_source_hash():
    h = hashlib.sha256()
    for f in ("conv.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "video_vae_decode_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per conv launch from the committed ncu summary, if it still
    describes the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "conv_traffic.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        return None
    e = d.get(workload)
    if not e or e.get("kernel_sha") != conv_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, index, period=0.01):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.error = str(e)
        return self

    def _run(self):
        nv = self._nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.reasons.update(k for k, bit in names.items() if r & bit)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------- CPU baseline

def oracle_baseline(layer, seconds):
    """Time the CPU oracle on a bounded sample of the layer: the activation
    quantisation over the whole tensor (its time scaled to the sampled share)
    plus the convolution and epilogue of a seeded subset of output pixels."""
    import numpy as np
    import oracle
    from video_vae_decode_b200 import synth

    s = layer.shape
    xb, wb, bb = synth.bits(layer.x), synth.bits(layer.w), synth.bits(layer.bias)
    qw, s_w = oracle.quantize_weights(wb)                  # one-time, not timed (as on the GPU)
    t0 = time.perf_counter()
    qx, s_a = oracle.act_quant(xb)
    t_act = time.perf_counter() - t0
    total_px = s.N * s.T * s.H * s.W
    rng = np.random.default_rng(0)

    def points(n):
        return np.stack([rng.integers(0, s.N, n), rng.integers(0, s.T, n), rng.integers(0, s.H, n),
                         rng.integers(0, s.W, n)], 1).astype(np.int64)

    def run(n):
        pts = points(n)
        t = time.perf_counter()
        acc = oracle.conv_acc_points(qx, qw, pts)
        oracle.epilogue(acc, s_a, s_w, bb)
        return time.perf_counter() - t, pts

    probe = 32
    dt, _ = run(probe)
    n = int(min(total_px, max(probe, probe * seconds / max(dt, 1e-6))))
    dt, pts = run(n)
    taps = np.array([min(t + 1, 3) for t in range(s.T)])[pts[:, 1]]
    ops = float(np.sum(2.0 * s.Cin * s.Cout * 9 * taps))
    t_total = dt + t_act * n / total_px
    return {
        "value": ops / t_total / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
        "sample": (f"{n} of {total_px} output pixels (all {s.Cout} channels) of {layer_name(layer)}: "
                   f"conv + epilogue {dt:.2f} s, plus the whole-tensor act quantisation "
                   f"({t_act:.3f} s) scaled by {n}/{total_px}"),
        "seconds": t_total,
    }


def layer_name(layer):
    s = layer.shape
    return f"{s.Cin}->{s.Cout} @{s.H}x{s.W} T={s.T} N={s.N}"


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from video_vae_decode_b200 import synth
    layer = synth.draw_workload(args.workload, only=[args.layer])[0]
    steps = []
    budget = min(args.cpu_seconds, max(1.0, 150.0 / max(args.steps + min(args.warmup, 1), 1)))
    if args.warmup:
        oracle_baseline(layer, min(budget, 1.0))          # untimed: page in the library and data
    for _ in range(args.steps):
        steps.append(oracle_baseline(layer, budget))
    v = statistics.median(r["value"] for r in steps)
    last = steps[-1]
    ops = layer.shape.ops()
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ops / (v * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8/int32/f32",
        "data": "synthetic (seeded stand-in for the decoder's latents and random-init weights)",
        "config": {"workload": args.workload, "layer": layer_name(layer), "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------- GPU arm

def run_ours(args):
    import torch
    import torch.distributed as dist
    from video_vae_decode_b200 import qvae, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    wl = synth.WORKLOADS[args.workload]
    layer = synth.draw_workload(args.workload, seed=wl.seed + rank, only=[args.layer])[0]
    s = layer.shape
    x = layer.x.to(dev)
    w, b = layer.w.to(dev), layer.bias.to(dev)
    packed, s_w = qvae.quantize_weights(w)                 # once, as at model load
    xq = torch.empty(x.shape, dtype=torch.int8, device=dev)
    x_scale = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(qvae.qvae_act_workspace_bytes(x.numel()), dtype=torch.uint8, device=dev)
    out = torch.empty((s.N, s.T, s.H, s.W, s.Cout), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        qvae.qvae_act_absmax_quant(x, xq, x_scale, ws, stream)
        e_mid.record(stream)
        qvae.qvae_causal_conv3d_w8a8(xq, x_scale, packed, s_w, b, out, stream)

    e_mid = torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if qvae.qvae_get_error() != 0:
        raise RuntimeError("device-side timeout during warm-up")

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for i in range(K):
            flush.zero_()                                   # L2 flush, outside the timed events
            a, m, z = ev[i]
            a.record(stream)
            e_mid = m
            step()
            z.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(z) for a, _, z in ev]
    act_ms = [a.elapsed_time(m) for a, m, _ in ev]
    conv_ms = [m.elapsed_time(z) for _, m, z in ev]
    total_ms = sum(step_ms)
    if qvae.qvae_get_error() != 0:
        raise RuntimeError("device-side timeout during timing")

    # ---- end to end: pinned host input -> device -> layer -> pinned host output
    x_host = layer.x.pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_steps = max(3, min(K, 200))
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(e2e_steps)]
    torch.cuda.synchronize()
    for i in range(e2e_steps):
        flush.zero_()
        a, z = e2e_ev[i]
        a.record(stream)
        x.copy_(x_host, non_blocking=True)
        e_mid = torch.cuda.Event(enable_timing=True)
        step()
        out_host.copy_(out, non_blocking=True)
        z.record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(z) for a, z in e2e_ev) / e2e_steps

    ops = s.ops()
    t = torch.tensor([total_ms, e2e_ms, statistics.mean(conv_ms)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms_max, e2e_ms_max, conv_ms_max = t.tolist()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    ms_per_step = total_ms_max / K
    value = ops * world / (ms_per_step * 1e-3) / 1e12
    bf16_burst, bf16_sust, peak_src = measured_peaks()
    peak = bf16_burst * INT8_PER_BF16
    conv_tops = ops / (statistics.mean(conv_ms) * 1e-3) / 1e12
    traffic = profiled_traffic(args.workload)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8 x int8 -> int32, f32 epilogue, bf16 io",
        "data": "synthetic (seeded stand-in for the decoder's latents and random-init weights)",
        "config": {"workload": args.workload, "layer": layer_name(layer),
                   "tiling": qvae.qvae_get_conv_tiling(s.N, s.T, s.H, s.W, s.Cin, s.Cout),
                   "l2": "flushed (256 MiB write) before every timed step", "ops_per_layer": ops},
        "ms_per_layer": {"act_absmax_quant": statistics.mean(act_ms), "conv": statistics.mean(conv_ms),
                         "total": statistics.mean(step_ms), "conv_median": statistics.median(conv_ms)},
        "conv_tops": conv_tops,
        "pct_datasheet_int8_peak": 100.0 * conv_tops / DATASHEET_INT8_TOPS,
        "roofline": {"bound": "tensor", "achieved": conv_tops, "peak": peak, "unit": "TOPS",
                     "frac": conv_tops / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 burst {bf16_burst} TFLOP/s x {INT8_PER_BF16} "
                                    "(nominal dense INT8/BF16 ratio)",
                     "kernel": "conv3d_w8a8_kernel"},
        "e2e": {"value": ops * world / (e2e_ms_max * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": out.numel() * 2},
        "gpu_launches": 3 * K,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        cb = oracle_baseline(layer, args.cpu_seconds)
        cb.pop("seconds", None)
        line["cpu_baseline"] = cb
    print(json.dumps(line))
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

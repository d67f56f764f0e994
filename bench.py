"""Benchmark of the W8A8 CausalConv3d layer on B200.

One step = the whole per-call path of one layer: activation absmax + INT8
quantisation, then the implicit-GEMM convolution with its fused epilogue
(weights are quantised and packed once, before timing, as a model load
would).  Default workload: the decoder top-stage layer for a 1024x1024 image
(Cin = Cout = 384, 128x128 latent, T = 1, 1% outliers at +-8).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]
                    [--layer I] [--chunk C | --bands B] [--chain I,J] [--launch graph|stream]

Rank 0 prints one JSON line.  With N > 1 (torchrun) every rank decodes its
own independently seeded layer (weak scaling, no collective on the data
path); the value is the ops of all ranks over the slowest rank's time.

Other modes of the same measurement (one GPU): --chunk C decodes a
multi-frame layer as a stream of C-frame chunks carrying two frames each;
--bands B decodes one image layer in B row bands (tiled decode); --chain I,J
runs consecutive layers of a workload through qvae_decode_layers, each
output feeding the next input.  --impl reference times the CPU oracle.
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
L2_BYTES = 126 * 10**6
ARITHMETIC = "int8 x int8 products, int32 accumulation, fp32 rescale + bias, bf16 in and out"
SPIN_CYCLES = 200_000                  # ~100 us of GPU spin ahead of each event-timed group


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
    ap.add_argument("--chunk", type=int, default=0,
                    help="decode a multi-frame layer as a stream of chunks of this many frames, each "
                         "carrying the previous chunk's last two input frames (0: whole layer at once)")
    ap.add_argument("--bands", type=int, default=0,
                    help="decode one image layer in this many row bands (tiled decode: whole-image "
                         "absmax, then per band quantise + band convolution)")
    ap.add_argument("--chain", default="",
                    help="comma-separated consecutive layers of the workload run as one qvae_decode_layers "
                         "chain, each output feeding the next input (one GPU)")
    ap.add_argument("--launch", default="graph", choices=["graph", "stream"],
                    help="timed steps as CUDA-graph replays (one graph per buffer set) or direct launches")
    return ap.parse_args()


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes its own independently seeded layer (weak scaling)."""
    return base_seed + rank


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings (a no-op on one process)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def code_only(src: str) -> str:
    """C/C++ source without comments and blank lines (comment edits keep the hash)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in src.splitlines())
    return "\n".join(ln for ln in lines if ln.strip())


def conv_source_hash():
    """Hash of the convolution kernel's code (conv.cuh + ptx.cuh, comments stripped)."""
    h = hashlib.sha256()
    for f in ("conv.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "video_vae_decode_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode())
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
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded stand-in for the decoder's latents and random-init weights)",
        "config": {"workload": args.workload, "layer": layer_name(layer), "l2": "n/a (CPU)",
                   "arithmetic": ARITHMETIC},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------- GPU arm

def run_ours(args):
    import math
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
    layer = synth.draw_workload(args.workload, seed=rank_seed(wl.seed, rank), only=[args.layer])[0]
    s = layer.shape
    w, b = layer.w.to(dev), layer.bias.to(dev)
    packed0, s_w = qvae.quantize_weights(w)                # once, as at model load
    torch.cuda.synchronize()
    # A side stream (CUDA graphs cannot capture the legacy default stream);
    # every launch and copy below runs on it.
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    # Buffer sets (input, codes, output, packed weights) rotate so that every
    # step reads and writes memory that is not in L2, as a decoder layer does:
    # together the sets are more than three times the 126 MB L2.
    per_set = x_bytes = layer.x.numel() * 2
    per_set += layer.x.numel() + s.pixels * s.Cout * 2 + packed0.numel()
    n_sets = max(2, math.ceil(3 * L2_BYTES / per_set))
    sets = []
    for _ in range(n_sets):
        sets.append(dict(
            x=layer.x.to(dev), xq=torch.empty(layer.x.shape, dtype=torch.int8, device=dev),
            x_scale=torch.empty(1, dtype=torch.float32, device=dev),
            ws=torch.empty(qvae.qvae_act_workspace_bytes(layer.x.numel()), dtype=torch.uint8, device=dev),
            out=torch.empty((s.N, s.T, s.H, s.W, s.Cout), dtype=torch.bfloat16, device=dev),
            packed=packed0.clone()))

    # Streamed decode (--chunk C, one video): chunk k covers frames
    # [kC, kC + C); its input is the view x[:, kC - 2 : kC + C] (the two frames
    # before it carried), quantised as one tensor, then the carried-frame
    # convolution; chunk 0 has no history and runs the causal convolution.
    chunk = args.chunk if (args.chunk > 0 and s.T > args.chunk) else 0
    if chunk and s.N != 1:
        raise SystemExit("--chunk streams one video (N = 1)")
    starts = list(range(0, s.T, chunk)) if chunk else [0]
    if chunk:
        for st in sets:
            st["chunks"] = []
            for k, t0 in enumerate(starts):
                t1 = min(t0 + chunk, s.T)
                xv = st["x"][:, (t0 - 2 if k else 0):t1]
                st["chunks"].append(dict(
                    k=k, x=xv, xq=torch.empty(xv.shape, dtype=torch.int8, device=dev),
                    x_scale=torch.empty(1, dtype=torch.float32, device=dev),
                    ws=torch.empty(qvae.qvae_act_workspace_bytes(xv.numel()), dtype=torch.uint8, device=dev),
                    out=st["out"][:, t0:t1]))
            del st["xq"]

    # Tiled decode (--bands B, one image): the whole image's absmax into a
    # word, then per band its rows plus halo rows quantised from that word and
    # the band convolution into the band's output rows.
    nb = args.bands if args.bands > 1 else 0
    if nb and s.N * s.T != 1:
        raise SystemExit("--bands decodes one image (N = T = 1)")
    if nb and chunk:
        raise SystemExit("--bands and --chunk do not combine")
    if nb:
        from video_vae_decode_b200 import bands as bandlib
        for st in sets:
            st["amax"] = torch.empty(1, dtype=torch.int32, device=dev)
            st["bands"] = []
            for k in range(nb):
                r0, r1 = bandlib.band_rows(s.H, nb, k)
                lo, hi, ht, hb = bandlib.band_input(s.H, r0, r1)
                xv = st["x"][:, :, lo:hi]
                st["bands"].append(dict(x=xv, xq=torch.empty(xv.shape, dtype=torch.int8, device=dev),
                                        x_scale=torch.empty(1, dtype=torch.float32, device=dev),
                                        ht=ht, hb=hb, out=st["out"][:, :, r0:r1]))
            del st["xq"]

    def act_one(c):
        qvae.qvae_act_absmax_quant(c["x"], c["xq"], c["x_scale"], c["ws"], stream)

    def band_quant(st, c):
        qvae.qvae_act_quant_from_absmax(c["x"], st["amax"], c["xq"], c["x_scale"], stream)

    def band_conv(st, c):
        qvae.qvae_causal_conv3d_w8a8_band(c["xq"], c["ht"], c["hb"], c["x_scale"], st["packed"], s_w, b,
                                          c["out"], stream)

    def conv_one(c, packed):
        if c.get("k", 0) == 0:
            qvae.qvae_causal_conv3d_w8a8(c["xq"], c["x_scale"], packed, s_w, b, c["out"], stream)
        else:
            qvae.qvae_causal_conv3d_w8a8_carry(c["xq"], c["x_scale"], packed, s_w, b, c["out"], stream)

    def parts(st):
        return st["chunks"] if chunk else [st]

    def act(st):
        if nb:
            qvae.qvae_act_absmax(st["x"], st["amax"], stream)
            for c in st["bands"]:
                band_quant(st, c)
            return
        for c in parts(st):
            act_one(c)

    def conv(st):
        if nb:
            for c in st["bands"]:
                band_conv(st, c)
            return
        for c in parts(st):
            conv_one(c, st["packed"])

    def step(st):
        if nb:
            qvae.qvae_act_absmax(st["x"], st["amax"], stream)
            for c in st["bands"]:
                band_quant(st, c)
                band_conv(st, c)
            return
        for c in parts(st):
            act_one(c)
            conv_one(c, st["packed"])

    # One CUDA graph per buffer set holds that set's step (the three kernels,
    # with their programmatic launch dependencies): a replay costs the host one
    # call, so the timed loop measures the device, not the Python launch path.
    # First call of the layer in this process (tiling choice, tensor-map
    # encoding, kernel attributes and module load included), host wall clock.
    torch.cuda.synchronize()
    t_first = time.perf_counter()
    step(sets[0])
    torch.cuda.synchronize()
    first_call_ms = (time.perf_counter() - t_first) * 1e3
    if args.launch == "graph":
        graphs = []
        for st in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(st)
            graphs.append(g)
        torch.cuda.synchronize()

        def run_step(i):
            graphs[i % n_sets].replay()
    else:
        def run_step(i):
            step(sets[i % n_sets])

    for i in range(args.warmup):
        run_step(i)
    torch.cuda.synchronize()
    if qvae.qvae_get_error() != 0:
        raise RuntimeError("device-side timeout during warm-up")

    # ---- timed region: K steps back to back
    K = args.steps
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        e_start.record(stream)
        for i in range(K):
            run_step(i)
        e_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms = e_start.elapsed_time(e_end)
    if qvae.qvae_get_error() != 0:
        raise RuntimeError("device-side timeout during timing")

    # ---- per-kernel durations (for the roofline): events around each launch.
    # A GPU spin ahead of each group keeps the device behind the host, so the
    # events time the kernels and not the host's launch gaps.
    R = max(20, min(K, 400))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(R)]
    for i in range(R):
        st = sets[i % n_sets]
        torch.cuda._sleep(SPIN_CYCLES)
        ev[i][0].record(stream)
        act(st)
        ev[i][1].record(stream)
        conv(st)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    act_ms = [a.elapsed_time(m) for a, m, _ in ev]

    # A resolution switch: the first call of the same layer at the spatial size
    # scaled by 840/1024 (the pages' switch from 1024x1024 to 840x1256 output),
    # in this warm process; nothing is compiled per shape.
    Hs, Ws = max(1, (s.H * 840) // 1024), max(1, (s.W * 1256) // 1024)
    xs = torch.randn((s.N, s.T, Hs, Ws, s.Cin), device=dev).to(torch.bfloat16)
    xqs = torch.empty(xs.shape, dtype=torch.int8, device=dev)
    scs = torch.empty(1, dtype=torch.float32, device=dev)
    wss = torch.empty(qvae.qvae_act_workspace_bytes(xs.numel()), dtype=torch.uint8, device=dev)
    outs = torch.empty((s.N, s.T, Hs, Ws, s.Cout), dtype=torch.bfloat16, device=dev)
    switch_ms = []
    for _ in range(2):                            # first call, then the same call warm
        torch.cuda.synchronize()
        t_sw = time.perf_counter()
        qvae.qvae_act_absmax_quant(xs, xqs, scs, wss, stream)
        qvae.qvae_causal_conv3d_w8a8(xqs, scs, packed0, s_w, b, outs, stream)
        torch.cuda.synchronize()
        switch_ms.append((time.perf_counter() - t_sw) * 1e3)
    del xs, xqs, wss, outs
    conv_ms = [m.elapsed_time(z) for _, m, z in ev]

    # ---- end to end: pinned host input -> device -> layer -> pinned host output.
    # Every step copies its own input in and its own output back; as in a
    # serving loop, the copies run on their own streams (one per direction)
    # and overlap the neighbouring steps' compute: step i + 1's input lands
    # in its buffer set while step i computes and step i - 1's output leaves.
    x_host = layer.x.pin_memory()
    out_hosts = [torch.empty(sets[0]["out"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d_stream, d2h_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e2e_steps = max(3, min(K, 200))
    loaded = [torch.cuda.Event() for _ in range(n_sets)]
    computed = [torch.cuda.Event() for _ in range(n_sets)]
    drained = [torch.cuda.Event() for _ in range(n_sets)]
    for ev_ in drained:
        ev_.record(d2h_stream)
    torch.cuda.synchronize()
    e2e_a, e2e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_a.record(h2d_stream)
    for i in range(e2e_steps):
        k = i % n_sets
        st = sets[k]
        h2d_stream.wait_event(drained[k])           # the set's previous output has left the device
        with torch.cuda.stream(h2d_stream):
            st["x"].copy_(x_host, non_blocking=True)
        loaded[k].record(h2d_stream)
        stream.wait_event(loaded[k])
        act(st)
        conv(st)
        computed[k].record(stream)
        d2h_stream.wait_event(computed[k])
        with torch.cuda.stream(d2h_stream):
            out_hosts[i % 2].copy_(st["out"], non_blocking=True)
        drained[k].record(d2h_stream)
    e2e_b.record(d2h_stream)
    torch.cuda.synchronize()
    e2e_ms = e2e_a.elapsed_time(e2e_b) / e2e_steps

    ops = s.ops()
    total_ms_max, e2e_ms_max, conv_ms_max = max_over_ranks([total_ms, e2e_ms, statistics.mean(conv_ms)], dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    ms_per_step = total_ms_max / K
    value = ops * world / (ms_per_step * 1e-3) / 1e12
    bf16_burst, bf16_sust, peak_src = measured_peaks()
    peak = bf16_burst * INT8_PER_BF16
    conv_mean = statistics.mean(conv_ms)
    conv_tops = ops / (conv_mean * 1e-3) / 1e12
    traffic = profiled_traffic(args.workload)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded stand-in for the decoder's latents and random-init weights)",
        "config": {"workload": args.workload, "layer": layer_name(layer), "arithmetic": ARITHMETIC,
                   "tiling": qvae.qvae_get_conv_tiling(s.N, s.T, s.H, s.W, s.Cin, s.Cout),
                   "l2": (f"inputs, codes, outputs and packed weights rotate over {n_sets} buffer sets "
                          f"({n_sets * per_set / 2**20:.0f} MiB > 3x the 126 MB L2); no flush in the timed region"),
                   "launch": ("one CUDA graph replay per step (act absmax, act quantise, conv)"
                              if args.launch == "graph" else "direct launches from Python"),
                   "ops_per_layer": ops,
                   "stream_chunk": (f"{chunk} frames, two carried" if chunk else None),
                   "row_bands": nb or None},
        "ms_per_layer": {"step": ms_per_step, "act_absmax_quant": statistics.mean(act_ms),
                         "conv": conv_mean, "conv_median": statistics.median(conv_ms)},
        "conv_tops": conv_tops,
        "act_gbs": {"moved_5B": 5 * layer.x.numel() / (statistics.mean(act_ms) * 1e-3) / 1e9,
                    "algorithmic_3B": 3 * layer.x.numel() / (statistics.mean(act_ms) * 1e-3) / 1e9,
                    "note": "activation passes: 5 B per element moved (bf16 read twice, int8 written; "
                            "the second read hits L2 when x fits), 3 B algorithmic; measured copy "
                            "bandwidth 6557 GB/s"},
        "first_call_ms": {"process_first": first_call_ms,
                          "resolution_switch": {"shape": f"{Hs}x{Ws}", "first": switch_ms[0],
                                                "warm": switch_ms[1]},
                          "note": "host wall clock, act + conv with a device synchronise"},
        "pct_datasheet_int8_peak": 100.0 * conv_tops / DATASHEET_INT8_TOPS,
        "roofline": {"bound": "tensor", "achieved": conv_tops, "peak": peak, "unit": "TOPS",
                     "frac": conv_tops / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 burst {bf16_burst} TFLOP/s x {INT8_PER_BF16} "
                                    "(nominal dense INT8/BF16 ratio)",
                     "kernel": "conv3d_w8a8_kernel", "kernel_ms_mean": conv_mean, "launches": R},
        "e2e": {"value": ops * world / (e2e_ms_max * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": x_bytes, "d2h_bytes_per_step": s.pixels * s.Cout * 2},
        "gpu_launches": K * (1 + 2 * nb if nb else 3 * len(starts)),
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        cb = oracle_baseline(layer, args.cpu_seconds)
        cb.pop("seconds", None)
        line["cpu_baseline"] = cb
    print(json.dumps(line))
    return 0


def run_chain(args):
    """Layers of a workload as one qvae_decode_layers chain on one GPU.

    Each layer's output buffer is the next layer's input, so the library takes
    each input's absmax from the previous convolution's epilogue and runs only
    the quantise pass.  The same layers with separate input buffers (no
    chaining) are timed too, as `unchained_ms_per_step`.
    """
    import math
    import torch
    from video_vae_decode_b200 import qvae, synth

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    idx = [int(v) for v in args.chain.split(",")]
    wl = synth.WORKLOADS[args.workload]
    tens = synth.draw_workload(args.workload, seed=wl.seed, only=idx)
    for a, b in zip(tens, tens[1:]):
        sa, sb = a.shape, b.shape
        if (sa.N, sa.T, sa.H, sa.W, sa.Cout) != (sb.N, sb.T, sb.H, sb.W, sb.Cin):
            raise SystemExit(f"layers {idx} do not chain: {sa} -> {sb}")
    weights = []
    for t in tens:
        packed, s_w = qvae.quantize_weights(t.w.to(dev))
        weights.append((packed, s_w, t.bias.to(dev)))
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    per_set = sum(t.x.numel() * 2 + t.shape.pixels * t.shape.Cout * 2 for t in tens)
    n_sets = max(2, math.ceil(3 * L2_BYTES / per_set))

    def make_set(chained):
        x0 = tens[0].x.to(dev)
        specs, x = [], x0
        for k, t in enumerate(tens):
            if k and not chained:
                x = torch.empty_like(x)  # a separate input buffer: no chaining
            out = torch.empty((t.shape.N, t.shape.T, t.shape.H, t.shape.W, t.shape.Cout),
                              dtype=torch.bfloat16, device=dev)
            packed, s_w, b = weights[k]
            specs.append(dict(x=x, out=out, wq_packed=packed.clone(), w_scale=s_w, bias=b, quantized=True))
            x = out
        layers = qvae.make_layers(specs)
        ws = torch.empty(qvae.qvae_decode_workspace_bytes(layers), dtype=torch.uint8, device=dev)
        return dict(specs=specs, layers=layers, ws=ws)

    def timed(chained):
        sets = [make_set(chained) for _ in range(n_sets)]
        graphs = []
        qvae.qvae_decode_layers(sets[0]["layers"], sets[0]["ws"], stream)
        torch.cuda.synchronize()
        for st in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                qvae.qvae_decode_layers(st["layers"], st["ws"], stream)
            graphs.append(g)
        for i in range(args.warmup):
            graphs[i % n_sets].replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(0) as clk:
            e0.record(stream)
            for i in range(args.steps):
                graphs[i % n_sets].replay()
            e1.record(stream)
            torch.cuda.synchronize()
        if qvae.qvae_get_error() != 0:
            raise RuntimeError("device-side timeout")
        del graphs, sets
        return e0.elapsed_time(e1) / args.steps, clk.summary()

    ms, clocks = timed(True)
    ms_unchained, _ = timed(False)
    ops = sum(t.shape.ops() for t in tens)
    line = {
        "metric": METRIC + ", layer chain", "value": ops / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded stand-in for the decoder's latents and random-init weights)",
        "config": {"workload": args.workload, "chain": [layer_name(t) for t in tens], "arithmetic": ARITHMETIC,
                   "l2": f"{n_sets} buffer sets rotate ({n_sets * per_set / 2**20:.0f} MiB)",
                   "launch": "one CUDA graph replay per chain (qvae_decode_layers)", "ops": ops},
        "unchained_ms_per_step": ms_unchained,
        "gpu_launches": 3 * len(tens) * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line))
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.chain:
        return run_chain(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

"""Benchmark of the W8A8 CausalConv3d layers of the VAE decoder on B200.

One step = the whole per-call path of every layer of the workload: for each
layer the activation absmax + INT8 quantisation, then the implicit-GEMM
convolution with its fused epilogue (weights are quantised and packed once,
before timing, as a model load would).  --fused times the other form of a
layer: the absmax pass, then the convolution that quantises its bf16 input
itself.  Default workload: the six decoder
layer shapes of a 1024x1024 decode (384->384 @128x128 and @256x256, 384->192
and 192->192 @512x512, 192->96 and 96->96 @1024x1024, 1% outliers at +-8);
its first layer is the same tensors as the single decoder top-stage layer
(384->384, 128x128).  The line reports the whole sweep's TOPS and, per layer,
ms, conv TOPS and the fraction of the INT8 tensor peak.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]
                    [--layer I] [--chunk C | --bands B | --split] [--chain I,J] [--launch graph|stream]

Rank 0 prints one JSON line.  With N > 1 (torchrun) every rank decodes its
own independently seeded layers (weak scaling, no collective on the data
path); the value is the ops of all ranks over the slowest rank's time.

Other modes (one layer, --layer I): --chunk C decodes a multi-frame layer as
a stream of C-frame chunks carrying two frames each; --bands B decodes one
image layer in B row bands (tiled decode); --split splits one image layer
across the ranks by row bands (an all-reduce MAX of the activation maximum and
one halo row to and from each neighbour over NCCL; strong scaling); --chain
I,J runs consecutive layers of a workload through qvae_decode_layers, each
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
HBM_GBS_MEASURED = 6557.0
ARITHMETIC = "int8 x int8 products, int32 accumulation, fp32 rescale + bias, bf16 in and out"
DATA = "synthetic (seeded stand-in for the decoder's latents and random-init weights)"
SPIN_CYCLES = 200_000                  # ~100 us of GPU spin ahead of each event-timed group


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decoder_sweep_1024")
    ap.add_argument("--layer", type=int, default=-1, help="one layer of the workload (-1: all of them)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=18.0)
    ap.add_argument("--chunk", type=int, default=0,
                    help="decode a multi-frame layer as a stream of chunks of this many frames, each "
                         "carrying the previous chunk's last two input frames (0: whole layer at once)")
    ap.add_argument("--bands", type=int, default=0,
                    help="decode one image layer in this many row bands (tiled decode: whole-image "
                         "absmax, then per band quantise + band convolution)")
    ap.add_argument("--split", action="store_true",
                    help="split one image layer across the ranks by row bands (strong scaling)")
    ap.add_argument("--native", action="store_true",
                    help="time the native-precision (bf16 kind::f16) convolution of the workload's layers")
    ap.add_argument("--fused", action="store_true",
                    help="layers as absmax + the convolution quantising its bf16 input in the kernel")
    ap.add_argument("--chain", default="",
                    help="comma-separated consecutive layers of the workload run as one qvae_decode_layers "
                         "chain, each output feeding the next input (one GPU)")
    ap.add_argument("--launch", default="graph", choices=["graph", "stream"],
                    help="timed steps as CUDA-graph replays (one graph per buffer set) or direct launches")
    return ap.parse_args()


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes its own independently seeded layers (weak scaling)."""
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


def profiled_traffic(key):
    """DRAM bytes per conv launch of one layer from the committed ncu summaries,
    if they still describe the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "conv_traffic.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        return None
    e = d.get(key)
    if not e or e.get("kernel_sha") != conv_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for ln in fh:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


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


def layer_name(layer):
    s = layer.shape
    return f"{s.Cin}->{s.Cout} @{s.H}x{s.W} T={s.T} N={s.N}"


def pick_layers(args):
    from video_vae_decode_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    idx = list(range(len(wl.layers))) if args.layer < 0 else [args.layer]
    return wl, idx


# ------------------------------------------------------------- CPU baseline

def oracle_sample(layer, seconds, threads=None):
    """Time the CPU oracle on a bounded sample of one layer: the activation
    quantisation over the whole tensor (its time scaled to the sampled share)
    plus the convolution and epilogue of a seeded subset of output pixels.
    Returns (ops, seconds, description)."""
    import numpy as np
    import oracle
    from video_vae_decode_b200 import synth

    s = layer.shape
    if threads:
        oracle.set_num_threads(threads)
    try:
        xb, wb, bb = synth.bits(layer.x), synth.bits(layer.w), synth.bits(layer.bias)
        qw, s_w = oracle.quantize_weights(wb)              # one-time, not timed (as on the GPU)
        t0 = time.perf_counter()
        qx, s_a = oracle.act_quant(xb)
        t_act = time.perf_counter() - t0
        total_px = s.N * s.T * s.H * s.W
        rng = np.random.default_rng(0)

        def run(n):
            pts = np.stack([rng.integers(0, s.N, n), rng.integers(0, s.T, n), rng.integers(0, s.H, n),
                            rng.integers(0, s.W, n)], 1).astype(np.int64)
            t = time.perf_counter()
            acc = oracle.conv_acc_points(qx, qw, pts)
            oracle.epilogue(acc, s_a, s_w, bb)
            return time.perf_counter() - t, pts

        probe = 16
        dt, _ = run(probe)
        n = int(min(total_px, max(probe, probe * seconds / max(dt, 1e-6))))
        dt, pts = run(n)
        taps = np.array([min(t + 1, 3) for t in range(s.T)])[pts[:, 1]]
        ops = float(np.sum(2.0 * s.Cin * s.Cout * 9 * taps))
        t_total = dt + t_act * n / total_px
        desc = (f"{n} of {total_px} output pixels of {layer_name(layer)}: conv + epilogue {dt:.2f} s, "
                f"plus the whole-tensor act quantisation ({t_act:.3f} s) scaled by {n}/{total_px}")
        return ops, t_total, desc
    finally:
        if threads:
            oracle.set_num_threads(os.cpu_count() or 1)


def oracle_baseline(layers, seconds, one_thread=True):
    """The oracle over a bounded sample of every layer of the workload (about
    `seconds` of CPU work in all), plus a 1-thread rate on the decoder
    top-stage layer and the 96-channel 64x64 layer."""
    import oracle
    from video_vae_decode_b200 import synth
    ops = tsec = 0.0
    parts = []
    for layer in layers:
        o, t, d = oracle_sample(layer, seconds / len(layers))
        ops += o
        tsec += t
        parts.append(d)
    out = {"value": ops / tsec / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
           "sample": "; ".join(parts), "cpu_model": cpu_model(), "seconds": tsec}
    if one_thread:
        single = {}
        for name in ("decoder_top_384_128x128", "single_96_64x64"):
            o, t, d = oracle_sample(synth.draw_workload(name)[0], 1.5, threads=1)
            single[name] = {"value": o / t / 1e12, "unit": UNIT, "sample": d}
        out["one_thread"] = single
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from video_vae_decode_b200 import synth
    wl, idx = pick_layers(args)
    layers = synth.draw_workload(args.workload, only=idx)
    steps = []
    budget = min(args.cpu_seconds, max(2.0, 150.0 / max(args.steps + min(args.warmup, 1), 1)))
    if args.warmup:
        oracle_baseline(layers, min(budget, 2.0), one_thread=False)   # untimed: page in library and data
    for _ in range(args.steps):
        steps.append(oracle_baseline(layers, budget, one_thread=False))
    v = statistics.median(r["value"] for r in steps)
    last = steps[-1]
    ops = sum(l.shape.ops() for l in layers)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ops / (v * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": DATA,
        "config": {"workload": args.workload, "layers": [layer_name(l) for l in layers], "l2": "n/a (CPU)",
                   "arithmetic": ARITHMETIC},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"], "cpu_model": last["cpu_model"]},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------- GPU arm

def int8_cublas_tops(dev, n=8192, iters=20):
    """Dense INT8 GEMM rate of the library GEMM (torch._int_mm, cuBLAS) at n^3: a
    measured INT8 reference beside the bf16-derived peak.  None if unavailable."""
    import torch
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        return 2.0 * n ** 3 * iters / (e0.elapsed_time(e1) * 1e-3) / 1e12
    except Exception:
        return None


class LayerJob:
    """Buffers and launches of one layer (plain, streamed chunks or row bands)."""

    def __init__(self, layer, dev, stream, qvae, args, single):
        import torch
        self.layer, self.s, self.stream, self.qvae = layer, layer.shape, stream, qvae
        s = self.s
        self.w, self.b = layer.w.to(dev), layer.bias.to(dev)
        self.packed0, self.s_w = qvae.quantize_weights(self.w)   # once, as at model load
        self.chunk = args.chunk if (single and args.chunk > 0 and s.T > args.chunk) else 0
        if self.chunk and s.N != 1:
            raise SystemExit("--chunk streams one video (N = 1)")
        self.nb = args.bands if (single and args.bands > 1) else 0
        if self.nb and s.N * s.T != 1:
            raise SystemExit("--bands decodes one image (N = T = 1)")
        if self.nb and self.chunk:
            raise SystemExit("--bands and --chunk do not combine")
        self.starts = list(range(0, s.T, self.chunk)) if self.chunk else [0]
        self.dev = dev
        self.fused = bool(args.fused) and not (self.chunk or self.nb)

    def set_bytes(self):
        s = self.s
        return self.layer.x.numel() * 3 + s.pixels * s.Cout * 2 + self.packed0.numel()

    def make_set(self):
        import torch
        qvae, s, dev = self.qvae, self.s, self.dev
        st = dict(x=self.layer.x.to(dev), xq=torch.empty(self.layer.x.shape, dtype=torch.int8, device=dev),
                  x_scale=torch.empty(1, dtype=torch.float32, device=dev),
                  amax=torch.empty(1, dtype=torch.int32, device=dev),
                  ws=torch.empty(qvae.qvae_act_workspace_bytes(self.layer.x.numel()), dtype=torch.uint8,
                                 device=dev),
                  out=torch.empty((s.N, s.T, s.H, s.W, s.Cout), dtype=torch.bfloat16, device=dev),
                  packed=self.packed0.clone())
        if self.chunk:
            # chunk k covers frames [kC, kC + C); its input is the view x[:, kC - 2 : kC + C]
            # (the two frames before it carried), quantised as one tensor
            st["chunks"] = []
            for k, t0 in enumerate(self.starts):
                t1 = min(t0 + self.chunk, s.T)
                xv = st["x"][:, (t0 - 2 if k else 0):t1]
                st["chunks"].append(dict(
                    k=k, x=xv, xq=torch.empty(xv.shape, dtype=torch.int8, device=dev),
                    x_scale=torch.empty(1, dtype=torch.float32, device=dev),
                    ws=torch.empty(qvae.qvae_act_workspace_bytes(xv.numel()), dtype=torch.uint8, device=dev),
                    out=st["out"][:, t0:t1]))
            del st["xq"]
        if self.nb:
            from video_vae_decode_b200 import bands as bandlib
            st["amax"] = torch.empty(1, dtype=torch.int32, device=dev)
            st["bands"] = []
            for k in range(self.nb):
                r0, r1 = bandlib.band_rows(s.H, self.nb, k)
                lo, hi, ht, hb = bandlib.band_input(s.H, r0, r1)
                xv = st["x"][:, :, lo:hi]
                st["bands"].append(dict(x=xv, xq=torch.empty(xv.shape, dtype=torch.int8, device=dev),
                                        x_scale=torch.empty(1, dtype=torch.float32, device=dev),
                                        ht=ht, hb=hb, out=st["out"][:, :, r0:r1]))
            del st["xq"]
        return st

    def launches_per_step(self):
        if self.nb:
            return 1 + 2 * self.nb
        return 2 if self.fused else 3 * len(self.starts)  # fused: absmax + convolution

    def _parts(self, st):
        return st["chunks"] if self.chunk else [st]

    def act(self, st):
        q = self.qvae
        if self.fused:
            q.qvae_act_absmax(st["x"], st["amax"], self.stream)
            return
        if self.nb:
            q.qvae_act_absmax(st["x"], st["amax"], self.stream)
            for c in st["bands"]:
                q.qvae_act_quant_from_absmax(c["x"], st["amax"], c["xq"], c["x_scale"], self.stream)
            return
        for c in self._parts(st):
            q.qvae_act_absmax_quant(c["x"], c["xq"], c["x_scale"], c["ws"], self.stream)

    def _conv_one(self, st, c):
        q = self.qvae
        if c.get("k", 0) == 0:
            q.qvae_causal_conv3d_w8a8(c["xq"], c["x_scale"], st["packed"], self.s_w, self.b, c["out"], self.stream)
        else:
            q.qvae_causal_conv3d_w8a8_carry(c["xq"], c["x_scale"], st["packed"], self.s_w, self.b, c["out"],
                                            self.stream)

    def conv(self, st):
        q = self.qvae
        if self.fused:
            q.qvae_causal_conv3d_w8a8_fused(st["x"], st["amax"], st["packed"], self.s_w, self.b, st["out"],
                                            st["x_scale"], self.stream)
            return
        if self.nb:
            for c in st["bands"]:
                q.qvae_causal_conv3d_w8a8_band(c["xq"], c["ht"], c["hb"], c["x_scale"], st["packed"], self.s_w,
                                               self.b, c["out"], self.stream)
            return
        for c in self._parts(st):
            self._conv_one(st, c)

    def step(self, st):
        q = self.qvae
        if self.fused:
            self.act(st)
            self.conv(st)
            return
        if self.nb:
            q.qvae_act_absmax(st["x"], st["amax"], self.stream)
            for c in st["bands"]:
                q.qvae_act_quant_from_absmax(c["x"], st["amax"], c["xq"], c["x_scale"], self.stream)
                q.qvae_causal_conv3d_w8a8_band(c["xq"], c["ht"], c["hb"], c["x_scale"], st["packed"], self.s_w,
                                               self.b, c["out"], self.stream)
            return
        for c in self._parts(st):
            q.qvae_act_absmax_quant(c["x"], c["xq"], c["x_scale"], c["ws"], self.stream)
            self._conv_one(st, c)


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

    wl, idx = pick_layers(args)
    layers = synth.draw_workload(args.workload, seed=rank_seed(wl.seed, rank), only=idx)
    single = len(layers) == 1
    if not single and (args.chunk or args.bands):
        raise SystemExit("--chunk and --bands take one layer (--layer I)")
    # A side stream (CUDA graphs cannot capture the legacy default stream);
    # every launch and copy below runs on it.
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    jobs = [LayerJob(l, dev, stream, qvae, args, single) for l in layers]
    torch.cuda.synchronize()

    # Buffer sets (inputs, codes, outputs, packed weights of every layer) rotate
    # so that every step reads and writes memory that is not in L2, as a
    # decoder does: together the sets are more than three times the 126 MB L2.
    per_set = sum(j.set_bytes() for j in jobs)
    n_sets = max(2, math.ceil(3 * L2_BYTES / per_set))
    sets = [[j.make_set() for j in jobs] for _ in range(n_sets)]

    def step(ss):
        for j, st in zip(jobs, ss):
            j.step(st)

    # First call of the first layer in this process (tiling choice, tensor-map
    # encoding, kernel attributes and module load included), host wall clock.
    torch.cuda.synchronize()
    t_first = time.perf_counter()
    jobs[0].step(sets[0][0])
    torch.cuda.synchronize()
    first_call_ms = (time.perf_counter() - t_first) * 1e3
    for j, st in zip(jobs, sets[0]):
        j.step(st)
    torch.cuda.synchronize()
    # One CUDA graph per buffer set holds that set's step (every layer's
    # kernels, with their programmatic launch dependencies): a replay costs the
    # host one call, so the timed loop measures the device.
    if args.launch == "graph":
        graphs = []
        for ss in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(ss)
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

    # ---- per-layer durations: events around each layer's activation passes,
    # its convolution, and both back to back.  A GPU spin ahead of each group
    # keeps the device behind the host, so the events time kernels and not
    # the host's launch gaps.
    R = max(10, min(K, 100 if single else 40))
    per_layer = []
    for li, j in enumerate(jobs):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(R)]
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(R)]
        for i in range(R):
            st = sets[i % n_sets][li]
            torch.cuda._sleep(SPIN_CYCLES)
            ev[i][0].record(stream)
            j.act(st)
            ev[i][1].record(stream)
            j.conv(st)
            ev[i][2].record(stream)
            torch.cuda._sleep(SPIN_CYCLES)
            ev2[i][0].record(stream)
            j.step(st)
            ev2[i][1].record(stream)
        torch.cuda.synchronize()
        act_ms = [a.elapsed_time(m) for a, m, _ in ev]
        conv_ms = [m.elapsed_time(z) for _, m, z in ev]
        layer_ms = [a.elapsed_time(z) for a, z in ev2]
        per_layer.append(dict(act=statistics.mean(act_ms), conv=statistics.mean(conv_ms),
                              conv_median=statistics.median(conv_ms), layer=statistics.mean(layer_ms)))
    conv_launches = R

    # A resolution switch: the first call of the first layer at the spatial size
    # scaled by 840/1024 (the pages' switch from 1024x1024 to 840x1256 output),
    # in this warm process; nothing is compiled per shape.
    s0 = jobs[0].s
    Hs, Ws = max(1, (s0.H * 840) // 1024), max(1, (s0.W * 1256) // 1024)
    xs = torch.randn((s0.N, s0.T, Hs, Ws, s0.Cin), device=dev).to(torch.bfloat16)
    ams = torch.empty(1, dtype=torch.int32, device=dev)
    scs = torch.empty(1, dtype=torch.float32, device=dev)
    outs = torch.empty((s0.N, s0.T, Hs, Ws, s0.Cout), dtype=torch.bfloat16, device=dev)
    switch_ms = []
    xqs = torch.empty(xs.shape, dtype=torch.int8, device=dev)
    wss = torch.empty(qvae.qvae_act_workspace_bytes(xs.numel()), dtype=torch.uint8, device=dev)
    for _ in range(2):                            # first call, then the same call warm
        torch.cuda.synchronize()
        t_sw = time.perf_counter()
        if jobs[0].fused:
            qvae.qvae_act_absmax(xs, ams, stream)
            qvae.qvae_causal_conv3d_w8a8_fused(xs, ams, jobs[0].packed0, jobs[0].s_w, jobs[0].b, outs, scs, stream)
        else:
            qvae.qvae_act_absmax_quant(xs, xqs, scs, wss, stream)
            qvae.qvae_causal_conv3d_w8a8(xqs, scs, jobs[0].packed0, jobs[0].s_w, jobs[0].b, outs, stream)
        torch.cuda.synchronize()
        switch_ms.append((time.perf_counter() - t_sw) * 1e3)
    del xs, outs

    # ---- end to end: pinned host inputs -> device -> layers -> pinned host outputs.
    # Every step copies its own inputs in and its own outputs back; as in a
    # serving loop, the copies run on their own streams (one per direction)
    # and overlap the neighbouring steps' compute: step i + 1's inputs land
    # in its buffer set while step i computes and step i - 1's outputs leave.
    x_hosts = [j.layer.x.pin_memory() for j in jobs]
    out_hosts = [[torch.empty(sets[0][li]["out"].shape, dtype=torch.bfloat16).pin_memory()
                  for li in range(len(jobs))] for _ in range(2)]
    h2d_stream, d2h_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e2e_steps = max(3, min(K, 200 if single else 12))
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
        ss = sets[k]
        h2d_stream.wait_event(drained[k])           # the set's previous outputs have left the device
        with torch.cuda.stream(h2d_stream):
            for st, xh in zip(ss, x_hosts):
                st["x"].copy_(xh, non_blocking=True)
        loaded[k].record(h2d_stream)
        stream.wait_event(loaded[k])
        for j, st in zip(jobs, ss):
            j.act(st)
            j.conv(st)
        computed[k].record(stream)
        d2h_stream.wait_event(computed[k])
        with torch.cuda.stream(d2h_stream):
            for st, oh in zip(ss, out_hosts[i % 2]):
                oh.copy_(st["out"], non_blocking=True)
        drained[k].record(d2h_stream)
    e2e_b.record(d2h_stream)
    torch.cuda.synchronize()
    e2e_ms = e2e_a.elapsed_time(e2e_b) / e2e_steps

    int8_tops = int8_cublas_tops(dev) if rank == 0 else None

    ops = sum(j.s.ops() for j in jobs)
    conv_total = sum(p["conv"] for p in per_layer)
    total_ms_max, e2e_ms_max, conv_total_max = max_over_ranks([total_ms, e2e_ms, conv_total], dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    ms_per_step = total_ms_max / K
    value = ops * world / (ms_per_step * 1e-3) / 1e12
    bf16_burst, bf16_sust, peak_src = measured_peaks()
    peak = bf16_burst * INT8_PER_BF16
    conv_tops = ops / (conv_total_max * 1e-3) / 1e12
    layer_entries = []
    traffic = []
    for li, (j, p) in enumerate(zip(jobs, per_layer)):
        lops = j.s.ops()
        key = args.workload if single and len(wl.layers) == 1 else f"{args.workload}[{idx[li]}]"
        # the committed counters describe one whole-layer launch of the two-pass
        # kernel; the fused kernel, row bands and streamed chunks launch otherwise
        tr = None if (j.fused or j.nb or j.chunk) else profiled_traffic(key)
        traffic.append(tr)
        numel = j.layer.x.numel()
        layer_entries.append({
            "layer": layer_name(j.layer), "index": idx[li], "ops": lops,
            "ms": p["layer"], "act_ms": p["act"], "conv_ms": p["conv"], "conv_ms_median": p["conv_median"],
            "layer_tops": lops / (p["layer"] * 1e-3) / 1e12, "conv_tops": lops / (p["conv"] * 1e-3) / 1e12,
            "conv_frac": lops / (p["conv"] * 1e-3) / 1e12 / peak,
            "act_gbs": (2 if j.fused else 5) * numel / (p["act"] * 1e-3) / 1e9,
            "tiling": qvae.qvae_get_conv_tiling(j.s.N, j.s.T, j.s.H, j.s.W, j.s.Cin, j.s.Cout,
                                                1 if j.fused else 0),
            "dram_bytes_per_conv_launch": tr})
    traffic_mean = (sum(traffic) / len(traffic)) if all(t is not None for t in traffic) else None
    h2d = sum(j.layer.x.numel() * 2 for j in jobs)
    d2h = sum(j.s.pixels * j.s.Cout * 2 for j in jobs)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": DATA,
        "config": {"workload": args.workload, "layers": [layer_name(j.layer) for j in jobs],
                   "arithmetic": ARITHMETIC,
                   "l2": (f"inputs, codes, outputs and packed weights rotate over {n_sets} buffer sets "
                          f"({n_sets * per_set / 2**20:.0f} MiB > 3x the 126 MB L2); no flush in the timed region"),
                   "launch": (("one CUDA graph replay per step (per layer: act absmax, conv quantising in its "
                               "producer)" if jobs[0].fused else
                               "one CUDA graph replay per step (per layer: act absmax, act quantise, conv)")
                              if args.launch == "graph" else "direct launches from Python"),
                   "ops_per_step": ops,
                   "stream_chunk": (f"{jobs[0].chunk} frames, two carried" if jobs[0].chunk else None),
                   "row_bands": jobs[0].nb or None},
        "ms_per_layer": {e["layer"]: e["ms"] for e in layer_entries},
        "per_layer": layer_entries,
        "conv_tops": conv_tops,
        "pct_datasheet_int8_peak": 100.0 * conv_tops / DATASHEET_INT8_TOPS,
        "first_call_ms": {"process_first": first_call_ms,
                          "resolution_switch": {"shape": f"{Hs}x{Ws}", "first": switch_ms[0], "warm": switch_ms[1]},
                          "note": "host wall clock, act + conv of the first layer with a device synchronise"},
        "roofline": {"bound": "tensor", "achieved": conv_tops, "peak": peak, "unit": "TOPS",
                     "kernel_variant": ("conv3d_w8a8_fused_kernel (bf16 in, codes made in shared memory)"
                                        if jobs[0].fused else "conv3d_w8a8_kernel (INT8 codes in)"),
                     "frac": conv_tops / peak, "traffic": traffic_mean,
                     "peak_source": f"{peak_src} bf16 burst {bf16_burst} TFLOP/s x {INT8_PER_BF16} "
                                    "(nominal dense INT8/BF16 ratio)",
                     "int8_cublas_tops": int8_tops,
                     "frac_of_int8_cublas": (conv_tops / int8_tops) if int8_tops else None,
                     "kernel": "conv3d_w8a8_fused_kernel" if jobs[0].fused else "conv3d_w8a8_kernel",
                     "kernel_ms_mean": conv_total_max / len(jobs), "launches": conv_launches * len(jobs),
                     "note": ("achieved = the layers' ops over the sum of their convolutions' mean CUDA-event "
                              "times; traffic = mean DRAM bytes per conv launch over the layers")},
        "e2e": {"value": ops * world / (e2e_ms_max * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": K * sum(j.launches_per_step() for j in jobs),
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        cb = oracle_baseline([j.layer for j in jobs], args.cpu_seconds)
        cb.pop("seconds", None)
        line["cpu_baseline"] = cb
    print(json.dumps(line))
    return 0


def run_split(args):
    """One image layer split across the ranks by row bands (bands.decode_split):
    per step, the local absmax, an all-reduce MAX of one 4-byte word, one halo
    row to and from each neighbour, then this rank's band quantisation and band
    convolution.  Strong scaling: every step decodes the same one image."""
    import torch
    import torch.distributed as dist
    from video_vae_decode_b200 import bands, qvae, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from datetime import timedelta
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wl = synth.WORKLOADS[args.workload]
    li = args.layer if args.layer >= 0 else len(wl.layers) - 1
    layer = synth.draw_workload(args.workload, only=[li])[0]      # the same image on every rank
    s = layer.shape
    if s.N * s.T != 1:
        raise SystemExit("--split decodes one image (N = T = 1)")
    r0, r1 = bands.band_rows(s.H, world, rank)
    x_rows = layer.x[:, :, r0:r1].contiguous().to(dev)
    packed, s_w = qvae.quantize_weights(layer.w.to(dev))
    ops_ = bands.QvaeBandOps(packed, s_w, layer.bias.to(dev), s.Cout)
    out = torch.empty((1, 1, r1 - r0, s.W, s.Cout), dtype=torch.bfloat16, device=dev)
    for _ in range(max(args.warmup, 3)):
        bands.decode_split(x_rows, ops_, rank, world, s.Cout, out=out)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record()
        for _ in range(args.steps):
            bands.decode_split(x_rows, ops_, rank, world, s.Cout, out=out)
        e1.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if qvae.qvae_get_error() != 0:
        raise RuntimeError("device-side timeout")
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev)[0]
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    ops = s.ops()
    line = {
        "metric": METRIC + ", one image split across GPUs by row bands", "value": ops / (ms * 1e-3) / 1e12,
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "int8", "data": DATA,
        "config": {"workload": args.workload, "layer": layer_name(layer), "arithmetic": ARITHMETIC,
                   "split": f"{world} row bands; all-reduce MAX of the activation maximum, one halo row per "
                            "neighbour (NCCL point-to-point), band quantise + band conv",
                   "launch": "direct launches from Python (NCCL calls between the kernels)"},
        "gpu_launches": args.steps * 3,
        "clocks": clk.summary(),
    }
    print(json.dumps(line))
    return 0


def run_native(args):
    """The native-precision convolution (bf16 operands on kind::f16, fp32
    accumulators, bf16 output: the layers the release note keeps unquantised)
    over the workload's layers on one GPU, in TFLOP/s against the bf16 peak.

    A step is every layer's convolution (no activation passes: the layer reads
    bf16 x directly).  Buffer sets larger than 3x L2 rotate; one CUDA graph per
    set; per-layer CUDA-event times from a second pass behind a GPU spin.
    """
    import math
    import statistics
    import torch
    from video_vae_decode_b200 import qvae, synth

    if int(os.environ.get("WORLD_SIZE", "1")) != 1:
        raise SystemExit("--native runs on one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    qvae.lib()
    wl = synth.WORKLOADS[args.workload]
    idx = [args.layer] if args.layer >= 0 else list(range(len(wl.layers)))
    layers = synth.draw_workload(args.workload, only=idx)
    layers = [layers[i] for i in idx] if len(layers) > len(idx) else layers
    packed = [qvae.pack_weights_bf16(l.w.to(dev)) for l in layers]
    bias = [l.bias.to(dev) for l in layers]
    per_set = sum(l.x.numel() * 2 + l.shape.pixels * l.shape.Cout * 2 for l in layers)
    n_sets = max(2, math.ceil(3 * 126e6 / per_set))
    sets = [[dict(x=l.x.to(dev), out=torch.empty((l.shape.N, l.shape.T, l.shape.H, l.shape.W, l.shape.Cout),
                                                dtype=torch.bfloat16, device=dev)) for l in layers]
            for _ in range(n_sets)]
    stream = torch.cuda.Stream(device=dev)   # graphs are captured on a side stream

    def step(ss):
        for st, wp, b in zip(ss, packed, bias):
            qvae.qvae_causal_conv3d_bf16(st["x"], wp, b, st["out"], stream)

    with torch.cuda.stream(stream):
        step(sets[0])
    torch.cuda.synchronize()
    graphs = []
    for ss in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(ss)
        graphs.append(g)
    with torch.cuda.stream(stream):            # replays launch on the current stream
        for i in range(max(args.warmup, 3)):
            graphs[i % n_sets].replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk, torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(args.steps):
            graphs[i % n_sets].replay()
        e1.record(stream)
        torch.cuda.synchronize()
    if qvae.qvae_get_error() != 0:
        raise RuntimeError("device-side timeout")
    ms = e0.elapsed_time(e1) / args.steps
    R = max(10, min(args.steps, 100))
    per_layer = []
    for li, l in enumerate(layers):
        ts = []
        with torch.cuda.stream(stream):
            for i in range(R):
                st = sets[i % n_sets][li]
                torch.cuda._sleep(SPIN_CYCLES)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                qvae.qvae_causal_conv3d_bf16(st["x"], packed[li], bias[li], st["out"], stream)
                b.record(stream)
                ts.append((a, b))
        torch.cuda.synchronize()
        t = statistics.mean(a.elapsed_time(b) for a, b in ts)
        per_layer.append({"layer": layer_name(l), "ms": t, "tflops": l.shape.ops() / (t * 1e-3) / 1e12,
                          "tiling": qvae.qvae_get_conv_tiling(l.shape.N, l.shape.T, l.shape.H, l.shape.W,
                                                              l.shape.Cin, l.shape.Cout, 2)})
    ops = sum(l.shape.ops() for l in layers)
    bf16_burst, _, peak_src = measured_peaks()
    conv_sum = sum(p["ms"] for p in per_layer)
    achieved = ops / (conv_sum * 1e-3) / 1e12
    line = {
        "metric": "native-precision CausalConv3d TFLOP/s (bf16 operands, fp32 accumulation, bf16 out)",
        "value": ops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": DATA,
        "config": {"workload": args.workload, "layers": [layer_name(l) for l in layers],
                   "arithmetic": "bf16 x bf16 products, fp32 accumulation, fp32 bias add, bf16 out",
                   "l2": f"inputs and outputs rotate over {n_sets} buffer sets (> 3x the 126 MB L2)",
                   "launch": "one CUDA graph replay per step (one convolution per layer)"},
        "per_layer": per_layer,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": bf16_burst, "unit": "TFLOP/s",
                     "frac": achieved / bf16_burst, "traffic": None, "peak_source": peak_src,
                     "kernel": "conv3d_bf16_kernel"},
        "gpu_launches": args.steps * len(layers),
        "clocks": clk.summary(),
    }
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
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": DATA,
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
    if args.split:
        return run_split(args)
    if args.native:
        return run_native(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

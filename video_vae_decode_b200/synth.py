"""Seeded synthetic inputs for the W8A8 CausalConv3d layer.

This module holds no arithmetic of the method: it only draws random tensors
of the decoder's layer shapes, so that the CUDA path and the CPU oracle can be
fed identical bytes.  Both sides may import it.

The trained VAE weights and real latents are not available, so these tensors
stand in for them (the release note of ComfyUI-Qwen-VAE-Triton v0.2.0 measures
a Qwen-Image decode at 1024x1024 and after a switch to 840x1256; the Wan video
decoder is named in its opening paragraph).

Recipe (one CPU ``torch.Generator`` per workload, drawn in this order per
layer, all in float32 and only then rounded to bf16):
  1. x ~ N(0, 1), shape [N, T, H, W, Cin] (channels_last order);
  2. outliers (when enabled): u ~ U[0,1) per element, then v ~ U[0,1) per
     element; where u < 0.01 the element becomes +8 if v < 0.5 else -8;
  3. drift (when enabled): d_t ~ N(0, 0.2) per frame (std), added to frame t;
  4. w ~ N(0, 1/sqrt(27 Cin)) (std), shape [Cout, Cin, 3, 3, 3];
  5. bias ~ N(0, 0.01) (std), shape [Cout].
Layers of one workload are drawn one after another from the same generator.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass(frozen=True)
class LayerShape:
    Cin: int
    Cout: int
    H: int
    W: int
    T: int = 1
    N: int = 1

    @property
    def pixels(self) -> int:
        return self.N * self.T * self.H * self.W

    def real_temporal_taps(self) -> int:
        """Sum over output frames of the temporal taps that meet a real frame."""
        return self.N * sum(min(t + 1, 3) for t in range(self.T))

    def ops(self) -> int:
        """Algorithmic INT8 ops (2 per multiply-add) of the convolution.

        Taps that meet the causal zero frames are excluded (the method never
        computes them); spatial border taps count as dense.
        """
        return 2 * self.Cin * self.Cout * 9 * self.H * self.W * self.real_temporal_taps()


@dataclass(frozen=True)
class Workload:
    name: str
    layers: tuple
    seed: int
    outliers: bool = False
    drift: bool = False
    description: str = ""


def _sweep(dims):
    chans = [(384, 384), (384, 384), (384, 192), (192, 192), (192, 96), (96, 96)]
    return tuple(LayerShape(ci, co, h, w) for (ci, co), (h, w) in zip(chans, dims))


WORKLOADS = {
    "single_96_64x64": Workload(
        "single_96_64x64", (LayerShape(96, 96, 64, 64),), seed=0,
        description="one CausalConv3d, Cin=Cout=96, T=1, 64x64"),
    "decoder_top_384_128x128": Workload(
        "decoder_top_384_128x128", (LayerShape(384, 384, 128, 128),), seed=0, outliers=True,
        description="decoder top-stage layer for a 1024x1024 image: Cin=Cout=384, T=1, "
                    "128x128, 1% outliers at +-8"),
    "decoder_sweep_1024": Workload(
        "decoder_sweep_1024",
        _sweep([(128, 128), (256, 256), (512, 512), (512, 512), (1024, 1024), (1024, 1024)]),
        seed=0, outliers=True,
        description="six decoder layer shapes for a 1024x1024 output"),
    "decoder_sweep_840x1256": Workload(
        "decoder_sweep_840x1256",
        _sweep([(105, 157), (210, 314), (420, 628), (420, 628), (840, 1256), (840, 1256)]),
        seed=1,
        description="the same six shapes after a resolution switch to 840x1256"),
    "wan_video_192_240x416_t8": Workload(
        "wan_video_192_240x416_t8", (LayerShape(192, 192, 240, 416, T=8),), seed=4, drift=True,
        description="video decode layer: Cin=Cout=192, T=8 (+2 causal zero frames), "
                    "240x416, per-frame mean drift"),
}


@dataclass
class LayerTensors:
    shape: LayerShape
    x: torch.Tensor      # bf16 [N, T, H, W, Cin], CPU
    w: torch.Tensor      # bf16 [Cout, Cin, 3, 3, 3], CPU
    bias: torch.Tensor   # bf16 [Cout], CPU


def draw_layer(gen: torch.Generator, s: LayerShape, outliers: bool = False,
               drift: bool = False) -> LayerTensors:
    x = torch.randn((s.N, s.T, s.H, s.W, s.Cin), generator=gen, dtype=torch.float32)
    if outliers:
        u = torch.rand(x.shape, generator=gen, dtype=torch.float32)
        v = torch.rand(x.shape, generator=gen, dtype=torch.float32)
        spike = torch.where(v < 0.5, torch.tensor(8.0), torch.tensor(-8.0))
        x = torch.where(u < 0.01, spike, x)
        del u, v, spike
    if drift:
        d = torch.randn((s.T,), generator=gen, dtype=torch.float32) * 0.2
        x = x + d.view(1, s.T, 1, 1, 1)
    std = 1.0 / (27.0 * s.Cin) ** 0.5
    w = torch.randn((s.Cout, s.Cin, 3, 3, 3), generator=gen, dtype=torch.float32) * std
    b = torch.randn((s.Cout,), generator=gen, dtype=torch.float32) * 0.01
    return LayerTensors(s, x.to(torch.bfloat16), w.to(torch.bfloat16), b.to(torch.bfloat16))


def draw_workload(name: str, seed: Optional[int] = None, only: Optional[List[int]] = None):
    """All layers of a named workload (optionally only some layer indices).

    Skipped layers are still drawn so that the rest keep their bytes.
    """
    wl = WORKLOADS[name]
    gen = torch.Generator("cpu")
    gen.manual_seed(wl.seed if seed is None else seed)
    out = []
    for i, s in enumerate(wl.layers):
        t = draw_layer(gen, s, wl.outliers, wl.drift)
        if only is None or i in only:
            out.append(t)
        else:
            del t
    return out


def draw_custom(shape: LayerShape, seed: int, outliers: bool = False, drift: bool = False):
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    return draw_layer(gen, shape, outliers, drift)


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (no copy of values' meaning)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")

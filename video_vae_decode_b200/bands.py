"""Row bands of one image: tiled decode for memory, and one image split across GPUs.

A layer's output rows [r0, r1) need its input rows [r0 - 1, r1 + 1) (one halo
row on each side, none past the image edge) and codes quantised with the
scale of the WHOLE image.  So a banded layer is:

  1. the maximum |x| of every band, combined (an unsigned max of bf16
     magnitude words: in place on one GPU, an all-reduce MAX across GPUs);
  2. per band: its rows plus the halo rows (on several GPUs, the neighbours'
     boundary rows arrive by point-to-point messages), quantised with that
     maximum (qvae_act_quant_from_absmax);
  3. the band convolution (qvae_causal_conv3d_w8a8_band) into the band's
     output rows.

The result equals the whole-image layer exactly.  Tiled decode for memory is
the page's fallback when a VAE decode runs out of memory (the dsh-qwen-paint
plugin README); only one band's codes are held at a time.

The compute steps go through a small ops object so that the multi-rank
orchestration can be exercised on CPU processes as well; `QvaeBandOps` is the
GPU implementation through the C ABI.
"""
from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import qvae


def band_rows(H: int, nbands: int, k: int) -> Tuple[int, int]:
    """Rows [r0, r1) of band k when H rows are split into nbands near-equal bands."""
    if not 0 <= k < nbands or nbands > max(H, 1):
        raise ValueError(f"band {k} of {nbands} for {H} rows")
    base, extra = divmod(H, nbands)
    r0 = k * base + min(k, extra)
    return r0, r0 + base + (1 if k < extra else 0)


def band_input(H: int, r0: int, r1: int) -> Tuple[int, int, int, int]:
    """Input rows [lo, hi) of output rows [r0, r1), and the halo rows above / below."""
    lo, hi = max(r0 - 1, 0), min(r1 + 1, H)
    return lo, hi, r0 - lo, hi - r1


class QvaeBandOps:
    """The three steps of a banded layer on the GPU (C ABI calls on `stream`)."""

    def __init__(self, wq_packed, w_scale, bias, Cout: int, stream=None):
        self.wq_packed, self.w_scale, self.bias, self.Cout, self.stream = wq_packed, w_scale, bias, Cout, stream

    def absmax(self, x: torch.Tensor) -> torch.Tensor:
        amax = torch.empty(1, dtype=torch.int32, device=x.device)
        qvae.qvae_act_absmax(x, amax, self.stream)
        return amax

    def quant(self, x_band: torch.Tensor, amax: torch.Tensor):
        xq = torch.empty(x_band.shape, dtype=torch.int8, device=x_band.device)
        scale = torch.empty(1, dtype=torch.float32, device=x_band.device)
        qvae.qvae_act_quant_from_absmax(x_band, amax, xq, scale, self.stream)
        return xq, scale

    def conv(self, xq_band, scale, halo_top: int, halo_bot: int, out: torch.Tensor) -> None:
        qvae.qvae_causal_conv3d_w8a8_band(xq_band, halo_top, halo_bot, scale, self.wq_packed, self.w_scale,
                                          self.bias, out, self.stream)


def decode_tiled(x: torch.Tensor, out: torch.Tensor, ops, nbands: int) -> None:
    """One GPU, one image in row bands: x [1, T, H, W, Cin] -> out [1, T, H, W, Cout].

    Bands of one frame's rows are contiguous only for N = T = 1 (decoder
    layers of an image); the views below rely on it.
    """
    N, T, H, _, _ = x.shape
    if N * T != 1:
        raise ValueError("row bands of one image: N = T = 1")
    amax = ops.absmax(x)  # the whole image's maximum, without its codes
    for k in range(nbands):
        r0, r1 = band_rows(H, nbands, k)
        lo, hi, ht, hb = band_input(H, r0, r1)
        xq, scale = ops.quant(x[:, :, lo:hi], amax)
        ops.conv(xq, scale, ht, hb, out[:, :, r0:r1])


def exchange_halo_rows(x_rows: torch.Tensor, rank: int, world: int, group=None) -> Tuple[torch.Tensor, int, int]:
    """This rank's rows [N, T, Hr, W, C] with its neighbours' boundary rows attached.

    Rank r holds band r of the image (band_rows); it sends its first row up
    and its last row down and receives the rows next to its band.  Returns
    (band input, halo rows above, halo rows below).
    """
    reqs, top, bot = [], None, None
    if rank > 0:
        top = torch.empty_like(x_rows[:, :, :1])
        reqs.append(dist.isend(x_rows[:, :, :1].contiguous(), rank - 1, group=group))
        reqs.append(dist.irecv(top, rank - 1, group=group))
    if rank < world - 1:
        bot = torch.empty_like(x_rows[:, :, -1:])
        reqs.append(dist.isend(x_rows[:, :, -1:].contiguous(), rank + 1, group=group))
        reqs.append(dist.irecv(bot, rank + 1, group=group))
    for r in reqs:
        r.wait()
    parts = [p for p in (top, x_rows, bot) if p is not None]
    return torch.cat(parts, dim=2).contiguous(), int(top is not None), int(bot is not None)


def decode_split(x_rows: torch.Tensor, ops, rank: int, world: int, Cout: int, group=None,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One image split across ranks by rows: this rank's rows in, its output rows out.

    The only exchanges are one all-reduce MAX of a 4-byte word (the global
    activation scale) and one row to and from each neighbour.
    """
    amax = ops.absmax(x_rows)
    if world > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    x_band, ht, hb = exchange_halo_rows(x_rows, rank, world, group)
    xq, scale = ops.quant(x_band, amax)
    if out is None:
        N, T, Hr, W, _ = x_rows.shape
        out = torch.empty((N, T, Hr, W, Cout), dtype=torch.bfloat16, device=x_rows.device)
    ops.conv(xq, scale, ht, hb, out)
    return out

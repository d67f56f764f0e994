"""Row bands of one image on CPU: tiled decode and the multi-rank split (gloo).

The orchestration in video_vae_decode_b200/bands.py (band rows, halo rows,
the global activation maximum, point-to-point halo exchange) is run with the
compute steps done by the oracle, so the whole split layer can be compared
with the oracle's whole-image layer bit for bit.  The GPU kernels of the
same steps are compared with the oracle in tests/test_gpu_bands.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from video_vae_decode_b200 import bands, synth


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


class OracleBandOps:
    """The three steps of a banded layer, done by the oracle (test infrastructure)."""

    def __init__(self, w, bias):
        self.qw, self.s_w = oracle.quantize_weights(bits(w))
        self.bias = bits(bias)

    def absmax(self, x):
        a = np.float32(oracle.act_absmax(bits(x)))
        return torch.tensor([int(a.view(np.uint32) >> 16) & 0x7FFF], dtype=torch.int32)

    def quant(self, x_band, amax):
        amax_f = np.uint32(int(amax.item()) << 16).view(np.float32)
        qx, s = oracle.act_quant_amax(bits(x_band), amax_f)
        return qx, s

    def conv(self, xq_band, scale, halo_top, halo_bot, out):
        acc = oracle.conv_acc(xq_band, self.qw)
        acc = acc[:, :, halo_top:acc.shape[2] - halo_bot]
        out.copy_(from_bits(oracle.epilogue(acc, scale, self.s_w, self.bias)).reshape(out.shape))


def test_band_rows_tile_the_image():
    for H in (1, 2, 7, 37, 128):
        for nb in range(1, min(H, 9) + 1):
            rows = [bands.band_rows(H, nb, k) for k in range(nb)]
            assert rows[0][0] == 0 and rows[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))
            assert max(r1 - r0 for r0, r1 in rows) - min(r1 - r0 for r0, r1 in rows) <= 1
            for r0, r1 in rows:
                lo, hi, ht, hb = bands.band_input(H, r0, r1)
                assert (ht, hb) == (int(r0 > 0), int(r1 < H)) and hi - lo == r1 - r0 + ht + hb
    with pytest.raises(ValueError):
        bands.band_rows(4, 5, 0)


@pytest.mark.parametrize("nbands", [1, 2, 3, 7])
def test_tiled_decode_equals_the_whole_layer(nbands):
    t = synth.draw_custom(synth.LayerShape(32, 32, 13, 9), seed=61, outliers=True)
    want = oracle.layer(bits(t.x), bits(t.w), bits(t.bias))["out"]
    out = torch.empty((1, 1, 13, 9, 32), dtype=torch.bfloat16)
    bands.decode_tiled(t.x, out, OracleBandOps(t.w, t.bias), nbands)
    assert np.array_equal(bits(out), want)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _split_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = synth.draw_custom(synth.LayerShape(32, 64, 11, 6, T=2), seed=62, outliers=True)
        r0, r1 = bands.band_rows(11, world, rank)
        mine = t.x[:, :, r0:r1].contiguous()
        got = bands.decode_split(mine, OracleBandOps(t.w, t.bias), rank, world, Cout=64)
        gathered = [None] * world
        dist.all_gather_object(gathered, bits(got))
        if rank == 0:
            out["split"] = np.concatenate(gathered, axis=2)
            out["want"] = oracle.layer(bits(t.x), bits(t.w), bits(t.bias))["out"]
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_split_across_ranks_equals_the_whole_layer(world):
    # the only exchanges: an all-reduce MAX of the activation maximum and one
    # halo row to and from each neighbour
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_split_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert np.array_equal(out["split"], out["want"])

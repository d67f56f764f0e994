"""Row-band decode on a B200: the activation maximum and quantise-from-maximum
entry points, the band convolution against the oracle, and tiled decode
against the whole-image layer (bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
from video_vae_decode_b200 import bands, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from video_vae_decode_b200 import qvae
    qvae.lib()
    yield qvae


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("numel", [1, 15, 16, 4097, 1 << 20, 3_000_001])
def test_absmax_word_and_quant_from_it_match_the_one_call_quantiser(q, numel):
    gen = torch.Generator().manual_seed(numel)
    x = (torch.randn(numel, generator=gen) * 3).to(torch.bfloat16)
    x[numel // 2] = -9.75
    x = x.cuda()
    amax = torch.full((1,), 12345, dtype=torch.int32, device="cuda")   # overwritten
    q.qvae_act_absmax(x, amax)
    want = np.float32(oracle.act_absmax(bits(x)))
    assert int(amax.item()) == int(want.view(np.uint32) >> 16) & 0x7FFF
    xq = torch.empty(numel, dtype=torch.int8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    q.qvae_act_quant_from_absmax(x, amax, xq, s)
    xq2, s2 = q.act_absmax_quant(x)
    assert q.qvae_get_error() == 0
    assert torch.equal(xq, xq2) and torch.equal(s, s2)


def test_quant_from_a_larger_maximum_matches_the_oracle(q):
    t = synth.draw_custom(synth.LayerShape(64, 32, 9, 14), seed=63)
    x = t.x.cuda()
    big = torch.tensor([0x4120], dtype=torch.int32, device="cuda")     # bf16 bits of 10.0
    xq = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    q.qvae_act_quant_from_absmax(x, big, xq, s)
    want_q, want_s = oracle.act_quant_amax(bits(x), np.float32(10.0))
    assert np.array_equal(xq.cpu().numpy(), want_q) and s.item() == want_s


@pytest.mark.parametrize("halo_top,halo_bot", [(0, 0), (1, 0), (0, 1), (1, 1)])
def test_band_conv_matches_the_oracle(q, halo_top, halo_bot):
    t = synth.draw_custom(synth.LayerShape(64, 96, 21, 19, T=2), seed=64, outliers=True)
    qx, _ = oracle.act_quant(bits(t.x))
    qw, _ = oracle.quantize_weights(bits(t.w))
    packed, _ = q.quantize_weights(t.w.cuda())
    acc = q.conv_acc32(torch.from_numpy(qx).cuda(), packed, 96)        # whole image
    # band of output rows [5, 17): input rows [5 - halo_top, 17 + halo_bot)
    xq_band = torch.from_numpy(np.ascontiguousarray(qx[:, :, 5 - halo_top:17 + halo_bot])).cuda()
    got = torch.empty((1, 2, 12, 19, 96), dtype=torch.int32, device="cuda")
    q.qvae_causal_conv3d_w8a8_band_acc32(xq_band, halo_top, halo_bot, packed, got)
    assert q.qvae_get_error() == 0
    band_ref = oracle.conv_acc(np.ascontiguousarray(qx[:, :, 5 - halo_top:17 + halo_bot]), qw)
    band_ref = band_ref[:, :, halo_top:band_ref.shape[2] - halo_bot]
    assert np.array_equal(got.cpu().numpy(), band_ref)
    if halo_top and halo_bot:   # with both halos the band is exactly rows 5..16 of the image
        assert torch.equal(got, acc[:, :, 5:17])


@pytest.mark.parametrize("shape,nbands", [(synth.LayerShape(192, 192, 100, 120), 3),
                                          (synth.LayerShape(384, 192, 64, 72), 5),
                                          (synth.LayerShape(96, 96, 33, 40), 1)])
def test_tiled_decode_equals_the_whole_layer(q, shape, nbands):
    t = synth.draw_custom(shape, seed=65, outliers=True)
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    packed, s_w = q.quantize_weights(w)
    xq, s_a = q.act_absmax_quant(x)
    want = q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, shape.Cout)
    out = torch.zeros_like(want)
    bands.decode_tiled(x, out, bands.QvaeBandOps(packed, s_w, b, shape.Cout), nbands)
    torch.cuda.synchronize()
    assert q.qvae_get_error() == 0
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))


def test_band_rejects_a_halo_beyond_one_row(q):
    xq = torch.zeros((1, 1, 8, 8, 32), dtype=torch.int8, device="cuda")
    acc = torch.zeros((1, 1, 4, 8, 32), dtype=torch.int32, device="cuda")
    with pytest.raises(q.QvaeError):
        q.qvae_causal_conv3d_w8a8_band_acc32(xq, 2, 2, torch.zeros(1 << 20, dtype=torch.int8, device="cuda"), acc)

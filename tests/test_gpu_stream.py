"""Streamed temporal decode: the convolution of a chunk whose input carries the
previous chunk's last two input frames (qvae_causal_conv3d_w8a8_carry), on a B200.

The bar is the same as for the causal conv: INT32 accumulators bit-exact with
the oracle (oracle.conv_acc_carry), bf16 outputs bit-exact with
oracle.layer_carry.  Two identities tie it to the causal conv: zero carried
frames give the causal conv of the chunk, and with the same codes the chunks
of a video reproduce the whole sequence's accumulators.
"""
import numpy as np
import pytest
import torch

import oracle
from video_vae_decode_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from video_vae_decode_b200 import qvae
    qvae.lib()
    yield qvae
    qvae.qvae_set_conv_tiling()
    qvae.qvae_set_conv_cta_limit(0)


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def chunk_case(q, Cin, Cout, H, W, T, seed, tiling=None, ctas=0):
    """One streamed chunk of T frames (T + 2 input frames) against the oracle."""
    t = synth.draw_custom(synth.LayerShape(Cin, Cout, H, W, T=T + 2), seed=seed, outliers=True)
    x_ext, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    if tiling:
        q.qvae_set_conv_tiling(**tiling)
    q.qvae_set_conv_cta_limit(ctas)
    try:
        packed, s_w = q.quantize_weights(w)
        xq, s_a = q.act_absmax_quant(x_ext)
        acc = q.conv_carry_acc32(xq, packed, Cout)
        out = q.conv_carry(xq, s_a, packed, s_w, b, Cout)
        assert q.qvae_get_error() == 0
    finally:
        q.qvae_set_conv_tiling()
        q.qvae_set_conv_cta_limit(0)
    ref = oracle.layer_carry(bits(x_ext), bits(w), bits(b))
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(bits(out), ref["out"])


@pytest.mark.parametrize("tiling,ctas", [(None, 0), (dict(mode=1, MS=1), 0), (dict(mode=2, MS=2, G=3), 0),
                                         (dict(mode=2, MS=2, NT=192, G=3, SB=3), 0), (dict(mode=1, MS=2), 3)])
def test_carry_chunk_exact(q, tiling, ctas):
    Cout = 192 if tiling and tiling.get("NT") == 192 else 64
    chunk_case(q, 64, Cout, 19, 37, 3, seed=7, tiling=tiling, ctas=ctas)


def test_carry_chunk_two_channel_chunks_one_frame(q):
    chunk_case(q, 192, 96, 21, 30, 1, seed=8)


def test_zero_history_equals_the_causal_conv(q):
    t = synth.draw_custom(synth.LayerShape(96, 96, 24, 40, T=3), seed=9, outliers=True)
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    x_ext = torch.cat([torch.zeros_like(x[:, :2]), x], dim=1)
    packed, s_w = q.quantize_weights(w)
    xq, s_a = q.act_absmax_quant(x)
    xq_e, s_e = q.act_absmax_quant(x_ext)
    assert torch.equal(s_a, s_e)
    want = q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, 96)
    got = q.conv_carry(xq_e, s_e, packed, s_w, b, 96)
    assert q.qvae_get_error() == 0
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("Cin,Cout,H,W,T,chunk", [(64, 64, 20, 24, 7, 2), (192, 192, 120, 208, 6, 2),
                                                  (384, 192, 64, 64, 5, 3)])
def test_chunked_stream_reproduces_the_sequence(q, Cin, Cout, H, W, T, chunk):
    # the whole video quantised once: chunk k reads frames k*chunk - 2 .. of the
    # same codes, so the chunks' accumulators must equal the whole sequence's
    t = synth.draw_custom(synth.LayerShape(Cin, Cout, H, W, T=T), seed=10, drift=True)
    x, w = t.x.cuda(), t.w.cuda()
    packed, _ = q.quantize_weights(w)
    xq, _ = q.act_absmax_quant(x)
    full = q.conv_acc32(xq, packed, Cout)
    parts = [q.conv_acc32(xq[:, :chunk].contiguous(), packed, Cout)]
    for t0 in range(chunk, T, chunk):
        parts.append(q.conv_carry_acc32(xq[:, t0 - 2:min(t0 + chunk, T)].contiguous(), packed, Cout))
    assert q.qvae_get_error() == 0
    assert torch.equal(torch.cat(parts, dim=1), full)
    if H * W <= 1024:
        assert np.array_equal(full.cpu().numpy(), oracle.conv_acc(xq.cpu().numpy(), oracle_w(q, w)))


def oracle_w(q, w):
    return oracle.quantize_weights(bits(w))[0]


def test_carry_rejects_a_chunk_without_history(q):
    xq = torch.zeros((1, 1, 8, 8, 32), dtype=torch.int8, device="cuda")
    with pytest.raises(ValueError):
        q.conv_carry_acc32(xq, torch.zeros(1 << 20, dtype=torch.int8, device="cuda"), 32)

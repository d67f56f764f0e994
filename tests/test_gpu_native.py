"""The native-precision (bf16) convolution against the oracle, on a B200.

The release note's Aggressive preset keeps two decoder convolutions in their
original precision (its exclusion rule names decoder.upsamples.14.residual.2
and .residual.6; the Balanced preset describes that stage as the 96-channel
one).  The library runs them on the same tiled convolution with bf16
operands (tcgen05 kind::f16) and fp32 accumulation.

Tolerance, from the arithmetic: the oracle's sum y is exact (binary64 of
exact bf16 products).  The kernel accumulates the products in fp32 over at
most 27 * Cin / 16 MMA steps (648 for Cin = 384); with at most two roundings
of at most 2^-23 relative per step, measured against S = sum |x * w| + |b|,
its sum is within 648 * 2^-22 * S < 2^-12 * S of y.  Adding the bias in fp32
and rounding to bf16 adds at most half a bf16 ulp.  So every output must
satisfy |out - y| <= ulp_bf16(y) + 2^-12 * S, and every raw fp32 sum
|acc - (y - b)| <= 2^-12 * S.  A dropped tap, a wrong frame or a transposed
operand moves outputs by a sizeable fraction of S and fails it.
"""
import numpy as np
import pytest
import torch

import oracle
from video_vae_decode_b200 import synth

pytestmark = pytest.mark.gpu

REL = 2.0 ** -12


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from video_vae_decode_b200 import qvae
    qvae.lib()
    yield qvae
    qvae.qvae_set_conv_tiling()
    qvae.qvae_set_conv_cta_limit(0)


def dev_bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def b2f(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_ulp(y):
    a = np.maximum(np.abs(y), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def check_outputs(got_bits, ref):
    y, S = ref["y"], ref["s_abs"]
    err = np.abs(b2f(got_bits).astype(np.float64) - y)
    bound = bf16_ulp(y) + REL * S
    bad = np.nonzero(err > bound)
    assert bad[0].size == 0, (f"{bad[0].size} outputs beyond ulp + 2^-12 S; worst ratio "
                              f"{np.max(err / bound):.3f} at {tuple(b[0] for b in bad)}")
    return float(np.mean(got_bits == ref["out"]))


def check_sums(acc, y_nobias, S):
    err = np.abs(acc.astype(np.float64) - y_nobias)
    assert np.all(err <= REL * S), f"worst fp32 sum error {np.max(err / (REL * S)):.3f} of the bound"
    return float(np.max(err / np.maximum(S, 1e-30)))


def run_case(q, shape, seed, tiling=None, ctas=0, drift=False):
    t = synth.draw_custom(shape, seed=seed, outliers=True, drift=drift)
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    if tiling:
        q.qvae_set_conv_tiling(**tiling)
    q.qvae_set_conv_cta_limit(ctas)
    try:
        packed = q.pack_weights_bf16(w)
        out = q.causal_conv3d_bf16(x, packed, b, shape.Cout)
        acc = q.conv_bf16_acc32(x, packed, shape.Cout)
        assert q.qvae_get_error() == 0
    finally:
        q.qvae_set_conv_tiling()
        q.qvae_set_conv_cta_limit(0)
    xb, wb, bb = dev_bits(x), dev_bits(w), dev_bits(b)
    ref = oracle.layer_bf16(xb, wb, bb)
    y0, S0 = oracle.conv_bf16(xb, wb, None)
    rel = check_sums(acc.cpu().numpy(), y0, S0)
    exact = check_outputs(dev_bits(out), ref)
    return exact, rel


def unpack_bf16(packed_bytes, Cin, Cout):
    """[tap][chunk][Cout][64] swizzled bf16 -> [Cout, Cin, 3, 3, 3] bits."""
    nch = (Cin + 63) // 64
    p = packed_bytes.view(np.uint16).reshape(27, nch, Cout, 8, 8)
    out = np.zeros((Cout, 27, nch * 64), dtype=np.uint16)
    for co in range(Cout):
        perm = [g ^ (co % 8) for g in range(8)]
        out[co] = p[:, :, co][:, :, perm, :].reshape(27, nch * 64)
    assert not out[:, :, Cin:].any()
    return out[:, :, :Cin].transpose(0, 2, 1).reshape(Cout, Cin, 3, 3, 3)


@pytest.mark.parametrize("Cin,Cout", [(96, 96), (384, 192), (32, 64), (160, 32)])
def test_bf16_weight_packing(q, Cin, Cout):
    t = synth.draw_custom(synth.LayerShape(Cin, Cout, 2, 2), seed=Cin * 3 + Cout)
    w = t.w.cuda()
    packed = q.pack_weights_bf16(w)
    torch.cuda.synchronize()
    assert np.array_equal(unpack_bf16(packed.cpu().numpy(), Cin, Cout), dev_bits(w))


TILINGS = [None, dict(mode=1), dict(mode=2), dict(mode=1, MS=1, G=3), dict(mode=2, MS=2, NT=32),
           dict(mode=1, MS=3, SA=1, SB=9), dict(mode=2, MS=2, G=1, SA=2, SB=9)]


@pytest.mark.parametrize("tiling", TILINGS)
def test_bf16_conv_tilings(q, tiling):
    exact, _ = run_case(q, synth.LayerShape(64, 64, 19, 37, T=4), seed=3, tiling=tiling)
    assert exact > 0.9


@pytest.mark.parametrize("shape", [
    synth.LayerShape(96, 96, 64, 64),                  # the native stage's channel count
    synth.LayerShape(192, 192, 21, 30, T=3),           # three 64-channel chunks
    synth.LayerShape(384, 384, 17, 18),                # six chunks, two N tiles
    synth.LayerShape(32, 96, 9, 11, T=5, N=2),         # a half chunk, batch > 1
    synth.LayerShape(160, 256, 8, 40),                 # NT = 256
])
@pytest.mark.parametrize("mode", [1, 2])
def test_bf16_conv_shapes(q, shape, mode):
    run_case(q, shape, seed=shape.Cin + shape.H, tiling=dict(mode=mode), drift=shape.T > 1)


@pytest.mark.parametrize("H,W,T", [(1, 1, 1), (3, 5, 2), (17, 9, 1), (1, 130, 3)])
def test_bf16_conv_tiny_and_odd(q, H, W, T):
    run_case(q, synth.LayerShape(32, 32, H, W, T=T), seed=H * 7 + W, tiling=dict(mode=1))
    run_case(q, synth.LayerShape(32, 32, H, W, T=T), seed=H * 7 + W, tiling=dict(mode=2))


def test_bf16_conv_few_ctas_walk_many_tiles(q):
    run_case(q, synth.LayerShape(96, 96, 40, 37, T=3), seed=9, ctas=4)


def test_bf16_conv_zero_input_gives_bias(q):
    t = synth.draw_custom(synth.LayerShape(96, 96, 16, 16), seed=2)
    packed = q.pack_weights_bf16(t.w.cuda())
    b = t.bias.cuda()
    out = q.causal_conv3d_bf16(torch.zeros_like(t.x).cuda(), packed, b, 96)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), b.view(1, 1, 1, 1, 96).expand_as(out).view(torch.int16))


def test_bf16_full_size_native_layer(q):
    """96->96 at 1024x1024: the native layers of a 1024x1024 decode, every element."""
    shape = synth.LayerShape(96, 96, 1024, 1024)
    exact, rel = run_case(q, shape, seed=14)
    assert exact > 0.9


def test_decode_layers_run_a_native_layer_inside_a_chain(q):
    """quantised -> native -> quantised, each output feeding the next input.  The
    native layer's epilogue takes the maximum the third layer's quantiser needs.
    Layer 0 and the codes of layer 2 are exact against the oracle; layer 1 within
    the native tolerance; layer 2 exact against the oracle run on its actual input."""
    shapes = [synth.LayerShape(96, 96, 37, 21, T=2)] * 3
    gen = torch.Generator().manual_seed(41)
    tens = [synth.draw_layer(gen, s, outliers=(i == 0)) for i, s in enumerate(shapes)]
    x = tens[0].x.cuda()
    specs = []
    for i, t in enumerate(tens):
        w, b = t.w.cuda(), t.bias.cuda()
        out = torch.zeros((1, 2, 37, 21, 96), dtype=torch.bfloat16, device="cuda")
        if i == 1:
            specs.append(dict(x=x, out=out, wq_packed=q.pack_weights_bf16(w), w_scale=None, bias=b,
                              quantized=False, w=w))
        else:
            packed, s_w = q.quantize_weights(w)
            specs.append(dict(x=x, out=out, wq_packed=packed, w_scale=s_w, bias=b, quantized=True, w=w))
        x = out
    layers = q.make_layers(specs)
    ws = torch.zeros(q.qvae_decode_workspace_bytes(layers), dtype=torch.uint8, device="cuda")
    q.qvae_decode_layers(layers, ws)
    torch.cuda.synchronize()
    assert q.qvae_get_error() == 0
    r0 = oracle.layer(dev_bits(specs[0]["x"]), dev_bits(specs[0]["w"]), dev_bits(specs[0]["bias"]))
    assert np.array_equal(dev_bits(specs[0]["out"]), r0["out"])
    r1 = oracle.layer_bf16(r0["out"], dev_bits(specs[1]["w"]), dev_bits(specs[1]["bias"]))
    check_outputs(dev_bits(specs[1]["out"]), r1)
    x2 = dev_bits(specs[2]["x"])
    r2 = oracle.layer(x2, dev_bits(specs[2]["w"]), dev_bits(specs[2]["bias"]))
    # layer 2's input maximum, taken by the native layer's epilogue (word 2 % 3), and its scale
    amax_bits = int(np.array([oracle.act_absmax(x2)], np.float32).view(np.uint32)[0] >> 16) & 0x7FFF
    assert int(ws[64 + 64 * 2:64 + 64 * 2 + 4].view(torch.int32).item()) == amax_bits
    assert ws[0:4].view(torch.float32).item() == r2["s_a"]
    assert np.array_equal(dev_bits(specs[2]["out"]), r2["out"])

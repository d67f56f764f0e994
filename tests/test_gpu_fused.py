"""The W8A8 convolution that quantises its bf16 input itself, against the oracle.

The quantise step runs inside the convolution (its producer side): the bf16
input is staged in shared memory and turned into codes there, never written
to device memory.  Codes, scale, INT32 accumulators and outputs must be those
of the method (oracle.layer): exact.  The codes are not observable directly,
so one test makes them so: with a delta kernel (weight 1 at the centre tap of
channel co = ci) every weight code is 127 and each accumulator is exactly 127
times one activation code -- over every positive and negative bf16 value up
to the maximum, for maxima at many exponents and mantissas.
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


def dev_bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def fused_case(q, x, w, b, tiling=None, ctas=0):
    Cout = w.shape[0]
    if tiling:
        q.qvae_set_conv_tiling(**tiling)
    q.qvae_set_conv_cta_limit(ctas)
    try:
        packed, s_w = q.quantize_weights(w)
        amax = torch.empty(1, dtype=torch.int32, device="cuda")
        q.qvae_act_absmax(x, amax)
        out = torch.empty(tuple(x.shape[:-1]) + (Cout,), dtype=torch.bfloat16, device="cuda")
        scale = torch.full((1,), -1.0, device="cuda")
        q.qvae_causal_conv3d_w8a8_fused(x, amax, packed, s_w, b, out, scale)
        acc = torch.empty(tuple(x.shape[:-1]) + (Cout,), dtype=torch.int32, device="cuda")
        q.qvae_causal_conv3d_w8a8_fused_acc32(x, amax, packed, acc)
        assert q.qvae_get_error() == 0
    finally:
        q.qvae_set_conv_tiling()
        q.qvae_set_conv_cta_limit(0)
    return out, acc, scale


def check(q, shape, seed, tiling=None, ctas=0, outliers=True, drift=False):
    t = synth.draw_custom(shape, seed=seed, outliers=outliers, drift=drift)
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    out, acc, scale = fused_case(q, x, w, b, tiling, ctas)
    ref = oracle.layer(dev_bits(x), dev_bits(w), dev_bits(b))
    assert np.array([scale.item()], np.float32).view(np.uint32)[0] == np.array([ref["s_a"]], np.float32).view(np.uint32)[0]
    mism = np.count_nonzero(acc.cpu().numpy() != ref["acc"])
    assert mism == 0, f"{mism} accumulators differ"
    got = dev_bits(out)
    assert np.array_equal(got, ref["out"]), f"{np.count_nonzero(got != ref['out'])} outputs differ"


TILINGS = [None, dict(mode=1), dict(mode=2), dict(mode=1, MS=1), dict(mode=2, MS=1), dict(mode=1, MS=3, G=1),
           dict(mode=2, MS=4, G=1), dict(mode=2, MS=2, NT=32), dict(mode=1, MS=2, SA=1, SB=2),
           dict(mode=2, MS=2, NT=64, G=3, SA=2, SB=2)]


@pytest.mark.parametrize("tiling", TILINGS)
def test_fused_tilings_exact(q, tiling):
    check(q, synth.LayerShape(64, 64, 19, 37, T=4), seed=1, tiling=tiling)


@pytest.mark.parametrize("shape", [
    synth.LayerShape(96, 96, 64, 64),                 # one partial chunk (96 of 128 channels)
    synth.LayerShape(192, 192, 21, 30, T=3),          # a full and a half chunk
    synth.LayerShape(384, 384, 17, 18),               # three chunks, two N tiles
    synth.LayerShape(32, 96, 9, 11, T=5, N=2),        # a quarter chunk, batch > 1
    synth.LayerShape(160, 256, 8, 40),                # NT = 256
    synth.LayerShape(192, 192, 37, 21, T=3),          # sub-tile hand-off shapes
])
@pytest.mark.parametrize("mode", [1, 2])
def test_fused_shapes_exact(q, shape, mode):
    check(q, shape, seed=shape.Cin + shape.H, tiling=dict(mode=mode), drift=shape.T > 1)


@pytest.mark.parametrize("H,W,T", [(1, 1, 1), (1, 2, 3), (3, 5, 1), (7, 9, 3), (17, 17, 2), (1, 130, 1), (130, 1, 1)])
def test_fused_tiny_and_odd(q, H, W, T):
    for mode in (1, 2):
        check(q, synth.LayerShape(32, 32, H, W, T=T), seed=H * 31 + W, tiling=dict(mode=mode))


def test_fused_few_ctas_walk_many_tiles(q):
    check(q, synth.LayerShape(64, 64, 19, 37, T=4), seed=2, tiling=dict(mode=2, MS=1, G=3), ctas=4)
    check(q, synth.LayerShape(192, 96, 40, 37, T=2), seed=3, ctas=2)


def test_fused_zero_input_gives_bias(q):
    t = synth.draw_custom(synth.LayerShape(96, 96, 16, 16), seed=2)
    x = torch.zeros_like(t.x).cuda()
    out, acc, scale = fused_case(q, x, t.w.cuda(), t.bias.cuda())
    assert scale.item() == 0.0 and not acc.any()
    b = t.bias.cuda()
    assert torch.equal(out.view(torch.int16), b.view(1, 1, 1, 1, 96).expand_as(out).view(torch.int16))


def test_fused_full_size_decoder_layers(q):
    """The decoder top-stage layer and 192->96 at 1024x1024, every element."""
    for name, i in (("decoder_top_384_128x128", 0), ("decoder_sweep_1024", 4)):
        t = synth.draw_workload(name, only=[i])[0]
        x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
        out, acc, scale = fused_case(q, x, w, b)
        qx, s_a = oracle.act_quant(dev_bits(x))
        qw, s_w = oracle.quantize_weights(dev_bits(w))
        assert scale.item() == s_a
        acc_ref = oracle.conv_acc(qx, qw)
        assert np.array_equal(acc.cpu().numpy(), acc_ref)
        assert np.array_equal(dev_bits(out), oracle.epilogue(acc_ref, s_a, s_w, dev_bits(b)))


def test_fused_codes_of_every_bf16_value(q):
    """Delta kernel: acc = 127 * code.  Every bf16 magnitude up to the maximum,
    both signs, for maxima of every mantissa at several exponents (the scale's
    reciprocal path) and a subnormal maximum (the plain-divide path)."""
    C = 64
    w = torch.zeros((C, C, 3, 3, 3))
    for c in range(C):
        w[c, c, 2, 1, 1] = 1.0
    w = w.to(torch.bfloat16).cuda()
    pos = (np.arange(0x0001, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    rng = np.random.default_rng(7)
    cases = [(e, m) for k, m in enumerate(range(0, 128, 5)) for e in [[0x3F, 0x41, 0x3B, 0x47, 0x30][k % 5]]]
    cases.append((0x00, 0x40))                         # a subnormal maximum
    for e, m in cases:
        amax = np.array([((e << 7) | m) << 16], dtype=np.uint32).view(np.float32)[0]
        xs = pos[pos <= amax]
        vals = np.concatenate([xs, -xs, [0.0, amax]]).astype(np.float32)
        rng.shuffle(vals)
        npx = -(-vals.size // C)
        H = -(-npx // 64)
        full = np.zeros(H * 64 * C, dtype=np.float32)
        full[:vals.size] = vals
        x = torch.from_numpy(full).to(torch.bfloat16).view(1, 1, H, 64, C).cuda()
        _, acc, scale = fused_case(q, x, w, None)
        codes, s_ref = oracle.act_quant(dev_bits(x))
        assert scale.item() == s_ref
        a = acc.cpu().numpy()
        assert np.array_equal(a, codes.astype(np.int32) * 127), f"codes differ for amax bits {(e << 7) | m:#x}"

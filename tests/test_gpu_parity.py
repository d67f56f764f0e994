"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200.

The bar: INT8 codes, scales and INT32 accumulators bit-exact; bf16 outputs
within 1 bf16 ulp (ordered-bit distance <= 1) or 1e-3 absolute -- the kernel
uses the oracle's operation order, so the tests also report exact matches.
Every case, the full-size decoder workloads included, compares every code,
scale, accumulator and output element with the oracle.
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


def dev_bits(t):
    """CUDA bf16 tensor -> numpy uint16 bits."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def ordered(bits):
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def assert_bf16_close(got_bits, want_bits):
    """Within 1 bf16 ulp (ordered distance) or 1e-3 absolute; returns exact-match fraction."""
    gf = (got_bits.astype(np.uint32) << 16).view(np.float32)
    wf = (want_bits.astype(np.uint32) << 16).view(np.float32)
    ulp = np.abs(ordered(got_bits) - ordered(want_bits))
    ok = (ulp <= 1) | (np.abs(gf - wf) <= 1e-3)
    bad = np.nonzero(~ok)
    assert ok.all(), f"{len(bad[0])} outputs off by more than 1 ulp, first at {tuple(b[0] for b in bad)}"
    return float(np.mean(got_bits == want_bits))


def oracle_w(qw):
    """oracle codes [Cout, Cin, 3, 3, 3] -> [Cout, 27, Cin] (tap-major)."""
    Cout, Cin = qw.shape[:2]
    return qw.reshape(Cout, Cin, 27).transpose(0, 2, 1)


def unpack(packed, Cin, Cout):
    """Undo the packed [tap][chunk][Cout][128] swizzled layout -> [Cout, 27, Cin]."""
    nch = (Cin + 127) // 128
    p = packed.reshape(27, nch, Cout, 8, 16)
    out = np.zeros((Cout, 27, nch * 128), dtype=np.int8)
    for co in range(Cout):
        rows = p[:, :, co]                       # [27, nch, 8, 16]
        perm = [g ^ (co % 8) for g in range(8)]  # logical group g sits at physical g ^ (co % 8)
        logical = rows[:, :, perm, :]            # [27, nch, 8, 16]
        out[co] = logical.reshape(27, nch * 128)
    assert not out[:, :, Cin:].any(), "channels beyond Cin must be zero"
    return out[:, :, :Cin]


# ------------------------------------------------------------------ weights

@pytest.mark.parametrize("Cin,Cout", [(96, 96), (384, 384), (384, 192), (192, 96), (32, 64), (160, 32)])
def test_weight_codes_scales_and_packing(q, Cin, Cout):
    t = synth.draw_custom(synth.LayerShape(Cin, Cout, 2, 2), seed=Cin + Cout)
    w = t.w.cuda()
    if Cout >= 64:
        w[5] = 0                                             # a zero output channel
    packed, s_w, plain = q.quantize_weights(w, plain=True)
    torch.cuda.synchronize()
    qw, s_ref = oracle.quantize_weights(dev_bits(w))
    assert np.array_equal(s_w.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(plain.cpu().numpy(), oracle_w(qw))
    assert np.array_equal(unpack(packed.cpu().numpy(), Cin, Cout), oracle_w(qw))


# -------------------------------------------------------------- activations

def check_act(q, x_dev, workspace=None):
    xq, s = q.act_absmax_quant(x_dev, workspace=workspace)
    torch.cuda.synchronize()
    qx, s_ref = oracle.act_quant(dev_bits(x_dev))
    assert np.array_equal(s.cpu().numpy().view(np.uint32), np.array([s_ref]).view(np.uint32))
    got = xq.cpu().numpy()
    mism = np.count_nonzero(got != qx)
    assert mism == 0, f"{mism} codes differ"


@pytest.mark.parametrize("name", ["single_96_64x64", "decoder_top_384_128x128"])
def test_act_quant_workloads(q, name):
    check_act(q, synth.draw_workload(name)[0].x.cuda())


@pytest.mark.parametrize("numel", [1, 7, 8, 15, 16, 17, 1000, 4095, 65537, 1 << 20, 3 * (1 << 20) + 5,
                                   7_000_003, 9_700_000, 12_000_001])
def test_act_quant_ragged_lengths(q, numel):
    g = torch.Generator().manual_seed(numel)
    x = (torch.randn(numel, generator=g) * 3).to(torch.bfloat16)
    check_act(q, x.cuda())


def test_act_quant_every_bf16_value_many_scales(q):
    """All bf16 inputs up to the absmax, for amax of every bf16 mantissa at several
    exponents: the fast quotient must reproduce the IEEE divide code for code."""
    pos = (np.arange(0x0001, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    rng = np.random.default_rng(3)
    mants = list(range(128))
    for k, m in enumerate(mants):
        e = [0x3F, 0x41, 0x3B, 0x47, 0x30][k % 5]         # exponents around 1, 4, 2^-8, 2^16, 2^-31
        am_bits = (e << 7 | m) & 0x7FFF
        amax = np.array([am_bits << 16], dtype=np.uint32).view(np.float32)[0]
        xs = pos[pos <= amax]
        vals = np.concatenate([xs, -xs, [0.0]]).astype(np.float32)
        rng.shuffle(vals)
        check_act(q, torch.from_numpy(vals).to(torch.bfloat16).cuda())


def test_act_quant_shared_workspace_many_calls(q):
    """Reuse one workspace across calls of different sizes (different numbers of
    partial maxima) and absmax positions."""
    ws = torch.empty(q.qvae_act_workspace_bytes(1), dtype=torch.uint8, device="cuda")
    g = torch.Generator().manual_seed(5)
    for k, n in enumerate([4096, 6_291_456, 17, 1_000_000, 6_291_456, 333_333]):
        x = torch.randn(n, generator=g).to(torch.bfloat16)
        x[(k * 7919) % n] = 20.0 + k
        check_act(q, x.cuda(), workspace=ws)


def test_act_quant_zero_and_empty(q):
    check_act(q, torch.zeros(1000, dtype=torch.bfloat16, device="cuda"))
    x = torch.zeros(0, dtype=torch.bfloat16, device="cuda")
    xq, s = q.act_absmax_quant(x)
    torch.cuda.synchronize()
    assert s.item() == 0.0


def test_act_quant_tiny_scales(q):
    """Subnormal absmax takes the plain-divide branch."""
    vals = np.array([1e-39, -5e-40, 3e-41, 0.0, 2e-39], dtype=np.float32)
    check_act(q, torch.from_numpy(vals).to(torch.bfloat16).cuda())


# --------------------------------------------------------------- convolution

def conv_case(q, shape, seed, tiling=None, outliers=False, drift=False):
    """Run codes -> acc32 and bf16 output on the GPU and compare with the oracle everywhere."""
    t = synth.draw_custom(shape, seed=seed, outliers=outliers, drift=drift)
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    if tiling:
        q.qvae_set_conv_tiling(**tiling)
    try:
        packed, s_w = q.quantize_weights(w)
        xq, s_a = q.act_absmax_quant(x)
        acc = q.conv_acc32(xq, packed, shape.Cout)
        out = q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, shape.Cout)
        assert q.qvae_get_error() == 0
    finally:
        if tiling:
            q.qvae_set_conv_tiling()
    ref = oracle.layer(dev_bits(x), dev_bits(w), dev_bits(b))
    got_acc = acc.cpu().numpy()
    mism = np.count_nonzero(got_acc != ref["acc"])
    assert mism == 0, f"{mism} accumulators differ"
    return assert_bf16_close(dev_bits(out), ref["out"])


TILINGS = [None,
           dict(mode=1), dict(mode=1, MS=1), dict(mode=1, MS=3), dict(mode=1, MS=4, NT=64, SA=1, SB=2),
           dict(mode=1, MS=1, SA=1, SB=1), dict(mode=1, NT=32),
           dict(mode=2), dict(mode=2, MS=1), dict(mode=2, MS=2), dict(mode=2, MS=3), dict(mode=2, MS=4),
           dict(mode=2, MS=1, SA=1, SB=1), dict(mode=2, NT=32), dict(mode=2, MS=2, NT=64, SA=2, SB=9),
           dict(mode=1, MS=1, G=3), dict(mode=1, MS=2, G=3, SA=1, SB=1), dict(mode=2, MS=1, G=3),
           dict(mode=2, MS=2, NT=32, G=3, SA=2, SB=2), dict(mode=2, MS=1, G=3, SA=1, SB=1)]


@pytest.mark.parametrize("tiling", [dict(mode=1, MS=1), dict(mode=2, MS=1, G=3), dict(mode=1, MS=4, NT=64)])
def test_conv_few_ctas_many_tiles_exact(q, tiling):
    # three CTAs (one pair in mode 2) walk all tiles: accumulator buffers and
    # ring phases wrap many times
    q.qvae_set_conv_cta_limit(3)
    try:
        assert conv_case(q, synth.LayerShape(64, 64, 19, 37, T=4), seed=2, tiling=tiling) == 1.0
    finally:
        q.qvae_set_conv_cta_limit(0)


@pytest.mark.parametrize("Cin", [32, 96, 160, 192])
@pytest.mark.parametrize("tiling", [dict(mode=2, MS=2, NT=96, G=3), dict(mode=1, MS=1, NT=96, G=3, SB=2)])
def test_conv_one_pair_every_kstep_count_exact(q, Cin, tiling):
    # one CTA pair (or two single CTAs) walks every tile, so the MMA warp's
    # lookahead probes of the next weight stage, activation stage and
    # accumulator buffer cross chunk, tile and ring boundaries many times;
    # the last 128-channel chunk has 1, 3, 1 and 2 k-steps of 32 channels
    q.qvae_set_conv_cta_limit(2)
    try:
        assert conv_case(q, synth.LayerShape(Cin, 96, 21, 19, T=3), seed=Cin, tiling=tiling) == 1.0
    finally:
        q.qvae_set_conv_cta_limit(0)


@pytest.mark.parametrize("tiling", TILINGS)
def test_conv_tilings_exact(q, tiling):
    # spans several tiles in h, w and channels, with ragged edges and T > 2
    exact = conv_case(q, synth.LayerShape(64, 64, 19, 37, T=4), seed=1, tiling=tiling)
    assert exact == 1.0


# One accumulator buffer of several sub-tiles, handed to the epilogue one by
# one (the first and last chunk of a tile issued sub-tile by sub-tile): CTA
# pairs with 3- and 1-tap weight stages, single CTAs with 3 and 4 sub-tiles.
SPLIT_TILINGS = [dict(mode=2, MS=2, NT=192, G=3, SA=2, SB=3), dict(mode=2, MS=2, NT=192, G=1, SA=2, SB=9),
                 dict(mode=1, MS=3, NT=96, G=1, SA=1, SB=9), dict(mode=1, MS=4, NT=96, G=1, SA=1, SB=9)]


@pytest.mark.parametrize("tiling", SPLIT_TILINGS)
@pytest.mark.parametrize("shape", [
    synth.LayerShape(192, 192, 37, 21, T=3),          # 2 chunks (128 + 64): 2, 4 and 6 chunks per tile
    synth.LayerShape(128, 192, 20, 24, T=2),          # 1 chunk: first and last chunk coincide at t = 0
])
@pytest.mark.parametrize("ctas", [0, 4])
def test_conv_subtile_handoff_exact(q, tiling, shape, ctas):
    # ctas = 4: every CTA walks several tiles, so hand-offs cross tile boundaries
    q.qvae_set_conv_cta_limit(ctas)
    try:
        assert conv_case(q, shape, seed=5, tiling=tiling, outliers=True) == 1.0
    finally:
        q.qvae_set_conv_cta_limit(0)


@pytest.mark.parametrize("shape", [
    synth.LayerShape(96, 96, 64, 64),                 # the 96-channel single layer
    synth.LayerShape(192, 192, 21, 30, T=3),          # two channel chunks, the second half-full
    synth.LayerShape(384, 384, 17, 18),               # three chunks, two N tiles
    synth.LayerShape(32, 96, 9, 11, T=5, N=2),        # batch > 1, all causal tap counts
    synth.LayerShape(160, 256, 8, 40),                # partial chunk of 32, NT = 256
    synth.LayerShape(96, 320, 6, 6),                  # NT = 160
])
@pytest.mark.parametrize("mode", [1, 2])
def test_conv_shapes_exact(q, shape, mode):
    conv_case(q, shape, seed=shape.Cin * 7 + shape.H, tiling=dict(mode=mode))


@pytest.mark.parametrize("H,W,T", [(1, 1, 1), (1, 2, 3), (2, 1, 2), (3, 5, 1), (5, 3, 2), (7, 9, 3),
                                   (9, 7, 1), (17, 17, 2), (1, 130, 1), (130, 1, 1)])
def test_conv_tiny_and_odd(q, H, W, T):
    conv_case(q, synth.LayerShape(32, 32, H, W, T=T), seed=H * 100 + W * 10 + T, tiling=dict(mode=1))
    conv_case(q, synth.LayerShape(32, 32, H, W, T=T), seed=H * 100 + W * 10 + T, tiling=dict(mode=2))


def test_conv_outliers_and_drift(q):
    conv_case(q, synth.LayerShape(64, 32, 12, 20), seed=5, outliers=True)
    conv_case(q, synth.LayerShape(64, 32, 12, 20, T=4), seed=6, drift=True)


def test_conv_zero_input_gives_bias(q):
    t = synth.draw_custom(synth.LayerShape(96, 96, 16, 16), seed=2)
    x = torch.zeros_like(t.x).cuda()
    packed, s_w = q.quantize_weights(t.w.cuda())
    xq, s_a = q.act_absmax_quant(x)
    b = t.bias.cuda()
    out = q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, 96)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), b.view(1, 1, 1, 1, 96).expand_as(out).view(torch.int16))
    out0 = q.causal_conv3d_w8a8(xq, s_a, packed, s_w, None, 96)
    torch.cuda.synchronize()
    assert not out0.view(torch.int16).any()


def test_conv_empty_is_noop(q):
    xq = torch.zeros((1, 0, 4, 4, 32), dtype=torch.int8, device="cuda")
    packed, s_w = q.quantize_weights(torch.zeros((32, 32, 3, 3, 3), dtype=torch.bfloat16, device="cuda"))
    s_a = torch.zeros(1, device="cuda")
    out = torch.empty((1, 0, 4, 4, 32), dtype=torch.bfloat16, device="cuda")
    q.qvae_causal_conv3d_w8a8(xq, s_a, packed, s_w, None, out)


# ----------------------------------------------------- full-size workloads

def full_layer_check(q, t):
    """Every code, scale, INT32 accumulator and bf16 output of a full-size layer
    against the oracle (the threaded oracle covers the largest layer, the video
    layer's 1.4 T ops, in well under a minute on a 16-core host)."""
    s = t.shape
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    packed, s_w = q.quantize_weights(w)
    xq, s_a = q.act_absmax_quant(x)
    out = q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, s.Cout)
    acc = q.conv_acc32(xq, packed, s.Cout)
    assert q.qvae_get_error() == 0
    xb, wb, bb = dev_bits(x), dev_bits(w), dev_bits(b)
    qx, s_ref = oracle.act_quant(xb)
    qw, sw_ref = oracle.quantize_weights(wb)
    assert np.array([s_a.item()], np.float32).view(np.uint32) == np.array([s_ref]).view(np.uint32)
    assert np.array_equal(s_w.cpu().numpy().view(np.uint32), sw_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), qx)
    del x, xq
    acc_ref = oracle.conv_acc(qx, qw)
    got_acc = acc.cpu().numpy()
    del acc
    mism = np.count_nonzero(got_acc != acc_ref)
    assert mism == 0, f"{mism} of {acc_ref.size} accumulators differ"
    del got_acc
    want = oracle.epilogue(acc_ref, s_ref, sw_ref, bb)
    exact = assert_bf16_close(dev_bits(out), want)
    assert exact == 1.0, f"outputs within 1 ulp but only {exact:.6f} bit-identical"


def test_full_single_96_64x64(q):
    full_layer_check(q, synth.draw_workload("single_96_64x64")[0])


def test_full_decoder_top_layer(q):
    full_layer_check(q, synth.draw_workload("decoder_top_384_128x128")[0])


@pytest.mark.parametrize("i", range(6))
def test_full_decoder_sweep_1024(q, i):
    full_layer_check(q, synth.draw_workload("decoder_sweep_1024", only=[i])[0])


@pytest.mark.parametrize("i", range(6))
def test_full_resolution_switch_840x1256(q, i):
    full_layer_check(q, synth.draw_workload("decoder_sweep_840x1256", only=[i])[0])


def test_full_video_layer(q):
    full_layer_check(q, synth.draw_workload("wan_video_192_240x416_t8")[0])


# --------------------------------------------------------------- layer chain

def test_decode_layers_matches_single_calls_and_skips_passthrough(q):
    shapes = [synth.LayerShape(96, 192, 20, 24), synth.LayerShape(192, 192, 20, 24),
              synth.LayerShape(192, 96, 40, 48)]
    gen = torch.Generator().manual_seed(11)
    specs, refs = [], []
    for i, s in enumerate(shapes):
        t = synth.draw_layer(gen, s, outliers=True)
        x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
        packed, s_w = q.quantize_weights(w)
        out = torch.full((s.N, s.T, s.H, s.W, s.Cout), 7.0, dtype=torch.bfloat16, device="cuda")
        # layer 1 is a native layer without weights: the library skips it
        specs.append(dict(x=x, out=out, wq_packed=None if i == 1 else packed, w_scale=s_w, bias=b,
                          quantized=(i != 1)))
        xq, s_a = q.act_absmax_quant(x)
        refs.append(q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, s.Cout))
    layers = q.make_layers(specs)
    ws = torch.empty(q.qvae_decode_workspace_bytes(layers), dtype=torch.uint8, device="cuda")
    q.qvae_decode_layers(layers, ws)
    assert q.qvae_get_error() == 0
    for i, (sp, ref) in enumerate(zip(specs, refs)):
        if i == 1:
            assert torch.all(sp["out"] == 7.0)             # pass-through layer untouched
        else:
            assert torch.equal(sp["out"].view(torch.int16), ref.view(torch.int16))


# --------------------------------------------------------- failure handling

def test_bounded_wait_reports_timeout_and_context_survives(q):
    assert q.qvae_get_error() == 0
    q.qvae_selftest_wait_timeout(2_000_000)                # 2 ms wait that nothing satisfies
    assert q.qvae_get_error() == q.QVAE_ERR_TIMEOUT
    assert q.qvae_get_error() == 0                         # cleared
    conv_case(q, synth.LayerShape(32, 32, 8, 8), seed=1)    # the context still works


# ------------------------------------------------- ordering after the packer

def test_conv_right_after_weight_packing(q):
    """The convolution loads packed weights before it waits for the kernel in
    front of it; qvae_quantize_weights ends with a launch that keeps the packer
    out of that overlap.  Repack new weights into the same buffer and run the
    convolution directly after, several times: a conv that read the previous
    weights would differ from the oracle."""
    shape = synth.LayerShape(384, 384, 40, 48)
    gen = torch.Generator().manual_seed(77)
    t = synth.draw_layer(gen, shape, outliers=True)
    x = t.x.cuda()
    xq, s_a = q.act_absmax_quant(x)
    packed = torch.empty(q.qvae_packed_weight_bytes(384, 384), dtype=torch.int8, device="cuda")
    s_w = torch.empty(384, dtype=torch.float32, device="cuda")
    out = torch.empty((1, 1, 40, 48, 384), dtype=torch.bfloat16, device="cuda")
    qx, s_ref = oracle.act_quant(dev_bits(x))
    for k in range(3):
        w = (torch.randn((384, 384, 3, 3, 3), generator=gen) * (0.02 * (k + 1))).to(torch.bfloat16)
        b = (torch.randn(384, generator=gen) * 0.01).to(torch.bfloat16)
        w_dev, b_dev = w.cuda(), b.cuda()
        torch.cuda.synchronize()
        q.qvae_quantize_weights(w_dev, packed, s_w)
        q.qvae_causal_conv3d_w8a8(xq, s_a, packed, s_w, b_dev, out)
        torch.cuda.synchronize()
        assert q.qvae_get_error() == 0
        qw, sw_ref = oracle.quantize_weights(dev_bits(w_dev))
        want = oracle.epilogue(oracle.conv_acc(qx, qw), s_ref, sw_ref, dev_bits(b_dev))
        assert assert_bf16_close(dev_bits(out), want) == 1.0


@pytest.mark.parametrize("mode", [1, 2])
def test_conv_large_accumulators_exact(q, mode):
    """Accumulators beyond 2^22 in magnitude (codes of +-127 against weights of
    +-127 over many taps reach 55.7 M for Cin = 384) take the epilogue's other
    int32 -> float path; a constant image region next to a small-valued one
    mixes both paths inside one warp.  Every output must still equal the
    oracle's bit for bit."""
    shape = synth.LayerShape(384, 192, 20, 24, T=2)
    g = torch.Generator().manual_seed(99)
    x = (torch.randn((1, 2, 20, 24, 384), generator=g) * 0.01)
    x[:, :, :10] = 1.0                                     # codes 127 in the upper half
    x[:, 1, 5:8, 3:9] = -1.0                               # and a negative patch
    w = torch.full((192, 384, 3, 3, 3), 0.02)
    w[::3] *= -1.0                                          # both signs of the maximum
    w[1::5, ::7] = 0.0013
    b = (torch.randn(192, generator=g) * 0.01)
    x, w, b = x.to(torch.bfloat16).cuda(), w.to(torch.bfloat16).cuda(), b.to(torch.bfloat16).cuda()
    q.qvae_set_conv_tiling(mode=mode)
    try:
        packed, s_w = q.quantize_weights(w)
        xq, s_a = q.act_absmax_quant(x)
        acc = q.conv_acc32(xq, packed, 192)
        out = q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, 192)
        assert q.qvae_get_error() == 0
    finally:
        q.qvae_set_conv_tiling()
    ref = oracle.layer(dev_bits(x), dev_bits(w), dev_bits(b))
    assert np.abs(ref["acc"]).max() > 2 ** 22 and np.abs(ref["acc"]).min() < 2 ** 20
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(dev_bits(out), ref["out"])

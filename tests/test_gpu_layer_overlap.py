"""The overlapped layer (qvae_layer_w8a8: the quantise pass runs inside the
convolution, beside the tensor cores) against the CPU oracle, on a B200.

Codes, scale, INT32 accumulators and bf16 outputs must all be bit-identical
to the oracle's -- the same bar as the two-call path (qvae_act_absmax_quant +
qvae_causal_conv3d_w8a8), whose codes and scale this path reproduces.  The
cases cover several tiles and ragged edges, CTA pairs and single CTAs, few
CTAs walking many tiles (the band waits and unit claims interleave), more
input rows than band counters (several rows per band), T > 2 and N > 1, the
full-size decoder layers, and the argument errors.
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


def f32_bits(t):
    return np.array([t.item()], np.float32).view(np.uint32)[0]


def run_layer(q, t, tiling=None, ctas=0, workspace=None):
    """(out, acc, codes, scale) of the overlapped layer, plus the packed weights' scales."""
    s = t.shape
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    if tiling:
        q.qvae_set_conv_tiling(**tiling)
    q.qvae_set_conv_cta_limit(ctas)
    try:
        packed, s_w = q.quantize_weights(w)
        out, xq, s_a = q.layer_w8a8(x, packed, s_w, b, s.Cout, workspace=workspace)
        acc, xq2, s_a2 = q.layer_w8a8(x, packed, s_w, b, s.Cout, workspace=workspace, acc32=True)
        assert q.qvae_get_error() == 0
    finally:
        q.qvae_set_conv_tiling()
        q.qvae_set_conv_cta_limit(0)
    assert torch.equal(xq, xq2) and f32_bits(s_a) == f32_bits(s_a2)
    return x, w, b, out, acc, xq, s_a


def check_against_oracle(q, t, **kw):
    x, w, b, out, acc, xq, s_a = run_layer(q, t, **kw)
    ref = oracle.layer(dev_bits(x), dev_bits(w), dev_bits(b))
    assert f32_bits(s_a) == np.array([ref["s_a"]], np.float32).view(np.uint32)[0], "activation scale differs"
    mism = np.count_nonzero(xq.cpu().numpy() != ref["qx"])
    assert mism == 0, f"{mism} codes differ"
    mism = np.count_nonzero(acc.cpu().numpy() != ref["acc"])
    assert mism == 0, f"{mism} accumulators differ"
    mism = np.count_nonzero(dev_bits(out) != ref["out"])
    assert mism == 0, f"{mism} outputs differ"


@pytest.mark.parametrize("shape", [
    synth.LayerShape(64, 64, 19, 37, T=4),            # several tiles in h, w, channels; ragged edges
    synth.LayerShape(192, 192, 21, 30, T=3),          # two channel chunks, the second half-full
    synth.LayerShape(384, 384, 17, 18),               # three chunks, two N tiles
    synth.LayerShape(32, 96, 9, 11, T=5, N=2),        # batch > 1, all causal tap counts
    synth.LayerShape(96, 96, 64, 64),                 # the 96-channel single layer
])
@pytest.mark.parametrize("mode", [1, 2])
def test_layer_overlap_shapes_exact(q, shape, mode):
    check_against_oracle(q, synth.draw_custom(shape, seed=shape.Cin + shape.H), tiling=dict(mode=mode))


@pytest.mark.parametrize("H,W,T", [(1, 1, 1), (1, 2, 3), (3, 5, 1), (7, 9, 3), (17, 17, 2), (1, 130, 1),
                                   (130, 1, 1)])
def test_layer_overlap_tiny_and_odd(q, H, W, T):
    check_against_oracle(q, synth.draw_custom(synth.LayerShape(32, 32, H, W, T=T), seed=H * 10 + W + T))


@pytest.mark.parametrize("tiling,ctas", [(dict(mode=1, MS=1), 3), (dict(mode=2, MS=1, G=3), 2),
                                         (dict(mode=2, MS=2, NT=96, G=3), 4), (dict(mode=1, MS=4, NT=64), 1)])
def test_layer_overlap_few_ctas_many_tiles(q, tiling, ctas):
    # few CTAs: each producer walks many tiles and band waits, and the few
    # quantising warps claim every unit of the tensor
    check_against_oracle(q, synth.draw_custom(synth.LayerShape(96, 96, 37, 21, T=3), seed=9),
                         tiling=tiling, ctas=ctas)


def test_layer_overlap_several_rows_per_band(q):
    # 2 x 3 x 700 = 4200 input rows > 4095 band counters: two rows per band
    check_against_oracle(q, synth.draw_custom(synth.LayerShape(32, 32, 700, 9, T=3, N=2), seed=4))


def test_layer_overlap_outliers_and_zero(q):
    check_against_oracle(q, synth.draw_custom(synth.LayerShape(64, 32, 12, 20), seed=5, outliers=True))
    t = synth.draw_custom(synth.LayerShape(96, 96, 16, 16), seed=2)
    t.x.zero_()
    x, w, b, out, acc, xq, s_a = run_layer(q, t)
    assert s_a.item() == 0.0 and not xq.any() and not acc.any()
    assert torch.equal(out.view(torch.int16), b.view(1, 1, 1, 1, 96).expand_as(out).view(torch.int16))


def test_layer_overlap_two_calls_and_reused_workspace(q):
    # the absmax pass and the convolution as two calls equal the one call, and
    # a workspace reused by consecutive layers on one stream needs no clearing
    t = synth.draw_custom(synth.LayerShape(128, 64, 33, 40, T=2), seed=8)
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    packed, s_w = q.quantize_weights(w)
    ws = torch.empty(q.qvae_layer_workspace_bytes(), dtype=torch.uint8, device="cuda")
    out1, xq1, s1 = q.layer_w8a8(x, packed, s_w, b, 64, workspace=ws)
    xq2 = torch.empty_like(xq1)
    s2 = torch.empty(1, device="cuda")
    out2 = torch.empty_like(out1)
    for _ in range(3):
        q.qvae_layer_w8a8_absmax(x, 64, ws)
        q.qvae_layer_w8a8_conv(x, xq2, s2, packed, s_w, b, out2, ws)
    assert q.qvae_get_error() == 0
    assert torch.equal(xq1, xq2) and f32_bits(s1) == f32_bits(s2)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_layer_overlap_matches_two_call_path_in_a_graph(q):
    # captured in a CUDA graph and replayed: the same bits as the two-call path
    t = synth.draw_custom(synth.LayerShape(192, 96, 40, 48, T=1), seed=12)
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    packed, s_w = q.quantize_weights(w)
    xq_ref, s_ref = q.act_absmax_quant(x)
    out_ref = q.causal_conv3d_w8a8(xq_ref, s_ref, packed, s_w, b, 96)
    ws = torch.empty(q.qvae_layer_workspace_bytes(), dtype=torch.uint8, device="cuda")
    xq = torch.empty_like(xq_ref)
    s = torch.empty(1, device="cuda")
    out = torch.empty_like(out_ref)
    stream = torch.cuda.Stream()
    q.qvae_layer_w8a8(x, xq, s, packed, s_w, b, out, ws, stream)   # first call outside the capture
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        q.qvae_layer_w8a8(x, xq, s, packed, s_w, b, out, ws, stream)
    out.zero_()
    xq.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert q.qvae_get_error() == 0
    assert torch.equal(xq, xq_ref) and f32_bits(s) == f32_bits(s_ref)
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))


@pytest.mark.parametrize("i", range(6))
def test_layer_overlap_full_decoder_sweep_1024(q, i):
    # every code, the scale, every accumulator and every output of a full-size
    # decoder layer against the oracle
    t = synth.draw_workload("decoder_sweep_1024", only=[i])[0]
    x, w, b, out, acc, xq, s_a = run_layer(q, t)
    xb, wb, bb = dev_bits(x), dev_bits(w), dev_bits(b)
    qx, s_ref = oracle.act_quant(xb)
    qw, sw_ref = oracle.quantize_weights(wb)
    assert f32_bits(s_a) == np.array([s_ref], np.float32).view(np.uint32)[0]
    assert np.array_equal(xq.cpu().numpy(), qx)
    del x, xq
    acc_ref = oracle.conv_acc(qx, qw)
    mism = np.count_nonzero(acc.cpu().numpy() != acc_ref)
    assert mism == 0, f"{mism} of {acc_ref.size} accumulators differ"
    del acc
    want = oracle.epilogue(acc_ref, s_ref, sw_ref, bb)
    mism = np.count_nonzero(dev_bits(out) != want)
    assert mism == 0, f"{mism} outputs differ"


def test_layer_overlap_argument_errors(q):
    x = torch.zeros((1, 1, 4, 4, 32), dtype=torch.bfloat16, device="cuda")
    packed, s_w = q.quantize_weights(torch.zeros((32, 32, 3, 3, 3), dtype=torch.bfloat16, device="cuda"))
    small = torch.empty(q.qvae_layer_workspace_bytes() - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QvaeError) as e:
        q.layer_w8a8(x, packed, s_w, None, 32, workspace=small)
    assert e.value.status == q.QVAE_ERR_ARG
    ws = torch.empty(q.qvae_layer_workspace_bytes() + 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QvaeError) as e:
        q.layer_w8a8(x, packed, s_w, None, 32, workspace=ws[1:])
    assert e.value.status == q.QVAE_ERR_ALIGN
    # nothing to compute: the scale is 0 and nothing else is written
    empty = torch.zeros((1, 0, 4, 4, 32), dtype=torch.bfloat16, device="cuda")
    out, xq, s = q.layer_w8a8(empty, packed, s_w, None, 32)
    torch.cuda.synchronize()
    assert s.item() == 0.0 and out.numel() == 0

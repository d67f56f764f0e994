"""The per-layer path (act quantiser + conv) and qvae_decode_layers: CUDA-graph replay and
layer chains.

The library's calls launch on the caller's stream, allocate nothing and never
synchronise, so a decoder can capture them once and replay.  A replay must
give bit-identical results to direct calls on the same data, including data
written into the captured input buffers after the capture.
"""
import numpy as np
import pytest
import torch

from video_vae_decode_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from video_vae_decode_b200 import qvae
    qvae.lib()
    yield qvae


def bits(t):
    return t.view(torch.int16)


def test_layer_step_replays_in_a_cuda_graph(q):
    s = synth.LayerShape(192, 192, 24, 40, T=2)
    gen = torch.Generator().manual_seed(21)
    t0 = synth.draw_layer(gen, s, outliers=True)
    t1 = synth.draw_layer(gen, s, outliers=False, drift=True)
    x = t0.x.cuda()
    w, b = t0.w.cuda(), t0.bias.cuda()
    packed, s_w = q.quantize_weights(w)
    xq = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    sa = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(q.qvae_act_workspace_bytes(x.numel()), dtype=torch.uint8, device="cuda")
    out = torch.empty((s.N, s.T, s.H, s.W, s.Cout), dtype=torch.bfloat16, device="cuda")

    def direct(xin):
        xq_r, sa_r = q.act_absmax_quant(xin)
        return q.causal_conv3d_w8a8(xq_r, sa_r, packed, s_w, b, s.Cout), xq_r, sa_r

    ref0, xq0, sa0 = direct(t0.x.cuda())
    ref1, _, _ = direct(t1.x.cuda())
    torch.cuda.synchronize()

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        q.qvae_act_absmax_quant(x, xq, sa, ws, stream)
        q.qvae_causal_conv3d_w8a8(xq, sa, packed, s_w, b, out, stream)
    g.replay()
    torch.cuda.synchronize()
    assert q.qvae_get_error() == 0
    assert torch.equal(xq, xq0) and torch.equal(sa, sa0)
    assert torch.equal(bits(out), bits(ref0))

    x.copy_(t1.x.cuda())                                     # new data, same buffers
    out.fill_(0)
    torch.cuda.synchronize()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert q.qvae_get_error() == 0
    assert torch.equal(bits(out), bits(ref1))


def test_decode_layers_replays_in_a_cuda_graph(q):
    shapes = [synth.LayerShape(96, 192, 20, 24), synth.LayerShape(192, 96, 20, 24)]
    gen = torch.Generator().manual_seed(22)
    specs, refs = [], []
    for s in shapes:
        t = synth.draw_layer(gen, s, outliers=True)
        x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
        packed, s_w = q.quantize_weights(w)
        out = torch.zeros((s.N, s.T, s.H, s.W, s.Cout), dtype=torch.bfloat16, device="cuda")
        specs.append(dict(x=x, out=out, wq_packed=packed, w_scale=s_w, bias=b, quantized=True))
        xq, s_a = q.act_absmax_quant(x)
        refs.append(q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, s.Cout))
    layers = q.make_layers(specs)
    ws = torch.empty(q.qvae_decode_workspace_bytes(layers), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        q.qvae_decode_layers(layers, ws, stream)
    g.replay()
    torch.cuda.synchronize()
    assert q.qvae_get_error() == 0
    for sp, ref in zip(specs, refs):
        assert torch.equal(bits(sp["out"]), bits(ref))


def _chain(q, shapes, passthrough=(), seed=31):
    """Layers whose outputs feed the next layer's input (same buffer)."""
    gen = torch.Generator().manual_seed(seed)
    t0 = synth.draw_layer(gen, shapes[0], outliers=True)
    x = t0.x.cuda()
    specs, weights = [], []
    for i, s in enumerate(shapes):
        t = t0 if i == 0 else synth.draw_layer(gen, s, outliers=False)
        w, b = t.w.cuda(), t.bias.cuda()
        packed, s_w = q.quantize_weights(w)
        out = torch.zeros((s.N, s.T, s.H, s.W, s.Cout), dtype=torch.bfloat16, device="cuda")
        quantized = i not in passthrough
        # a pass-through layer without weights is skipped by the library (the caller runs it)
        specs.append(dict(x=x, out=out, wq_packed=packed if quantized else None, w_scale=s_w, bias=b,
                          quantized=quantized, w=w))
        weights.append((packed, s_w, b, s.Cout))
        x = out
    return specs, weights


def _layer_by_layer(q, specs, weights):
    """Reference: each layer on its actual input with the standalone absmax pass."""
    outs = []
    for sp, (packed, s_w, b, Cout) in zip(specs, weights):
        if not sp["quantized"]:
            outs.append(sp["out"].clone())
            continue
        xq, s_a = q.act_absmax_quant(sp["x"])
        outs.append(q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, Cout))
    return outs


def _np_bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _check_chain_against_oracle(q, specs, weights, fused=False):
    """Every quantised layer of a qvae_decode_layers chain against the oracle.

    The oracle chain starts from the first input alone: layer k's reference
    input is the oracle's own output of layer k - 1 (the chain is bit-exact,
    so the GPU's input bits must equal it).  For each k the chain is run
    again on its first k + 1 layers.  The workspace then holds layer k's
    activation scale (fp32 at byte 0) and its input maximum (word k % 3 at
    byte 64 + 64 * (k % 3)): for k > 0 the maximum the previous layer's
    epilogue took over what it wrote.  Maximum, scale, the INT32 accumulators
    (the fused convolution's accumulator variant on the same input and word)
    and the bf16 output are compared element by element.  Layer k's output as
    the chain writes it when it also feeds layer k + 1 (with the epilogue
    maximum) is checked as layer k + 1's input."""
    import oracle
    ref_in = _np_bits(specs[0]["x"])
    for k, (sp, (packed, s_w, b, Cout)) in enumerate(zip(specs, weights)):
        assert sp["quantized"]
        for j in range(k + 1):
            specs[j]["out"].fill_(0)
        layers = q.make_layers(specs[:k + 1])
        ws = torch.zeros(q.qvae_decode_workspace_bytes(layers), dtype=torch.uint8, device="cuda")
        q.qvae_decode_layers(layers, ws)
        torch.cuda.synchronize()
        assert q.qvae_get_error() == 0
        x_bits = _np_bits(sp["x"])
        assert np.array_equal(x_bits, ref_in), f"layer {k}: input differs from the oracle chain"
        ref = oracle.layer(ref_in, _np_bits(sp["w"]), _np_bits(b))
        amax_bits = int(np.array([oracle.act_absmax(ref_in)], np.float32).view(np.uint32)[0] >> 16) & 0x7FFF
        word = ws[64 + 64 * (k % 3):64 + 64 * (k % 3) + 4].view(torch.int32)
        if k > 0 or fused:   # a chained maximum (or the absmax pass's word on the fused path)
            assert int(word.item()) == amax_bits, f"layer {k}: input maximum differs"
        word = torch.tensor([amax_bits], dtype=torch.int32, device="cuda")
        scale = ws[0:4].view(torch.float32)
        assert scale.cpu().numpy().view(np.uint32)[0] == np.array([ref["s_a"]], np.float32).view(np.uint32)[0]
        acc = torch.empty(tuple(sp["x"].shape[:-1]) + (Cout,), dtype=torch.int32, device="cuda")
        q.qvae_causal_conv3d_w8a8_fused_acc32(sp["x"], word.clone(), packed, acc)
        assert np.array_equal(acc.cpu().numpy(), ref["acc"]), f"layer {k}: accumulators differ"
        got = _np_bits(sp["out"])
        assert np.array_equal(got, ref["out"]), f"layer {k}: {np.count_nonzero(got != ref['out'])} outputs differ"
        ref_in = ref["out"]


@pytest.fixture(params=[0, 1], ids=["two-pass", "fused"])
def fused(q, request):
    q.qvae_set_fused_quant(request.param)
    yield request.param
    q.qvae_set_fused_quant(0)


def test_decode_chain_matches_the_oracle_at_every_layer(q, fused):
    # ragged sizes: the epilogue's maximum must skip rows and columns beyond the image
    shapes = [synth.LayerShape(96, 192, 37, 21, T=2), synth.LayerShape(192, 192, 37, 21, T=2),
              synth.LayerShape(192, 96, 37, 21, T=2)]
    specs, weights = _chain(q, shapes)
    _check_chain_against_oracle(q, specs, weights, fused)


def test_decode_chain_full_size_sweep_layers(q, fused):
    """384->192 then 192->192 at 512x512 (two layers of the 1024x1024 decoder sweep),
    chained, every element against the oracle."""
    tens = synth.draw_workload("decoder_sweep_1024", only=[2, 3])
    x = tens[0].x.cuda()
    specs, weights = [], []
    for t in tens:
        s = t.shape
        w, b = t.w.cuda(), t.bias.cuda()
        packed, s_w = q.quantize_weights(w)
        out = torch.zeros((s.N, s.T, s.H, s.W, s.Cout), dtype=torch.bfloat16, device="cuda")
        specs.append(dict(x=x, out=out, wq_packed=packed, w_scale=s_w, bias=b, quantized=True, w=w))
        weights.append((packed, s_w, b, s.Cout))
        x = out
    _check_chain_against_oracle(q, specs, weights, fused)


@pytest.mark.parametrize("passthrough", [(), (1,)])
def test_decode_chain_takes_each_input_absmax_from_the_previous_epilogue(q, passthrough):
    # ragged sizes: the epilogue's maximum must skip rows and columns beyond the image
    shapes = [synth.LayerShape(96, 192, 37, 21, T=2), synth.LayerShape(192, 192, 37, 21, T=2),
              synth.LayerShape(192, 96, 37, 21, T=2)]
    specs, weights = _chain(q, shapes, passthrough)
    layers = q.make_layers(specs)
    ws = torch.empty(q.qvae_decode_workspace_bytes(layers), dtype=torch.uint8, device="cuda")
    q.qvae_decode_layers(layers, ws)
    torch.cuda.synchronize()
    assert q.qvae_get_error() == 0
    got = [sp["out"].clone() for sp in specs]
    want = _layer_by_layer(q, specs, weights)
    for g, w_ in zip(got, want):
        assert torch.equal(g.view(torch.int16), w_.view(torch.int16))
    # and the first layer against the oracle
    ref = oracle_layer(specs[0], q)
    assert np.array_equal(got[0].cpu().view(torch.int16).numpy().view(np.uint16), ref)


def oracle_layer(sp, q):
    import oracle
    gen = torch.Generator().manual_seed(31)
    t = synth.draw_layer(gen, synth.LayerShape(96, 192, 37, 21, T=2), outliers=True)
    b = lambda v: v.contiguous().view(torch.int16).numpy().view(np.uint16)
    return oracle.layer(b(t.x), b(t.w), b(t.bias))["out"]

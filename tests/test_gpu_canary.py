"""Guard bytes around every output buffer (a stand-in for a memory checker).

The convolution writes bf16 outputs with TMA stores whose tensor map clips
rows and columns beyond the image, and INT32 accumulators with plain stores
behind a bounds check.  On ragged shapes (H, W not multiples of the 16 x 8
pixel sub-tile, channel counts that leave a partial 128-channel chunk) the
tests place each output between two guard regions filled with a pattern and
check that no byte of either region changes, for the whole-layer, streamed-
chunk, row-band and layer-chain entry points.
"""
import numpy as np
import pytest
import torch

from video_vae_decode_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 64 * 1024        # bytes on each side
PATTERN = 0x5AA5


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from video_vae_decode_b200 import qvae
    qvae.lib()
    yield qvae
    qvae.qvae_set_conv_tiling()


def guarded(shape, dtype):
    """A tensor of `shape` between two guard regions; returns (tensor, guard record)."""
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    total = GUARD + ((n + 255) // 256) * 256 + GUARD
    buf = torch.full((total // 2,), PATTERN, dtype=torch.int16, device="cuda")
    view = buf.view(torch.uint8)[GUARD:GUARD + n].view(dtype).view(shape)
    return view, (buf, n)


def assert_guards(rec):
    """No byte outside [GUARD, GUARD + n) of the buffer has changed."""
    buf, n = rec
    torch.cuda.synchronize()
    b = buf.view(torch.uint8).cpu().numpy()
    want = np.full(b.size // 2, PATTERN, dtype=np.int16).view(np.uint8)
    outside = np.ones(b.size, dtype=bool)
    outside[GUARD:GUARD + n] = False
    changed = np.nonzero((b != want) & outside)[0]
    assert changed.size == 0, f"{changed.size} guard bytes changed, first at offset {changed[0] - GUARD} from the output"


SHAPES = [synth.LayerShape(32, 32, 1, 1), synth.LayerShape(64, 96, 17, 9), synth.LayerShape(160, 64, 5, 130, T=2),
          synth.LayerShape(192, 192, 37, 21, T=3), synth.LayerShape(96, 32, 130, 3)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s.Cin}-{s.Cout}-{s.H}x{s.W}-T{s.T}")
@pytest.mark.parametrize("mode", [1, 2])
def test_conv_outputs_stay_inside_their_buffers(q, shape, mode):
    t = synth.draw_custom(shape, seed=shape.H + shape.W, outliers=True)
    x, w, b = t.x.cuda(), t.w.cuda(), t.bias.cuda()
    packed, s_w = q.quantize_weights(w)
    xq, s_a = q.act_absmax_quant(x)
    oshape = (shape.N, shape.T, shape.H, shape.W, shape.Cout)
    q.qvae_set_conv_tiling(mode=mode)
    try:
        out, buf = guarded(oshape, torch.bfloat16)
        q.qvae_causal_conv3d_w8a8(xq, s_a, packed, s_w, b, out)
        assert_guards(buf)
        acc, abuf = guarded(oshape, torch.int32)
        q.qvae_causal_conv3d_w8a8_acc32(xq, packed, acc)
        assert_guards(abuf)
        ref = q.causal_conv3d_w8a8(xq, s_a, packed, s_w, b, shape.Cout)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        if shape.H >= 3:
            # a row band of the middle rows, halos on both sides
            r0, r1 = 1, shape.H - 1
            xq_band = xq[:, :, r0 - 1:r1 + 1].contiguous()
            bout, bbuf = guarded((shape.N, shape.T, r1 - r0, shape.W, shape.Cout), torch.bfloat16)
            q.qvae_causal_conv3d_w8a8_band(xq_band, 1, 1, s_a, packed, s_w, b, bout)
            assert_guards(bbuf)
            assert torch.equal(bout.view(torch.int16), ref[:, :, r0:r1].view(torch.int16))
        # a streamed chunk with two carried frames (zero history)
        zeros = torch.zeros((shape.N, 2, shape.H, shape.W, shape.Cin), dtype=torch.int8, device="cuda")
        xq_ext = torch.cat([zeros, xq], 1).contiguous()
        cout, cbuf = guarded(oshape, torch.bfloat16)
        q.qvae_causal_conv3d_w8a8_carry(xq_ext, s_a, packed, s_w, b, cout)
        assert_guards(cbuf)
        assert torch.equal(cout.view(torch.int16), ref.view(torch.int16))
        assert q.qvae_get_error() == 0
    finally:
        q.qvae_set_conv_tiling()


def test_activation_codes_stay_inside_their_buffer(q):
    for n in (1, 15, 17, 4097, 1_000_003):
        x = torch.randn(n).to(torch.bfloat16).cuda()
        xq, rec = guarded((n,), torch.int8)
        s = torch.empty(1, device="cuda")
        ws = torch.empty(q.qvae_act_workspace_bytes(n), dtype=torch.uint8, device="cuda")
        q.qvae_act_absmax_quant(x, xq, s, ws)
        assert_guards(rec)

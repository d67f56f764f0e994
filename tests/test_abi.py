"""The C ABI library: it loads, exports every declared symbol, and rejects bad
arguments before touching the GPU (no compute calls here; runs without a GPU)."""
import ctypes
import os
import re

import pytest

from video_vae_decode_b200 import qvae

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qvae.h")

FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced
FAKE_ODD = ctypes.c_void_p(0x10008)      # misaligned


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qvae_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(qvae.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = qvae.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_release_library_has_no_debug_checks():
    # the in-tree library is the release build unless QVAE_LIBRARY names another
    if not os.environ.get("QVAE_LIBRARY"):
        assert qvae.lib().qvae_build_flags() == 0


def test_status_strings():
    L = qvae.lib()
    for code in range(8):
        assert L.qvae_status_string(code) not in (None, b"", b"unknown status")
    assert L.qvae_status_string(99) == b"unknown status"


def test_packed_weight_bytes():
    assert qvae.qvae_packed_weight_bytes(384, 384) == 27 * 3 * 384 * 128
    assert qvae.qvae_packed_weight_bytes(96, 96) == 27 * 1 * 96 * 128
    assert qvae.qvae_packed_weight_bytes(192, 96) == 27 * 2 * 96 * 128
    assert qvae.qvae_packed_weight_bytes(0, 96) == 0


def conv(shape, xq=FAKE, xs=FAKE, wq=FAKE, ws=FAKE, b=None, out=FAKE):
    return qvae.lib().qvae_causal_conv3d_w8a8(ctypes.byref(shape), xq, xs, wq, ws, b, out, None)


def test_conv_argument_checks():
    ok = qvae.make_shape(1, 1, 8, 8, 64, 64)
    assert conv(qvae.make_shape(1, 1, 8, 8, 48, 64)) == qvae.QVAE_ERR_SHAPE
    assert conv(qvae.make_shape(1, 1, 8, 8, 64, 40)) == qvae.QVAE_ERR_SHAPE
    assert conv(qvae.make_shape(1, 1, 8, 8, 16, 64)) == qvae.QVAE_ERR_SHAPE
    assert conv(qvae.make_shape(-1, 1, 8, 8, 64, 64)) == qvae.QVAE_ERR_ARG
    assert conv(ok, xq=None) == qvae.QVAE_ERR_ARG
    assert conv(ok, xs=None) == qvae.QVAE_ERR_ARG
    assert conv(ok, out=FAKE_ODD) == qvae.QVAE_ERR_ALIGN
    assert conv(ok, xq=FAKE_ODD) == qvae.QVAE_ERR_ALIGN
    assert conv(qvae.make_shape(1, 0, 8, 8, 64, 64), xq=None) == qvae.QVAE_OK   # empty: no-op
    L = qvae.lib()
    assert L.qvae_causal_conv3d_w8a8(None, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_causal_conv3d_w8a8_acc32(ctypes.byref(ok), FAKE, FAKE, None, None) == qvae.QVAE_ERR_ARG


def test_act_and_weight_argument_checks():
    L = qvae.lib()
    ws = qvae.qvae_act_workspace_bytes(1000)
    assert L.qvae_act_absmax_quant(FAKE, -1, FAKE, FAKE, FAKE, ws, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_act_absmax_quant(FAKE, 100, FAKE, FAKE, FAKE, 16, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_act_absmax_quant(FAKE_ODD, 100, FAKE, FAKE, FAKE, ws, None) == qvae.QVAE_ERR_ALIGN
    assert L.qvae_act_absmax_quant(FAKE, 100, FAKE, None, FAKE, ws, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_quantize_weights(48, 64, FAKE, FAKE, FAKE, None, None) == qvae.QVAE_ERR_SHAPE
    assert L.qvae_quantize_weights(64, 64, None, FAKE, FAKE, None, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_quantize_weights(64, 64, FAKE, FAKE_ODD, FAKE, None, None) == qvae.QVAE_ERR_ALIGN


def test_decode_layers_validates_everything_first():
    L = qvae.lib()
    arr = (qvae.qvae_layer * 2)()
    for i in range(2):
        arr[i].shape = qvae.make_shape(1, 1, 8, 8, 64, 64)
        arr[i].quantized = 1
        arr[i].x = arr[i].out = arr[i].wq_packed = arr[i].w_scale = 0x10000
    arr[1].shape = qvae.make_shape(1, 1, 8, 8, 48, 64)
    need = L.qvae_decode_workspace_bytes(arr, 2)
    assert L.qvae_decode_layers(arr, 2, FAKE, need, None) == qvae.QVAE_ERR_SHAPE
    arr[1].quantized = 0                                   # a native layer with weights is run: checked
    assert L.qvae_decode_layers(arr, 2, FAKE, need, None) == qvae.QVAE_ERR_SHAPE
    arr[1].shape = qvae.make_shape(1, 1, 8, 8, 64, 64)
    arr[1].x = 0x10008
    assert L.qvae_decode_layers(arr, 2, FAKE, need, None) == qvae.QVAE_ERR_ALIGN
    arr[1].shape = qvae.make_shape(1, 1, 8, 8, 48, 64)
    arr[1].wq_packed = None                                # without weights it is skipped: not checked
    need = L.qvae_decode_workspace_bytes(arr, 2)
    # scale + maximum words, partial maxima, the codes of the largest quantised input (8 x 8 x 64)
    assert need == 256 + qvae.qvae_act_workspace_bytes(1) + 8 * 8 * 64
    qvae.qvae_set_fused_quant(1)
    try:
        assert L.qvae_decode_workspace_bytes(arr, 2) == 256       # the fused path keeps no codes
    finally:
        qvae.qvae_set_fused_quant(0)
    assert L.qvae_set_fused_quant(2) == qvae.QVAE_ERR_ARG
    assert L.qvae_decode_layers(arr, 2, FAKE, need - 1, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_decode_layers(arr, -1, FAKE, need, None) == qvae.QVAE_ERR_ARG


def test_tiling_choice_is_valid():
    for (N, T, H, W, Cin, Cout) in [(1, 1, 128, 128, 384, 384), (1, 1, 64, 64, 96, 96),
                                    (1, 1, 105, 157, 384, 384), (1, 8, 240, 416, 192, 192),
                                    (1, 1, 1024, 1024, 192, 96), (1, 1, 840, 1256, 96, 96)]:
        t = qvae.qvae_get_conv_tiling(N, T, H, W, Cin, Cout)
        assert 1 <= t["MS"] <= 4 and t["MS"] * t["NT"] <= 512 and t["mode"] in (1, 2)
        assert Cout % t["NT"] == 0 and t["NT"] % 32 == 0 and t["NT"] <= 256
        assert 1 <= t["SA"] <= 12 and 1 <= t["SB"] <= 12
        assert t["G"] == 1 or (t["G"] == 3 and t["MS"] <= 2)
        assert t["acc_buffers"] == (2 if 2 * t["MS"] * t["NT"] <= 512 else 1)
        rows = 16 * t["MS"] * t["mode"]
        tiles = N * T * -(-H // rows) * -(-W // 8) * (Cout // t["NT"])
        assert t["ctas"] == tiles * t["mode"]
    qvae.qvae_set_conv_tiling(MS=1, NT=64, SA=2, SB=3, mode=1)
    try:
        t = qvae.qvae_get_conv_tiling(1, 1, 100, 100, 128, 128)
        assert (t["MS"], t["NT"], t["SA"], t["SB"], t["mode"]) == (1, 64, 2, 3, 1)
        qvae.qvae_set_conv_tiling(MS=1, NT=192, mode=2, G=3)
        t = qvae.qvae_get_conv_tiling(1, 1, 100, 100, 192, 192)
        assert (t["MS"], t["NT"], t["mode"], t["G"]) == (1, 192, 2, 3)
    finally:
        qvae.qvae_set_conv_tiling()
    with pytest.raises(qvae.QvaeError):
        qvae.qvae_set_conv_tiling(MS=5)
    with pytest.raises(qvae.QvaeError):
        qvae.qvae_set_conv_tiling(NT=48)
    with pytest.raises(qvae.QvaeError):
        qvae.qvae_set_conv_tiling(MS=3, NT=256)
    with pytest.raises(qvae.QvaeError):
        qvae.qvae_set_conv_tiling(mode=3)
    with pytest.raises(qvae.QvaeError):
        qvae.qvae_set_conv_tiling(G=2)
    with pytest.raises(qvae.QvaeError):
        qvae.qvae_set_conv_tiling(MS=3, G=3)


@pytest.mark.parametrize("variant", [0, 1, 2], ids=["codes", "fused", "native"])
def test_tiling_choice_is_valid_over_the_supported_shapes(variant):
    """The cost model picks a launchable tiling for every shape each kernel accepts."""
    chans = (32, 64, 96, 128, 160, 192, 256, 384, 512)
    for Cin in chans:
        for Cout in chans:
            for H, W in ((1, 1), (7, 33), (16, 8), (33, 7), (128, 128), (517, 300)):
                for T in (1, 3):
                    t = qvae.qvae_get_conv_tiling(1, T, H, W, Cin, Cout, variant)
                    assert 1 <= t["MS"] <= 4 and t["MS"] * t["NT"] <= 512 and t["mode"] in (1, 2)
                    assert Cout % t["NT"] == 0 and t["NT"] % 32 == 0 and t["NT"] <= 256
                    assert 1 <= t["SA"] <= 12 and 1 <= t["SB"] <= 12
                    assert t["G"] == 1 or (t["G"] == 3 and t["MS"] <= 2)
                    assert t["acc_buffers"] == (2 if 2 * t["MS"] * t["NT"] <= 512 else 1)
                    rows = 16 * t["MS"] * t["mode"]
                    assert t["ctas"] == T * -(-H // rows) * -(-W // 8) * (Cout // t["NT"]) * t["mode"]


def test_stream_band_and_split_activation_argument_checks():
    L = qvae.lib()
    ok = qvae.make_shape(1, 2, 8, 8, 64, 64)
    bad = qvae.make_shape(1, 2, 8, 8, 48, 64)
    # streamed chunk (two carried frames)
    assert L.qvae_causal_conv3d_w8a8_carry(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                           None) == qvae.QVAE_ERR_SHAPE
    assert L.qvae_causal_conv3d_w8a8_carry(ctypes.byref(ok), FAKE, None, FAKE, FAKE, None, FAKE,
                                           None) == qvae.QVAE_ERR_ARG
    assert L.qvae_causal_conv3d_w8a8_carry_acc32(ctypes.byref(ok), FAKE, FAKE, None, None) == qvae.QVAE_ERR_ARG
    # row band: halos of 0 or 1 rows only
    for ht, hb in ((2, 0), (0, 2), (-1, 0)):
        assert L.qvae_causal_conv3d_w8a8_band(ctypes.byref(ok), ht, hb, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                              None) == qvae.QVAE_ERR_ARG
    assert L.qvae_causal_conv3d_w8a8_band(ctypes.byref(ok), 1, 1, None, FAKE, FAKE, FAKE, None, FAKE,
                                          None) == qvae.QVAE_ERR_ARG
    assert L.qvae_causal_conv3d_w8a8_band(ctypes.byref(ok), 1, 1, FAKE_ODD, FAKE, FAKE, FAKE, None, FAKE,
                                          None) == qvae.QVAE_ERR_ALIGN
    assert L.qvae_causal_conv3d_w8a8_band_acc32(ctypes.byref(ok), 0, 0, FAKE, FAKE, None, None) == qvae.QVAE_ERR_ARG
    # the two activation steps apart
    assert L.qvae_act_absmax(FAKE, -1, FAKE, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_act_absmax(FAKE, 100, None, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_act_absmax(None, 100, FAKE, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_act_absmax(FAKE_ODD, 100, FAKE, None) == qvae.QVAE_ERR_ALIGN
    assert L.qvae_act_quant_from_absmax(FAKE, 100, None, FAKE, FAKE, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_act_quant_from_absmax(FAKE, 100, FAKE, FAKE, None, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_act_quant_from_absmax(FAKE, 100, FAKE, None, FAKE, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_act_quant_from_absmax(FAKE, 100, FAKE, FAKE_ODD, FAKE, None) == qvae.QVAE_ERR_ALIGN


def test_native_layer_argument_checks():
    L = qvae.lib()
    assert qvae.qvae_packed_weight_bytes_bf16(96, 96) == 27 * 2 * 96 * 128
    assert qvae.qvae_packed_weight_bytes_bf16(384, 192) == 27 * 6 * 192 * 128
    assert qvae.qvae_packed_weight_bytes_bf16(32, 32) == 27 * 1 * 32 * 128
    assert qvae.qvae_packed_weight_bytes_bf16(0, 32) == 0
    assert L.qvae_pack_weights_bf16(48, 64, FAKE, FAKE, None) == qvae.QVAE_ERR_SHAPE
    assert L.qvae_pack_weights_bf16(64, 64, None, FAKE, None) == qvae.QVAE_ERR_ARG
    assert L.qvae_pack_weights_bf16(64, 64, FAKE, FAKE_ODD, None) == qvae.QVAE_ERR_ALIGN
    ok = qvae.make_shape(1, 1, 8, 8, 64, 64)
    conv = L.qvae_causal_conv3d_bf16
    assert conv(ctypes.byref(qvae.make_shape(1, 1, 8, 8, 48, 64)), FAKE, FAKE, None, FAKE, None) == qvae.QVAE_ERR_SHAPE
    assert conv(ctypes.byref(ok), None, FAKE, None, FAKE, None) == qvae.QVAE_ERR_ARG
    assert conv(ctypes.byref(ok), FAKE, None, None, FAKE, None) == qvae.QVAE_ERR_ARG
    assert conv(ctypes.byref(ok), FAKE, FAKE, None, None, None) == qvae.QVAE_ERR_ARG
    assert conv(ctypes.byref(ok), FAKE_ODD, FAKE, None, FAKE, None) == qvae.QVAE_ERR_ALIGN
    assert conv(ctypes.byref(ok), FAKE, FAKE, None, FAKE_ODD, None) == qvae.QVAE_ERR_ALIGN
    assert conv(ctypes.byref(qvae.make_shape(1, 1, 0, 8, 64, 64)), None, None, None, None, None) == qvae.QVAE_OK
    assert L.qvae_causal_conv3d_bf16_acc32(ctypes.byref(ok), FAKE, FAKE, None, None) == qvae.QVAE_ERR_ARG


# Tilings measured best on a B200 for the decoder layer shapes (forced-tiling
# sweeps with bench-style timing): a change to the cost model that picks
# another one for these shapes must come with a new measurement.
MEASURED_BEST = [
    # (T, H, W, Cin, Cout) -> (mode, MS, NT, G, accumulator buffers)
    ((1, 128, 128, 384, 384), (2, 1, 192, 3, 2)),
    ((1, 256, 256, 384, 384), (2, 1, 192, 3, 2)),
    ((1, 512, 512, 384, 192), (2, 1, 192, 3, 2)),
    ((1, 512, 512, 192, 192), (2, 1, 192, 3, 2)),
    ((1, 1024, 1024, 192, 96), (2, 2, 96, 3, 2)),
    ((1, 1024, 1024, 96, 96), (2, 2, 96, 3, 2)),
    ((1, 105, 157, 384, 384), (1, 1, 192, 3, 2)),
    ((1, 420, 628, 384, 192), (2, 1, 192, 3, 2)),
    ((1, 840, 1256, 96, 96), (2, 2, 96, 3, 2)),
    ((8, 240, 416, 192, 192), (2, 2, 192, 3, 1)),
]


@pytest.mark.parametrize("shape,want", MEASURED_BEST, ids=[str(s) for s, _ in MEASURED_BEST])
def test_cost_model_picks_the_measured_best_tiling(shape, want):
    T, H, W, Cin, Cout = shape
    t = qvae.qvae_get_conv_tiling(1, T, H, W, Cin, Cout, 0)
    assert (t["mode"], t["MS"], t["NT"], t["G"], t["acc_buffers"]) == want

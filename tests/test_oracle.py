"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: values
derived by hand from the method (tests/golden/), a float64 library
convolution, brute force on tiny shapes, exact rational arithmetic, and
invariants that a plausible mistake (a dropped term, a wrong sign or index,
a transposed operand, the wrong rounding) would break.

Method: ComfyUI-Qwen-VAE-Triton v0.2.0 release note (sd114.wiki), "three
presets" section (symmetric per-output-channel INT8 weights, dynamic
symmetric INT8 activations, INT32 accumulation, FP32 rescale, output in the
activation dtype; clip ratios 1.0, channels_last) and the opening paragraph
(CausalConv3d).
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from video_vae_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f2b(values):
    """float -> bf16 bits through torch's own conversion."""
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def b2f(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rn32(r: Fraction) -> Fraction:
    """Exact rational -> nearest binary32 (ties to even), normal range only."""
    if r == 0:
        return Fraction(0)
    sign = -1 if r < 0 else 1
    r = abs(r)
    e = r.numerator.bit_length() - r.denominator.bit_length()
    while Fraction(2) ** e > r:
        e -= 1
    while Fraction(2) ** (e + 1) <= r:
        e += 1
    assert e >= -126, "subnormal results are outside this helper"
    scaled = r / Fraction(2) ** (e - 23)          # in [2^23, 2^24)
    q, rem = divmod(scaled.numerator, scaled.denominator)
    if 2 * rem > scaled.denominator or (2 * rem == scaled.denominator and q % 2 == 1):
        q += 1
    return sign * Fraction(q) * Fraction(2) ** (e - 23)


def exact_code(x: float, amax: float) -> int:
    """Code the reading prescribes, evaluated with exact rationals:
    s = RN32(amax / 127); code = clamp(half-even-round(RN32(x / s)), +-127)."""
    s = rn32(Fraction(amax) / 127)
    if s == 0:
        return 0
    q = rn32(Fraction(x) / s)
    fl = q.numerator // q.denominator
    frac = q - fl
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return max(-127, min(127, fl))


# ----------------------------------------------------------------- bf16 cast

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 10,
        # exact ties: bf16 value + half an ulp
        (b2f(rng.integers(0x3000, 0x5000, 500).astype(np.uint16)).view(np.uint32)
         + np.uint32(0x8000)).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-30], dtype=np.float32),
    ])
    assert np.array_equal(oracle.f32_to_bf16(vals), f2b(vals))


# ------------------------------------------------------------- quantisation

def load_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    return rows


def test_act_codes_unit_scale_golden():
    rows = load_golden("quant_unit_scale.txt")
    x = np.array([float(r[0]) for r in rows], dtype=np.float32)
    want = np.array([int(r[1]) for r in rows], dtype=np.int8)
    qx, s = oracle.act_quant(f2b(x))
    assert s == np.float32(1.0)
    assert np.array_equal(qx, want)


def test_act_codes_exact_rational_division():
    """Codes equal the exactly-rounded quotient, including inputs where
    multiplying by a rounded reciprocal would give a different code."""
    pos = (np.arange(0x0080, 0x7f80, dtype=np.uint32) << 16).view(np.float32)
    rng = np.random.default_rng(7)
    checked = discriminating = 0
    for am_bits in rng.integers(0x3c00, 0x4300, 120):
        amax = float(b2f(np.array([am_bits], dtype=np.uint16))[0])
        xs = pos[pos <= amax]
        s32 = np.float32(amax) / np.float32(127.0)
        recip = np.rint(xs * (np.float32(1.0) / s32))
        div = np.rint(xs / s32)
        pick = np.nonzero(recip != div)[0].tolist()
        pick += rng.choice(len(xs), 6, replace=False).tolist()
        sample = np.concatenate([[amax, -amax], xs[pick], -xs[pick]]).astype(np.float32)
        qx, s = oracle.act_quant(f2b(sample))
        assert Fraction(float(s)) == rn32(Fraction(amax) / 127)
        for xv, qv in zip(sample, qx):
            assert int(qv) == exact_code(float(xv), amax), (amax, float(xv))
        checked += len(sample)
        discriminating += int(np.sum(recip != div))
    assert discriminating > 0, "the sample must contain reciprocal-vs-divide cases"
    assert checked > 1000


def test_act_quant_invariants():
    t = synth.draw_custom(synth.LayerShape(32, 16, 9, 7, T=3), seed=3, outliers=True).x
    x = synth.bits(t)
    qx, s = oracle.act_quant(x)
    xf = b2f(x)
    amax = np.abs(xf).max()
    assert amax == np.float32(8.0)                # the outliers set the absmax
    assert s == np.float32(8.0) / np.float32(127.0)
    assert qx.min() >= -127 and qx.max() <= 127
    assert np.all(qx[xf == amax] == 127) and np.all(qx[xf == -amax] == -127)
    # symmetric: q(-x) = -q(x)
    qn, sn = oracle.act_quant(x ^ np.uint16(0x8000))
    assert sn == s and np.array_equal(qn, -qx)
    # scaling by a power of two changes only the scale
    x4 = f2b(xf * np.float32(4.0))
    q4, s4 = oracle.act_quant(x4)
    assert s4 == s * np.float32(4.0) and np.array_equal(q4, qx)
    # |x/s - q| <= 1/2 away from the clamp
    assert np.all(np.abs(xf / s - qx) <= 0.5 + 1e-5)


def test_act_quant_zero_tensor():
    qx, s = oracle.act_quant(np.zeros((2, 3, 5), dtype=np.uint16))
    assert s == 0.0 and not qx.any()


def test_weight_quant_is_per_output_channel():
    rng = np.random.default_rng(5)
    base = rng.standard_normal((6, 3, 3, 3)).astype(np.float32)
    base[2, 1, 0, 2] = 3.0                        # single largest element
    # channel co = base * 2^(co - 2): codes identical, scales exact powers of two
    w = np.stack([base * np.float32(2.0 ** (co - 2)) for co in range(5)])
    qw, s_w = oracle.quantize_weights(f2b(w))
    ref = qw[2]
    for co in range(5):
        assert np.array_equal(qw[co], ref)
        assert s_w[co] == s_w[2] * np.float32(2.0 ** (co - 2))
    assert np.all(qw[:, 2, 1, 0, 2] == 127)
    amax = float(b2f(f2b(base)).__abs__().max())
    assert Fraction(float(s_w[2])) == rn32(Fraction(amax) / 127)
    # a zero channel has scale 0 and zero codes
    w[3] = 0.0
    qz, sz = oracle.quantize_weights(f2b(w))
    assert sz[3] == 0.0 and not qz[3].any()
    assert np.array_equal(qz[4], ref)


def test_weight_codes_exact_rational():
    t = synth.draw_custom(synth.LayerShape(16, 8, 4, 4), seed=11).w
    wb = synth.bits(t)
    qw, s_w = oracle.quantize_weights(wb)
    wf = b2f(wb)
    for co in range(8):
        amax = float(np.abs(wf[co]).max())
        flat_w, flat_q = wf[co].ravel(), qw[co].ravel()
        for i in range(0, flat_w.size, 7):
            assert int(flat_q[i]) == exact_code(float(flat_w[i]), amax)


# ------------------------------------------------------------ accumulators

def brute_force_acc(qx, qw):
    """Seven nested Python loops over the zero-padded causal window."""
    N, T, H, W, Cin = qx.shape
    Cout = qw.shape[0]
    acc = np.zeros((N, T, H, W, Cout), dtype=np.int64)
    for n in range(N):
        for t in range(T):
            for h in range(H):
                for w in range(W):
                    for co in range(Cout):
                        total = 0
                        for kt in range(3):
                            for kh in range(3):
                                for kw in range(3):
                                    ti, hi, wi = t - 2 + kt, h - 1 + kh, w - 1 + kw
                                    if 0 <= ti < T and 0 <= hi < H and 0 <= wi < W:
                                        for ci in range(Cin):
                                            total += int(qx[n, ti, hi, wi, ci]) * int(qw[co, ci, kt, kh, kw])
                        acc[n, t, h, w, co] = total
    return acc


def rand_codes(rng, shape):
    return rng.integers(-127, 128, size=shape).astype(np.int8)


@pytest.mark.parametrize("N,T,H,W,Cin,Cout", [
    (1, 1, 3, 3, 2, 3), (1, 3, 4, 5, 3, 2), (2, 4, 3, 2, 2, 2), (1, 2, 1, 1, 4, 3), (1, 5, 2, 3, 1, 1)])
def test_conv_acc_brute_force(N, T, H, W, Cin, Cout):
    rng = np.random.default_rng(N * 1000 + T * 100 + H * 10 + W)
    qx, qw = rand_codes(rng, (N, T, H, W, Cin)), rand_codes(rng, (Cout, Cin, 3, 3, 3))
    assert np.array_equal(oracle.conv_acc(qx, qw), brute_force_acc(qx, qw))


def torch_conv_f64(qx, qw):
    """float64 library convolution on explicitly zero-padded codes."""
    x = torch.from_numpy(qx.astype(np.float64)).permute(0, 4, 1, 2, 3)   # N C T H W
    x = F.pad(x, (1, 1, 1, 1, 2, 0))
    w = torch.from_numpy(qw.astype(np.float64))
    y = F.conv3d(x, w)
    return y.permute(0, 2, 3, 4, 1).numpy()


@pytest.mark.parametrize("N,T,H,W,Cin,Cout", [
    (1, 1, 9, 11, 32, 16), (2, 4, 17, 5, 48, 32), (1, 3, 6, 7, 96, 48)])
def test_conv_acc_matches_float64_library_conv(N, T, H, W, Cin, Cout):
    rng = np.random.default_rng(Cin + Cout)
    qx, qw = rand_codes(rng, (N, T, H, W, Cin)), rand_codes(rng, (Cout, Cin, 3, 3, 3))
    acc = oracle.conv_acc(qx, qw)
    ref = torch_conv_f64(qx, qw)
    assert np.array_equal(acc.astype(np.float64), ref)


def test_conv_t1_equals_2d_conv_with_last_slice():
    rng = np.random.default_rng(21)
    qx, qw = rand_codes(rng, (1, 1, 12, 10, 32)), rand_codes(rng, (24, 32, 3, 3, 3))
    acc = oracle.conv_acc(qx, qw)
    x2 = torch.from_numpy(qx[:, 0].astype(np.float64)).permute(0, 3, 1, 2)
    y2 = F.conv2d(x2, torch.from_numpy(qw[:, :, 2].astype(np.float64)), padding=1)
    assert np.array_equal(acc[:, 0].astype(np.float64), y2.permute(0, 2, 3, 1).numpy())


def test_conv_first_frame_and_causality():
    rng = np.random.default_rng(22)
    qx, qw = rand_codes(rng, (1, 5, 6, 6, 32)), rand_codes(rng, (16, 32, 3, 3, 3))
    acc = oracle.conv_acc(qx, qw)
    # frame 0 only meets slice kt = 2
    x2 = torch.from_numpy(qx[:, 0].astype(np.float64)).permute(0, 3, 1, 2)
    y2 = F.conv2d(x2, torch.from_numpy(qw[:, :, 2].astype(np.float64)), padding=1)
    assert np.array_equal(acc[:, 0].astype(np.float64), y2.permute(0, 2, 3, 1).numpy())
    # changing frames after t0 leaves outputs at t <= t0 unchanged
    t0 = 2
    qx2 = qx.copy()
    qx2[:, t0 + 1:] = rand_codes(rng, qx2[:, t0 + 1:].shape)
    acc2 = oracle.conv_acc(qx2, qw)
    assert np.array_equal(acc2[:, :t0 + 1], acc[:, :t0 + 1])
    assert not np.array_equal(acc2[:, t0 + 1:], acc[:, t0 + 1:])
    # changing frame t0 reaches exactly frames t0, t0+1, t0+2
    qx3 = qx.copy()
    qx3[:, t0] = rand_codes(rng, qx3[:, t0].shape)
    acc3 = oracle.conv_acc(qx3, qw)
    assert np.array_equal(acc3[:, :t0], acc[:, :t0])
    for t in (t0, t0 + 1, t0 + 2):
        assert not np.array_equal(acc3[:, t], acc[:, t])


def test_conv_delta_kernel_and_symmetry():
    rng = np.random.default_rng(23)
    C = 16
    qx = rand_codes(rng, (1, 2, 5, 4, C))
    qw = np.zeros((C, C, 3, 3, 3), dtype=np.int8)
    for c in range(C):
        qw[c, c, 2, 1, 1] = 1                    # centre tap of the current frame
    assert np.array_equal(oracle.conv_acc(qx, qw), qx.astype(np.int32))
    qw2 = rand_codes(rng, (8, C, 3, 3, 3))
    a = oracle.conv_acc(qx, qw2)
    qneg = (-qx.astype(np.int16)).astype(np.int8)
    assert np.array_equal(oracle.conv_acc(qneg, qw2), -a)


def test_conv_shift_equivariance_interior():
    rng = np.random.default_rng(24)
    qx, qw = rand_codes(rng, (1, 1, 10, 10, 16)), rand_codes(rng, (8, 16, 3, 3, 3))
    a = oracle.conv_acc(qx, qw)
    b = oracle.conv_acc(np.roll(qx, (2, 3), axis=(2, 3)), qw)
    # away from the borders a shift of the input shifts the output
    assert np.array_equal(b[0, 0, 3:9, 4:9], a[0, 0, 1:7, 1:6])


def test_conv_points_match_full():
    rng = np.random.default_rng(25)
    qx, qw = rand_codes(rng, (2, 3, 7, 9, 32)), rand_codes(rng, (16, 32, 3, 3, 3))
    acc = oracle.conv_acc(qx, qw)
    pts = np.array([[0, 0, 0, 0], [1, 2, 6, 8], [0, 1, 3, 4], [1, 0, 6, 0]], dtype=np.int64)
    got = oracle.conv_acc_points(qx, qw, pts)
    for p, row in zip(pts, got):
        assert np.array_equal(row, acc[tuple(p)])


# ---------------------------------------------------------------- epilogue

def test_epilogue_pow2_golden():
    rows = load_golden("epilogue_pow2.txt")
    for acc_s, b_s, want_s in rows:
        acc = np.array([[int(acc_s)]], dtype=np.int32)
        bias = np.array([int(b_s, 16)], dtype=np.uint16)
        s_w = np.array([2.0 ** -4], dtype=np.float32)
        out = oracle.epilogue(acc, np.float32(2.0 ** -3), s_w, bias)
        assert int(out[0, 0]) == int(want_s, 16), (acc_s, b_s, hex(int(out[0, 0])))


def test_epilogue_null_bias_and_zero_acc():
    acc = np.zeros((3, 4), dtype=np.int32)
    out = oracle.epilogue(acc, np.float32(0.5), np.ones(4, dtype=np.float32))
    assert not out.any()


def test_layer_zero_input_returns_bias():
    t = synth.draw_custom(synth.LayerShape(32, 16, 5, 6, T=2), seed=9)
    x = np.zeros(synth.bits(t.x).shape, dtype=np.uint16)
    r = oracle.layer(x, synth.bits(t.w), synth.bits(t.bias))
    assert r["s_a"] == 0.0
    assert np.array_equal(r["out"], np.broadcast_to(synth.bits(t.bias), r["out"].shape))
    r2 = oracle.layer(synth.bits(t.x), np.zeros_like(synth.bits(t.w)), synth.bits(t.bias))
    assert np.array_equal(r2["out"], np.broadcast_to(synth.bits(t.bias), r2["out"].shape))


def test_layer_close_to_float64_conv_of_bf16_inputs():
    """The quantised layer approximates the float convolution it replaces."""
    t = synth.draw_custom(synth.LayerShape(64, 32, 8, 8, T=2), seed=10)
    r = oracle.layer(synth.bits(t.x), synth.bits(t.w), synth.bits(t.bias))
    x = t.x.to(torch.float64).permute(0, 4, 1, 2, 3)
    y = F.conv3d(F.pad(x, (1, 1, 1, 1, 2, 0)), t.w.to(torch.float64), t.bias.to(torch.float64))
    y = y.permute(0, 2, 3, 4, 1).numpy()
    got = b2f(r["out"]).astype(np.float64)
    err = np.abs(got - y).max() / np.abs(y).max()
    assert err < 0.05


# ------------------------------------------------- streamed chunks (carried frames)

def _brute_carry(qx_ext, qw):
    """Pure-Python reference for one streamed chunk: output frame t reads input frames
    t, t+1, t+2 of the extended input (two carried frames first), spatial padding 1."""
    N, T2, H, W, Cin = qx_ext.shape
    Cout = qw.shape[0]
    out = np.zeros((N, T2 - 2, H, W, Cout), dtype=np.int64)
    for n in range(N):
        for t in range(T2 - 2):
            for h in range(H):
                for w in range(W):
                    for co in range(Cout):
                        s = 0
                        for kt in range(3):
                            for kh in range(3):
                                for kw in range(3):
                                    hi, wi = h + kh - 1, w + kw - 1
                                    if 0 <= hi < H and 0 <= wi < W:
                                        for ci in range(Cin):
                                            s += int(qx_ext[n, t + kt, hi, wi, ci]) * int(qw[co, ci, kt, kh, kw])
                        out[n, t, h, w, co] = s
    return out


def test_carry_matches_brute_force_tiny():
    rng = np.random.default_rng(41)
    qx_ext = rng.integers(-127, 128, size=(2, 4, 2, 3, 3), dtype=np.int8)   # T = 2 chunk frames
    qw = rng.integers(-127, 128, size=(2, 3, 3, 3, 3), dtype=np.int8)
    assert np.array_equal(oracle.conv_acc_carry(qx_ext, qw), _brute_carry(qx_ext, qw))


def test_carry_with_zero_history_is_the_causal_conv():
    rng = np.random.default_rng(42)
    qx = rng.integers(-127, 128, size=(1, 3, 5, 6, 32), dtype=np.int8)
    qw = rng.integers(-127, 128, size=(8, 32, 3, 3, 3), dtype=np.int8)
    ext = np.concatenate([np.zeros_like(qx[:, :2]), qx], axis=1)
    assert np.array_equal(oracle.conv_acc_carry(ext, qw), oracle.conv_acc(qx, qw))


def test_chunked_stream_reproduces_the_whole_sequence():
    # with the same codes, chunks of two frames that carry the previous chunk's
    # last two input frames give the whole sequence's accumulators exactly
    rng = np.random.default_rng(43)
    qx = rng.integers(-127, 128, size=(2, 7, 4, 5, 32), dtype=np.int8)
    qw = rng.integers(-127, 128, size=(8, 32, 3, 3, 3), dtype=np.int8)
    full = oracle.conv_acc(qx, qw)
    parts = [oracle.conv_acc(qx[:, 0:2], qw)]
    for t0 in range(2, 7, 2):
        parts.append(oracle.conv_acc_carry(qx[:, t0 - 2:min(t0 + 2, 7)], qw))
    assert np.array_equal(np.concatenate(parts, axis=1), full)


def test_layer_carry_zero_history_equals_layer():
    # zero frames leave the absmax, hence the scale and codes, unchanged
    t = synth.draw_custom(synth.LayerShape(32, 32, 6, 5, T=2), seed=44, outliers=True)
    xb, wb, bb = (t.x.view(torch.int16).numpy().view(np.uint16), t.w.view(torch.int16).numpy().view(np.uint16),
                  t.bias.view(torch.int16).numpy().view(np.uint16))
    ext = np.concatenate([np.zeros_like(xb[:, :2]), xb], axis=1)
    a, b = oracle.layer_carry(ext, wb, bb), oracle.layer(xb, wb, bb)
    assert a["s_a"] == b["s_a"] and np.array_equal(a["out"], b["out"])


def test_epilogue_rounds_the_product_before_adding_the_bias():
    # A bf16 tie met on B200: acc = 135 with this scale and bias gives
    # y + b = -2.8405339e-07 exactly (0xb4988000), which rounds to even
    # (0xb498).  A fused multiply-add (one rounding) lands at 0xb4988c80 and
    # rounds to 0xb499: the oracle must keep the two roundings.
    s_a = np.float32(1.0)
    s_w = np.array([np.float32(3.3906315e-05)], dtype=np.float32)
    bias = np.array([np.uint32(np.float32(-0.0045776367).view(np.uint32) >> 16)], dtype=np.uint16)
    out = oracle.epilogue(np.array([[135]], dtype=np.int32), s_a, s_w, bias)
    y = np.float32(np.float32(135.0) * np.float32(s_w[0] * s_a))
    b = np.uint32(int(bias[0]) << 16).view(np.float32)
    sep = np.float32(y + b)
    assert sep.view(np.uint32) == 0xB4988000
    fused = np.float32(135.0 * np.float64(s_w[0]) + np.float64(b))
    assert fused.view(np.uint32) != sep.view(np.uint32)
    assert int(out[0, 0]) == 0xB498


# ------------------------------------------- property tests against a library conv

from hypothesis import given, settings, strategies as st  # noqa: E402


def _torch_conv(qx_padded_t, qw, pad_hw=1):
    """float64 conv3d of codes already padded in time; spatial zero padding 1."""
    x = torch.from_numpy(qx_padded_t.astype(np.float64)).permute(0, 4, 1, 2, 3)   # N C T H W
    w = torch.from_numpy(qw.astype(np.float64))                                     # Co Ci kt kh kw
    y = torch.nn.functional.conv3d(x, w, padding=(0, pad_hw, pad_hw))
    return y.permute(0, 2, 3, 4, 1).numpy()


@settings(max_examples=25, deadline=None)
@given(N=st.integers(1, 2), T=st.integers(1, 4), H=st.integers(1, 6), W=st.integers(1, 6),
       Cin=st.integers(1, 6), Cout=st.integers(1, 4), seed=st.integers(0, 2**31 - 1))
def test_conv_acc_matches_a_library_conv(N, T, H, W, Cin, Cout, seed):
    rng = np.random.default_rng(seed)
    qx = rng.integers(-127, 128, size=(N, T, H, W, Cin), dtype=np.int8)
    qw = rng.integers(-127, 128, size=(Cout, Cin, 3, 3, 3), dtype=np.int8)
    padded = np.concatenate([np.zeros((N, 2, H, W, Cin), np.int8), qx], axis=1)   # two causal zero frames
    assert np.array_equal(oracle.conv_acc(qx, qw), _torch_conv(padded, qw).astype(np.int64))


@settings(max_examples=25, deadline=None)
@given(T=st.integers(1, 3), H=st.integers(1, 5), W=st.integers(1, 5), Cin=st.integers(1, 5),
       Cout=st.integers(1, 3), seed=st.integers(0, 2**31 - 1))
def test_conv_acc_carry_matches_a_library_conv(T, H, W, Cin, Cout, seed):
    rng = np.random.default_rng(seed)
    ext = rng.integers(-127, 128, size=(1, T + 2, H, W, Cin), dtype=np.int8)      # carried frames first
    qw = rng.integers(-127, 128, size=(Cout, Cin, 3, 3, 3), dtype=np.int8)
    assert np.array_equal(oracle.conv_acc_carry(ext, qw), _torch_conv(ext, qw).astype(np.int64))

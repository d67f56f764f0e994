"""Pins for the oracle's native-precision layer (no GPU).

The release note's Aggressive preset (section on the three presets, and its
exclusion rule) keeps two decoder convolutions, decoder.upsamples.14.residual.2
and .residual.6, in their original precision.  The oracle evaluates such a
layer exactly -- the causal 3x3x3 convolution of the bf16 values in binary64
plus the bias -- and rounds once to bf16.  These tests pin it to things other
than itself: a float64 library convolution, a pure-Python loop over a tiny
case, exact rational rounding, and invariants (zero input gives the bias, a
delta kernel returns the input, T = 1 is a 2-D convolution with the last
temporal slice, causality).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from video_vae_decode_b200 import synth


def b2f(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f2bits(values):
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_layer(seed, N, T, H, W, Cin, Cout):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((N, T, H, W, Cin), generator=g).to(torch.bfloat16)
    w = (torch.randn((Cout, Cin, 3, 3, 3), generator=g) / (27 * Cin) ** 0.5).to(torch.bfloat16)
    b = (torch.randn(Cout, generator=g) * 0.1).to(torch.bfloat16)
    return synth.bits(x), synth.bits(w), synth.bits(b)


def library_conv(xb, wb, bb=None, magnitudes=False):
    """float64 torch conv3d on explicitly padded inputs: pad (2, 0) frames, 1 pixel."""
    x = torch.from_numpy(b2f(xb).astype(np.float64))
    w = torch.from_numpy(b2f(wb).astype(np.float64))
    if magnitudes:
        x, w = x.abs(), w.abs()
    xp = F.pad(x.permute(0, 4, 1, 2, 3), (1, 1, 1, 1, 2, 0))
    y = F.conv3d(xp, w).permute(0, 2, 3, 4, 1)
    if bb is not None:
        b = torch.from_numpy(b2f(bb).astype(np.float64))
        y = y + (b.abs() if magnitudes else b)
    return y.numpy()


# ------------------------------------------------------- the exact sum

@pytest.mark.parametrize("N,T,H,W,Cin,Cout", [(1, 1, 5, 7, 8, 4), (2, 3, 4, 3, 16, 8), (1, 4, 6, 5, 32, 32),
                                              (1, 2, 9, 1, 3, 5)])
def test_sum_matches_a_float64_library_conv(N, T, H, W, Cin, Cout):
    xb, wb, bb = rand_layer(N * 100 + T * 10 + H, N, T, H, W, Cin, Cout)
    y, s_abs = oracle.conv_bf16(xb, wb, bb)
    ref = library_conv(xb, wb, bb)
    mag = library_conv(xb, wb, bb, magnitudes=True)
    # both are binary64 sums of the same exact products in different orders
    assert np.all(np.abs(y - ref) <= 1e-12 * mag)
    assert np.allclose(s_abs, mag, rtol=1e-12, atol=0)


def test_sum_matches_a_python_loop_tiny():
    N, T, H, W, Cin, Cout = 1, 3, 3, 2, 2, 3
    xb, wb, bb = rand_layer(5, N, T, H, W, Cin, Cout)
    x, w, b = b2f(xb), b2f(wb), b2f(bb)
    y, _ = oracle.conv_bf16(xb, wb, bb)
    for t in range(T):
        for h in range(H):
            for ww in range(W):
                for co in range(Cout):
                    acc = Fraction(float(b[co]))
                    for kt in range(3):
                        for kh in range(3):
                            for kw in range(3):
                                ti, hi, wi = t + kt - 2, h + kh - 1, ww + kw - 1
                                if ti < 0 or not (0 <= hi < H) or not (0 <= wi < W):
                                    continue
                                for ci in range(Cin):
                                    acc += Fraction(float(x[0, ti, hi, wi, ci])) * Fraction(float(w[co, ci, kt, kh, kw]))
                    assert abs(Fraction(float(y[0, t, h, ww, co])) - acc) <= abs(acc) * Fraction(1, 2 ** 50)


def test_zero_input_gives_the_bias_and_no_bias_gives_zero():
    xb, wb, bb = rand_layer(7, 1, 2, 4, 4, 16, 8)
    y, s = oracle.conv_bf16(np.zeros_like(xb), wb, bb)
    assert np.array_equal(y, np.broadcast_to(b2f(bb).astype(np.float64), y.shape))
    y0, _ = oracle.conv_bf16(np.zeros_like(xb), wb, None)
    assert not y0.any()


def test_delta_kernel_returns_the_input():
    Cin = 8
    xb, _, bb = rand_layer(8, 1, 3, 5, 6, Cin, Cin)
    w = np.zeros((Cin, Cin, 3, 3, 3), dtype=np.float32)
    for c in range(Cin):
        w[c, c, 2, 1, 1] = 1.0                       # current frame, centre pixel
    y, _ = oracle.conv_bf16(xb, f2bits(w), bb)
    assert np.array_equal(y, b2f(xb).astype(np.float64) + b2f(bb).astype(np.float64))


def test_t1_is_a_2d_conv_with_the_last_temporal_slice():
    xb, wb, _ = rand_layer(9, 1, 1, 7, 6, 16, 8)
    y, _ = oracle.conv_bf16(xb, wb)
    x = torch.from_numpy(b2f(xb)[:, 0].astype(np.float64)).permute(0, 3, 1, 2)
    w2 = torch.from_numpy(b2f(wb)[:, :, 2].astype(np.float64))
    ref = F.conv2d(x, w2, padding=1).permute(0, 2, 3, 1).numpy()
    assert np.allclose(y[:, 0], ref, rtol=0, atol=1e-12)


def test_causality():
    xb, wb, bb = rand_layer(10, 1, 5, 4, 4, 8, 8)
    y, _ = oracle.conv_bf16(xb, wb, bb)
    x2 = xb.copy()
    x2[:, 3:] = f2bits(np.random.default_rng(0).standard_normal(x2[:, 3:].shape))
    y2, _ = oracle.conv_bf16(x2, wb, bb)
    assert np.array_equal(y[:, :3], y2[:, :3])
    assert not np.array_equal(y[:, 3:], y2[:, 3:])


# ------------------------------------------------------- one rounding to bf16

def nearest_bf16(v: float) -> int:
    """Exact rational search over the bf16 grid (ties to even)."""
    if v == 0:
        return 0x8000 if np.signbit(v) else 0
    a = Fraction(abs(v))
    best = None
    # candidates: the bf16 values around |v|, taken from the binary32 neighbours
    f = np.float32(abs(v))
    base = int(np.array([f], np.float32).view(np.uint32)[0] >> 16)
    for c in range(max(0, base - 2), base + 3):
        cv = Fraction(float(b2f(np.array([c], np.uint16))[0]))
        d = abs(cv - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1] | (0x8000 if v < 0 else 0)


def test_f64_to_bf16_rounds_once():
    rng = np.random.default_rng(11)
    vals = list(rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000))
    # ties of bf16 and values just off them that a detour through binary32 rounds onto the tie
    for m in range(0, 128, 7):
        tie = (1.0 + (2 * m + 1) / 256.0) * 2.0 ** rng.integers(-20, 20)
        vals += [tie, -tie, tie * (1 + 2.0 ** -40), tie * (1 - 2.0 ** -40)]
    vals += [0.0, -0.0, 1e-39, 3e-40, 2.0 ** -133, 1.5 * 2.0 ** -133]
    got = oracle.f64_to_bf16(np.array(vals))
    want = np.array([nearest_bf16(v) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)
    # the detour through binary32 does round twice on some of these values
    twice = f2bits(np.array(vals, dtype=np.float32))
    assert np.count_nonzero(twice != want) > 0


def test_layer_bf16_is_the_rounded_sum():
    xb, wb, bb = rand_layer(12, 1, 3, 6, 5, 32, 16)
    r = oracle.layer_bf16(xb, wb, bb)
    assert np.array_equal(r["out"], oracle.f64_to_bf16(r["y"]))
    # and it is within half a bf16 ulp of the library convolution
    ref = library_conv(xb, wb, bb)
    got = b2f(r["out"]).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    assert np.all(np.abs(got - ref) <= 0.5 * ulp * (1 + 1e-9))

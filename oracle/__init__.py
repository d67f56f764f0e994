"""CPU oracle for the W8A8 CausalConv3d layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never does, and the oracle never imports the product package.

The arithmetic lives in ``qvae_oracle.c`` (plain C, one function per step of
the method, each citing the passage it follows).  This module only marshals
numpy arrays.  bf16 tensors travel as ``uint16`` bit patterns.

Every function here is pinned by ``tests/test_oracle.py`` against things other
than itself: brute force on tiny shapes, a float64 library convolution,
closed-form golden values (``tests/golden/``) and invariants of the method.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        p = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        L.oracle_quantize_weights.argtypes = [p, i32, i32, p, p]
        L.oracle_quantize_weights.restype = ctypes.c_int
        L.oracle_act_absmax.argtypes = [p, i64, p]
        L.oracle_act_absmax.restype = ctypes.c_int
        L.oracle_act_quant.argtypes = [p, i64, p, p]
        L.oracle_act_quant_amax.argtypes = [p, i64, f32, p, p]
        L.oracle_act_quant_amax.restype = ctypes.c_int
        L.oracle_act_quant.restype = ctypes.c_int
        L.oracle_conv_acc.argtypes = [p, p, i64, i64, i64, i64, i32, i32, p]
        L.oracle_conv_acc.restype = ctypes.c_int
        L.oracle_conv_acc_carry.argtypes = [p, p, i64, i64, i64, i64, i32, i32, p]
        L.oracle_conv_acc_carry.restype = ctypes.c_int
        L.oracle_conv_acc_points.argtypes = [p, p, i64, i64, i64, i64, i32, i32, p, i64, p]
        L.oracle_conv_acc_points.restype = ctypes.c_int
        L.oracle_epilogue.argtypes = [p, i64, i32, f32, p, p, p]
        L.oracle_epilogue.restype = None
        L.oracle_f32_to_bf16.argtypes = [f32]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_conv_bf16.argtypes = [p, p, p, i64, i64, i64, i64, i32, i32, p, p]
        L.oracle_conv_bf16.restype = ctypes.c_int
        L.oracle_f64_to_bf16.argtypes = [p, i64, p]
        L.oracle_f64_to_bf16.restype = None
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        L.oracle_set_num_threads.restype = None
        _lib = L
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def quantize_weights(w_bits):
    """Per-output-channel symmetric INT8.

    w_bits: uint16 [Cout, Cin, 3, 3, 3] (bf16 bits, PyTorch Conv3d layout).
    Returns (qw int8 same shape, s_w float32 [Cout]).
    """
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    Cout, Cin = w.shape[0], w.shape[1]
    assert w.shape[2:] == (3, 3, 3)
    qw = np.empty(w.shape, dtype=np.int8)
    s_w = np.empty(Cout, dtype=np.float32)
    _check(lib().oracle_quantize_weights(_ptr(w), Cout, Cin, _ptr(qw), _ptr(s_w)), "quantize_weights")
    return qw, s_w


def act_absmax(x_bits) -> np.float32:
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    out = np.zeros(1, dtype=np.float32)
    _check(lib().oracle_act_absmax(_ptr(x), x.size, _ptr(out)), "act_absmax")
    return out[0]


def act_quant(x_bits):
    """Dynamic per-tensor symmetric INT8. Returns (qx int8 same shape, s_a float32)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    qx = np.empty(x.shape, dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    _check(lib().oracle_act_quant(_ptr(x), x.size, _ptr(qx), _ptr(s)), "act_quant")
    return qx, s[0]


def act_quant_amax(x_bits, amax):
    """Codes and scale of x for a maximum |value| taken over a larger tensor."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    qx = np.empty(x.shape, dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    _check(lib().oracle_act_quant_amax(_ptr(x), x.size, float(amax), _ptr(qx), _ptr(s)), "act_quant_amax")
    return qx, s[0]


def conv_acc(qx, qw):
    """Exact INT32 causal conv. qx int8 [N,T,H,W,Cin]; qw int8 [Cout,Cin,3,3,3]."""
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    N, T, H, W, Cin = qx.shape
    Cout = qw.shape[0]
    assert qw.shape == (Cout, Cin, 3, 3, 3)
    acc = np.empty((N, T, H, W, Cout), dtype=np.int32)
    _check(lib().oracle_conv_acc(_ptr(qx), _ptr(qw), N, T, H, W, Cin, Cout, _ptr(acc)), "conv_acc")
    return acc


def conv_acc_carry(qx_ext, qw):
    """Exact INT32 conv of a streamed chunk. qx_ext int8 [N,T+2,H,W,Cin] whose first
    two frames are the previous chunk's last two input frames; returns [N,T,H,W,Cout]."""
    qx_ext = np.ascontiguousarray(qx_ext, dtype=np.int8)
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    N, T2, H, W, Cin = qx_ext.shape
    T = T2 - 2
    assert T >= 1, "a chunk needs at least one frame after the two carried ones"
    Cout = qw.shape[0]
    assert qw.shape == (Cout, Cin, 3, 3, 3)
    acc = np.empty((N, T, H, W, Cout), dtype=np.int32)
    _check(lib().oracle_conv_acc_carry(_ptr(qx_ext), _ptr(qw), N, T, H, W, Cin, Cout, _ptr(acc)),
           "conv_acc_carry")
    return acc


def conv_acc_points(qx, qw, pts):
    """INT32 accumulators at selected pixels. pts int64 [P, 4] of (n, t, h, w)."""
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    pts = np.ascontiguousarray(pts, dtype=np.int64).reshape(-1, 4)
    N, T, H, W, Cin = qx.shape
    Cout = qw.shape[0]
    acc = np.empty((pts.shape[0], Cout), dtype=np.int32)
    _check(lib().oracle_conv_acc_points(_ptr(qx), _ptr(qw), N, T, H, W, Cin, Cout,
                                        _ptr(pts), pts.shape[0], _ptr(acc)), "conv_acc_points")
    return acc


def epilogue(acc, s_a, s_w, bias_bits=None):
    """bf16_rne(float(acc) * (s_a * s_w[co]) + bias[co]); acc int32 [..., Cout]."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    Cout = acc.shape[-1]
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    assert s_w.shape == (Cout,)
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    out = np.empty(acc.shape, dtype=np.uint16)
    lib().oracle_epilogue(_ptr(acc), acc.size // Cout, Cout, ctypes.c_float(float(s_a)),
                          _ptr(s_w), _ptr(b), _ptr(out))
    return out


def f32_to_bf16(values):
    """Round float32 values to bf16 bits (nearest, ties to even)."""
    v = np.asarray(values, dtype=np.float32).ravel()
    L = lib()
    return np.array([L.oracle_f32_to_bf16(ctypes.c_float(float(f))) for f in v],
                    dtype=np.uint16).reshape(np.shape(values))


def layer_carry(x_ext_bits, w_bits, bias_bits=None):
    """One streamed chunk: x_ext (bf16 bits [N,T+2,H,W,Cin], the two carried frames
    first) is quantised as one tensor; the output covers the T chunk frames."""
    qw, s_w = quantize_weights(w_bits)
    qx, s_a = act_quant(x_ext_bits)
    acc = conv_acc_carry(qx, qw)
    out = epilogue(acc, s_a, s_w, bias_bits)
    return {"qw": qw, "s_w": s_w, "qx": qx, "s_a": s_a, "acc": acc, "out": out}


def layer(x_bits, w_bits, bias_bits=None):
    """The whole layer: codes, scales, accumulators and bf16 output."""
    qw, s_w = quantize_weights(w_bits)
    qx, s_a = act_quant(x_bits)
    acc = conv_acc(qx, qw)
    out = epilogue(acc, s_a, s_w, bias_bits)
    return {"qw": qw, "s_w": s_w, "qx": qx, "s_a": s_a, "acc": acc, "out": out}


def conv_bf16(x_bits, w_bits, bias_bits=None):
    """Native-precision causal conv, exact: returns (y float64, s_abs float64), both
    [N,T,H,W,Cout]; y = bias + sum of x*w, s_abs = |bias| + sum of |x*w|."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    N, T, H, W, Cin = x.shape
    Cout = w.shape[0]
    assert w.shape == (Cout, Cin, 3, 3, 3)
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    y = np.empty((N, T, H, W, Cout), dtype=np.float64)
    s_abs = np.empty_like(y)
    _check(lib().oracle_conv_bf16(_ptr(x), _ptr(w), _ptr(b), N, T, H, W, Cin, Cout, _ptr(y), _ptr(s_abs)),
           "conv_bf16")
    return y, s_abs


def f64_to_bf16(values):
    """Round float64 values to bf16 bits once (nearest, ties to even)."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_f64_to_bf16(_ptr(v), v.size, _ptr(out))
    return out


def layer_bf16(x_bits, w_bits, bias_bits=None):
    """A native-precision layer: exact sum, then one rounding to bf16."""
    y, s_abs = conv_bf16(x_bits, w_bits, bias_bits)
    return {"y": y, "s_abs": s_abs, "out": f64_to_bf16(y)}

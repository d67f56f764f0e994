"""ctypes binding of libqvae (declarations in include/qvae.h).

Argument marshalling only: every step of the layer runs in the CUDA library.
Tensors are torch CUDA tensors (device memory and streams come from PyTorch);
their data pointers are handed to the C entry points of the same names.
Each wrapper raises ``QvaeError`` on a non-zero status.  ``lib()`` raises if
``libqvae.so`` has not been built: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# QVAE_LIBRARY names another build of the same ABI (libqvae_debug.so: the
# bounds-checked kernels); the default is the in-tree release library.
LIB_PATH = os.environ.get("QVAE_LIBRARY") or os.path.join(HERE, "libqvae.so")

QVAE_OK, QVAE_ERR_ARG, QVAE_ERR_SHAPE, QVAE_ERR_ALIGN = 0, 1, 2, 3
QVAE_ERR_CUDA, QVAE_ERR_TIMEOUT, QVAE_ERR_UNSUPPORTED, QVAE_ERR_BOUNDS = 4, 5, 6, 7

# Every symbol include/qvae.h declares.
EXPORTS = (
    "qvae_status_string", "qvae_last_error_message", "qvae_packed_weight_bytes",
    "qvae_quantize_weights", "qvae_act_workspace_bytes", "qvae_act_absmax_quant",
    "qvae_causal_conv3d_w8a8", "qvae_causal_conv3d_w8a8_acc32", "qvae_decode_workspace_bytes",
    "qvae_decode_layers", "qvae_get_error", "qvae_set_wait_limit_ns",
    "qvae_selftest_wait_timeout", "qvae_build_flags", "qvae_set_conv_tiling", "qvae_get_conv_tiling", "qvae_set_conv_cta_limit",
    "qvae_act_absmax_quant_noalloc",
    "qvae_causal_conv3d_w8a8_carry", "qvae_causal_conv3d_w8a8_carry_acc32",
    "qvae_act_absmax", "qvae_act_quant_from_absmax",
    "qvae_causal_conv3d_w8a8_band", "qvae_causal_conv3d_w8a8_band_acc32",
    "qvae_packed_weight_bytes_bf16", "qvae_pack_weights_bf16", "qvae_causal_conv3d_bf16",
    "qvae_causal_conv3d_bf16_acc32", "qvae_causal_conv3d_w8a8_fused", "qvae_causal_conv3d_w8a8_fused_acc32",
    "qvae_set_fused_quant",
)


class QvaeError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} failed: {message} (status {status})")
        self.status = status


class qvae_shape(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("T", ctypes.c_int64), ("H", ctypes.c_int64),
                ("W", ctypes.c_int64), ("Cin", ctypes.c_int32), ("Cout", ctypes.c_int32)]


class qvae_layer(ctypes.Structure):
    _fields_ = [("shape", qvae_shape), ("quantized", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("x", ctypes.c_void_p), ("out", ctypes.c_void_p), ("wq_packed", ctypes.c_void_p),
                ("w_scale", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


_lib = None


def lib():
    """Load libqvae.so; raises when it has not been built (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m video_vae_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        p, i32, i64, u64, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                ctypes.c_size_t)
        sig = {
            "qvae_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "qvae_last_error_message": ([], ctypes.c_char_p),
            "qvae_packed_weight_bytes": ([i32, i32], sz),
            "qvae_quantize_weights": ([i32, i32, p, p, p, p, p], ctypes.c_int),
            "qvae_act_workspace_bytes": ([i64], sz),
            "qvae_act_absmax_quant": ([p, i64, p, p, p, sz, p], ctypes.c_int),
            "qvae_act_absmax_quant_noalloc": ([p, i64, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_w8a8": ([ctypes.POINTER(qvae_shape), p, p, p, p, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_w8a8_acc32": ([ctypes.POINTER(qvae_shape), p, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_w8a8_carry": ([ctypes.POINTER(qvae_shape), p, p, p, p, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_w8a8_carry_acc32": ([ctypes.POINTER(qvae_shape), p, p, p, p], ctypes.c_int),
            "qvae_act_absmax": ([p, i64, p, p], ctypes.c_int),
            "qvae_act_quant_from_absmax": ([p, i64, p, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_w8a8_band": ([ctypes.POINTER(qvae_shape), i32, i32, p, p, p, p, p, p, p],
                                             ctypes.c_int),
            "qvae_causal_conv3d_w8a8_band_acc32": ([ctypes.POINTER(qvae_shape), i32, i32, p, p, p, p],
                                                   ctypes.c_int),
            "qvae_packed_weight_bytes_bf16": ([i32, i32], sz),
            "qvae_pack_weights_bf16": ([i32, i32, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_bf16": ([ctypes.POINTER(qvae_shape), p, p, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_bf16_acc32": ([ctypes.POINTER(qvae_shape), p, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_w8a8_fused": ([ctypes.POINTER(qvae_shape), p, p, p, p, p, p, p, p], ctypes.c_int),
            "qvae_causal_conv3d_w8a8_fused_acc32": ([ctypes.POINTER(qvae_shape), p, p, p, p, p], ctypes.c_int),
            "qvae_decode_workspace_bytes": ([ctypes.POINTER(qvae_layer), i32], sz),
            "qvae_decode_layers": ([ctypes.POINTER(qvae_layer), i32, p, sz, p], ctypes.c_int),
            "qvae_get_error": ([p], ctypes.c_int),
            "qvae_set_wait_limit_ns": ([u64], ctypes.c_int),
            "qvae_selftest_wait_timeout": ([u64, p], ctypes.c_int),
            "qvae_build_flags": ([], ctypes.c_int),
            "qvae_set_conv_tiling": ([i32, i32, i32, i32, i32, i32], ctypes.c_int),
            "qvae_set_conv_cta_limit": ([i32], ctypes.c_int),
            "qvae_set_fused_quant": ([i32], ctypes.c_int),
            "qvae_get_conv_tiling": ([ctypes.POINTER(qvae_shape), i32, ctypes.POINTER(i32)], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(name: str, status: int):
    if status != QVAE_OK:
        L = lib()
        msg = L.qvae_status_string(status).decode()
        extra = L.qvae_last_error_message().decode()
        raise QvaeError(name, status, msg + (f": {extra}" if extra and status == QVAE_ERR_CUDA else ""))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_shape(N, T, H, W, Cin, Cout) -> qvae_shape:
    return qvae_shape(int(N), int(T), int(H), int(W), int(Cin), int(Cout))


def shape_of(x: torch.Tensor, Cout: int) -> qvae_shape:
    N, T, H, W, Cin = x.shape
    return make_shape(N, T, H, W, Cin, Cout)


# ---------------------------------------------------------------- weights

def qvae_packed_weight_bytes(Cin: int, Cout: int) -> int:
    return int(lib().qvae_packed_weight_bytes(Cin, Cout))


def qvae_quantize_weights(w: torch.Tensor, wq_packed: torch.Tensor, w_scale: torch.Tensor,
                          wq_plain: Optional[torch.Tensor] = None, stream=None) -> None:
    Cout, Cin = int(w.shape[0]), int(w.shape[1])
    _check("qvae_quantize_weights",
           lib().qvae_quantize_weights(Cin, Cout, _ptr(w), _ptr(wq_packed), _ptr(w_scale),
                                       _ptr(wq_plain), _stream(stream)))


def quantize_weights(w: torch.Tensor, plain: bool = False, stream=None):
    """Allocate and fill (wq_packed, w_scale[, wq_plain [Cout, 27, Cin]]) for a bf16 weight."""
    Cout, Cin = int(w.shape[0]), int(w.shape[1])
    packed = torch.empty(qvae_packed_weight_bytes(Cin, Cout), dtype=torch.int8, device=w.device)
    scale = torch.empty(Cout, dtype=torch.float32, device=w.device)
    pl = torch.zeros((Cout, 27, Cin), dtype=torch.int8, device=w.device) if plain else None
    qvae_quantize_weights(w, packed, scale, pl, stream)
    return (packed, scale, pl) if plain else (packed, scale)


# ------------------------------------------------------------ activations

def qvae_act_workspace_bytes(numel: int) -> int:
    return int(lib().qvae_act_workspace_bytes(numel))


def qvae_act_absmax_quant(x: torch.Tensor, xq: torch.Tensor, x_scale: torch.Tensor,
                          workspace: torch.Tensor, stream=None) -> None:
    _check("qvae_act_absmax_quant",
           lib().qvae_act_absmax_quant(_ptr(x), x.numel(), _ptr(xq), _ptr(x_scale), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)))


def qvae_act_absmax_quant_noalloc(x: torch.Tensor, xq: torch.Tensor, x_scale: torch.Tensor,
                                  stream=None) -> None:
    """Same as qvae_act_absmax_quant with the library's fixed scratch (no workspace)."""
    _check("qvae_act_absmax_quant_noalloc",
           lib().qvae_act_absmax_quant_noalloc(_ptr(x), x.numel(), _ptr(xq), _ptr(x_scale), _stream(stream)))


def act_absmax_quant(x: torch.Tensor, stream=None, workspace: Optional[torch.Tensor] = None):
    xq = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    s = torch.empty(1, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(qvae_act_workspace_bytes(x.numel()), dtype=torch.uint8, device=x.device)
    qvae_act_absmax_quant(x, xq, s, workspace, stream)
    return xq, s


# ------------------------------------------------------------ convolution

def qvae_causal_conv3d_w8a8(xq: torch.Tensor, x_scale: torch.Tensor, wq_packed: torch.Tensor,
                            w_scale: torch.Tensor, bias: Optional[torch.Tensor], out: torch.Tensor,
                            stream=None) -> None:
    shp = shape_of(xq, int(out.shape[-1]))
    _check("qvae_causal_conv3d_w8a8",
           lib().qvae_causal_conv3d_w8a8(ctypes.byref(shp), _ptr(xq), _ptr(x_scale), _ptr(wq_packed),
                                         _ptr(w_scale), _ptr(bias), _ptr(out), _stream(stream)))


def qvae_causal_conv3d_w8a8_acc32(xq: torch.Tensor, wq_packed: torch.Tensor, acc: torch.Tensor,
                                  stream=None) -> None:
    shp = shape_of(xq, int(acc.shape[-1]))
    _check("qvae_causal_conv3d_w8a8_acc32",
           lib().qvae_causal_conv3d_w8a8_acc32(ctypes.byref(shp), _ptr(xq), _ptr(wq_packed), _ptr(acc),
                                               _stream(stream)))


def causal_conv3d_w8a8(xq, x_scale, wq_packed, w_scale, bias, Cout: int, stream=None):
    out = torch.empty(tuple(xq.shape[:-1]) + (Cout,), dtype=torch.bfloat16, device=xq.device)
    qvae_causal_conv3d_w8a8(xq, x_scale, wq_packed, w_scale, bias, out, stream)
    return out


def _chunk_shape(xq_ext: torch.Tensor, Cout: int) -> qvae_shape:
    """Shape of a streamed chunk: xq_ext holds two carried frames before the chunk's."""
    N, T2, H, W, Cin = xq_ext.shape
    if T2 < 2:
        raise ValueError("a streamed chunk's input holds two carried frames before its own")
    return make_shape(N, T2 - 2, H, W, Cin, Cout)


def qvae_causal_conv3d_w8a8_carry(xq_ext: torch.Tensor, x_scale: torch.Tensor, wq_packed: torch.Tensor,
                                  w_scale: torch.Tensor, bias: Optional[torch.Tensor], out: torch.Tensor,
                                  stream=None) -> None:
    shp = _chunk_shape(xq_ext, int(out.shape[-1]))
    _check("qvae_causal_conv3d_w8a8_carry",
           lib().qvae_causal_conv3d_w8a8_carry(ctypes.byref(shp), _ptr(xq_ext), _ptr(x_scale), _ptr(wq_packed),
                                               _ptr(w_scale), _ptr(bias), _ptr(out), _stream(stream)))


def qvae_causal_conv3d_w8a8_carry_acc32(xq_ext: torch.Tensor, wq_packed: torch.Tensor, acc: torch.Tensor,
                                        stream=None) -> None:
    shp = _chunk_shape(xq_ext, int(acc.shape[-1]))
    _check("qvae_causal_conv3d_w8a8_carry_acc32",
           lib().qvae_causal_conv3d_w8a8_carry_acc32(ctypes.byref(shp), _ptr(xq_ext), _ptr(wq_packed),
                                                     _ptr(acc), _stream(stream)))


def conv_carry(xq_ext, x_scale, wq_packed, w_scale, bias, Cout: int, stream=None):
    _chunk_shape(xq_ext, Cout)
    N, T2, H, W, _ = xq_ext.shape
    out = torch.empty((N, T2 - 2, H, W, Cout), dtype=torch.bfloat16, device=xq_ext.device)
    qvae_causal_conv3d_w8a8_carry(xq_ext, x_scale, wq_packed, w_scale, bias, out, stream)
    return out


def conv_carry_acc32(xq_ext, wq_packed, Cout: int, stream=None):
    _chunk_shape(xq_ext, Cout)
    N, T2, H, W, _ = xq_ext.shape
    acc = torch.empty((N, T2 - 2, H, W, Cout), dtype=torch.int32, device=xq_ext.device)
    qvae_causal_conv3d_w8a8_carry_acc32(xq_ext, wq_packed, acc, stream)
    return acc


def qvae_act_absmax(x: torch.Tensor, amax: torch.Tensor, stream=None) -> None:
    """amax: a 4-byte device tensor (int32 or uint32) that receives max |x| as bf16 magnitude bits."""
    _check("qvae_act_absmax", lib().qvae_act_absmax(_ptr(x), x.numel(), _ptr(amax), _stream(stream)))


def qvae_act_quant_from_absmax(x: torch.Tensor, amax: torch.Tensor, xq: torch.Tensor, x_scale: torch.Tensor,
                               stream=None) -> None:
    _check("qvae_act_quant_from_absmax",
           lib().qvae_act_quant_from_absmax(_ptr(x), x.numel(), _ptr(amax), _ptr(xq), _ptr(x_scale),
                                            _stream(stream)))


def _band_shape(xq_band: torch.Tensor, halo_top: int, halo_bot: int, Cout: int) -> qvae_shape:
    N, T, Hin, W, Cin = xq_band.shape
    H = Hin - halo_top - halo_bot
    if H < 0:
        raise ValueError("a band holds its halo rows and its own")
    return make_shape(N, T, H, W, Cin, Cout)


def qvae_causal_conv3d_w8a8_band(xq_band: torch.Tensor, halo_top: int, halo_bot: int, x_scale: torch.Tensor,
                                 wq_packed: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor],
                                 out: torch.Tensor, stream=None) -> None:
    shp = _band_shape(xq_band, halo_top, halo_bot, int(out.shape[-1]))
    _check("qvae_causal_conv3d_w8a8_band",
           lib().qvae_causal_conv3d_w8a8_band(ctypes.byref(shp), int(halo_top), int(halo_bot), _ptr(xq_band),
                                              _ptr(x_scale), _ptr(wq_packed), _ptr(w_scale), _ptr(bias),
                                              _ptr(out), _stream(stream)))


def qvae_causal_conv3d_w8a8_band_acc32(xq_band: torch.Tensor, halo_top: int, halo_bot: int,
                                       wq_packed: torch.Tensor, acc: torch.Tensor, stream=None) -> None:
    shp = _band_shape(xq_band, halo_top, halo_bot, int(acc.shape[-1]))
    _check("qvae_causal_conv3d_w8a8_band_acc32",
           lib().qvae_causal_conv3d_w8a8_band_acc32(ctypes.byref(shp), int(halo_top), int(halo_bot),
                                                    _ptr(xq_band), _ptr(wq_packed), _ptr(acc), _stream(stream)))


def qvae_causal_conv3d_w8a8_fused(x: torch.Tensor, x_amax: torch.Tensor, wq_packed: torch.Tensor,
                                  w_scale: torch.Tensor, bias: Optional[torch.Tensor], out: torch.Tensor,
                                  x_scale_out: Optional[torch.Tensor] = None, stream=None) -> None:
    """x bf16; x_amax a 4-byte device word from qvae_act_absmax (bf16 magnitude bits of max |x|)."""
    shp = shape_of(x, int(out.shape[-1]))
    _check("qvae_causal_conv3d_w8a8_fused",
           lib().qvae_causal_conv3d_w8a8_fused(ctypes.byref(shp), _ptr(x), _ptr(x_amax), _ptr(wq_packed),
                                               _ptr(w_scale), _ptr(bias), _ptr(out), _ptr(x_scale_out),
                                               _stream(stream)))


def qvae_causal_conv3d_w8a8_fused_acc32(x: torch.Tensor, x_amax: torch.Tensor, wq_packed: torch.Tensor,
                                        acc: torch.Tensor, stream=None) -> None:
    shp = shape_of(x, int(acc.shape[-1]))
    _check("qvae_causal_conv3d_w8a8_fused_acc32",
           lib().qvae_causal_conv3d_w8a8_fused_acc32(ctypes.byref(shp), _ptr(x), _ptr(x_amax), _ptr(wq_packed),
                                                     _ptr(acc), _stream(stream)))


def layer_w8a8(x, wq_packed, w_scale, bias, Cout: int, stream=None, amax=None, scale=None):
    """One quantised layer the fused way: qvae_act_absmax, then the convolution quantising x itself.
    Returns (out, scale)."""
    if amax is None:
        amax = torch.empty(1, dtype=torch.int32, device=x.device)
    if scale is None:
        scale = torch.empty(1, dtype=torch.float32, device=x.device)
    out = torch.empty(tuple(x.shape[:-1]) + (Cout,), dtype=torch.bfloat16, device=x.device)
    qvae_act_absmax(x, amax, stream)
    qvae_causal_conv3d_w8a8_fused(x, amax, wq_packed, w_scale, bias, out, scale, stream)
    return out, scale


def conv_acc32(xq, wq_packed, Cout: int, stream=None):
    acc = torch.empty(tuple(xq.shape[:-1]) + (Cout,), dtype=torch.int32, device=xq.device)
    qvae_causal_conv3d_w8a8_acc32(xq, wq_packed, acc, stream)
    return acc


# ------------------------------------------------- native-precision layer

def qvae_packed_weight_bytes_bf16(Cin: int, Cout: int) -> int:
    return int(lib().qvae_packed_weight_bytes_bf16(Cin, Cout))


def qvae_pack_weights_bf16(w: torch.Tensor, w_packed: torch.Tensor, stream=None) -> None:
    Cout, Cin = int(w.shape[0]), int(w.shape[1])
    _check("qvae_pack_weights_bf16",
           lib().qvae_pack_weights_bf16(Cin, Cout, _ptr(w), _ptr(w_packed), _stream(stream)))


def pack_weights_bf16(w: torch.Tensor, stream=None) -> torch.Tensor:
    """Allocate and fill the packed bf16 weights of a native-precision layer."""
    Cout, Cin = int(w.shape[0]), int(w.shape[1])
    packed = torch.empty(qvae_packed_weight_bytes_bf16(Cin, Cout), dtype=torch.uint8, device=w.device)
    qvae_pack_weights_bf16(w, packed, stream)
    return packed


def qvae_causal_conv3d_bf16(x: torch.Tensor, w_packed: torch.Tensor, bias: Optional[torch.Tensor],
                            out: torch.Tensor, stream=None) -> None:
    shp = shape_of(x, int(out.shape[-1]))
    _check("qvae_causal_conv3d_bf16",
           lib().qvae_causal_conv3d_bf16(ctypes.byref(shp), _ptr(x), _ptr(w_packed), _ptr(bias), _ptr(out),
                                         _stream(stream)))


def qvae_causal_conv3d_bf16_acc32(x: torch.Tensor, w_packed: torch.Tensor, acc: torch.Tensor,
                                  stream=None) -> None:
    shp = shape_of(x, int(acc.shape[-1]))
    _check("qvae_causal_conv3d_bf16_acc32",
           lib().qvae_causal_conv3d_bf16_acc32(ctypes.byref(shp), _ptr(x), _ptr(w_packed), _ptr(acc),
                                               _stream(stream)))


def causal_conv3d_bf16(x, w_packed, bias, Cout: int, stream=None):
    out = torch.empty(tuple(x.shape[:-1]) + (Cout,), dtype=torch.bfloat16, device=x.device)
    qvae_causal_conv3d_bf16(x, w_packed, bias, out, stream)
    return out


def conv_bf16_acc32(x, w_packed, Cout: int, stream=None):
    acc = torch.empty(tuple(x.shape[:-1]) + (Cout,), dtype=torch.float32, device=x.device)
    qvae_causal_conv3d_bf16_acc32(x, w_packed, acc, stream)
    return acc


# ------------------------------------------------------------ layer chain

def make_layers(specs: Sequence[dict]):
    """specs: dicts with x, out, wq_packed, w_scale, bias (tensors), quantized (bool).

    A native-precision layer (quantized=False) carries the output of
    pack_weights_bf16 as wq_packed (the library runs it), or no weights (the
    library skips it)."""
    arr = (qvae_layer * len(specs))()
    for i, s in enumerate(specs):
        x, out = s["x"], s["out"]
        N, T, H, W, Cin = x.shape
        arr[i].shape = make_shape(N, T, H, W, Cin, out.shape[-1])
        arr[i].quantized = 1 if s.get("quantized", True) else 0
        arr[i].reserved = 0
        arr[i].x = x.data_ptr()
        arr[i].out = out.data_ptr()
        arr[i].wq_packed = s["wq_packed"].data_ptr() if s.get("wq_packed") is not None else None
        arr[i].w_scale = s["w_scale"].data_ptr() if s.get("w_scale") is not None else None
        arr[i].bias = s["bias"].data_ptr() if s.get("bias") is not None else None
    return arr


def qvae_decode_workspace_bytes(layers) -> int:
    return int(lib().qvae_decode_workspace_bytes(layers, len(layers)))


def qvae_decode_layers(layers, workspace: torch.Tensor, stream=None) -> None:
    _check("qvae_decode_layers",
           lib().qvae_decode_layers(layers, len(layers), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))


# ---------------------------------------------------------------- control

def qvae_get_error(stream=None) -> int:
    return int(lib().qvae_get_error(_stream(stream)))


def qvae_set_wait_limit_ns(limit_ns: int) -> None:
    _check("qvae_set_wait_limit_ns", lib().qvae_set_wait_limit_ns(int(limit_ns)))


def qvae_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check("qvae_selftest_wait_timeout", lib().qvae_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def qvae_set_conv_tiling(MS=0, NT=0, SA=0, SB=0, mode=0, G=0) -> None:
    _check("qvae_set_conv_tiling", lib().qvae_set_conv_tiling(MS, NT, SA, SB, mode, G))


def qvae_set_fused_quant(on: int = 0) -> None:
    _check("qvae_set_fused_quant", lib().qvae_set_fused_quant(int(on)))


def qvae_set_conv_cta_limit(max_ctas: int = 0) -> None:
    _check("qvae_set_conv_cta_limit", lib().qvae_set_conv_cta_limit(int(max_ctas)))


def qvae_get_conv_tiling(N, T, H, W, Cin, Cout, variant: int = 0) -> dict:
    """variant 0: convolution of INT8 codes; 1: fused (bf16 input quantised in the kernel); 2: native bf16."""
    shp = make_shape(N, T, H, W, Cin, Cout)
    out = (ctypes.c_int32 * 8)()
    _check("qvae_get_conv_tiling", lib().qvae_get_conv_tiling(ctypes.byref(shp), int(variant), out))
    return dict(zip(("MS", "NT", "SA", "SB", "acc_buffers", "ctas", "mode", "G"), list(out)))

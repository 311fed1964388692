"""Python binding of libmxmoe.so, the sm_100a MXFP4 MoE expert-layer library.

Argument marshalling only: each function below takes torch tensors (or raw
pointers), checks dtypes/shapes, and calls the C entry point of the same name
(declared in include/mxmoe.h) on the current CUDA stream. Every step of the
layer runs in the library's CUDA kernels; there is no Python or CPU fallback.
The library is loaded on first use; if it is missing that first call raises.

Layer (pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4
Quantization"; nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article, architecture
section): router GEMM -> top-k routing -> grouping by expert -> SwiGLU expert
FFN over MXFP4 weights -> weighted combine.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmxmoe.so")

OK = 0
ERR_INVALID_SHAPE = 1
ERR_ALIGNMENT = 2
ERR_NULL = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_DEVICE = 6
ERR_WORKSPACE = 7

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64

_SIGS = {
    "mxmoe_version": (ctypes.c_char_p, []),
    "mxmoe_last_error": (ctypes.c_char_p, []),
    "mxmoe_quantize": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "mxmoe_dequantize": (_I, [_P, _P, _I64, _I64, _P, _P]),
    "mxmoe_prepacked_size": (_I64, [_I, _I, _I]),
    "mxmoe_prepack_experts": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "mxmoe_router_gemm": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "mxmoe_route": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "mxmoe_permute": (_I, [_P, _I, _I, _I, _P, _P, _P, _P]),
    "mxmoe_ffn_workspace_size": (_I64, [_I, _I, _I, _I, _I]),
    "mxmoe_expert_ffn": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I64, _P]),
    "mxmoe_ffn_gate_up": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I64, _P]),
    "mxmoe_ffn_down": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _I64, _P]),
    "mxmoe_expert_ffn_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "mxmoe_combine": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "mxmoe_workspace_size": (_I64, [_I, _I, _I, _I, _I]),
    "mxmoe_layer_forward": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I64, _P]),
    "mxmoe_layer_forward_persistent": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I64, _P]),
    "mxmoe_layer_forward_chained": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I64, _P]),
    "mxmoe_read_status": (_I, [_P, _P, _P]),
    "mxmoe_selftest_wait_timeout": (_I, [_P, _I, _P]),
    "mxmoe_permute_ws": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I64, _P]),
    "mxmoe_permute_scratch_size": (_I64, [_I, _I, _I]),
    "mxmoe_quantize_fp8": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "mxmoe_dequantize_fp8": (_I, [_P, _P, _I64, _I64, _P, _P]),
    "mxmoe_prepacked_size_fp8": (_I64, [_I, _I, _I]),
    "mxmoe_prepack_experts_fp8": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "mxmoe_ffn_workspace_size_fp8": (_I64, [_I, _I, _I, _I, _I]),
    "mxmoe_expert_ffn_fp8": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I64, _P]),
    "mxmoe_workspace_size_fp8": (_I64, [_I, _I, _I, _I, _I]),
    "mxmoe_layer_forward_fp8": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I64, _P]),
    "mxmoe_ep_dispatch": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "mxmoe_ep_workspace_size": (_I64, [_I, _I, _I, _I]),
    "mxmoe_ep_expert_ffn": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _I64, _P]),
    "mxmoe_verify_workspace_size": (_I64, [_I, _I, _I64]),
    "mxmoe_verify_block": (_I, [_P, _P, _P, _P, _I, _I, _I64, ctypes.c_float, _P, _P, _P, _I64, _P]),
}

_lib = None


def load():
    """Load libmxmoe.so (once). Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                "libmxmoe.so is not built (expected at %s); run "
                "`python -m mxfp4_quantized_moe_router_b200.build` or __graft_entry__.build()" % LIB_PATH)
        lib_ = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(lib_, name)
            f.restype = res
            f.argtypes = args
        _lib = lib_
    return _lib


def __getattr__(name):
    if name == "lib":
        return load()
    raise AttributeError(name)


class MxmoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__("%s failed (status %d): %s" % (fn, code, last_error()))


def version() -> str:
    return load().mxmoe_version().decode()


def last_error() -> str:
    return load().mxmoe_last_error().decode()


def _check(fn: str, rc: int) -> None:
    if rc != OK:
        raise MxmoeError(fn, rc)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch

    return torch.cuda.current_stream().cuda_stream


def _need(t, dtype, shape, name):
    import torch

    if t.dtype != dtype:
        raise TypeError("%s: expected %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s: expected shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("%s: must be a contiguous CUDA tensor" % name)
    del torch


# ---------------------------------------------------------------------------
# Weight format
# ---------------------------------------------------------------------------
def mxmoe_quantize(w, packed, scales, stream=None):
    import torch

    rows, K = w.shape
    _need(w, torch.bfloat16, (rows, K), "w")
    _need(packed, torch.uint8, (rows, K // 2), "packed")
    _need(scales, torch.uint8, (rows, K // 32), "scales")
    _check("mxmoe_quantize", load().mxmoe_quantize(_ptr(w), rows, K, _ptr(packed), _ptr(scales), _stream(stream)))


def quantize(w, stream=None):
    """bf16 [rows, K] -> (packed uint8 [rows, K/2], scales uint8 [rows, K/32])."""
    import torch

    rows, K = w.shape
    packed = torch.empty((rows, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((rows, K // 32), dtype=torch.uint8, device=w.device)
    mxmoe_quantize(w.contiguous(), packed, scales, stream)
    return packed, scales


def mxmoe_dequantize(packed, scales, out, stream=None):
    import torch

    rows, K = out.shape
    _need(packed, torch.uint8, (rows, K // 2), "packed")
    _need(scales, torch.uint8, (rows, K // 32), "scales")
    _need(out, torch.float32, (rows, K), "out")
    _check("mxmoe_dequantize", load().mxmoe_dequantize(_ptr(packed), _ptr(scales), rows, K, _ptr(out), _stream(stream)))


def dequantize(packed, scales, stream=None):
    import torch

    rows = packed.shape[0]
    out = torch.empty((rows, packed.shape[1] * 2), dtype=torch.float32, device=packed.device)
    mxmoe_dequantize(packed, scales, out, stream)
    return out


def mxmoe_prepacked_size(E: int, H: int, I: int) -> int:
    return load().mxmoe_prepacked_size(E, H, I)


def mxmoe_prepack_experts(packed13, sc13, packed2, sc2, E, H, I, prepacked, stream=None):
    import torch

    _need(packed13, torch.uint8, (E, 2 * I, H // 2), "packed13")
    _need(sc13, torch.uint8, (E, 2 * I, H // 32), "sc13")
    _need(packed2, torch.uint8, (E, H, I // 2), "packed2")
    _need(sc2, torch.uint8, (E, H, I // 32), "sc2")
    _need(prepacked, torch.uint8, (mxmoe_prepacked_size(E, H, I),), "prepacked")
    _check("mxmoe_prepack_experts",
           load().mxmoe_prepack_experts(_ptr(packed13), _ptr(sc13), _ptr(packed2), _ptr(sc2), E, H, I, _ptr(prepacked),
                                     _stream(stream)))


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------
def mxmoe_router_gemm(x, wg, bias, logits, stream=None):
    import torch

    T, H = x.shape
    E = wg.shape[0]
    _need(x, torch.bfloat16, (T, H), "x")
    _need(wg, torch.bfloat16, (E, H), "wg")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    _need(logits, torch.float32, (T, E), "logits")
    _check("mxmoe_router_gemm",
           load().mxmoe_router_gemm(_ptr(x), _ptr(wg), _ptr(bias), T, H, E, _ptr(logits), _stream(stream)))


def mxmoe_route(logits, k, ids, w, stream=None):
    import torch

    T, E = logits.shape
    _need(logits, torch.float32, (T, E), "logits")
    _need(ids, torch.int32, (T, k), "ids")
    _need(w, torch.float32, (T, k), "w")
    _check("mxmoe_route", load().mxmoe_route(_ptr(logits), T, E, k, _ptr(ids), _ptr(w), _stream(stream)))


def mxmoe_permute(ids, E, offsets, src_row, dst_of, stream=None):
    import torch

    T, k = ids.shape
    _need(ids, torch.int32, (T, k), "ids")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(src_row, torch.int32, (T * k,), "src_row")
    _need(dst_of, torch.int32, (T * k,), "dst_of")
    _check("mxmoe_permute",
           load().mxmoe_permute(_ptr(ids), T, k, E, _ptr(offsets), _ptr(src_row), _ptr(dst_of), _stream(stream)))


# ---------------------------------------------------------------------------
# Experts / combine / layer
# ---------------------------------------------------------------------------
def mxmoe_ffn_workspace_size(T, k, E, H, I) -> int:
    return load().mxmoe_ffn_workspace_size(T, k, E, H, I)


def mxmoe_expert_ffn(x, offsets, src_row, prepacked, k, E, I, y_perm, workspace, stream=None):
    import torch

    T, H = x.shape
    _need(x, torch.bfloat16, (T, H), "x")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(src_row, torch.int32, (T * k,), "src_row")
    _need(y_perm, torch.float32, (T * k, H), "y_perm")
    _check("mxmoe_expert_ffn",
           load().mxmoe_expert_ffn(_ptr(x), _ptr(offsets), _ptr(src_row), _ptr(prepacked), T, k, E, H, I, _ptr(y_perm),
                                _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def mxmoe_ffn_gate_up(x, offsets, src_row, prepacked, k, E, I, workspace, stream=None):
    import torch

    T, H = x.shape
    _need(x, torch.bfloat16, (T, H), "x")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(src_row, torch.int32, (T * k,), "src_row")
    _check("mxmoe_ffn_gate_up",
           load().mxmoe_ffn_gate_up(_ptr(x), _ptr(offsets), _ptr(src_row), _ptr(prepacked), T, k, E, H, I,
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def mxmoe_ffn_down(offsets, prepacked, T, k, E, H, I, y_perm, workspace, stream=None):
    import torch

    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(y_perm, torch.float32, (T * k, H), "y_perm")
    _check("mxmoe_ffn_down",
           load().mxmoe_ffn_down(_ptr(offsets), _ptr(prepacked), T, k, E, H, I, _ptr(y_perm), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream)))


def mxmoe_expert_ffn_noalloc(x, offsets, src_row, prepacked, k, E, I, y_perm, status=None, stream=None):
    """mxmoe_expert_ffn without a workspace (scratch in the library's fixed
    8 MiB static device array); for callers that cannot allocate."""
    import torch

    T, H = x.shape
    _need(x, torch.bfloat16, (T, H), "x")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(src_row, torch.int32, (T * k,), "src_row")
    _need(y_perm, torch.float32, (T * k, H), "y_perm")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    _check("mxmoe_expert_ffn_noalloc",
           load().mxmoe_expert_ffn_noalloc(_ptr(x), _ptr(offsets), _ptr(src_row), _ptr(prepacked), T, k, E, H, I,
                                           _ptr(y_perm), _ptr(status), _stream(stream)))


def mxmoe_combine(y_perm, dst_of, w, y, stream=None):
    import torch

    T, k = w.shape
    H = y.shape[1]
    _need(y_perm, torch.float32, (T * k, H), "y_perm")
    _need(dst_of, torch.int32, (T * k,), "dst_of")
    _need(w, torch.float32, (T, k), "w")
    _need(y, torch.float32, (T, H), "y")
    _check("mxmoe_combine", load().mxmoe_combine(_ptr(y_perm), _ptr(dst_of), _ptr(w), T, k, H, _ptr(y), _stream(stream)))


def mxmoe_workspace_size(T, H, I, E, k) -> int:
    return load().mxmoe_workspace_size(T, H, I, E, k)


def mxmoe_layer_forward(x, wg, bias, prepacked, I, k, y, workspace, ids_out=None, w_out=None, stream=None):
    import torch

    T, H = x.shape
    E = wg.shape[0]
    _need(x, torch.bfloat16, (T, H), "x")
    _need(wg, torch.bfloat16, (E, H), "wg")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    _need(y, torch.float32, (T, H), "y")
    if ids_out is not None:
        _need(ids_out, torch.int32, (T, k), "ids_out")
    if w_out is not None:
        _need(w_out, torch.float32, (T, k), "w_out")
    _check("mxmoe_layer_forward",
           load().mxmoe_layer_forward(_ptr(x), _ptr(wg), _ptr(bias), _ptr(prepacked), T, H, I, E, k, _ptr(y),
                                   _ptr(ids_out), _ptr(w_out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))


def _layer_call(name, x, wg, bias, prepacked, I, k, y, workspace, ids_out, w_out, stream):
    import torch

    T, H = x.shape
    E = wg.shape[0]
    _need(x, torch.bfloat16, (T, H), "x")
    _need(wg, torch.bfloat16, (E, H), "wg")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    _need(y, torch.float32, (T, H), "y")
    if ids_out is not None:
        _need(ids_out, torch.int32, (T, k), "ids_out")
    if w_out is not None:
        _need(w_out, torch.float32, (T, k), "w_out")
    _check(name, getattr(load(), name)(_ptr(x), _ptr(wg), _ptr(bias), _ptr(prepacked), T, H, I, E, k, _ptr(y),
                                       _ptr(ids_out), _ptr(w_out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)))


def mxmoe_layer_forward_persistent(x, wg, bias, prepacked, I, k, y, workspace, ids_out=None, w_out=None, stream=None):
    """mxmoe_layer_forward as one persistent kernel (T <= 256, T*k <= 4096, E <= 384)."""
    _layer_call("mxmoe_layer_forward_persistent", x, wg, bias, prepacked, I, k, y, workspace, ids_out, w_out, stream)


def mxmoe_layer_forward_chained(x, wg, bias, prepacked, I, k, y, workspace, ids_out=None, w_out=None, stream=None):
    """mxmoe_layer_forward as chained launches at every size."""
    _layer_call("mxmoe_layer_forward_chained", x, wg, bias, prepacked, I, k, y, workspace, ids_out, w_out, stream)


def mxmoe_read_status(workspace, stream=None) -> int:
    st = ctypes.c_int(-1)
    _check("mxmoe_read_status", load().mxmoe_read_status(_ptr(workspace), ctypes.byref(st), _stream(stream)))
    return st.value


def mxmoe_permute_scratch_size(T, k, E) -> int:
    return int(load().mxmoe_permute_scratch_size(T, k, E))


def mxmoe_permute_ws(ids, E, offsets, src_row, dst_of, scratch, stream=None):
    """mxmoe_permute with caller scratch (the multi-block grouping for many pairs)."""
    import torch

    T, k = ids.shape
    _need(ids, torch.int32, (T, k), "ids")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(src_row, torch.int32, (T * k,), "src_row")
    _need(dst_of, torch.int32, (T * k,), "dst_of")
    _check("mxmoe_permute_ws",
           load().mxmoe_permute_ws(_ptr(ids), T, k, E, _ptr(offsets), _ptr(src_row), _ptr(dst_of), _ptr(scratch),
                                   scratch.numel() * scratch.element_size(), _stream(stream)))


def mxmoe_selftest_wait_timeout(status, limit_us: int, stream=None) -> None:
    """Make one bounded device-side wait run out (nothing arrives on its
    barrier); status (device int32 [1]) receives MXMOE_ERR_TIMEOUT."""
    import torch

    _need(status, torch.int32, (1,), "status")
    _check("mxmoe_selftest_wait_timeout",
           load().mxmoe_selftest_wait_timeout(_ptr(status), int(limit_us), _stream(stream)))


# ---------------------------------------------------------------------------
# Convenience: a whole expert set on the device
# ---------------------------------------------------------------------------
class ExpertWeights:
    """MXFP4 expert weights of one layer on the device: canonical packed codes
    and scales (the graded format) plus the prepacked blob the kernels stream."""

    def __init__(self, E: int, H: int, I: int, device="cuda", keep_canonical: bool = True):
        import torch

        self.E, self.H, self.I = E, H, I
        self.keep_canonical = keep_canonical
        self.packed13 = torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device=device)
        self.sc13 = torch.empty((E, 2 * I, H // 32), dtype=torch.uint8, device=device)
        self.packed2 = torch.empty((E, H, I // 2), dtype=torch.uint8, device=device)
        self.sc2 = torch.empty((E, H, I // 32), dtype=torch.uint8, device=device)
        self.prepacked = torch.empty((mxmoe_prepacked_size(E, H, I),), dtype=torch.uint8, device=device)

    def quantize_expert(self, e: int, w13, w2, stream=None):
        """Quantise one expert's bf16 gate/up [2I, H] and down [H, I] weights."""
        mxmoe_quantize(w13, self.packed13[e], self.sc13[e], stream)
        mxmoe_quantize(w2, self.packed2[e], self.sc2[e], stream)

    def prepack(self, stream=None):
        mxmoe_prepack_experts(self.packed13, self.sc13, self.packed2, self.sc2, self.E, self.H, self.I,
                              self.prepacked, stream)


# ---------------------------------------------------------------------------
# FP8 expert weights (E4M3, one E8M0 scale per 32)
# ---------------------------------------------------------------------------
def mxmoe_quantize_fp8(w, codes, scales, stream=None):
    import torch

    rows, K = w.shape
    _need(w, torch.bfloat16, (rows, K), "w")
    _need(codes, torch.uint8, (rows, K), "codes")
    _need(scales, torch.uint8, (rows, K // 32), "scales")
    _check("mxmoe_quantize_fp8",
           load().mxmoe_quantize_fp8(_ptr(w), rows, K, _ptr(codes), _ptr(scales), _stream(stream)))


def quantize_fp8(w, stream=None):
    """bf16 [rows, K] -> (E4M3 codes uint8 [rows, K], scales uint8 [rows, K/32])."""
    import torch

    rows, K = w.shape
    codes = torch.empty((rows, K), dtype=torch.uint8, device=w.device)
    scales = torch.empty((rows, K // 32), dtype=torch.uint8, device=w.device)
    mxmoe_quantize_fp8(w.contiguous(), codes, scales, stream)
    return codes, scales


def mxmoe_dequantize_fp8(codes, scales, out, stream=None):
    import torch

    rows, K = out.shape
    _need(codes, torch.uint8, (rows, K), "codes")
    _need(scales, torch.uint8, (rows, K // 32), "scales")
    _need(out, torch.float32, (rows, K), "out")
    _check("mxmoe_dequantize_fp8",
           load().mxmoe_dequantize_fp8(_ptr(codes), _ptr(scales), rows, K, _ptr(out), _stream(stream)))


def dequantize_fp8(codes, scales, stream=None):
    import torch

    out = torch.empty(tuple(codes.shape), dtype=torch.float32, device=codes.device)
    mxmoe_dequantize_fp8(codes, scales, out, stream)
    return out


def mxmoe_prepacked_size_fp8(E: int, H: int, I: int) -> int:
    return load().mxmoe_prepacked_size_fp8(E, H, I)


def mxmoe_prepack_experts_fp8(codes13, sc13, codes2, sc2, E, H, I, prepacked, stream=None):
    import torch

    _need(codes13, torch.uint8, (E, 2 * I, H), "codes13")
    _need(sc13, torch.uint8, (E, 2 * I, H // 32), "sc13")
    _need(codes2, torch.uint8, (E, H, I), "codes2")
    _need(sc2, torch.uint8, (E, H, I // 32), "sc2")
    _need(prepacked, torch.uint8, (mxmoe_prepacked_size_fp8(E, H, I),), "prepacked")
    _check("mxmoe_prepack_experts_fp8",
           load().mxmoe_prepack_experts_fp8(_ptr(codes13), _ptr(sc13), _ptr(codes2), _ptr(sc2), E, H, I,
                                            _ptr(prepacked), _stream(stream)))


def mxmoe_ffn_workspace_size_fp8(T, k, E, H, I) -> int:
    return load().mxmoe_ffn_workspace_size_fp8(T, k, E, H, I)


def mxmoe_expert_ffn_fp8(x, offsets, src_row, prepacked, k, E, I, y_perm, workspace, stream=None):
    import torch

    T, H = x.shape
    _need(x, torch.bfloat16, (T, H), "x")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(src_row, torch.int32, (T * k,), "src_row")
    _need(y_perm, torch.float32, (T * k, H), "y_perm")
    _check("mxmoe_expert_ffn_fp8",
           load().mxmoe_expert_ffn_fp8(_ptr(x), _ptr(offsets), _ptr(src_row), _ptr(prepacked), T, k, E, H, I,
                                       _ptr(y_perm), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)))


def mxmoe_workspace_size_fp8(T, H, I, E, k) -> int:
    return load().mxmoe_workspace_size_fp8(T, H, I, E, k)


def mxmoe_layer_forward_fp8(x, wg, bias, prepacked, I, k, y, workspace, ids_out=None, w_out=None, stream=None):
    import torch

    T, H = x.shape
    E = wg.shape[0]
    _need(x, torch.bfloat16, (T, H), "x")
    _need(wg, torch.bfloat16, (E, H), "wg")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    _need(y, torch.float32, (T, H), "y")
    if ids_out is not None:
        _need(ids_out, torch.int32, (T, k), "ids_out")
    if w_out is not None:
        _need(w_out, torch.float32, (T, k), "w_out")
    _check("mxmoe_layer_forward_fp8",
           load().mxmoe_layer_forward_fp8(_ptr(x), _ptr(wg), _ptr(bias), _ptr(prepacked), T, H, I, E, k, _ptr(y),
                                          _ptr(ids_out), _ptr(w_out), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)))


class ExpertWeightsFp8:
    """FP8 expert weights of one layer on the device: E4M3 codes and scales
    (canonical) plus the prepacked blob the FP8 FFN streams."""

    def __init__(self, E: int, H: int, I: int, device="cuda"):
        import torch

        self.E, self.H, self.I = E, H, I
        self.codes13 = torch.empty((E, 2 * I, H), dtype=torch.uint8, device=device)
        self.sc13 = torch.empty((E, 2 * I, H // 32), dtype=torch.uint8, device=device)
        self.codes2 = torch.empty((E, H, I), dtype=torch.uint8, device=device)
        self.sc2 = torch.empty((E, H, I // 32), dtype=torch.uint8, device=device)
        self.prepacked = torch.empty((mxmoe_prepacked_size_fp8(E, H, I),), dtype=torch.uint8, device=device)

    def quantize_expert(self, e: int, w13, w2, stream=None):
        mxmoe_quantize_fp8(w13, self.codes13[e], self.sc13[e], stream)
        mxmoe_quantize_fp8(w2, self.codes2[e], self.sc2[e], stream)

    def prepack(self, stream=None):
        mxmoe_prepack_experts_fp8(self.codes13, self.sc13, self.codes2, self.sc2, self.E, self.H, self.I,
                                  self.prepacked, stream)


# ---------------------------------------------------------------------------
# Expert parallelism (compute steps; the exchanges are in .ep)
# ---------------------------------------------------------------------------
def mxmoe_ep_dispatch(x, offsets, src_row, k, E, G, send_x, send_local, send_counts, stream=None):
    import torch

    T, H = x.shape
    _need(x, torch.bfloat16, (T, H), "x")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(src_row, torch.int32, (T * k,), "src_row")
    _need(send_x, torch.bfloat16, (T * k, H), "send_x")
    _need(send_local, torch.int32, (T * k,), "send_local")
    _need(send_counts, torch.int32, (G,), "send_counts")
    _check("mxmoe_ep_dispatch",
           load().mxmoe_ep_dispatch(_ptr(x), _ptr(offsets), _ptr(src_row), T, k, E, G, H, _ptr(send_x),
                                    _ptr(send_local), _ptr(send_counts), _stream(stream)))


def mxmoe_ep_workspace_size(n_recv, E_local, H, I) -> int:
    return load().mxmoe_ep_workspace_size(n_recv, E_local, H, I)


def mxmoe_ep_expert_ffn(x_recv, recv_local, E_local, I, prepacked_local, y_recv, workspace, stream=None):
    import torch

    n, H = x_recv.shape
    _need(x_recv, torch.bfloat16, (n, H), "x_recv")
    _need(recv_local, torch.int32, (n,), "recv_local")
    _need(y_recv, torch.float32, (n, H), "y_recv")
    _check("mxmoe_ep_expert_ffn",
           load().mxmoe_ep_expert_ffn(_ptr(x_recv), _ptr(recv_local), n, E_local, H, I, _ptr(prepacked_local),
                                      _ptr(y_recv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream)))


# ---------------------------------------------------------------------------
# Block verification of a speculative draft
# ---------------------------------------------------------------------------
def mxmoe_verify_workspace_size(B, K, V) -> int:
    return load().mxmoe_verify_workspace_size(B, K, V)


def mxmoe_verify_block(target_logits, draft_logits, draft_tokens, uniforms, temperature, accepted, tokens, workspace,
                       stream=None):
    """Verify B drafted blocks (see include/mxmoe.h). target_logits float32
    [B, K+1, V], draft_logits float32 [B, K, V] or None (greedy),
    draft_tokens int32 [B, K], uniforms float32 [B, K+1], accepted int32 [B],
    tokens int32 [B, K+1], workspace uint8 of mxmoe_verify_workspace_size."""
    import torch

    B, K1, V = target_logits.shape
    K = K1 - 1
    _need(target_logits, torch.float32, (B, K + 1, V), "target_logits")
    if draft_logits is not None:
        _need(draft_logits, torch.float32, (B, K, V), "draft_logits")
    _need(draft_tokens, torch.int32, (B, K), "draft_tokens")
    _need(uniforms, torch.float32, (B, K + 1), "uniforms")
    _need(accepted, torch.int32, (B,), "accepted")
    _need(tokens, torch.int32, (B, K + 1), "tokens")
    _check("mxmoe_verify_block",
           load().mxmoe_verify_block(_ptr(target_logits), _ptr(draft_logits), _ptr(draft_tokens), _ptr(uniforms), B,
                                     K, V, float(temperature), _ptr(accepted), _ptr(tokens), _ptr(workspace),
                                     workspace.numel(), _stream(stream)))

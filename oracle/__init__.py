"""Plain float64 CPU oracle for the MXFP4 MoE expert layer (test infrastructure).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers. The product library never imports this package and shares no code
with it.

The arithmetic lives in ``mxmoe_oracle.c`` (plain single-threaded C loops in
IEEE double, compiled with ``gcc -O2`` and no fast-math). This module only
compiles it, loads it with ctypes and marshals numpy arrays. ``moe_layer``
composes the C steps for a set of tokens, decoding one expert at a time so that
the 384-expert layer fits in host memory; its optional thread pool only runs
independent experts side by side (ctypes releases the GIL), which does not
change any arithmetic.

Pages followed (see the C file for the step-by-step readings):
  * "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization"
    (MXFP4 experts, block size 32);
  * nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article, architecture section
    (384 experts, 8 active per token, hidden size 6144).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxmoe_oracle.c")
_LIB = os.path.join(_HERE, "libmxmoe_oracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 32


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math) if missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I32 = ctypes.c_int
        lib.mxo_e2m1_value.restype = ctypes.c_double
        lib.mxo_e2m1_value.argtypes = [I32]
        lib.mxo_e8m0_value.restype = ctypes.c_double
        lib.mxo_e8m0_value.argtypes = [I32]
        lib.mxo_e2m1_round.restype = I32
        lib.mxo_e2m1_round.argtypes = [ctypes.c_double]
        lib.mxo_bf16_to_double.restype = ctypes.c_double
        lib.mxo_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.mxo_e4m3_value.restype = ctypes.c_double
        lib.mxo_e4m3_value.argtypes = [I32]
        lib.mxo_e4m3_round.restype = I32
        lib.mxo_e4m3_round.argtypes = [ctypes.c_double]
        lib.mxo_quantize_fp8.argtypes = [P, I64, I64, P, P]
        lib.mxo_dequantize_fp8.argtypes = [P, P, I64, I64, P]
        lib.mxo_expert_ffn_fp8.argtypes = [P, P, P, P, P, I64, I64, I64, P, P]
        lib.mxo_quantize.argtypes = [P, I64, I64, P, P]
        lib.mxo_dequantize.argtypes = [P, P, I64, I64, P]
        lib.mxo_router_logits.argtypes = [P, P, P, I64, I64, I64, P]
        lib.mxo_route.argtypes = [P, I64, I64, I32, P, P]
        lib.mxo_route_f32.argtypes = [P, I64, I64, I32, P, P]
        lib.mxo_permute.argtypes = [P, I64, I32, I64, P, P, P]
        lib.mxo_combine.argtypes = [P, P, P, I64, I32, I64, P]
        lib.mxo_expert_ffn.argtypes = [P, P, P, I64, I64, I64, P, P]
        lib.mxo_expert_ffn_mxfp4.argtypes = [P, P, P, P, P, I64, I64, I64, P, P]
        lib.mxo_verify_block.argtypes = [P, P, P, P, I64, I32, I64, ctypes.c_double, P, P, P, P]
        lib.mxo_draw_interval.argtypes = [P, P, I64, ctypes.c_double, I64, P, P]
        for f in ("mxo_quantize_fp8", "mxo_dequantize_fp8", "mxo_expert_ffn_fp8", "mxo_quantize", "mxo_dequantize", "mxo_router_logits", "mxo_route", "mxo_route_f32",
                  "mxo_permute", "mxo_combine", "mxo_expert_ffn", "mxo_expert_ffn_mxfp4", "mxo_verify_block",
                  "mxo_draw_interval"):
            getattr(lib, f).restype = None
        _lib = lib
        return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(x) -> np.ndarray:
    """Accept a torch bf16 tensor or a uint16 array of bf16 bits."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # plumbing only: view the bf16 bits

    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


# --- scalar encodings -------------------------------------------------------
def e2m1_value(code: int) -> float:
    return _load().mxo_e2m1_value(int(code))


def e8m0_value(s: int) -> float:
    return _load().mxo_e8m0_value(int(s))


def e2m1_round(q: float) -> int:
    return _load().mxo_e2m1_round(float(q))


def bf16_to_double(bits: int) -> float:
    return _load().mxo_bf16_to_double(int(bits))


# --- quantiser ----------------------------------------------------------------
def quantize(w) -> tuple[np.ndarray, np.ndarray]:
    """bf16 [rows, K] -> (packed uint8 [rows, K/2], scales uint8 [rows, K/32])."""
    wb = _bf16_bits(w)
    rows, K = wb.shape
    assert K % BLOCK == 0
    packed = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // BLOCK), np.uint8)
    _load().mxo_quantize(_p(wb), rows, K, _p(packed), _p(scales))
    return packed, scales


def dequantize(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows = packed.shape[0]
    K = packed.shape[1] * 2
    out = np.empty((rows, K), np.float64)
    _load().mxo_dequantize(_p(packed), _p(scales), rows, K, _p(out))
    return out


# --- FP8 expert weights (E4M3 elements, one E8M0 scale per 32) ---------------
def e4m3_value(code: int) -> float:
    return _load().mxo_e4m3_value(int(code))


def e4m3_round(q: float) -> int:
    return _load().mxo_e4m3_round(float(q))


def quantize_fp8(w) -> tuple[np.ndarray, np.ndarray]:
    """bf16 [rows, K] -> (E4M3 codes uint8 [rows, K], scales uint8 [rows, K/32])."""
    wb = _bf16_bits(w)
    rows, K = wb.shape
    assert K % BLOCK == 0
    codes = np.zeros((rows, K), np.uint8)
    scales = np.zeros((rows, K // BLOCK), np.uint8)
    _load().mxo_quantize_fp8(_p(wb), rows, K, _p(codes), _p(scales))
    return codes, scales


def dequantize_fp8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    _load().mxo_dequantize_fp8(_p(codes), _p(scales), rows, K, _p(out))
    return out


def expert_ffn_fp8(c13, s13, c2, s2, x, want_h: bool = False):
    """One FP8 expert (codes13 [2I, H], sc13 [2I, H/32], codes2 [H, I], sc2
    [H, I/32]) decoded to float64, on rows x."""
    c13, s13, c2, s2 = (np.ascontiguousarray(a, np.uint8) for a in (c13, s13, c2, s2))
    xb = _bf16_bits(x)
    n, H = xb.shape
    I = c13.shape[0] // 2
    y = np.empty((n, H), np.float64)
    h = np.empty((n, I), np.float64) if want_h else None
    _load().mxo_expert_ffn_fp8(_p(c13), _p(s13), _p(c2), _p(s2), _p(xb), n, H, I, _p(h) if want_h else None, _p(y))
    return (y, h) if want_h else y


# --- router -------------------------------------------------------------------
def router_logits(x, wg, bias=None) -> np.ndarray:
    xb, wb = _bf16_bits(x), _bf16_bits(wg)
    T, H = xb.shape
    E = wb.shape[0]
    out = np.empty((T, E), np.float64)
    bp = None
    if bias is not None:
        bias = np.ascontiguousarray(np.asarray(bias, np.float32))
        bp = _p(bias)
    _load().mxo_router_logits(_p(xb), _p(wb), bp, T, H, E, _p(out))
    return out


def route(logits: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """Top-k routing. float64 logits use them as they are; float32 logits are
    widened exactly first. Returns (ids int32 [T,k], w float64 [T,k])."""
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    if logits.dtype == np.float32:
        l32 = np.ascontiguousarray(logits)
        _load().mxo_route_f32(_p(l32), T, E, k, _p(ids), _p(w))
    else:
        l64 = np.ascontiguousarray(logits, np.float64)
        _load().mxo_route(_p(l64), T, E, k, _p(ids), _p(w))
    return ids, w


def permute(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, np.int32)
    T, k = ids.shape
    offsets = np.empty(E + 1, np.int32)
    src_row = np.empty(T * k, np.int32)
    dst_of = np.empty(T * k, np.int32)
    _load().mxo_permute(_p(ids), T, k, E, _p(offsets), _p(src_row), _p(dst_of))
    return offsets, src_row, dst_of


def combine(y_perm: np.ndarray, dst_of: np.ndarray, w: np.ndarray, T: int, k: int) -> np.ndarray:
    y_perm = np.ascontiguousarray(y_perm, np.float64)
    dst_of = np.ascontiguousarray(dst_of, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    H = y_perm.shape[1]
    y = np.empty((T, H), np.float64)
    _load().mxo_combine(_p(y_perm), _p(dst_of), _p(w), T, k, H, _p(y))
    return y


# --- expert FFN ---------------------------------------------------------------
def expert_ffn(w13: np.ndarray, w2: np.ndarray, x, want_h: bool = False):
    """Dense float64 expert: w13 [2I, H] (gate rows first), w2 [H, I]."""
    w13 = np.ascontiguousarray(w13, np.float64)
    w2 = np.ascontiguousarray(w2, np.float64)
    xb = _bf16_bits(x)
    n, H = xb.shape
    I = w13.shape[0] // 2
    y = np.empty((n, H), np.float64)
    h = np.empty((n, I), np.float64) if want_h else None
    _load().mxo_expert_ffn(_p(w13), _p(w2), _p(xb), n, H, I, _p(h) if want_h else None, _p(y))
    return (y, h) if want_h else y


def expert_ffn_mxfp4(p13, s13, p2, s2, x, want_h: bool = False):
    """One MXFP4 expert (canonical packed layout) decoded to float64, on rows x."""
    p13, s13, p2, s2 = (np.ascontiguousarray(a, np.uint8) for a in (p13, s13, p2, s2))
    xb = _bf16_bits(x)
    n, H = xb.shape
    I = p13.shape[0] // 2
    y = np.empty((n, H), np.float64)
    h = np.empty((n, I), np.float64) if want_h else None
    _load().mxo_expert_ffn_mxfp4(_p(p13), _p(s13), _p(p2), _p(s2), _p(xb), n, H, I,
                                 _p(h) if want_h else None, _p(y))
    return (y, h) if want_h else y


def moe_layer(x, wg, bias, expert_fetch, k: int, threads: int = 1, fmt: str = "mxfp4"):
    """Whole MoE layer on the tokens in ``x`` (bf16 [n, H]).

    ``expert_fetch(e)`` returns the canonical MXFP4 arrays of expert e as
    (packed13 [2I, H/2], sc13 [2I, H/32], packed2 [H, I/2], sc2 [H, I/32]),
    or with ``fmt="fp8"`` the FP8 arrays (codes13 [2I, H], sc13, codes2
    [H, I], sc2).
    Steps: router logits (float64) -> route -> per expert, the rows routed
    to it -> combine in slot order. Returns dict with y, ids, w, logits,
    offsets, src_row, dst_of.
    """
    xb = _bf16_bits(x)
    n, H = xb.shape
    logits = router_logits(xb, wg, bias)
    E = logits.shape[1]
    ids, w = route(logits, k)
    offsets, src_row, dst_of = permute(ids, E)
    y_perm = np.zeros((n * k, H), np.float64)
    touched = [e for e in range(E) if offsets[e + 1] > offsets[e]]

    def run(e):
        rows = src_row[offsets[e]:offsets[e + 1]]
        xe = np.ascontiguousarray(xb[rows // k])
        p13, s13, p2, s2 = expert_fetch(e)
        ffn = expert_ffn_fp8 if fmt == "fp8" else expert_ffn_mxfp4
        y_perm[offsets[e]:offsets[e + 1]] = ffn(p13, s13, p2, s2, xe)

    if threads > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, touched))
    else:
        for e in touched:
            run(e)
    y = combine(y_perm, dst_of, w, n, k)
    return dict(y=y, ids=ids, w=w, logits=logits, offsets=offsets, src_row=src_row, dst_of=dst_of,
                touched=len(touched))


# --- block verification of a speculative draft ----------------------------
def verify_block(target: np.ndarray, draft, dtok: np.ndarray, u: np.ndarray, tau: float):
    """Verify B drafted blocks of K tokens (see ``mxo_verify_block`` in the C
    file for the reading of the pages' rejection-sampling verification).

    target float32 [B, K+1, V]; draft float32 [B, K, V] (None when tau = 0);
    dtok int32 [B, K]; u float32 [B, K+1] in [0, 1); tau >= 0 (0: greedy).
    Returns (accepted int32 [B], tokens int32 [B, K+1], margin_acc float64
    [B], margin_draw float64 [B])."""
    target = np.ascontiguousarray(target, np.float32)
    B, K1, V = target.shape
    K = K1 - 1
    dtok = np.ascontiguousarray(dtok, np.int32)
    u = np.ascontiguousarray(u, np.float32)
    assert dtok.shape == (B, K) and u.shape == (B, K + 1)
    dp = None
    if tau != 0.0:
        draft = np.ascontiguousarray(draft, np.float32)
        assert draft.shape == (B, K, V)
        dp = _p(draft)
    acc = np.empty(B, np.int32)
    tokens = np.empty((B, K + 1), np.int32)
    m_acc = np.empty(B, np.float64)
    m_draw = np.empty(B, np.float64)
    _load().mxo_verify_block(_p(target), dp, _p(dtok), _p(u), B, K, V, float(tau), _p(acc), _p(tokens), _p(m_acc),
                             _p(m_draw))
    return acc, tokens, m_acc, m_draw


def draw_interval(z_row: np.ndarray, w_row, tau: float, v: int) -> tuple[float, float]:
    """[lo, hi) that token v covers in the normalised running sum of a draw's
    weights: the residual max(0, p - q) when a drafter row is given, else p."""
    z_row = np.ascontiguousarray(z_row, np.float32)
    wp = None
    if w_row is not None:
        w_row = np.ascontiguousarray(w_row, np.float32)
        wp = _p(w_row)
    lo, hi = ctypes.c_double(), ctypes.c_double()
    _load().mxo_draw_interval(_p(z_row), wp, z_row.size, float(tau), int(v), ctypes.byref(lo), ctypes.byref(hi))
    return lo.value, hi.value

"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/mxmoe.h declares, and rejects bad arguments on the
host (before anything would be enqueued)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxmoe.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"MXMOE_API\s+[\w\s\*]+?\b(mxmoe_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = set(declared_symbols())
    for n in ("mxmoe_quantize", "mxmoe_dequantize", "mxmoe_prepack_experts", "mxmoe_router_gemm", "mxmoe_route",
              "mxmoe_permute", "mxmoe_expert_ffn", "mxmoe_combine", "mxmoe_layer_forward", "mxmoe_workspace_size",
              "mxmoe_read_status", "mxmoe_last_error", "mxmoe_version"):
        assert n in names, n


def test_library_exports_every_declared_symbol(mx):
    lib = ctypes.CDLL(mx.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_binding_names_match_header(mx):
    for name in declared_symbols():
        if name in ("mxmoe_version", "mxmoe_last_error"):
            continue
        assert hasattr(mx, name), name


def test_version(mx):
    assert mx.version().startswith("mxmoe")


def test_prepacked_size_is_format_bytes(mx):
    # codes + scales, 3*H*I*E*(1/2 + 1/32), with H and I padded to multiples of 256
    def pad(v):
        return (v + 255) // 256 * 256
    for E, H, I in [(384, 6144, 2048), (16, 256, 256), (3, 512, 768), (16, 256, 128), (5, 640, 384)]:
        Hp, Ip = pad(H), pad(I)
        assert mx.mxmoe_prepacked_size(E, H, I) == E * (2 * I * Hp + Hp * Ip) * 17 // 32
    assert mx.mxmoe_prepacked_size(384, 6144, 2048) == 384 * 20_054_016  # no padding at the layer's shape
    assert mx.mxmoe_prepacked_size(4, 192, 128) == -1  # H % 128
    assert mx.mxmoe_prepacked_size(4, 256, 64) == -1  # I % 128


def test_workspace_queries(mx):
    assert mx.mxmoe_workspace_size(8, 6144, 2048, 384, 8) > 0
    assert mx.mxmoe_workspace_size(8, 6144, 2048, 384, 400) == -1
    assert mx.mxmoe_ffn_workspace_size(8, 8, 384, 6144, 2048) > 0
    assert mx.mxmoe_ffn_workspace_size(8, 8, 384, 6100, 2048) == -1
    assert mx.mxmoe_ffn_workspace_size(8, 8, 384, 6144, 32768 + 256) == -1
    assert mx.mxmoe_ffn_workspace_size(8, 8, 384, 6144, 2048 + 64) == -1  # I % 128
    assert mx.mxmoe_ffn_workspace_size((1 << 22) // 8 + 1, 8, 384, 6144, 2048) == -1
    # grows with T
    assert mx.mxmoe_workspace_size(256, 6144, 2048, 384, 8) > mx.mxmoe_workspace_size(8, 6144, 2048, 384, 8)
    # the layer's size query refuses exactly what the layer refuses: H and I multiples of 128
    assert mx.mxmoe_workspace_size(8, 192, 2048, 384, 8) == -1
    assert mx.mxmoe_workspace_size(8, 6144, 2048 + 64, 384, 8) == -1
    assert mx.mxmoe_workspace_size(8, 6144, 2048, 2000, 8) == -1  # E above the grouping's 1024
    assert mx.mxmoe_workspace_size(65536, 256, 128, 16, 2) == -1  # T above the combine's 65535
    assert mx.mxmoe_workspace_size(8, 256, 128, 4, 8) == -1  # k > E


def _lib(mx):
    return mx.lib


def test_quantize_rejects_on_host(mx):
    lib = _lib(mx)
    buf = ctypes.create_string_buffer(4096 + 16)
    base = (ctypes.addressof(buf) + 15) & ~15
    assert lib.mxmoe_quantize(base, 4, 33, base, base, None) == mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_quantize(base, 0, 32, base, base, None) == mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_quantize(None, 4, 32, base, base, None) == mx.ERR_NULL
    assert lib.mxmoe_quantize(base + 2, 4, 32, base, base, None) == mx.ERR_ALIGNMENT
    assert "multiple of 32" in mx.last_error() or mx.last_error()


def test_route_and_permute_reject_on_host(mx):
    lib = _lib(mx)
    assert lib.mxmoe_route(None, 4, 16, 0, None, None, None) == mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_route(None, 4, 16, 17, None, None, None) == mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_route(None, 4, 16, 2, None, None, None) == mx.ERR_NULL
    assert lib.mxmoe_route(None, 0, 16, 2, None, None, None) == mx.OK  # empty input is a no-op
    assert lib.mxmoe_permute(None, 4, 2, 5000, None, None, None, None) == mx.ERR_INVALID_SHAPE


def test_ffn_and_layer_reject_on_host(mx):
    lib = _lib(mx)
    assert lib.mxmoe_expert_ffn(None, None, None, None, 8, 8, 384, 6100, 2048, None, None, 0, None) == \
        mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_expert_ffn(None, None, None, None, 8, 8, 384, 6144, 2048, None, None, 0, None) == \
        mx.ERR_WORKSPACE
    need = mx.mxmoe_workspace_size(8, 6144, 2048, 384, 8)
    assert lib.mxmoe_layer_forward(None, None, None, None, 8, 6144, 2048, 384, 8, None, None, None, None, need - 1,
                                   None) == mx.ERR_WORKSPACE
    assert lib.mxmoe_layer_forward(None, None, None, None, 8, 6144, 2048, 384, 8, None, None, None, 256, need,
                                   None) == mx.ERR_NULL
    assert lib.mxmoe_layer_forward(None, None, None, None, 8, 6144, 2048, 384, 9, None, None, None, 256, need,
                                   None) != mx.OK


def test_combine_rejects_on_host(mx):
    lib = _lib(mx)
    assert lib.mxmoe_combine(None, None, None, 4, 2, 6, None, None) == mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_combine(None, None, None, 4, 2, 8, None, None) == mx.ERR_NULL


def test_cpu_only_box_reports_no_device(mx):
    """Without a GPU an otherwise valid call fails with a CUDA or device error,
    never silently succeeds (there is no CPU fallback)."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    lib = _lib(mx)
    buf = ctypes.create_string_buffer(4096 + 16)
    base = (ctypes.addressof(buf) + 15) & ~15
    rc = lib.mxmoe_quantize(base, 4, 32, base, base, None)
    assert rc in (mx.ERR_CUDA, mx.ERR_DEVICE)


def test_timeout_selftest_rejects_on_host(mx):
    lib = mx.load()
    base = 1 << 20  # never dereferenced: rejected before anything is enqueued
    assert lib.mxmoe_selftest_wait_timeout(None, 1000, None) == mx.ERR_NULL
    assert lib.mxmoe_selftest_wait_timeout(base, 0, None) == mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_selftest_wait_timeout(base, 1000001, None) == mx.ERR_INVALID_SHAPE


def test_grouping_expert_limit(mx):
    lib = mx.load()
    # the grouping kernels take up to 1024 experts (34 ints of shared memory each)
    assert lib.mxmoe_permute(None, 4, 2, 2000, None, None, None, None) == mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_permute_scratch_size(4, 2, 1025) == -1
    assert lib.mxmoe_permute_scratch_size(4, 2, 1024) > 0


def test_verify_block_queries_and_rejects_on_host(mx):
    lib = mx.load()
    V = 152064
    ws = lib.mxmoe_verify_workspace_size(32, 8, V)
    # partials of 17 rows x 19 chunks x 16 bytes per block, then per-block draw state and chunk sums
    assert ws >= 32 * 17 * 19 * 16 and ws < 32 * 17 * 19 * 16 + 8192
    assert lib.mxmoe_verify_workspace_size(1, 8, V) < ws
    assert lib.mxmoe_verify_workspace_size(1, 0, V) == -1
    assert lib.mxmoe_verify_workspace_size(1, 33, V) == -1
    assert lib.mxmoe_verify_workspace_size(1, 8, 0) == -1
    assert lib.mxmoe_verify_workspace_size(1, 8, (1 << 24) + 1) == -1
    assert lib.mxmoe_verify_workspace_size(1, 8, 1 << 24) > 0
    base = 1 << 20  # never dereferenced: rejected before anything is enqueued
    big = 1 << 40
    f = lib.mxmoe_verify_block
    assert f(base, base, base, base, 1, 0, V, 1.0, base, base, base, big, None) == mx.ERR_INVALID_SHAPE
    assert f(base, base, base, base, 1, 8, V, -1.0, base, base, base, big, None) == mx.ERR_INVALID_SHAPE
    assert f(base, base, base, base, 1, 8, V, float("inf"), base, base, base, big, None) == mx.ERR_INVALID_SHAPE
    assert f(base, base, base, base, 1, 8, V, float("nan"), base, base, base, big, None) == mx.ERR_INVALID_SHAPE
    # log2(e) / temperature overflows float below about 4e-39 (1e-40 is a float subnormal)
    assert f(base, base, base, base, 1, 8, V, 1e-40, base, base, base, big, None) == mx.ERR_INVALID_SHAPE
    assert "too small" in mx.last_error()
    assert f(base, base, base, base, 1, 8, V, 1.0, base, base, base, 16, None) == mx.ERR_WORKSPACE
    assert f(base, None, base, base, 1, 8, V, 1.0, base, base, base, big, None) == mx.ERR_NULL  # sampling needs q
    assert f(base, base, base, base, 1, 8, V, 1.0, base, base, base + 16, big, None) == mx.ERR_ALIGNMENT
    assert f(None, None, None, None, 0, 8, V, 0.0, None, None, None, 0, None) == mx.OK  # nothing to do


def test_grid_limits_reject_on_host(mx):
    # one grid row per token in the combine, per logit row in the verification's row pass
    lib = mx.load()
    base = 1 << 20  # never dereferenced: rejected before anything is enqueued
    assert lib.mxmoe_combine(base, base, base, 65536, 8, 6144, base, None) == mx.ERR_INVALID_SHAPE
    assert mx.mxmoe_workspace_size(65536, 6144, 2048, 384, 8) == -1
    assert mx.mxmoe_workspace_size(65535, 6144, 2048, 384, 1) > 0
    assert lib.mxmoe_layer_forward(base, base, None, base, 65536, 6144, 2048, 384, 8, base, None, None, base,
                                   1 << 40, None) == mx.ERR_INVALID_SHAPE
    assert lib.mxmoe_verify_workspace_size(3855, 8, 152064) > 0   # 3855 x 17 = 65535 rows
    assert lib.mxmoe_verify_workspace_size(3856, 8, 152064) == -1
    assert lib.mxmoe_verify_block(base, base, base, base, 3856, 8, 152064, 1.0, base, base, base, 1 << 40,
                                  None) == mx.ERR_INVALID_SHAPE

"""The C-ABI library loads, exports every symbol include/*.h declares, and its
host-side validation returns the documented status before touching the GPU."""
import ctypes
import glob
import os
import re

import pytest

from moe_decode_weight_router_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M):
            name = m.group(1)
            if name not in ("if", "return", "sizeof", "defined"):
                names.add(name)
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert {"moe_route", "moe_mxfp4_experts", "lm_head_fp8_quantize", "lm_head_fp8_gemv", "decode_step"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(_abi.SIGNATURES) == declared


def test_status_strings_and_version(lib):
    assert lib.moe_abi_version() == 2
    for code, name in _abi.STATUS_NAMES.items():
        assert lib.moe_status_string(code).decode() == name


A = 0x7f0000001000  # an aligned fake device address: validation must reject before any access


def test_route_validation(lib):
    ok_ws = lib.moe_route_workspace_bytes(1, 512)
    assert ok_ws > 0
    assert lib.moe_route_workspace_bytes(9, 512) == 0
    # NULL input
    assert lib.moe_route(None, 1, 2560, A, 512, 8, A, A, None, A, ok_ws, None) == 1
    # shapes
    assert lib.moe_route(A, 0, 2560, A, 512, 8, A, A, None, A, ok_ws, None) == 2
    assert lib.moe_route(A, 9, 2560, A, 512, 8, A, A, None, A, ok_ws, None) == 2
    assert lib.moe_route(A, 1, 2561, A, 512, 8, A, A, None, A, ok_ws, None) == 2
    assert lib.moe_route(A, 1, 2560, A, 520, 8, A, A, None, A, ok_ws, None) == 2
    assert lib.moe_route(A, 1, 2560, A, 512, 9, A, A, None, A, ok_ws, None) == 2
    assert lib.moe_route(A, 1, 2560, A, 512, 0, A, A, None, A, ok_ws, None) == 2
    # alignment
    assert lib.moe_route(A + 2, 1, 2560, A, 512, 8, A, A, None, A, ok_ws, None) == 3
    assert lib.moe_route(A, 1, 2560, A, 512, 8, A, A, A + 4, A, ok_ws, None) == 3
    # workspace
    assert lib.moe_route(A, 1, 2560, A, 512, 8, A, A, None, A, ok_ws - 1, None) == 4
    assert lib.moe_route(A, 1, 2560, A, 512, 8, A, A, None, None, ok_ws, None) == 4


def test_experts_validation(lib):
    need = lib.moe_experts_workspace_bytes(4, 2560, 768, 512, 8, 768)
    assert need > 0
    args = [A, 4, 2560, 768, 512, 8, A, A, A, A, A, A, A, A, 768, A, A, need, None]
    f = lib.moe_mxfp4_experts

    def call(**kw):
        a = list(args)
        names = ["x", "M", "H", "I", "E", "k", "ids", "w", "w13c", "w13s", "w2c", "w2s", "sw13", "sw2", "Is", "y",
                 "ws", "ws_bytes", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return f(*a)

    assert call(x=None) == 1
    assert call(y=None) == 1
    assert call(sw13=None) == 1          # shared weights must come as a pair with Is > 0
    assert call(Is=0) == 1               # ... and Is = 0 must come without them
    assert call(M=9) == 2
    assert call(I=770) == 2
    assert call(I=2048) == 2
    assert call(Is=40) == 2
    assert call(H=8192) == 2
    assert call(w2s=A + 8) == 3
    assert call(ws_bytes=need - 1) == 4
    # a chunk (M a multiple of 128) takes the block-scaled path under the caller's routing
    chunk = lib.moe_experts_workspace_bytes(2048, 2560, 768, 512, 8, 768)
    # ... and its workspace leaves out the router logits, ids and weights (M*E*4 + 2*M*k*4
    # bytes, each rounded to 256) that only moe_prefill_layer's own routing needs
    own = lib.moe_prefill_workspace_bytes(2048, 2560, 768, 512, 8, 768)
    assert 0 < chunk == own - (2048 * 512 * 4 + 2 * 2048 * 8 * 4)
    assert lib.moe_experts_workspace_bytes(200, 2560, 768, 512, 8, 768) == 0
    assert call(M=200) == 2
    assert call(M=2048, ws_bytes=chunk - 1) == 4
    assert call(M=2048, ws_bytes=chunk, w13c=A + 16) == 3   # 32-byte bases for the 4-bit tensor maps


def test_prefill_validation(lib):
    need = lib.moe_prefill_workspace_bytes(2048, 2560, 768, 512, 8, 768)
    assert need > 0
    assert lib.moe_prefill_workspace_bytes(100, 2560, 768, 512, 8, 768) == 0   # M % 128
    assert lib.moe_prefill_workspace_bytes(2048, 2560, 768, 1024, 8, 768) == 0  # E > 512
    args = [A, 2048, 2560, 768, 512, 8, A, A, A, A, A, A, A, 768, None, None, None, A, A, need, None]
    f = lib.moe_prefill_layer

    def call(**kw):
        a = list(args)
        names = ["x", "M", "H", "I", "E", "k", "wr", "w13c", "w13s", "w2c", "w2s", "sw13", "sw2", "Is", "ids", "w",
                 "logits", "y", "ws", "ws_bytes", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return f(*a)

    assert call(x=None) == 1
    assert call(y=None) == 1
    assert call(sw2=None) == 1           # shared weights are required when Is > 0
    assert call(M=64) == 2
    assert call(H=2600) == 2
    assert call(I=800) == 2
    assert call(E=640) == 2
    assert call(k=9) == 2
    assert call(Is=96) == 2
    assert call(w13c=A + 16) == 3        # the 4-bit tensor-map form needs 32-byte bases
    assert call(y=A + 4) == 3
    assert call(ws_bytes=need - 1) == 4
    q = lib.moe_mxfp8_quantize
    assert q(None, 4, 64, A, A, None) == 1
    assert q(A, 4, 48, A, A, None) == 2
    assert q(A, 4, 64, A + 2, A, None) == 3


def test_lm_head_validation(lib):
    need = lib.lm_head_workspace_bytes(1, 157184, 2560)
    assert need > 0
    f = lib.lm_head_fp8_gemv
    assert f(None, 1, 157184, 2560, A, A, A, A, A, need, None) == 1
    assert f(A, 1, 157184, 2560, A, A, A, None, A, need, None) == 1
    assert f(A, 0, 157184, 2560, A, A, A, A, A, need, None) == 2
    assert f(A, 1, 157184, 2500, A, A, A, A, A, need, None) == 2
    assert f(A, 1, 157184, 2560, A + 1, A, A, A, A, need, None) == 3
    assert f(A, 1, 157184, 2560, A, A, A, A, A, need - 1, None) == 4
    q = lib.lm_head_fp8_quantize
    assert q(None, 10, 64, A, A, None) == 1
    assert q(A, 0, 64, A, A, None) == 2
    assert q(A, 10, 60, A, A, None) == 2
    assert q(A, 10, 64, A + 3, A, None) == 3


def _model(n_layers=2, fmt_override=None, Is=768):
    layers = (_abi.Layer * n_layers)()
    for i in range(n_layers):
        layers[i].router = _abi.Buf(A, _abi.FMT_BF16)
        layers[i].w13_codes = _abi.Buf(A, _abi.FMT_MXFP4_CODES)
        layers[i].w13_scales = _abi.Buf(A, _abi.FMT_E8M0_SCALES)
        layers[i].w2_codes = _abi.Buf(A, _abi.FMT_MXFP4_CODES)
        layers[i].w2_scales = _abi.Buf(A, _abi.FMT_E8M0_SCALES)
        if Is:
            layers[i].shared_w13 = _abi.Buf(A, _abi.FMT_BF16)
            layers[i].shared_w2 = _abi.Buf(A, _abi.FMT_BF16)
    if fmt_override:
        li, field, fmt = fmt_override
        b = getattr(layers[li], field)
        setattr(layers[li], field, _abi.Buf(b.ptr, fmt))
    m = _abi.Model(n_layers, 2560, 768, 512, 8, Is, 157184, 1e-6, ctypes.cast(layers, ctypes.POINTER(_abi.Layer)),
                   _abi.Buf(A, _abi.FMT_E4M3), _abi.Buf(A, _abi.FMT_F32))
    return m, layers


def test_decode_step_rejects_format_mismatch(lib):
    m, keep = _model()
    need = lib.decode_step_workspace_bytes(ctypes.byref(m), 4)
    assert need > 0
    # the silent-fallback class of bug: FP8 LM-head bytes handed over as BF16
    m.lm_head = _abi.Buf(A, _abi.FMT_BF16)
    assert lib.decode_step(ctypes.byref(m), A, 4, A, A, None, A, need, None) == 5
    assert lib.decode_step_workspace_bytes(ctypes.byref(m), 4) == 0
    for field, bad in [("w13_codes", _abi.FMT_E4M3), ("w2_scales", _abi.FMT_MXFP4_CODES), ("router", _abi.FMT_F32),
                       ("shared_w2", _abi.FMT_E4M3)]:
        m2, keep2 = _model(fmt_override=(1, field, bad))
        assert lib.decode_step(ctypes.byref(m2), A, 4, A, A, None, A, need, None) == 5, field


def test_decode_step_other_errors(lib):
    m, keep = _model()
    need = lib.decode_step_workspace_bytes(ctypes.byref(m), 1)
    assert lib.decode_step(ctypes.byref(m), None, 1, A, A, None, A, need, None) == 1
    assert lib.decode_step(ctypes.byref(m), A, 1, A, None, None, A, need, None) == 1
    assert lib.decode_step(ctypes.byref(m), A, 0, A, A, None, A, need, None) == 2
    assert lib.decode_step(ctypes.byref(m), A + 8, 1, A, A, None, A, need, None) == 3
    assert lib.decode_step(ctypes.byref(m), A, 1, A, A, None, A, need - 1, None) == 4
    assert lib.decode_step(None, A, 1, A, A, None, A, need, None) == 1
    m.n_layers = 0
    assert lib.decode_step(ctypes.byref(m), A, 1, A, A, None, A, need, None) == 2
    m3, k3 = _model(Is=0)
    need3 = lib.decode_step_workspace_bytes(ctypes.byref(m3), 1)
    assert 0 < need3 < need
    m4, k4 = _model()
    tr = _abi.Trace(A + 4, None, None, None, None, 0, None)
    assert lib.decode_step(ctypes.byref(m4), A, 1, A, A, ctypes.byref(tr), A, need, None) == 3


def test_graph_create_rejects_null_out(lib):
    m, keep = _model()
    assert lib.decode_step_graph_create(ctypes.byref(m), A, 1, A, A, None, A, 1 << 20, None) == 1
    assert lib.decode_step_graph_launch(None, None) == 1
    lib.decode_step_graph_destroy(None)

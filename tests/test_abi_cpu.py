"""Host-side checks of the C ABI that need no GPU.

The library builds for sm_100a, loads, and exports every function that
``include/bitlinear.h`` declares; argument checks that run before any CUDA
call return the documented status codes; the workspace arithmetic matches
the documented layout.  No call here launches work.
"""
import ctypes
import os
import re

import pytest

import ternary_weight_a8_b200 as tb
from ternary_weight_a8_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return tb.lib()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(bitlinear_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for required in ("bitlinear_pack_weights", "bitlinear_quant_act", "bitlinear_forward",
                     "bitlinear_layer_chain"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_host_side_validation(L):
    vp = ctypes.c_void_p
    assert L.bitlinear_set_path(5) == tb.BL_ERR_INVALID_ARG
    assert "path" in tb.last_error()
    assert L.bitlinear_set_path(0) == tb.BL_OK
    # bad shapes are refused before any pointer is looked at
    assert L.bitlinear_forward(None, None, 0, 256, None, 0, 1, None, 0, None, None, 0, None) == tb.BL_ERR_UNSUPPORTED_SHAPE
    assert L.bitlinear_forward(None, None, 8, 100, None, 0, 1, None, 0, None, None, 0, None) == tb.BL_ERR_UNSUPPORTED_SHAPE
    assert "K = 100" in tb.last_error()
    assert L.bitlinear_forward(None, None, 8, 32, None, 0, 1, None, 0, None, None, 0, None) == tb.BL_ERR_UNSUPPORTED_SHAPE
    assert L.bitlinear_forward(None, None, 8, 256, None, 7, 1, None, 0, None, None, 0, None) == tb.BL_ERR_INVALID_ARG
    assert L.bitlinear_forward(None, None, 8, 256, None, 0, -1, None, 0, None, None, 0, None) == tb.BL_ERR_INVALID_ARG
    assert L.bitlinear_quant_act(None, 3, 1, 256, None, None, None, None) == tb.BL_ERR_INVALID_ARG
    assert L.bitlinear_pack_weights(None, 8, 48, None, None, None, 0, None) == tb.BL_ERR_UNSUPPORTED_SHAPE
    assert L.bitlinear_layer_chain(None, 1, 1, 0, 0, None, 0, None) == tb.BL_ERR_INVALID_ARG
    # empty inputs are a no-op that succeeds without touching memory
    assert L.bitlinear_forward(vp(16), vp(16), 8, 256, vp(16), 0, 0, vp(16), 0, None, vp(256), 0, None) == tb.BL_OK
    assert L.bitlinear_quant_act(vp(16), 0, 0, 256, vp(16), vp(16), None, None) == tb.BL_OK


def test_host_side_validation_of_the_next_rows(L):
    vp, f = ctypes.c_void_p, ctypes.c_float
    # fused norm: K, dtype and eps are checked before any pointer
    assert L.bitlinear_rmsnorm_quant(None, 0, 1, 48, None, f(1e-6), None, None, None, None, None) == tb.BL_ERR_UNSUPPORTED_SHAPE
    assert L.bitlinear_rmsnorm_quant(None, 5, 1, 64, None, f(1e-6), None, None, None, None, None) == tb.BL_ERR_INVALID_ARG
    for eps in (-1.0, float("inf"), float("nan")):
        assert L.bitlinear_rmsnorm_quant(None, 0, 1, 64, None, f(eps), None, None, None, None, None) == tb.BL_ERR_INVALID_ARG
    assert "eps" in tb.last_error()
    assert L.bitlinear_rmsnorm_quant(vp(16), 0, 0, 64, None, f(1e-6), None, vp(16), vp(16), None, None) == tb.BL_OK
    # gated activation: the width is the down BitLinear's K; unknown activations are refused
    assert L.bitlinear_glu_quant(None, None, 0, 1, 96, 0, None, None, None, None, None) == tb.BL_ERR_UNSUPPORTED_SHAPE
    assert L.bitlinear_glu_quant(None, None, 0, 1, 128, 2, None, None, None, None, None) == tb.BL_ERR_INVALID_ARG
    # lookup-table product: one token, K within the tables' shared memory
    assert L.bitlinear_forward_lut(None, None, 8, 256, None, None, None, 2, None, 0, None, None) == tb.BL_ERR_UNSUPPORTED_SHAPE
    assert L.bitlinear_forward_lut(None, None, 8, 24576 + 64, None, None, None, 1, None, 0, None, None) == \
        tb.BL_ERR_UNSUPPORTED_SHAPE
    # straight-through backward: N % 64, M % 8, dtype; nothing to do is a no-op
    assert L.bitlinear_ste_backward(None, None, 96, 64, None, None, None, 8, None, 0, None, None, 0, None) == \
        tb.BL_ERR_UNSUPPORTED_SHAPE
    assert L.bitlinear_ste_backward(None, None, 64, 64, None, None, None, 12, None, 0, None, None, 0, None) == \
        tb.BL_ERR_UNSUPPORTED_SHAPE
    assert L.bitlinear_ste_backward(None, None, 64, 64, None, None, None, 8, None, 9, None, None, 0, None) == \
        tb.BL_ERR_INVALID_ARG
    assert L.bitlinear_ste_backward(None, None, 64, 64, None, None, None, 8, None, 0, None, None, 0, None) == tb.BL_OK
    # its workspace: status block + t^T [K][N] + dy^T [N][M] + xhat^T [K][M] in bf16, each 256-rounded
    assert tb.ste_workspace_bytes(2048, 6912, 2560) == 256 + 2560 * 6912 * 2 + 6912 * 2048 * 2 + 2560 * 2048 * 2
    assert tb.ste_workspace_bytes(8, 64, 64) == 256 + 64 * 64 * 2 + 64 * 8 * 2 + 64 * 8 * 2


def test_workspace_layout(L):
    # status block (256) + q (M rows of K rounded up to 128, 256-rounded) + scale and
    # rowsum (4*M each, 256-rounded)
    assert tb.workspace_bytes(1, 6912, 2560) == 256 + 2560 + 256 + 256
    assert tb.workspace_bytes(2048, 6912, 2560) == 256 + 2048 * 2560 + 8192 + 8192
    assert tb.workspace_bytes(3, 10, 64) == 256 + 512 + 256 + 256
    assert tb.workspace_bytes(2, 10, 8640) == 256 + 2 * 8704 + 256 + 256
    assert tb.pack_workspace_bytes(6912, 2560) == 256 + 6912 * 8
    layers = (tb.bl_layer * 2)()
    layers[0].N, layers[0].K = 10240, 8192
    layers[1].N, layers[1].K = 8192, 28672
    # a chain gives every layer its own q, s, rowsum region (a decode group's layers run together)
    per_layer = lambda K: tb.workspace_bytes(8, 0, K) - 256
    assert L.bitlinear_chain_workspace_bytes(layers, 2, 8) == 256 + per_layer(8192) + per_layer(28672)
    # the fused gate/up call: codes of x, then h (4-byte elements at most), then (1 to 8
    # tokens) its counters: per token a 128-byte line of maxima and one of code sums, 256 more
    # bytes; (9 to 16 tokens) the gate and up outputs
    r = lambda v: (v + 255) // 256 * 256
    assert tb.gate_up_glu_workspace_bytes(8, 28672, 8192) == \
        tb.workspace_bytes(8, 0, 8192) + r(8 * 28672 * 4) + 2 * 16 * 128 + 256
    assert tb.gate_up_glu_workspace_bytes(16, 28672, 8192) == \
        tb.workspace_bytes(16, 0, 8192) + r(16 * 28672 * 4) + r(2 * 16 * 28672 * 4)
    assert tb.gate_up_glu_workspace_bytes(2048, 6912, 2560) == tb.workspace_bytes(2048, 0, 2560) + 2048 * 6912 * 4


def test_decode_split_setting(L):
    for bad in (-1, 9):
        assert L.bitlinear_set_decode_split(bad) == tb.BL_ERR_INVALID_ARG
        assert "ctas" in tb.last_error()
    assert L.bitlinear_set_decode_split(3) == tb.BL_OK
    assert L.bitlinear_set_decode_split(0) == tb.BL_OK


def test_decode_form_setting(L):
    for bad in (-1, 3):
        assert L.bitlinear_set_decode_form(bad) == tb.BL_ERR_INVALID_ARG
    for good in (tb.DECODE_FORM_TENSOR_CORES, tb.DECODE_FORM_CUDA_CORES, tb.DECODE_FORM_AUTO):
        assert L.bitlinear_set_decode_form(good) == tb.BL_OK


def test_chain_layer_struct_matches_the_header():
    text = open(os.path.join(ROOT, "include", "bitlinear.h")).read()
    body = re.search(r"typedef struct \{(.*?)\} bl_layer;", text, flags=re.S).group(1)
    fields = re.findall(r"(\w+);", body)
    assert fields == [f for f, _ in tb.bl_layer._fields_]


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(tb, "_lib", None)
    monkeypatch.setattr(tb, "LIB_PATH", "/nonexistent/libbitlinear.so")
    with pytest.raises(RuntimeError, match="not built"):
        tb.lib()


def test_package_does_not_import_oracle():
    import subprocess
    import sys
    code = "import sys, ternary_weight_a8_b200 as t; t.lib(); print('oracle' in sys.modules)"
    out = subprocess.check_output([sys.executable, "-c", code], cwd=ROOT, text=True).strip()
    assert out == "False"
    src_dir = os.path.join(ROOT, "ternary_weight_a8_b200")
    for dirpath, _, files in os.walk(src_dir):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "bitlinear_oracle" not in text, fn

"""The C-ABI library loads and exports every symbol include/quip.h declares;
host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from conftest import ROOT
from post_weight_quantization_09_b200 import _lib as L
from post_weight_quantization_09_b200.build import build

HEADER = os.path.join(ROOT, "include", "quip.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(quip_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build()
    return L.load()


def test_every_declared_symbol_is_exported_and_bound(lib):
    syms = declared_symbols()
    assert len(syms) >= 14
    for s in syms:
        assert hasattr(lib, s), f"{s} missing from libquip.so"
        assert s in L.SIGNATURES, f"{s} has no binding"
    assert set(L.SIGNATURES) == set(syms)


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.quip_version()
    assert L.status_string(L.QUIP_ERR_NOT_PD).startswith("matrix not positive definite")
    assert L.status_string(99) == "unknown status"


def test_host_argument_errors(lib):
    out = ctypes.c_void_p()
    # bad Hadamard size (not a power of two), bad Kronecker factorisation, null out
    assert lib.quip_transform_create(0, 6, 8, L.QUIP_T_HADAMARD, 0, 0, L.QUIP_T_IDENTITY, 0, 0,
                                     None, ctypes.byref(out)) == L.QUIP_ERR_SHAPE
    assert lib.quip_transform_create(0, 8, 12, L.QUIP_T_IDENTITY, 0, 0, L.QUIP_T_KRONECKER, 3, 5,
                                     None, ctypes.byref(out)) == L.QUIP_ERR_SHAPE
    assert lib.quip_transform_create(0, 8, 8, 7, 0, 0, L.QUIP_T_IDENTITY, 0, 0, None,
                                     ctypes.byref(out)) == L.QUIP_ERR_ARG
    assert lib.quip_transform_create(0, 8, 8, 0, 0, 0, 0, 0, 0, None, None) == L.QUIP_ERR_ARG
    fake = ctypes.c_void_p(0x1000)
    assert lib.quip_hessian_accumulate(None, L.QUIP_BF16, 8, 4, 4, fake, 0, None) == L.QUIP_ERR_ARG
    assert lib.quip_hessian_accumulate(fake, 9, 8, 4, 4, fake, 0, None) == L.QUIP_ERR_ARG
    assert lib.quip_hessian_accumulate(fake, L.QUIP_F32, 8, 4, 2, fake, 0, None) == L.QUIP_ERR_SHAPE
    assert lib.quip_hessian_finalize(fake, 4, 0, 0.01, None) == L.QUIP_ERR_SHAPE
    assert lib.quip_hessian_finalize(fake, 4, 8, -1.0, None) == L.QUIP_ERR_ARG
    assert lib.quip_ldl(None, fake, 4, None, 0, None) == L.QUIP_ERR_ARG
    assert lib.quip_ldl(fake, fake, 0, None, 0, None) == L.QUIP_ERR_SHAPE
    # LDLQ: bad bits, block not dividing n, block unsupported, workspace too small
    args = lambda bits, n, block, ws, wsb: lib.quip_ldlq_quantize(
        fake, fake, n, 4, n, bits, block, fake, fake, fake, ws, wsb, None)
    assert args(0, 64, 32, fake, 1 << 20) == L.QUIP_ERR_ARG
    assert args(9, 64, 32, fake, 1 << 20) == L.QUIP_ERR_ARG
    assert args(2, 96, 64, fake, 1 << 20) == L.QUIP_ERR_SHAPE
    assert args(2, 96, 48, fake, 1 << 20) == L.QUIP_ERR_SHAPE
    assert args(2, 64, 32, fake, 16) == L.QUIP_ERR_WORKSPACE
    assert args(2, 64, 32, ctypes.c_void_p(0x1004), 1 << 20) == L.QUIP_ERR_WORKSPACE
    assert lib.quip_dequantize(None, fake, fake, 2, 2, fake, None) == L.QUIP_ERR_ARG
    # the other rounding methods
    assert lib.quip_nearest_quantize(fake, 4, 8, 0, fake, fake, fake, None) == L.QUIP_ERR_ARG
    assert lib.quip_nearest_quantize(None, 4, 8, 2, fake, fake, fake, None) == L.QUIP_ERR_ARG
    assert lib.quip_nearest_quantize(fake, 0, 8, 2, fake, fake, fake, None) == L.QUIP_ERR_SHAPE
    assert lib.quip_diag_order(fake, 8, 8, None, None, None) == L.QUIP_ERR_ARG
    assert lib.quip_diag_order(fake, 4, 8, fake, None, None) == L.QUIP_ERR_SHAPE
    assert lib.quip_diag_order(fake, 70000, 70000, fake, None, None) == L.QUIP_ERR_SHAPE
    other = ctypes.c_void_p(0x100000)
    assert lib.quip_permute(fake, 7, 4, 4, 4, None, None, other, 4, None) == L.QUIP_ERR_ARG
    assert lib.quip_permute(fake, L.QUIP_F32, 4, 4, 4, None, None, fake, 4, None) == L.QUIP_ERR_ARG  # overlap
    assert lib.quip_permute(fake, L.QUIP_U8, 4, 4, 3, None, None, other, 4, None) == L.QUIP_ERR_SHAPE
    g = lambda W, m, n, bits, passes, ws, wsb: lib.quip_greedy_refine(
        W, fake, n, m, n, bits, fake, fake, fake, passes, ws, wsb, None)
    assert g(fake, 4, 64, 0, 1, fake, 1 << 30) == L.QUIP_ERR_ARG
    assert g(fake, 4, 64, 2, -1, fake, 1 << 30) == L.QUIP_ERR_ARG
    assert g(fake, 4, 96, 2, 1, fake, 1 << 30) == L.QUIP_ERR_SHAPE
    assert g(ctypes.c_void_p(0x1004), 4, 64, 2, 1, fake, 1 << 30) == L.QUIP_ERR_ARG
    assert g(fake, 4, 64, 2, 1, fake, 16) == L.QUIP_ERR_WORKSPACE
    assert g(fake, 4, 64, 2, 0, fake, 1 << 30) == L.QUIP_OK          # no pass: nothing launched
    # packing and the quantized product
    assert lib.quip_packed_words(4096, 2) == 256 and lib.quip_packed_words(5, 3) == 4
    assert lib.quip_packed_words(0, 2) == 0 and lib.quip_packed_words(8, 9) == 0
    assert lib.quip_pack_codes(fake, 4, 8, 9, fake, 4, None) == L.QUIP_ERR_ARG
    assert lib.quip_pack_codes(fake, 4, 64, 2, fake, 2, None) == L.QUIP_ERR_SHAPE      # ldp < 4
    assert lib.quip_pack_codes(fake, 4, 64, 2, ctypes.c_void_p(0x1004), 4, None) == L.QUIP_ERR_SHAPE
    assert lib.quip_qmatvec(None, fake, 4, fake, fake, 2, fake, L.QUIP_F32, 8, 1, fake, 8, fake, 1 << 20,
                            None) == L.QUIP_ERR_ARG


def test_layer_calls_reject_a_missing_transform(lib):
    # a transform cannot be made without a device; a null one is refused
    # before any argument is read
    fake = ctypes.c_void_p(0x1000)
    nb = ctypes.c_size_t(7)
    assert lib.quip_layer_workspace_size(None, 64, L.QUIP_BF16, L.QUIP_BF16, 32, 0,
                                         ctypes.byref(nb)) == L.QUIP_ERR_ARG
    rest = (0, fake, L.QUIP_BF16, 128, fake, L.QUIP_BF16, 64, 128, 2, 32, 0.01, fake, fake, fake,
            None, fake, 1 << 20, None)
    assert lib.quip_quantize_layer(None, *rest) == L.QUIP_ERR_ARG
    assert lib.quip_quantize_layer_host(None, *rest) == L.QUIP_ERR_ARG


def test_timing_calls_answer_on_the_host(lib):
    # no launches recorded: begin, trace and end report nothing, on any host
    assert lib.quip_timing_begin() == L.QUIP_OK
    n = ctypes.c_int(-1)
    assert lib.quip_timing_trace(None, None, None, None, 0, ctypes.byref(n)) == L.QUIP_OK
    assert n.value == 0
    n.value = -1
    assert lib.quip_timing_end(None, None, None, 0, ctypes.byref(n)) == L.QUIP_OK
    assert n.value == 0


def test_workspace_sizes(lib):
    nb = ctypes.c_size_t()
    assert lib.quip_workspace_size(L.QUIP_OP_LDLQ, None, 64, 128, 32, ctypes.byref(nb)) == 0
    assert nb.value >= (64 * 128 + 64 * 32) * 4 and nb.value % 256 == 0
    assert lib.quip_workspace_size(L.QUIP_OP_LDL, None, 64, 128, 0, ctypes.byref(nb)) == 0
    ldlq = ctypes.c_size_t()
    lib.quip_workspace_size(L.QUIP_OP_LDLQ, None, 64, 128, 128, ctypes.byref(ldlq))
    assert lib.quip_workspace_size(L.QUIP_OP_GREEDY, None, 64, 128, 0, ctypes.byref(nb)) == 0
    assert nb.value >= ldlq.value + (128 * 128 + 64 * 128) * 4 and nb.value % 256 == 0
    assert lib.quip_workspace_size(99, None, 1, 1, 1, ctypes.byref(nb)) == L.QUIP_ERR_ARG
    assert lib.quip_workspace_size(L.QUIP_OP_INCOHERENCE_FORWARD, None, 1, 1, 1,
                                   ctypes.byref(nb)) == L.QUIP_ERR_ARG


def test_package_refuses_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="libquip.so not found"):
        L._lib, saved = None, L._lib
        try:
            L.load(str(tmp_path / "missing.so"))
        finally:
            L._lib = saved

"""The C-ABI library loads, exports every symbol the header declares, and
validates arguments before touching the GPU (CPU only: no compute call is
made; every call below fails validation before any CUDA work)."""

import ctypes
import os
import re

import pytest

from compressed_sparse_long_compress_b200 import cslc

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "cslc.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


def test_header_declares_the_expected_entry_points():
    assert declared_functions() == sorted(cslc.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(cslc.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version():
    assert cslc.abi_version() == 1


def _err(st):
    return st, cslc.LIB.cslc_last_error().decode()


def test_validation_unsupported_dims():
    st, msg = _err(cslc.LIB.csa_compress(None, None, None, None, None, 1, 64, 96, 4, None, None))
    assert st == 4 and "D must be 128 or 64" in msg
    st, msg = _err(cslc.LIB.csa_compress(None, None, None, None, None, 1, 64, 128, 3, None, None))
    assert st == 4 and "power of two" in msg
    st, _ = _err(cslc.LIB.hca_dense_attn(None, None, 1, 8, 24, 128, 4, 128, 0, 0.1, None, None, None))
    assert st == 4
    st, _ = _err(cslc.LIB.csa_indexer_topk(None, None, None, 1, 8, 4, 4, 32, 4, 0, 16, None, None, None, 0, None))
    assert st == 4   # d_I != 64
    st, _ = _err(cslc.LIB.csa_topk(None, 1, 8, 4, 4, 0, 4096, None, None))
    assert st == 4   # topk > 2048


def test_validation_null_and_alignment():
    st, msg = _err(cslc.LIB.csa_compress(None, None, None, None, None, 1, 64, 128, 4, None, None))
    assert st == 1 and "NULL" in msg
    odd = ctypes.c_void_p(0x1008)   # never dereferenced: alignment is checked first
    st, msg = _err(cslc.LIB.hca_compress(odd, odd, odd, 1, 256, 128, 128, odd, None))
    assert st == 3 and "aligned" in msg
    st, _ = _err(cslc.LIB.csa_compress(ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000),
                                       None, ctypes.c_void_p(0x1000), 1, 64, 128, 4, ctypes.c_void_p(0x1000), None))
    assert st == 1   # c_b without z_b


def test_validation_shapes_and_workspace():
    st, _ = _err(cslc.LIB.csa_compress(None, None, None, None, None, -1, 64, 128, 4, None, None))
    assert st == 2
    # empty work returns OK without touching anything
    assert cslc.LIB.csa_compress(None, None, None, None, None, 1, 3, 128, 4, None, None) == 0
    assert cslc.LIB.hca_dense_attn(None, None, 0, 8, 16, 128, 4, 128, 0, 0.1, None, None, None) == 0
    # workspace: the blocked scores path needs one; none is given
    p = ctypes.c_void_p(0x1000)
    need = cslc.LIB.csa_indexer_topk_workspace_bytes(1, 4096, 1024, 4, 128, 0)
    assert need > 0 and cslc.LIB.csa_indexer_topk_workspace_bytes(1, 4096, 1024, 4, 128, 1) == 0
    st, msg = _err(cslc.LIB.csa_indexer_topk(p, p, p, 1, 4096, 1024, 4, 64, 4, 0, 128, None, p, None, 0, None))
    assert st == 5 and "workspace" in msg


def test_decode_validation():
    L = cslc.DecodeLayerC()
    L.kind = 3
    arr = (cslc.DecodeLayerC * 1)(L)
    st, _ = _err(cslc.LIB.cslc_decode_step(arr, 1, 2, 64, 128, 8, 64, None, 0, None))
    assert st == 4
    st, _ = _err(cslc.LIB.cslc_decode_step(arr, 1, 2, 60, 128, 8, 64, None, 0, None))
    assert st == 4   # H not a multiple of 16
    assert cslc.LIB.cslc_decode_topk_workspace_bytes(8, 262144, 1024) > 8 * 262144 * 8


def test_validation_decode_append():
    P = None
    # key arguments must be all given or all NULL
    st, msg = _err(cslc.LIB.cslc_decode_append(P, P, 16, P, P, P, P, 1, 4, 1, P, P, P, P, P, P, P, P, 8, P, P))
    assert st == 1 and "k_c" in msg
    st, msg = _err(cslc.LIB.cslc_decode_append(P, P, P, P, P, P, P, 1, 3, 1, P, P, P, P, P, P, P, P, 8, P, P))
    assert st == 4 and "power of two" in msg
    st, _ = _err(cslc.LIB.cslc_decode_append(P, P, P, P, P, P, P, 1, 4, 2, P, P, P, P, P, P, P, P, 8, P, P))
    assert st == 4
    st, _ = _err(cslc.LIB.cslc_decode_append(P, P, P, P, P, P, P, 2, 4, 1, P, P, P, P, P, P, P, P, 8, P, P))
    assert st == 1   # c is NULL
    assert cslc.LIB.cslc_decode_append(P, P, P, P, P, P, P, 0, 4, 1, P, P, P, P, P, P, P, P, 8, P, P) == 0


def test_fp8_entry_points_validation():
    p = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1004)
    # the row quantiser takes rows of 64 values only
    st, msg = _err(cslc.LIB.cslc_quantize_rows_e4m3(p, 10, 128, p, p, None))
    assert st == 4 and "d must be 64" in msg
    st, _ = _err(cslc.LIB.cslc_quantize_rows_e4m3(p, -1, 64, p, p, None))
    assert st == 2
    assert cslc.LIB.cslc_quantize_rows_e4m3(None, 0, 64, None, None, None) == 0   # nothing to do
    st, msg = _err(cslc.LIB.cslc_quantize_rows_e4m3(p, 10, 64, p, odd, None))
    assert st == 3 and "scales" in msg
    # FP8 indexer: scales are required, H_I in [1, 16], d_I = 64, workspace as the fp32 path
    args = lambda qs, ks, HI, dI, ws, nbytes: (p, qs, p, p, ks, 1, 4096, 1024, HI, dI, 4, 0, 128, None, p, ws,
                                                 nbytes, None)
    st, msg = _err(cslc.LIB.csa_indexer_topk_fp8(*args(None, p, 8, 64, None, 0)))
    assert st == 1 and "q_scale" in msg
    st, msg = _err(cslc.LIB.csa_indexer_topk_fp8(*args(p, None, 8, 64, None, 0)))
    assert st == 1 and "k_scale" in msg
    st, _ = _err(cslc.LIB.csa_indexer_topk_fp8(*args(p, p, 17, 64, None, 0)))
    assert st == 4
    st, _ = _err(cslc.LIB.csa_indexer_topk_fp8(*args(p, p, 8, 32, None, 0)))
    assert st == 4
    st, msg = _err(cslc.LIB.csa_indexer_topk_fp8(*args(p, p, 6, 64, None, 0)))
    assert st == 5 and "workspace" in msg   # H_I = 6 is accepted; only the workspace is missing

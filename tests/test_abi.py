"""The C-ABI library loads and exports every symbol include/qjl.h declares.

These run without a GPU. The calls here either touch no device at all (status
strings, defaults, workspace sizing) or fail argument checks on the host
before any CUDA call.
"""

import ctypes

import pytest

from bit_kv_cache_qjl_b200 import _lib
from bit_kv_cache_qjl_b200._lib import Options


@pytest.fixture(scope="module")
def L():
    return _lib.lib()


def test_exports_every_declared_function(L):
    names = _lib.header_functions()
    assert len(names) >= 14
    for name in names:
        assert hasattr(L, name), name
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_status_strings_and_version(L):
    assert L.qjl_status_string(0) == b"ok"
    assert L.qjl_status_string(-1) == b"invalid argument"
    assert L.qjl_status_string(-5) == b"workspace too small"
    assert b"sm_100a" in L.qjl_version()


def test_default_options(L):
    o = Options()
    L.qjl_default_options(ctypes.byref(o))
    assert abs(o.dither_sigma_rel - 0.5) < 1e-7 and o.dg_outer == 0 and o.s_bf16 == 1


@pytest.mark.parametrize("d,m,kind", [(128, 0, 0), (128, 48, 0), (0, 256, 0), (100, 256, 1),
                                      (128, 192, 2), (16, 32, 1), (2048, 2048, 2), (128, 256, 7)])
def test_make_projection_rejects_bad_shapes_on_host(L, d, m, kind):
    h = ctypes.c_void_p()
    st = L.qjl_make_projection(1, d, m, kind, None, ctypes.byref(h))
    assert st == -1
    assert not h.value
    assert len(L.qjl_last_error_message()) > 0


def test_null_projection_is_rejected(L):
    z = ctypes.c_void_p(0)
    assert L.qjl_quantize_keys(None, z, 1, 10, 128, 0, z, z, None) == -1
    assert L.qjl_project_queries(None, z, 1, 128, z, None) == -1
    assert L.qjl_scores(None, z, z, 1, 1, z, 1, z, None) == -1
    assert L.qjl_decode_attention(None, z, z, z, z, z, 1, 1, z, 1, 1.0, z, z, 0, None) == -1
    assert L.qjl_destroy_projection(None) == 0


def test_values_argument_checks(L):
    z = ctypes.c_void_p(0)
    assert L.qjl_quantize_values_2bit(z, 1, 4, 48, z, z, z, None) == -1      # d not a multiple of 32
    assert L.qjl_quantize_values_2bit(z, 5, 4, 128, z, z, z, None) == -1     # unknown dtype
    assert L.qjl_quantize_values_2bit(z, 1, 0, 128, z, z, z, None) == 0      # n = 0 is a no-op
    assert L.qjl_quantize_values_2bit(z, 1, 4, 128, z, z, z, None) == -1     # NULL pointers
    bad = ctypes.c_void_p(8)                                                  # misaligned
    assert L.qjl_quantize_values_2bit(bad, 1, 4, 128, bad, bad, bad, None) == -1


def test_workspace_sizing(L):
    assert L.qjl_decode_workspace_bytes(0, 1, 10, 128) == 0
    assert L.qjl_decode_workspace_bytes(4, 65, 10, 128) == 0
    b1 = L.qjl_decode_workspace_bytes(1024, 1, 16384, 128)
    b2 = L.qjl_decode_workspace_bytes(1024, 2, 16384, 128)
    # one query per group: partial slots of d + 2 floats for the persistent CTAs
    assert b1 > 0 and b1 % (130 * 4) == 0
    # 2-4 queries per group: groups x splits x queries slots of d + 2 floats
    assert b2 > 0 and b2 % (2 * 130 * 4) == 0
    assert L.qjl_decode_workspace_bytes(1024, 4, 16384, 128) == 2 * b2

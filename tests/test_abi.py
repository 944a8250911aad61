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


def test_kivi_key_argument_checks(L):
    z = ctypes.c_void_p(0)
    bad = ctypes.c_void_p(8)                                                  # misaligned
    q = L.qjl_kivi_quantize_keys_2bit
    assert q(z, 5, 2, 64, 128, z, z, z, None) == -1                           # unknown dtype
    assert q(z, 1, -1, 64, 128, z, z, z, None) == -1                          # negative groups
    assert q(z, 1, 2, 64, 96, z, z, z, None) == -2                            # d outside {64, 128, 256}
    assert q(z, 1, 0, 64, 128, z, z, z, None) == 0                            # no groups: a no-op
    assert q(z, 1, 2, 0, 128, z, z, z, None) == 0                             # no tokens: a no-op
    assert q(z, 1, 2, 64, 128, z, z, z, None) == -1                           # NULL pointers
    assert q(bad, 1, 2, 64, 128, bad, bad, bad, None) == -1
    assert b"aligned" in L.qjl_last_error_message()
    s = L.qjl_kivi_key_scores
    assert s(z, z, z, 2, 64, 128, z, 0, z, None) == -1                        # q_per_group < 1
    assert s(z, z, z, 2, 64, 128, z, 65, z, None) == -1                       # q_per_group > 64
    assert s(z, z, z, 2, 64, 32, z, 1, z, None) == -2                         # unsupported d
    assert s(z, z, z, 0, 64, 128, z, 1, z, None) == 0                         # no groups: a no-op
    assert s(z, z, z, 2, 64, 128, z, 1, z, None) == -1                        # NULL pointers
    assert s(bad, z, z, 2, 64, 128, z, 1, z, None) == -1


def test_paged_and_prefill_calls_reject_a_null_projection(L):
    z = ctypes.c_void_p(0)
    assert L.qjl_append_keys(None, z, 1, 1, 128, z, z, 1, 16, 1, z, z, None) == -1
    assert L.qjl_scores_paged(None, z, z, z, 1, 16, 1, z, 1, 16, z, 1, z, None) == -1
    assert L.qjl_decode_attention_paged(None, z, z, z, z, z, z, 1, 16, 1, z, 1, 16, z, 1.0, z, z, 0, None) == -1
    assert L.qjl_prefill_attention(None, z, z, z, z, z, 1, 16, z, 1.0, z, None) == -1
    assert b"NULL" in L.qjl_last_error_message() or b"projection" in L.qjl_last_error_message()


def test_only_projection_upload_allocates_device_memory():
    """The library's one device allocation site is the projection's parameter upload.

    Every other call works on caller-owned buffers, the fixed no-alloc scratch and
    the static error int. A new cudaMalloc (or an allocating runtime call) anywhere
    else in the sources fails this check.
    """
    import glob
    import os
    import re
    csrc = os.path.join(os.path.dirname(_lib.__file__), "csrc")
    sites = []
    for path in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.h*"))):
        for i, line in enumerate(open(path), 1):
            code = line.split("//")[0]
            if re.search(r"\bcuda(Malloc\w*|MallocAsync|MallocManaged|HostAlloc)\s*\(", code):
                sites.append((os.path.basename(path), i))
    assert len(sites) == 1 and sites[0][0] == "qjl_api.cu", sites

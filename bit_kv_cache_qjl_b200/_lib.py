"""ctypes loader for libqjl_b200.so: C-ABI signatures only, no computation."""

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqjl_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "qjl.h")

_lib = None

c_void_p, c_int, c_int64, c_uint64, c_size_t, c_float = (
    ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_float)


class Options(ctypes.Structure):
    _fields_ = [("dither_sigma_rel", ctypes.c_float), ("dg_outer", ctypes.c_int), ("s_bf16", ctypes.c_int)]


SIGNATURES = {
    "qjl_default_options": (None, [ctypes.POINTER(Options)]),
    "qjl_make_projection": (c_int, [c_uint64, c_int, c_int, c_int, ctypes.POINTER(Options), ctypes.POINTER(c_void_p)]),
    "qjl_destroy_projection": (c_int, [c_void_p]),
    "qjl_projection_info": (c_int, [c_void_p, ctypes.POINTER(c_int), ctypes.POINTER(c_int), ctypes.POINTER(c_int),
                                    ctypes.POINTER(c_float)]),
    "qjl_projection_export": (c_int, [c_void_p, c_int, c_void_p, c_size_t]),
    "qjl_quantize_keys": (c_int, [c_void_p, c_void_p, c_int, c_int64, c_int64, c_uint64, c_void_p, c_void_p, c_void_p]),
    "qjl_project_queries": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_void_p]),
    "qjl_scores": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_int, c_void_p, c_void_p]),
    "qjl_quantize_values_2bit": (c_int, [c_void_p, c_int, c_int64, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "qjl_decode_workspace_bytes": (c_size_t, [c_int64, c_int, c_int64, c_int]),
    "qjl_decode_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64,
                                     c_void_p, c_int, c_float, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qjl_decode_attention_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64,
                                             c_int64, c_void_p, c_int, c_float, c_void_p, c_void_p]),
    "qjl_append_keys": (c_int, [c_void_p, c_void_p, c_int, c_int64, c_int64, c_void_p, c_void_p, c_int, c_int, c_int64,
                                c_void_p, c_void_p, c_void_p]),
    "qjl_append_values_2bit": (c_int, [c_void_p, c_int, c_int64, c_int, c_void_p, c_void_p, c_int, c_int, c_int64,
                                       c_void_p, c_void_p, c_void_p, c_void_p]),
    "qjl_scores_paged": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int64, c_void_p, c_int64,
                                 c_int64, c_void_p, c_int, c_void_p, c_void_p]),
    "qjl_decode_paged_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int]),
    "qjl_decode_attention_paged": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                           c_int, c_int64, c_void_p, c_int64, c_int64, c_void_p, c_float, c_void_p,
                                           c_void_p, c_size_t, c_void_p]),
    "qjl_kivi_quantize_keys_2bit": (c_int, [c_void_p, c_int, c_int64, c_int64, c_int, c_void_p, c_void_p, c_void_p,
                                            c_void_p]),
    "qjl_kivi_key_scores": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int, c_void_p, c_int, c_void_p,
                                    c_void_p]),
    "qjl_device_errors": (c_int, [c_int, c_int, ctypes.POINTER(c_int)]),
    "qjl_selftest_bounded_wait": (c_int, [c_int, c_uint64]),
    "qjl_prefill_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64,
                                      c_void_p, c_float, c_void_p, c_void_p]),
    "qjl_status_string": (ctypes.c_char_p, [c_int]),
    "qjl_last_error_message": (ctypes.c_char_p, []),
    "qjl_version": (ctypes.c_char_p, []),
}


def header_functions():
    """Names of the functions include/qjl.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qjl_[a-z0-9_]+)\s*\(", text)))


def lib():
    """The loaded library. Raises if it has not been built: there is no fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libqjl_b200.so is missing; build it with `python -m bit_kv_cache_qjl_b200.build` "
                               "(the CUDA library is the only implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib

"""qjl_decode_attention_noalloc matches qjl_decode_attention.

The no-alloc entry point serves callers that may not allocate device memory
while decoding: an engine whose pool owns the whole GPU, or a latency-bound
loop that cannot take cudaMalloc's device-wide synchronisation. It takes its
split-N workspace from a fixed device array. This test calls both entry
points through the C ABI on the same inputs, twice in a row with different
inputs and sizes, so the second call runs on scratch that still holds the
first call's contents. Outputs must agree within the decode tolerance of the
other tests: 1e-3 * sum_n p_n |v_hat| + 1e-6, here against the workspace
entry point's output, computed from that same bound. Oversized requests must
be refused.

The file name sorts last, so a run that stops at the first failure has
already run every other test.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import bit_kv_cache_qjl_b200 as qjl
from bit_kv_cache_qjl_b200 import lib
from bit_kv_cache_qjl_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(P, G, N, J, seed):
    d, m = P.d, P.m
    keys = wl.normal((G * N, d), seed, "cuda", torch.bfloat16)
    vals = wl.normal((G * N, d), seed + 1, "cuda", torch.bfloat16)
    q = wl.normal((G * J, d), seed + 2, "cuda")
    bits, norms = qjl.quantize_keys(P, keys)
    codes, sc, zr = qjl.quantize_values_2bit(vals)
    sq = qjl.project_queries(P, q)
    return (bits.view(G, N, m // 32), norms.view(G, N), codes.view(G, N, d // 16), sc.view(G, N, d // 32),
            zr.view(G, N, d // 32), sq.view(G, J, m))


def _with_ws(P, inp, G, N, J, smx):
    bits, norms, codes, sc, zr, sq = inp
    out = torch.empty((G, J, P.d), dtype=torch.float32, device="cuda")
    need = lib().qjl_decode_workspace_bytes(G, J, N, P.d)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    st = lib().qjl_decode_attention(P.handle, _p(bits), _p(norms), _p(codes), _p(sc), _p(zr), G, N, _p(sq), J, smx,
                                    _p(out), _p(ws), need, None)
    assert st == 0, lib().qjl_last_error_message()
    return out


def _noalloc(P, inp, G, N, J, smx):
    bits, norms, codes, sc, zr, sq = inp
    out = torch.empty((G, J, P.d), dtype=torch.float32, device="cuda")
    st = lib().qjl_decode_attention_noalloc(P.handle, _p(bits), _p(norms), _p(codes), _p(sc), _p(zr), G, N, _p(sq),
                                            J, smx, _p(out), None)
    assert st == 0, lib().qjl_last_error_message()
    return out, st


def test_noalloc_matches_workspace_entry_two_calls(cuda_ok):
    P = qjl.Projection(5, 128, 256, "dfqjl")
    smx = 1.0 / math.sqrt(128)
    for (G, N, J, seed) in [(64, 4096, 1, 900), (24, 5000, 3, 901)]:
        inp = _inputs(P, G, N, J, seed)
        ref = _with_ws(P, inp, G, N, J, smx)
        got, _ = _noalloc(P, inp, G, N, J, smx)
        torch.cuda.synchronize()
        # decode tolerance of the other tests, with sum p |v_hat| bounded by max |v_hat|
        _, sc, zr = inp[2], inp[3], inp[4]
        vmax = (zr.float().abs() + 3 * sc.float().abs()).amax().item()
        tol = 1e-3 * vmax + 1e-6
        err = (got - ref).abs().max().item()
        assert err <= tol, (G, N, J, err, tol)


def test_noalloc_rejects_oversized_workspace(cuda_ok):
    P = qjl.Projection(5, 256, 256, "dense")
    G, J, N = 4096, 4, 1 << 16
    need = lib().qjl_decode_workspace_bytes(G, J, N, 256)
    assert need > (4 << 20)
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    st = lib().qjl_decode_attention_noalloc(P.handle, _p(z), _p(z), _p(z), _p(z), _p(z), G, N, _p(z), J, 1.0, _p(z),
                                            None)
    assert st == -5
    assert b"exceeds" in lib().qjl_last_error_message()

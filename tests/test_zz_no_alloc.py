"""qjl_decode_attention_noalloc against qjl_decode_attention and the oracle.

The no-alloc entry point serves callers that may not allocate device memory
while decoding: an engine whose pool owns the whole GPU, or a latency-bound
loop that cannot take cudaMalloc's device-wide synchronisation. It takes its
split-N workspace from a fixed device array, and the kernels' error int is
static device storage too.

Both entry points run the same kernels with the same split plan and a
fixed-order combine, so their outputs must be bit-identical: the tests assert
torch.equal. Each output is also held to the oracle under the fused-decode
bound of the other tests, |gpu - oracle| <= 1e-3 * sum_n p_n |v_hat| + 1e-6.
Calls come in a row on the shared array, a larger one before a smaller one
with the same queries per group, so later calls run on scratch that still
holds more of an earlier call's data than they write.

One test runs in a fresh process: the no-alloc call is the first compute call
of the library there, and every device allocation the library would make
after the projection's is made to fail on the host (QJL_FAIL_ALLOC_AFTER).
The call must still succeed.

The file name sorts last, so a run that stops at the first failure has
already run every other test.
"""

import ctypes
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import bit_kv_cache_qjl_b200 as qjl
from bit_kv_cache_qjl_b200 import lib
from helpers import host, oracle_projection

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _oracle_case(P, O, G, N, J, seed):
    """The oracle's bits, norms and 2-bit values, fp32 Sq, and the expected output with its bound."""
    d, m = P.d, P.m
    rng = np.random.default_rng(seed)
    keys = rng.standard_normal((G * N, d)).astype(np.float32)
    vals = rng.standard_normal((G * N, d)).astype(np.float32)
    vals = (vals.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    words, norms, _ = oracle.qjl.quantize_keys(O, keys)
    codes, sc, zr = oracle.kivi.quantize_values_2bit(vals)
    q = rng.standard_normal((G * J, d)).astype(np.float32)
    sq = oracle.qjl.project_queries(O, q).astype(np.float32).reshape(G, J, m)
    norms32 = norms.astype(np.float32).reshape(G, N)
    est = oracle.qjl.scores(O, words.reshape(G, N, m // 32), norms32.astype(np.float64), sq.astype(np.float64))
    vhat = oracle.kivi.dequantize_values(codes, sc, zr, d).reshape(G, N, d)
    smx = 1.0 / math.sqrt(d)
    want = oracle.attention.decode_attention(est, vhat, smx)
    bound = 1e-3 * np.einsum("gjn,gnd->gjd", oracle.attention.softmax(est * smx), np.abs(vhat)) + 1e-6

    def t(a, dt=None):
        return torch.from_numpy(np.ascontiguousarray(a if dt is None else a.view(dt))).cuda()

    inp = (t(words.reshape(G, N, m // 32), np.int32), t(norms32), t(codes.reshape(G, N, d // 16), np.int32),
           t(sc.reshape(G, N, d // 32)), t(zr.reshape(G, N, d // 32)), t(sq))
    return inp, smx, want, bound


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
    out = torch.full((G, J, P.d), float("nan"), dtype=torch.float32, device="cuda")
    st = lib().qjl_decode_attention_noalloc(P.handle, _p(bits), _p(norms), _p(codes), _p(sc), _p(zr), G, N, _p(sq),
                                            J, smx, _p(out), None)
    assert st == 0, lib().qjl_last_error_message()
    return out


def test_noalloc_matches_workspace_entry_calls_in_a_row(cuda_ok):
    P = qjl.Projection(5, 128, 256, "dfqjl")
    O = oracle_projection(P)
    # a larger call, then a smaller one with the same J on the same scratch, then 2-4 queries per group
    for (G, N, J, seed) in [(32, 4096, 1, 900), (6, 3001, 1, 901), (16, 2500, 3, 902), (4, 700, 3, 903)]:
        inp, smx, want, bound = _oracle_case(P, O, G, N, J, seed)
        ref = _with_ws(P, inp, G, N, J, smx)
        got = _noalloc(P, inp, G, N, J, smx)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (G, N, J, (got - ref).abs().max().item())
        err = np.abs(host(got) - want)
        assert np.all(err <= bound), (G, N, J, (err / bound).max())


_FRESH = r"""
import ctypes, math, sys, torch
sys.path.insert(0, sys.argv[1])
import bit_kv_cache_qjl_b200 as qjl
from bit_kv_cache_qjl_b200 import lib
torch.cuda.init()
P = qjl.Projection(5, 128, 256, "dfqjl")       # its five parameter uploads are the only ones allowed
G, N, J, d, m = 8, 1500, 1, 128, 256
g = torch.Generator(device="cuda").manual_seed(77)
bits = torch.randint(-2**31, 2**31 - 1, (G, N, m // 32), dtype=torch.int32, device="cuda", generator=g)
norms = torch.rand((G, N), device="cuda", generator=g) + 0.5
codes = torch.randint(-2**31, 2**31 - 1, (G, N, d // 16), dtype=torch.int32, device="cuda", generator=g)
sc = (torch.rand((G, N, d // 32), device="cuda", generator=g) * 0.5).half()
zr = (torch.rand((G, N, d // 32), device="cuda", generator=g) - 1.0).half()
sq = torch.randn((G, J, m), device="cuda", generator=g)
torch.cuda.synchronize()
p = lambda t: ctypes.c_void_p(t.data_ptr())
out = torch.full((G, J, d), float("nan"), device="cuda")
st = lib().qjl_decode_attention_noalloc(P.handle, p(bits), p(norms), p(codes), p(sc), p(zr), G, N, p(sq), J,
                                        1 / math.sqrt(d), p(out), None)
assert st == 0, (st, lib().qjl_last_error_message())
need = lib().qjl_decode_workspace_bytes(G, J, N, d)
ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
ref = torch.empty_like(out)
st = lib().qjl_decode_attention(P.handle, p(bits), p(norms), p(codes), p(sc), p(zr), G, N, p(sq), J,
                                1 / math.sqrt(d), p(ref), p(ws), need, None)
assert st == 0, (st, lib().qjl_last_error_message())
torch.cuda.synchronize()
assert torch.isfinite(out).all() and torch.equal(out, ref)
# the injection is live: a second projection's uploads are refused
h = ctypes.c_void_p()
assert lib().qjl_make_projection(6, 128, 256, 1, None, ctypes.byref(h)) == -4
print("fresh-process no-alloc ok")
"""


def test_noalloc_first_call_in_fresh_process_with_allocations_refused(cuda_ok):
    env = dict(os.environ, QJL_FAIL_ALLOC_AFTER="5")
    r = subprocess.run([sys.executable, "-c", _FRESH, ROOT], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert "fresh-process no-alloc ok" in r.stdout


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


def test_noalloc_range_checks_come_before_the_size_check(cuda_ok):
    P = qjl.Projection(5, 128, 256, "dense")
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    f = lib().qjl_decode_attention_noalloc
    assert f(P.handle, _p(z), _p(z), _p(z), _p(z), _p(z), (1 << 24) + 1, 16, _p(z), 1, 1.0, _p(z), None) == -1
    assert f(P.handle, _p(z), _p(z), _p(z), _p(z), _p(z), 1, (1 << 36) + 1, _p(z), 1, 1.0, _p(z), None) == -1
    assert f(P.handle, _p(z), _p(z), _p(z), _p(z), _p(z), 1, 16, _p(z), 0, 1.0, _p(z), None) == -1
    assert f(P.handle, _p(z), _p(z), _p(z), _p(z), _p(z), 1, 16, _p(z), 65, 1.0, _p(z), None) == -1
    assert b"range" in lib().qjl_last_error_message() or b"q_per_group" in lib().qjl_last_error_message()

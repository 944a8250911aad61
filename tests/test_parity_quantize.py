"""Key sketch on the GPU vs the oracle (bits under the margin rule, norms).

Covers the dense tcgen05/TMA kernel (bf16 keys, bf16 S_eff), the fp32 SIMT
kernel (fp32 keys or fp32 S_eff), and the fast Walsh-Hadamard kernel for
D-FQJL (with dither) and P-FQJL. Sizes span several 128-key tiles with a
ragged tail, single keys, strided rows, and the literal D_g-outside order.
"""

import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_qjl_b200 import Projection, quantize_keys
from bit_kv_cache_qjl_b200 import workloads as wl
from helpers import check_bits, host, oracle_projection

pytestmark = pytest.mark.gpu


def _run(P, keys, first_token=0):
    bits, norms = quantize_keys(P, keys, first_token=first_token)
    torch.cuda.synchronize()
    O = oracle_projection(P)
    K = host(keys)
    ow, onorm, y = oracle.qjl.quantize_keys(O, K, first_token)
    check_bits(host(bits), ow, y, onorm, P.m)
    np.testing.assert_allclose(host(norms), onorm, rtol=1e-5, atol=1e-30)
    return bits, norms


@pytest.mark.parametrize("d,m,n", [(128, 256, 4096), (128, 256, 129), (128, 256, 1), (128, 512, 1000),
                                   (64, 256, 300), (256, 256, 257), (128, 128, 200), (192, 512, 131)])
def test_dense_tensor_core_path(cuda_ok, d, m, n):
    P = Projection(2, d, m, "dense", s_bf16=True)
    keys = wl.normal((n, d), 1000 + n, "cuda", torch.bfloat16)
    _run(P, keys)


def test_dense_tensor_core_strided_rows(cuda_ok):
    P = Projection(2, 128, 256, "dense")
    big = wl.normal((700, 192), 5, "cuda", torch.bfloat16)
    keys = big[:, :128]
    assert keys.stride(0) == 192
    bits, norms = quantize_keys(P, keys.contiguous())
    O = oracle_projection(P)
    ow, onorm, y = oracle.qjl.quantize_keys(O, host(keys))
    # run on the strided view through the C ABI directly (ld = 192)
    import ctypes
    from bit_kv_cache_qjl_b200 import lib
    b2 = torch.empty_like(bits)
    n2 = torch.empty_like(norms)
    st = lib().qjl_quantize_keys(P.handle, ctypes.c_void_p(keys.data_ptr()), 1, 700, 192, 0,
                                 ctypes.c_void_p(b2.data_ptr()), ctypes.c_void_p(n2.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    check_bits(host(b2), ow, y, onorm, 256)
    assert torch.equal(b2, bits)


def test_dense_fp32_workload_full(cuda_ok):
    """The 1-head fp32 workload in full: 4096 keys, d=128, m=256, fp32 S."""
    w = wl.WORKLOADS["dense_1head"]
    P = Projection(w["proj_seed"], w["d"], w["m"], "dense", s_bf16=False)
    keys, _ = wl.dense_1head("cuda")
    bits, norms = _run(P, keys)
    assert bits.shape == (4096, 8) and norms.shape == (4096,)


def test_dense_bf16_keys_fp32_matrix_simt(cuda_ok):
    P = Projection(3, 128, 256, "dense", s_bf16=False)
    _run(P, wl.normal((333, 128), 9, "cuda", torch.bfloat16))


@pytest.mark.parametrize("kind,d,m,n,dtype,ft", [
    ("pfqjl", 256, 256, 1000, torch.bfloat16, 0),
    ("pfqjl", 256, 1024, 300, torch.bfloat16, 0),
    ("dfqjl", 128, 256, 1000, torch.bfloat16, 12345),
    ("dfqjl", 128, 256, 64, torch.float32, (1 << 32) + 7),
    ("pfqjl", 32, 64, 77, torch.float32, 0),
    ("dfqjl", 1024, 2048, 40, torch.bfloat16, 3),
    ("pfqjl", 512, 512, 33, torch.float32, 0),
    # every thread layout of the transform kernel (d = 32 ... 1024), both dtypes, ragged batches
    ("pfqjl", 64, 128, 129, torch.bfloat16, 0),
    ("dfqjl", 32, 64, 65, torch.bfloat16, 5),
    ("dfqjl", 64, 64, 31, torch.float32, 9),
    ("dfqjl", 256, 512, 301, torch.bfloat16, 7),
    ("pfqjl", 256, 256, 17, torch.float32, 0),
    ("dfqjl", 512, 1024, 45, torch.float32, 0),
    ("pfqjl", 1024, 1024, 9, torch.float32, 0),
    ("pfqjl", 128, 128, 1, torch.bfloat16, 0),
    # more blocks than one launch's table budget: several launches over block ranges
    ("pfqjl", 1024, 4096, 37, torch.bfloat16, 0),
    ("dfqjl", 128, 4096, 70, torch.float32, 11),
    # the tcgen05 kernel (bf16, d in {128, 256}, m a multiple of 256): one key; the dither past
    # 2^32 tokens; several 256-coordinate passes (the dither's coordinate offset per pass)
    ("pfqjl", 256, 256, 1, torch.bfloat16, 0),
    ("dfqjl", 128, 256, 129, torch.bfloat16, (1 << 32) + 7),
    ("dfqjl", 128, 512, 300, torch.bfloat16, 5),
    ("pfqjl", 128, 768, 200, torch.bfloat16, 0),
    # every CTA of the persistent grid takes two tiles or more (ring and TMEM phases wrap)
    ("dfqjl", 128, 256, 148 * 128 * 2 + 77, torch.bfloat16, 1),
    ("pfqjl", 256, 256, 148 * 128 * 2 + 5, torch.bfloat16, 0),
])
def test_fqjl(cuda_ok, kind, d, m, n, dtype, ft):
    P = Projection(4, d, m, kind)
    _run(P, wl.normal((n, d), 77 + n, "cuda", dtype), first_token=ft)


def test_fqjl_literal_order(cuda_ok):
    P = Projection(4, 128, 256, "pfqjl", dg_outer=True)
    _run(P, wl.normal((500, 128), 8, "cuda", torch.bfloat16))
    P = Projection(4, 256, 512, "dfqjl", dg_outer=True)
    _run(P, wl.normal((70, 256), 18, "cuda", torch.bfloat16), first_token=3)


def test_dfqjl_without_dither(cuda_ok):
    P = Projection(6, 128, 256, "dfqjl", dither_sigma_rel=0.0)
    _run(P, wl.normal((100, 128), 19, "cuda", torch.bfloat16))


@pytest.mark.parametrize("kind,d", [("pfqjl", 128), ("dfqjl", 128), ("pfqjl", 256), ("dfqjl", 512)])
def test_fqjl_zero_keys(cuda_ok, kind, d):
    """A zero key: the map is +0 everywhere, so every bit is 1 (sign(0) = +1), dither or not."""
    P = Projection(4, d, 2 * d, kind)
    keys = torch.zeros((40, d), dtype=torch.bfloat16, device="cuda")
    keys[7] = -0.0
    bits, norms = quantize_keys(P, keys)
    torch.cuda.synchronize()
    assert torch.all(norms == 0)
    assert torch.all(bits == -1)


def test_fqjl_strided_rows(cuda_ok):
    import ctypes
    from bit_kv_cache_qjl_b200 import lib
    P = Projection(4, 256, 512, "pfqjl")
    big = wl.normal((90, 320), 21, "cuda", torch.bfloat16)
    keys = big[:, :256]
    b2 = torch.empty((90, 16), dtype=torch.int32, device="cuda")
    n2 = torch.empty((90,), device="cuda")
    st = lib().qjl_quantize_keys(P.handle, ctypes.c_void_p(keys.data_ptr()), 1, 90, 320, 4,
                                 ctypes.c_void_p(b2.data_ptr()), ctypes.c_void_p(n2.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    ow, onorm, y = oracle.qjl.quantize_keys(oracle_projection(P), host(keys), 4)
    check_bits(host(b2), ow, y, onorm, 512)
    np.testing.assert_allclose(host(n2), onorm, rtol=1e-5)


def test_outlier_keys_dense(cuda_ok):
    """Keys with x10 outlier channels (the Llama-shaped decode workload's structure)."""
    P = Projection(2, 128, 256, "dense")
    keys = wl.llama_keys("cuda", B=1, H=2, N=1500).reshape(-1, 128)
    _run(P, keys)


def test_zero_keys_edge(cuda_ok):
    P = Projection(2, 128, 256, "dense")
    keys = torch.zeros((130, 128), dtype=torch.bfloat16, device="cuda")
    bits, norms = quantize_keys(P, keys)
    torch.cuda.synchronize()
    assert torch.all(norms == 0)
    # y = +0 everywhere: sign(0) = +1 in the oracle. -0.0 cannot arise from a
    # sum of +0 products, so every bit must be 1.
    assert torch.all(bits == -1)
    assert quantize_keys(P, keys[:0])[0].numel() == 0

"""The hot path runs the intended kernels of libqjl_b200.so.

The CUDA profiler (CUPTI, through torch.profiler) lists every kernel launched
in the process. Each call must launch its own library kernel, with no torch
kernels and no CPU work standing in.
"""

import pytest
import torch

import bit_kv_cache_qjl_b200 as qjl
from bit_kv_cache_qjl_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _kernels(fn):
    torch.cuda.synchronize()
    with torch.profiler.profile(activities=[torch.profiler.ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    return names


def _has(names, frag):
    return any(frag in n for n in names)


def test_dense_bf16_uses_tcgen05_kernel(cuda_ok):
    P = qjl.Projection(2, 128, 256, "dense")
    keys = wl.normal((4096, 128), 1, "cuda", torch.bfloat16)
    names = _kernels(lambda: qjl.quantize_keys(P, keys))
    assert _has(names, "dense_tc_kernel"), names
    assert not _has(names, "dense_simt_kernel")


def test_fp32_keys_use_simt_kernel(cuda_ok):
    P = qjl.Projection(2, 128, 256, "dense", s_bf16=False)
    keys = wl.normal((512, 128), 1, "cuda")
    assert _has(_kernels(lambda: qjl.quantize_keys(P, keys)), "dense_simt_kernel")


def test_fqjl_kernels(cuda_ok):
    # bf16 keys with d in {128, 256} and m a multiple of 256: the tcgen05 kernel, one launch for all
    # 256-coordinate passes
    P = qjl.Projection(4, 256, 1024, "pfqjl")
    keys = wl.normal((512, 256), 1, "cuda", torch.bfloat16)
    names = _kernels(lambda: qjl.quantize_keys(P, keys))
    assert sum("fqjl_tc_kernel" in n for n in names) == 1, names
    assert not _has(names, "fqjl_keys_kernel")
    D0 = qjl.Projection(5, 128, 256, "dfqjl", dither_sigma_rel=0.0)
    names = _kernels(lambda: qjl.quantize_keys(D0, wl.normal((300, 128), 3, "cuda", torch.bfloat16)))
    assert sum("fqjl_tc_kernel" in n for n in names) == 1, names
    D = qjl.Projection(5, 128, 256, "dfqjl")
    names = _kernels(lambda: qjl.quantize_keys(D, wl.normal((300, 128), 3, "cuda", torch.bfloat16)))
    assert sum("fqjl_tc_kernel" in n for n in names) == 1, names
    # the dither at d = 256, fp32 keys, other widths and the literal order keep the register
    # Walsh-Hadamard kernel
    D2 = qjl.Projection(5, 256, 256, "dfqjl")
    assert _has(_kernels(lambda: qjl.quantize_keys(D2, wl.normal((300, 256), 3, "cuda", torch.bfloat16))),
                "fqjl_keys_kernel")
    assert _has(_kernels(lambda: qjl.quantize_keys(P, keys.float())), "fqjl_keys_kernel")
    E = qjl.Projection(4, 512, 1024, "pfqjl")
    assert _has(_kernels(lambda: qjl.quantize_keys(E, wl.normal((64, 512), 4, "cuda", torch.bfloat16))),
                "fqjl_keys_kernel")
    F = qjl.Projection(4, 128, 256, "pfqjl", dg_outer=True)
    assert _has(_kernels(lambda: qjl.quantize_keys(F, wl.normal((64, 128), 5, "cuda", torch.bfloat16))),
                "fqjl_keys_kernel")
    q = wl.normal((3, 256), 2, "cuda")
    assert _has(_kernels(lambda: qjl.project_queries(P, q)), "fqjl_query_kernel")


def test_scores_and_projection_kernels(cuda_ok):
    P = qjl.Projection(2, 128, 256, "dense")
    bits = torch.zeros((4, 1000, 8), dtype=torch.int32, device="cuda")
    norms = torch.ones((4, 1000), device="cuda")
    q = wl.normal((4, 128), 3, "cuda")
    names = _kernels(lambda: qjl.scores(P, bits, norms, qjl.project_queries(P, q).view(4, 1, 256)))
    # one or two queries per group: the shift-window digit kernel
    assert _has(names, "scores_digit_kernel") and _has(names, "project_dense_kernel"), names
    sq2 = torch.ones((4, 2, 256), device="cuda")
    assert _has(_kernels(lambda: qjl.scores(P, bits, norms, sq2)), "scores_digit_kernel")
    # three or four: the weight-class kernel
    sq4 = torch.ones((4, 4, 256), device="cuda")
    assert _has(_kernels(lambda: qjl.scores(P, bits, norms, sq4)), "scores_decode_kernel")
    # more than 4 queries per group are a contraction for the tcgen05 kernel
    sq8 = torch.ones((4, 8, 256), device="cuda")
    assert _has(_kernels(lambda: qjl.scores(P, bits, norms, sq8)), "scores_many_kernel")
    # and so is any query count at m = 1024
    P1k = qjl.Projection(2, 128, 1024, "dense")
    b1k = torch.zeros((4, 1000, 32), dtype=torch.int32, device="cuda")
    sq1 = torch.ones((4, 1, 1024), device="cuda")
    assert _has(_kernels(lambda: qjl.scores(P1k, b1k, norms, sq1)), "scores_many_kernel")


def test_values_and_decode_kernels(cuda_ok):
    P = qjl.Projection(5, 128, 256, "dfqjl")
    v = wl.normal((2 * 300, 128), 4, "cuda", torch.bfloat16)
    bits = torch.zeros((2, 300, 8), dtype=torch.int32, device="cuda")
    norms = torch.ones((2, 300), device="cuda")

    def run(J):
        sq = torch.ones((2, J, 256), device="cuda")
        c, s, z = qjl.quantize_values_2bit(v)
        qjl.decode_attention(P, bits, norms, c.view(2, 300, 8), s.view(2, 300, 4), z.view(2, 300, 4), sq, 0.1)
    names = _kernels(lambda: run(1))
    for k in ("values_2bit_kernel", "decode_stream_kernel", "decode_combine_stream_kernel"):
        assert _has(names, k), (k, names)
    # several queries per group take the tile-per-warp kernel and the split combine
    names = _kernels(lambda: run(2))
    assert _has(names, "decode_partial_kernel") and _has(names, "decode_combine_kernel"), names


def test_many_query_projection_kernels(cuda_ok):
    # a prefill's projection of every position: the bf16 tensor-core kernel when S_eff is bf16,
    # the warp-per-row SIMT kernel when S is fp32
    q = wl.normal((2048, 128), 4, "cuda")
    Pb = qjl.Projection(2, 128, 256, "dense", s_bf16=True)
    assert _has(_kernels(lambda: qjl.project_queries(Pb, q)), "project_mma_kernel")
    Pf = qjl.Projection(2, 128, 256, "dense", s_bf16=False)
    assert _has(_kernels(lambda: qjl.project_queries(Pf, q)), "dense_simt_kernel")


def test_prefill_uses_tcgen05_kernel(cuda_ok):
    P = qjl.Projection(2, 128, 256, "dense")
    G, L = 2, 200
    bits = torch.zeros((G, L, 8), dtype=torch.int32, device="cuda")
    norms = torch.ones((G, L), device="cuda")
    codes = torch.zeros((G, L, 8), dtype=torch.int32, device="cuda")
    sc = torch.ones((G, L, 4), dtype=torch.float16, device="cuda")
    zr = torch.zeros((G, L, 4), dtype=torch.float16, device="cuda")
    sq = torch.ones((G, L, 256), device="cuda")
    names = _kernels(lambda: qjl.prefill_attention(P, bits, norms, codes, sc, zr, sq, 0.1))
    assert _has(names, "prefill_tc_kernel"), names

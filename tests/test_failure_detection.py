"""Failure detection without a GPU fault.

* A bounded wait that expires: qjl_selftest_bounded_wait waits on a barrier
  nothing completes, with a 20 ms limit. The kernel records bit 128 and
  returns, the host reads it through qjl_device_errors, and the context keeps
  working.
* A bad paged-cache entry: the kernels skip it and record bit 64.
* A device allocation that fails: QJL_FAIL_ALLOC_AFTER=k makes the projection's
  allocations after the first k report failure on the host. qjl_make_projection
  returns QJL_ERR_OOM, frees what it had, and later calls in the process keep
  failing cleanly. It runs in a child process, since the limit is read once.
The argument checks of both calls need no GPU.
"""

import ctypes
import os
import subprocess
import sys

import pytest
import torch

import bit_kv_cache_qjl_b200 as qjl
from bit_kv_cache_qjl_b200 import workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_argument_checks_without_gpu():
    L = qjl.lib()
    assert L.qjl_device_errors(0, 1, None) == -1
    assert L.qjl_selftest_bounded_wait(0, 0) == -1
    assert L.qjl_selftest_bounded_wait(0, 2 * 10**9) == -1


@pytest.mark.gpu
def test_bounded_wait_expires_and_reports(cuda_ok):
    qjl.device_errors(0, clear=True)
    assert qjl.lib().qjl_selftest_bounded_wait(0, 20_000_000) == 0
    flags = ctypes.c_int(0)
    assert qjl.lib().qjl_device_errors(0, 1, ctypes.byref(flags)) == -6      # QJL_ERR_DEVICE
    assert flags.value & 128
    assert qjl.device_errors(0) == 0                                         # cleared
    # the context still works
    P = qjl.Projection(1, 128, 256, "dense")
    bits, norms = qjl.quantize_keys(P, wl.normal((64, 128), 1, "cuda", torch.bfloat16))
    torch.cuda.synchronize()
    assert torch.isfinite(norms).all() and qjl.device_errors(0) == 0


@pytest.mark.gpu
def test_bad_page_entry_sets_its_bit(cuda_ok):
    qjl.device_errors(0, clear=True)
    T, d, m = 32, 128, 256
    P = qjl.Projection(2, d, m, "dense")
    table = torch.tensor([[0], [7]], dtype=torch.int32, device="cuda")        # page 7 does not exist
    bits = torch.zeros((2 * T, m // 32), dtype=torch.int32, device="cuda")
    norms = torch.zeros((2 * T,), dtype=torch.float32, device="cuda")
    cache = qjl.PagedCache(T, table, None, bits, norms)
    qjl.append_keys(P, cache, wl.normal((2, d), 3, "cuda", torch.bfloat16),
                    torch.tensor([1, 2], dtype=torch.int32, device="cuda"))
    assert qjl.device_errors(0) & 64
    assert norms[1] > 0 and (norms[T:] == 0).all()


_CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import bit_kv_cache_qjl_b200 as qjl
out = []
for kind in ("dense", "pfqjl"):
    try:
        qjl.Projection(3, 128, 256, kind)
        out.append("ok")
    except qjl.QJLError as e:
        out.append(str(e.status))
print(",".join(out))
"""


@pytest.mark.gpu
@pytest.mark.parametrize("after", [0, 1, 2])
def test_injected_allocation_failure(cuda_ok, after):
    env = dict(os.environ, QJL_FAIL_ALLOC_AFTER=str(after))
    r = subprocess.run([sys.executable, "-c", _CHILD.format(root=ROOT)], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    # the dense projection makes two device allocations, so it survives only after >= 2; either way
    # every failure is QJL_ERR_OOM (-4) and later projections in the process fail the same way
    got = r.stdout.strip().split(",")
    assert got == (["-4", "-4"] if after < 2 else ["ok", "-4"]), got

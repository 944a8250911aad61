"""The alternative estimator kernels stay correct.

QJL_SCORES_KERNEL=tc selects the tcgen05 kind::i8 kernel, and
QJL_SCORES_KERNEL=stream selects the generic streaming kernel. The library
reads the switch once per process, so each variant reruns the estimator
parity tests in a child process.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("variant", ["tc", "stream"])
def test_scores_variant_parity(cuda_ok, variant):
    env = dict(os.environ, QJL_SCORES_KERNEL=variant)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_parity_scores.py")], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]

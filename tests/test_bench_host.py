"""Host-side pieces of bench.py that need no GPU: the source hash that keys the ncu traffic
lines, and the format of profiles/traffic.txt."""

import glob
import hashlib
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_kv_cache_qjl_b200", "csrc")
BENCH_SRC = open(os.path.join(ROOT, "bench.py")).read()


def test_source_hash_of_one_file_and_of_a_list():
    a = os.path.join(CSRC, "fqjl_tc.cu")
    b = os.path.join(CSRC, "key_math.cuh")
    one = hashlib.sha256(open(a, "rb").read()).hexdigest()[:16]
    both = hashlib.sha256(open(a, "rb").read() + open(b, "rb").read()).hexdigest()[:16]
    assert bench.source_hash(a) == one
    assert bench.source_hash([a]) == one
    assert bench.source_hash([a, b]) == both
    assert both != one


def test_traffic_lines_are_well_formed_and_name_real_kernels():
    sources = "".join(open(p).read() for p in glob.glob(os.path.join(CSRC, "*.cu")))
    lines = [l.split() for l in open(os.path.join(ROOT, "profiles", "traffic.txt"))
             if l.strip() and not l.startswith("#")]
    assert lines
    for f in lines:
        kernel, workload, nbytes, h = f[:4]
        assert re.search(r"\b%s\b" % re.escape(kernel), sources), kernel
        assert int(nbytes) > 0
        assert re.fullmatch(r"[0-9a-f]{16}", h), h
        assert re.search(r'"%s"' % re.escape(workload), BENCH_SRC), workload


def test_traffic_lookup_follows_the_source_hash():
    # the lookup returns a line's bytes only while the named sources hash to its key
    for f in (l.split() for l in open(os.path.join(ROOT, "profiles", "traffic.txt"))
              if l.strip() and not l.startswith("#")):
        kernel, workload, nbytes, h = f[:4]
        srcs = ("fqjl_tc.cu", "key_math.cuh") if kernel == "fqjl_tc_kernel" else None
        if srcs is None:
            continue
        got = bench.ncu_traffic(kernel, workload, srcs)
        if bench.source_hash([os.path.join(CSRC, s) for s in srcs]) == h:
            assert got == float(nbytes)
        else:
            assert got is None
        assert bench.ncu_traffic(kernel, workload, "values.cu") is None

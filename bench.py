"""Throughput of the QJL key-quantize + decode-score hot path on B200.

One step is a whole pass of the path over one batch of the Llama-2-7B-shaped
decode workload: B=8, 32 heads, N=32768 cached keys per head, d=128,
m=256, dense bf16 S. The step:
  (1) sketches every key (tcgen05 kernel): bits + ||k||;
  (2) projects one query per head (unquantised JL map);
  (3) scores every cached key against its head's query (estimator).
`value` is cached keys processed per second over whole steps, with inputs
already resident in HBM. The 2.1 GB keys exceed the 126 MB L2, so no flush
is needed. `e2e` is the same metric through the same C-ABI calls with host
buffers: each step copies the keys and queries in from pinned host memory and
copies the scores back.

Multi-GPU (torchrun): the (batch, head) groups are independent, so every
rank processes its own copy of the workload (weak scaling). No collective
touches the data path. Ranks meet at a barrier around the timed region, and
the time is the max over ranks.

--impl reference times the CPU oracle on a bounded sample of the same
workload (the reference arm). It runs on rank 0 only.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QJL decode scores keys/s (HBM GB/s vs ~8 TB/s); key-quantize vectors/s"
WORKLOAD = "decode_llama7b"
B, H, N, D, M = 8, 32, 32768, 128, 256
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# FP32 issue ceiling of the ALU-bound transform: 148 SMs x 128 FP32 lanes x 1.965 GHz (max SM clock),
# one add or multiply per lane per clock.
FP32_TFLOPS = 148 * 128 * 1.965e9 / 1e12


def fqjl_flops_per_key(d, m):
    """Algorithmic fp32 operations of the FQJL map per key: per block, D_r and D_g (d multiplies
    each) and two Walsh-Hadamard transforms (d log2 d additions each)."""
    return 2 * m * (int(math.log2(d)) + 1)



def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(paths):
    """sha256 prefix of a kernel's source file, or of several concatenated (the .cu and the headers
    whose arithmetic it runs)."""
    h = hashlib.sha256()
    for path in ([paths] if isinstance(paths, str) else paths):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload, src):
    """Per-launch DRAM bytes from profiles/traffic.txt, valid only for the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    srcs = [src] if isinstance(src, str) else list(src)
    h = source_hash([os.path.join(ROOT, "bit_kv_cache_qjl_b200", "csrc", f) for f in srcs])
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == kernel and f[1] == workload and f[3] == h:
            return float(f[2])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled around a timed region.

    A reader thread collects samples every `period_ms`. Entering waits (up to 5 s) for the first
    sample, so the region is never timed before sampling runs; mark() records the region's start
    and end on the host clock, and leaving waits for one sample past the end. The summary takes the
    samples that fall in the region plus the last one before it and the first one after it, so a
    region shorter than the period is still bracketed by two samples under load.
    """

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index, period_ms=50):
        self.index, self.period_ms = index, period_ms
        self.proc, self.samples, self.marks = None, [], []
        import threading
        self._cv = threading.Condition()

    def _reader(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            reasons = [n for n, v in zip(self.NAMES, f[5:9]) if v.lower() == "active"]
            with self._cv:
                self.samples.append((time.monotonic(), mhz, mx, reasons))
                self._cv.notify_all()

    def _wait_for(self, count, timeout):
        with self._cv:
            self._cv.wait_for(lambda: len(self.samples) >= count, timeout=timeout)

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        threading.Thread(target=self._reader, daemon=True).start()
        self._wait_for(1, 5.0)
        return self

    def mark(self):
        """Record the host time of a region boundary (call after a synchronize)."""
        self.marks.append(time.monotonic())

    def __exit__(self, *a):
        if self.proc is None:
            return
        with self._cv:
            n = len(self.samples)
        self._wait_for(n + 1, 2.0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()

    def summary(self):
        with self._cv:
            smp = list(self.samples)
        if len(self.marks) >= 2:
            t0, t1 = self.marks[0], self.marks[-1]
            inside = [s for s in smp if t0 <= s[0] <= t1]
            before = [s for s in smp if s[0] < t0][-1:]
            after = [s for s in smp if s[0] > t1][:1]
            use = before + inside + after
            region_ms = 1e3 * (t1 - t0)
        else:
            use, inside, region_ms = smp, smp, None
        reasons = sorted({r for s in use for r in s[3]})
        return {"sm_mhz": statistics.median([s[1] for s in use]) if use else None,
                "sm_max_mhz": use[-1][2] if use else None, "reasons": reasons, "samples": len(use),
                "samples_inside": len(inside), "region_ms": region_ms, "period_ms": self.period_ms,
                "rule": "samples inside the timed region plus the last before and the first after it"}


def dist_setup(backend=None):
    """One process per GPU under torchrun: (world, rank, local rank). NCCL on GPUs; gloo when no
    GPU is visible (the CPU tests of the multi-rank path)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x, world):
    """The max of a per-rank scalar over all ranks (the job's time is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def job_throughput(units_per_rank, world, ms_step_max):
    """Whole-job units per second: every rank processed units_per_rank in the slowest rank's time."""
    return world * units_per_rank / (ms_step_max * 1e-3)


_ORACLE_PROJ = {}


def oracle_prepare(name, units):
    """The oracle's path over a `units`-sized slice of workload `name`, ready to run: the projection
    is drawn and the inputs generated here (setup, not timed). Returns (run, units): run() takes
    every step of that workload's path in the fp64 oracle, as it stands."""
    import numpy as np

    import oracle
    from bit_kv_cache_qjl_b200 import workloads as wl

    class P:                                       # the oracle's projections, drawn once per process
        KIND_DENSE, KIND_DFQJL, KIND_PFQJL = (oracle.params.KIND_DENSE, oracle.params.KIND_DFQJL,
                                              oracle.params.KIND_PFQJL)

        @staticmethod
        def make_projection(*a, **k):
            key = (a, tuple(sorted(k.items())))
            if key not in _ORACLE_PROJ:
                _ORACLE_PROJ[key] = oracle.params.make_projection(*a, **k)
            return _ORACLE_PROJ[key]
    if name == "dense_1head":
        O = P.make_projection(1, D, M, P.KIND_DENSE, s_bf16=False)
        n = max(16, min(units, 4096))
        keys, q = wl.dense_1head("cpu", n=n)
        keys, q = keys.double().numpy(), q.double().numpy()

        def run():
            words, norms, _ = oracle.qjl.quantize_keys(O, keys)
            sq = oracle.qjl.project_queries(O, q)
            oracle.qjl.scores(O, words[None], norms[None], sq[None])
        return run, n
    if name in ("decode_llama7b", "gqa_decode"):
        dense = name == "decode_llama7b"
        m, J = (M, 1) if dense else (512, 4)
        O = P.make_projection(2 if dense else 3, D, m, P.KIND_DENSE, s_bf16=True)
        n = max(64, min(units, N if dense else 131072))
        if dense:
            keys = wl.llama_keys("cpu", B=1, H=1, N=n).reshape(n, D)
            q = wl.llama_queries("cpu", B=1, H=1).reshape(1, D)
        else:
            keys = wl.gqa_keys("cpu", B=1, Hkv=1, N=n).reshape(n, D)
            q = wl.gqa_queries("cpu", B=1, Hq=J).reshape(J, D)
        keys, q = keys.double().numpy(), q.double().numpy()

        def run():
            words, norms, _ = oracle.qjl.quantize_keys(O, keys)
            sq = oracle.qjl.project_queries(O, q)
            oracle.qjl.scores(O, words[None], norms[None], sq[None])
        return run, n
    if name in ("pfqjl_bulk_m256", "pfqjl_bulk_m1024"):
        m = 256 if name.endswith("256") else 1024
        O = P.make_projection(4, 256, m, P.KIND_PFQJL)
        n = max(256, min(units, 1 << 16))
        keys = wl.bulk_keys("cpu", n=n, d=256).double().numpy()
        q = wl.bulk_queries("cpu", nq=64, d=256).double().numpy()
        ns = max(1, n // 16)                       # the workload scores 2^20 of its 2^24 keys

        def run():
            words, norms, _ = oracle.qjl.quantize_keys(O, keys)
            sq = oracle.qjl.project_queries(O, q)
            oracle.qjl.scores(O, words[None, :ns], norms[None, :ns], sq[None])
        return run, n
    if name == "dfqjl_decode":
        O = P.make_projection(5, D, M, P.KIND_DFQJL, sigma_rel=0.5)
        n = max(64, min(units, 16384))
        keys, vals = wl.decode_kv("cpu", B=1, H=1, N=n, d=D)
        keys, vals = keys.reshape(n, D).double().numpy(), vals.reshape(n, D).float().numpy()
        q = wl.decode_queries("cpu", B=1, H=1).reshape(1, D).double().numpy()

        def run():
            words, norms, _ = oracle.qjl.quantize_keys(O, keys)
            codes, sc, zr = oracle.kivi.quantize_values_2bit(vals)
            sq = oracle.qjl.project_queries(O, q)
            est = oracle.qjl.scores(O, words[None], norms[None], sq[None])
            vhat = oracle.kivi.dequantize_values(codes, sc, zr, D)[None]
            oracle.attention.decode_attention(est, vhat, 1.0 / math.sqrt(D))
        return run, n
    raise ValueError(name)


ORACLE_UNIT = {"dense_1head": "keys/s", "decode_llama7b": "keys/s", "gqa_decode": "keys/s",
               "pfqjl_bulk_m256": "vectors/s", "pfqjl_bulk_m1024": "vectors/s", "dfqjl_decode": "tokens/s"}


def _timed(run, threads, warm=None):
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=threads):
        (warm or run)()                                    # warm: BLAS threads, caches, allocations
        t0 = time.perf_counter()
        run()
        return time.perf_counter() - t0


# oracle slice per config: one head (or the whole small config), or a key count that takes a few seconds
ORACLE_SAMPLE = {"dense_1head": 4096, "decode_llama7b": N, "gqa_decode": 16384, "pfqjl_bulk_m256": 32768,
                 "pfqjl_bulk_m1024": 8192, "dfqjl_decode": 16384}


def cpu_baseline(name):
    """The oracle timed on this host's cores over a fixed slice of workload `name` (ORACLE_SAMPLE), in
    two modes: one BLAS thread, and as many threads as the process may run on. Each mode takes one
    untimed warm call on a 512-unit slice, then one timed pass."""
    affinity = len(os.sched_getaffinity(0))
    small, _ = oracle_prepare(name, 512)
    run, units = oracle_prepare(name, ORACLE_SAMPLE[name])
    res = {"kind": "oracle", "unit": ORACLE_UNIT[name], "nproc": os.cpu_count(), "affinity": affinity}
    for mode, threads in (("all_cores", affinity), ("single_thread", 1)):
        dt = _timed(run, threads, warm=small)
        res[mode] = {"value": units / dt, "cores": threads, "seconds": dt}
    res["value"] = res["all_cores"]["value"]
    res["cores"] = affinity
    res["sample"] = ("%d %s of the workload (one head or key slice, same shapes and generators on the host); "
                     "the fp64 oracle's quantize, projection and scoring (and, for the fused decode, values "
                     "and attention), one timed pass per mode after a 512-unit warm call" %
                     (units, ORACLE_UNIT[name].split("/")[0]))
    return res


def default_desc():
    """The workload text of the default step (decode_llama7b), shared by both arms' config."""
    return ("%s: B=%d, heads=%d, N=%d, d=%d, m=%d dense bf16 S; quantize all keys, project 1 query/head, "
            "score all keys" % (WORKLOAD, B, H, N, D, M))


def run_config(desc, units, world):
    """The JSON line's config: the same dict for our arm and the reference arm."""
    return {"workload": desc, "units_per_step": units * world,
            "l2": "inputs larger than L2 (126 MB) in every step, no flush",
            "parallelism": "replicas (weak)" if world > 1 else "single GPU"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    threads = len(os.sched_getaffinity(0))
    run, sample = oracle_prepare(WORKLOAD, args.ref_sample)
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=threads):
        for _ in range(args.warmup):
            run()
        total_keys, total_t = 0, 0.0
        for _ in range(args.steps):
            t0 = time.perf_counter()
            run()
            total_t += time.perf_counter() - t0
            total_keys += sample
    value = total_keys / total_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": run_config(default_desc(), B * H * N, world),
            "cpu_baseline": {"value": value, "unit": "keys/s", "cores": threads, "kind": "oracle",
                             "nproc": os.cpu_count(),
                             "sample": "%d keys (one head slice of the workload) per step: oracle quantize + "
                                       "project + score" % sample},
            "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def profile_case(case, n):
    """A small case of one kernel for ncu: inputs > L2 (126 MB) but a few GB at most; 2 + 3 launches."""
    import torch
    import bit_kv_cache_qjl_b200 as qjl
    from bit_kv_cache_qjl_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    if case == "quantize":
        P = qjl.Projection(2, D, M, "dense")
        keys = wl.llama_keys(dev, B=1, H=max(1, n // N), N=min(N, n), d=D).reshape(-1, D)
        run = lambda: qjl.quantize_keys(P, keys)
    elif case in ("fqjl", "fqjl1024"):
        m = 256 if case == "fqjl" else 1024
        P = qjl.Projection(4, 256, m, "pfqjl")
        keys = wl.bulk_keys(dev, n=n, d=256)
        run = lambda: qjl.quantize_keys(P, keys)
    elif case == "dfqjl":
        P = qjl.Projection(5, D, M, "dfqjl", dither_sigma_rel=0.5)
        keys, _ = wl.decode_kv(dev, B=1, H=max(1, n // 16384), N=min(16384, n), d=D)
        keys = keys.reshape(-1, D)
        run = lambda: qjl.quantize_keys(P, keys)
    elif case == "scores":
        P = qjl.Projection(2, D, M, "dense")
        G = max(1, n // N)
        keys = wl.llama_keys(dev, B=1, H=G, N=N, d=D).reshape(-1, D)
        bits, norms = qjl.quantize_keys(P, keys)
        sq = qjl.project_queries(P, wl.llama_queries(dev, B=1, H=G, d=D).reshape(-1, D))
        run = lambda: qjl.scores(P, bits.view(G, N, M // 32), norms.view(G, N), sq.view(G, 1, M))
    elif case in ("many256", "many1024"):
        # many-query scores: 2^18 keys against 64 queries (a quarter of the bulk workload's scored keys)
        m = 256 if case == "many256" else 1024
        P = qjl.Projection(4, 256, m, "pfqjl")
        keys = wl.bulk_keys(dev, n=n, d=256)
        bits, norms = qjl.quantize_keys(P, keys)
        sq = qjl.project_queries(P, wl.bulk_queries(dev, nq=64, d=256))
        run = lambda: qjl.scores(P, bits.view(1, n, m // 32), norms.view(1, n), sq.view(1, 64, m))
    elif case == "values":
        v = wl.normal((n, D), 506, dev, torch.bfloat16)
        run = lambda: qjl.quantize_values_2bit(v)
    elif case == "prefill":
        # 8 heads x 4096 tokens of the prefill workload (n is ignored)
        Gp, Lp = 8, 4096
        P = qjl.Projection(2, D, M, "dense")
        keys, vals = wl.decode_kv(dev, B=1, H=Gp, N=Lp, d=D)
        bits, norms = qjl.quantize_keys(P, keys.reshape(-1, D))
        codes, sc, zr = qjl.quantize_values_2bit(vals.reshape(-1, D))
        sq = qjl.project_queries(P, wl.normal((Gp * Lp, D), 407, dev))
        run = lambda: qjl.prefill_attention(P, bits.view(Gp, Lp, -1), norms.view(Gp, Lp), codes.view(Gp, Lp, -1),
                                            sc.view(Gp, Lp, -1), zr.view(Gp, Lp, -1), sq.view(Gp, Lp, M),
                                            1 / math.sqrt(D))
    else:
        P = qjl.Projection(5, D, M, "dfqjl")
        G = max(1, n // 16384)
        keys, vals = wl.decode_kv(dev, B=1, H=G, N=16384, d=D)
        bits, norms = qjl.quantize_keys(P, keys.reshape(-1, D))
        codes, sc, zr = qjl.quantize_values_2bit(vals.reshape(-1, D))
        sq = qjl.project_queries(P, wl.decode_queries(dev, B=1, H=G, d=D).reshape(-1, D))
        run = lambda: qjl.decode_attention(P, bits.view(G, 16384, M // 32), norms.view(G, 16384),
                                           codes.view(G, 16384, D // 16), sc.view(G, 16384, D // 32),
                                           zr.view(G, 16384, D // 32), sq.view(G, 1, M), 1 / math.sqrt(D))
    torch.cuda.synchronize()
    for _ in range(5):
        run()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": case, "n": n, "status": "ok"}))
    return 0


class Stage:
    """One library call of a step: name, callable, units it processes, algorithmic bytes (and flops) per unit."""

    def __init__(self, name, fn, units, bytes_per_unit, flops_per_unit=0, kernel=None, src=None, bound="hbm",
                 launches=1, peak_scale=1.0, alu_ops_per_unit=0):
        # peak_scale: the stage's tensor peak relative to the measured bf16 one (2 for an int8
        # contraction: the nominal int8 : bf16 dense ratio). alu_ops_per_unit: fp32 lane operations
        # a tensor-bound stage also runs (reported beside, against the FP32 lane ceiling)
        self.name, self.fn, self.units, self.launches = name, fn, units, launches
        self.peak_scale, self.alu_ops_per_unit = peak_scale, alu_ops_per_unit
        self.bytes_per_unit, self.flops_per_unit = bytes_per_unit, flops_per_unit
        self.kernel, self.src, self.bound = kernel, src, bound


def build_workload(name, dev, qjl, wl, torch):
    """Inputs resident on `dev`, the step's stages, the host-side copies for the e2e leg, and a description."""
    W = {}
    if name == "decode_llama7b":
        P = qjl.Projection(2, D, M, "dense", s_bf16=True)
        G = B * H
        keys = wl.llama_keys(dev, B=B, H=H, N=N, d=D).reshape(-1, D)
        q = wl.llama_queries(dev, B=B, H=H, d=D).reshape(-1, D)
        bits = torch.empty((G * N, M // 32), dtype=torch.int32, device=dev)
        norms = torch.empty((G * N,), dtype=torch.float32, device=dev)
        sq = torch.empty((G, M), dtype=torch.float32, device=dev)
        out = torch.empty((G, 1, N), dtype=torch.float32, device=dev)
        stages = [
            Stage("quantize_keys", lambda: qjl.quantize_keys(P, keys, bits=bits, norms=norms), G * N,
                  2 * D + M // 8 + 4, 2 * D * M, "dense_tc_kernel", "dense_tc.cu"),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), G, 4 * D + 4 * M, bound="launch"),
            Stage("scores", lambda: qjl.scores(P, bits.view(G, N, M // 32), norms.view(G, N), sq.view(G, 1, M), out=out),
                  G * N, M // 8 + 4 + 4, 0, "scores_digit_kernel", "scores.cu"),
        ]
        W.update(units=G * N, unit="keys/s", inputs=[keys, q], outputs=[out], dtype="bf16", desc=default_desc())
    elif name == "gqa_decode":
        Bq, Hq, Hkv, Nq, m = 16, 32, 8, 131072, 512
        G, J = Bq * Hkv, Hq // Hkv
        P = qjl.Projection(3, D, m, "dense", s_bf16=True)
        keys = wl.gqa_keys(dev, B=Bq, Hkv=Hkv, N=Nq, d=D).reshape(-1, D)
        q = wl.gqa_queries(dev, B=Bq, Hq=Hq, d=D).reshape(-1, D)
        bits = torch.empty((G * Nq, m // 32), dtype=torch.int32, device=dev)
        norms = torch.empty((G * Nq,), dtype=torch.float32, device=dev)
        sq = torch.empty((G * J, m), dtype=torch.float32, device=dev)
        out = torch.empty((G, J, Nq), dtype=torch.float32, device=dev)
        stages = [
            Stage("quantize_keys", lambda: qjl.quantize_keys(P, keys, bits=bits, norms=norms), G * Nq,
                  2 * D + m // 8 + 4, 2 * D * m, "dense_tc_kernel", "dense_tc.cu", "tensor"),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), G * J, 4 * D + 4 * m, bound="launch"),
            Stage("scores", lambda: qjl.scores(P, bits.view(G, Nq, m // 32), norms.view(G, Nq), sq.view(G, J, m),
                                               out=out), G * Nq, m // 8 + 4 + 4 * J, 0, "scores_decode_kernel",
                  "scores.cu"),
        ]
        W.update(units=G * Nq, unit="keys/s", inputs=[keys, q], outputs=[out], dtype="bf16",
                 desc="%s: B=16, 32 query heads over 8 KV heads (4 per KV head), N=131072, d=128, m=512 dense bf16 S; "
                      "quantize, project, score" % name)
    elif name == "dense_1head":
        P = qjl.Projection(1, D, M, "dense", s_bf16=False)
        keys, q = wl.dense_1head(dev)
        n, J = keys.shape[0], q.shape[0]
        bits = torch.empty((n, M // 32), dtype=torch.int32, device=dev)
        norms = torch.empty((n,), dtype=torch.float32, device=dev)
        sq = torch.empty((J, M), dtype=torch.float32, device=dev)
        out = torch.empty((1, J, n), dtype=torch.float32, device=dev)
        stages = [
            Stage("quantize_keys", lambda: qjl.quantize_keys(P, keys, bits=bits, norms=norms), n, 4 * D + M // 8 + 4,
                  2 * D * M, "dense_simt_kernel", "dense_simt.cu", "launch"),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), J, 4 * D + 4 * M, bound="launch"),
            Stage("scores", lambda: qjl.scores(P, bits.view(1, n, M // 32), norms.view(1, n), sq.view(1, J, M), out=out),
                  n, M // 8 + 4 + 4 * J, 0, "scores_many_kernel", "scores_many.cu", "launch"),
        ]
        W.update(units=n, unit="keys/s", inputs=[keys, q], outputs=[out], dtype="f32",
                 desc="%s: 4096 fp32 keys, 16 queries, d=128, m=256 fp32 S (launch-bound)" % name)
    elif name in ("pfqjl_bulk_m256", "pfqjl_bulk_m1024"):
        m = 256 if name.endswith("256") else 1024
        d, n, ns, J = 256, 1 << 24, 1 << 20, 64
        P = qjl.Projection(4, d, m, "pfqjl")
        keys = wl.bulk_keys(dev, n=n, d=d)
        q = wl.bulk_queries(dev, nq=J, d=d)
        bits = torch.empty((n, m // 32), dtype=torch.int32, device=dev)
        norms = torch.empty((n,), dtype=torch.float32, device=dev)
        sq = torch.empty((J, m), dtype=torch.float32, device=dev)
        out = torch.empty((1, J, ns), dtype=torch.float32, device=dev)
        stages = [
            # the first Hadamard factor runs as an exact +-1 contraction on tcgen05 (2 d m flops per
            # key), the second (D_g and d log2 d additions per block) on the FP32 lanes
            Stage("quantize_keys", lambda: qjl.quantize_keys(P, keys, bits=bits, norms=norms), n,
                  2 * d + m // 8 + 4, 2 * d * m, "fqjl_tc_kernel", ("fqjl_tc.cu", "key_math.cuh"), "tensor",
                  alu_ops_per_unit=(m // d) * (d + d * int(math.log2(d)))),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), J, 4 * d + 4 * m, bound="launch"),
            Stage("scores", lambda: qjl.scores(P, bits[:ns].view(1, ns, m // 32), norms[:ns].view(1, ns),
                                               sq.view(1, J, m), out=out), ns, m // 8 + 4 + 4 * J, 2 * J * m,
                  "scores_many_kernel", "scores_many.cu", "hbm" if m == 256 else "tensor", peak_scale=2.0),
        ]
        W.update(units=n, unit="vectors/s", inputs=[keys, q], outputs=[out], dtype="bf16",
                 desc="%s: P-FQJL, 2^24 keys d=256 bf16, m=%d; quantize all, project 64 queries, score the first "
                      "2^20 keys against them" % (name, m))
    elif name == "dfqjl_decode":
        Bd, Hd, Nd, m = 32, 32, 16384, 256
        G = Bd * Hd
        P = qjl.Projection(5, D, m, "dfqjl", dither_sigma_rel=0.5)
        keys, vals = wl.decode_kv(dev, B=Bd, H=Hd, N=Nd, d=D)
        keys, vals = keys.reshape(-1, D), vals.reshape(-1, D)
        q = wl.decode_queries(dev, B=Bd, H=Hd, d=D).reshape(-1, D)
        bits = torch.empty((G * Nd, m // 32), dtype=torch.int32, device=dev)
        norms = torch.empty((G * Nd,), dtype=torch.float32, device=dev)
        codes = torch.empty((G * Nd, D // 16), dtype=torch.int32, device=dev)
        sc = torch.empty((G * Nd, D // 32), dtype=torch.float16, device=dev)
        zr = torch.empty((G * Nd, D // 32), dtype=torch.float16, device=dev)
        sq = torch.empty((G, m), dtype=torch.float32, device=dev)
        out = torch.empty((G, 1, D), dtype=torch.float32, device=dev)
        ws = torch.empty((qjl.decode_workspace_bytes(G, 1, Nd, D),), dtype=torch.uint8, device=dev)
        smx = 1.0 / math.sqrt(D)
        stages = [
            # the first Hadamard factor on tcgen05, the second and the dither on the lanes: reported
            # against the FP32 lane ceiling with the second factor's fp32 operations only (the
            # dither's Philox multiplies and Box-Muller are not fp32 adds or multiplies)
            Stage("quantize_keys", lambda: qjl.quantize_keys(P, keys, bits=bits, norms=norms), G * Nd,
                  2 * D + m // 8 + 4, (m // D) * (D + D * int(math.log2(D))), "fqjl_tc_kernel", ("fqjl_tc.cu", "key_math.cuh"), "alu"),
            Stage("quantize_values", lambda: qjl.quantize_values_2bit(vals, codes=codes, scale=sc, zero=zr), G * Nd,
                  2 * D + D // 4 + D // 8, 0, "values_2bit_kernel", "values.cu"),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), G, 4 * D + 4 * m, bound="launch"),
            Stage("decode_attention", lambda: qjl.decode_attention(
                P, bits.view(G, Nd, m // 32), norms.view(G, Nd), codes.view(G, Nd, D // 16), sc.view(G, Nd, D // 32),
                zr.view(G, Nd, D // 32), sq.view(G, 1, m), smx, out=out, workspace=ws), G * Nd,
                m // 8 + 4 + D // 4 + D // 8, 0, "decode_stream_kernel", "decode.cu", launches=2),
        ]
        W.update(units=G * Nd, unit="tokens/s", inputs=[keys, vals, q], outputs=[out], dtype="bf16",
                 desc="%s: D-FQJL sigma_rel 0.5, B=32, 32 heads, N=16384, d=128, m=256; quantize keys and 2-bit "
                      "values, project queries, fused softmax(QK)V decode" % name)
    elif name == "paged_decode":
        # the dfqjl_decode cache in 256-token pages under a shuffled block table; a step appends one
        # key and one value per group (at the last position, so the length stays N) and attends over
        # all N tokens through the table
        Bd, Hd, Nd, m, T = 32, 32, 16384, 256, 256
        G, pages = Bd * Hd, Nd // T
        P = qjl.Projection(5, D, m, "dfqjl", dither_sigma_rel=0.5)
        keys, vals = wl.decode_kv(dev, B=Bd, H=Hd, N=Nd, d=D)
        keys, vals = keys.reshape(-1, D), vals.reshape(-1, D)
        num_pages = G * pages + 64
        perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(509))[:G * pages]
        table = perm.view(G, pages).to(torch.int32).to(dev)
        t = torch.arange(Nd, device=dev)
        rows = (table.long()[:, t // T] * T + (t % T)[None, :]).reshape(-1)
        R = num_pages * T
        pool = dict(bits=torch.zeros((R, m // 32), dtype=torch.int32, device=dev),
                    norms=torch.zeros((R,), dtype=torch.float32, device=dev),
                    codes=torch.zeros((R, D // 16), dtype=torch.int32, device=dev),
                    scale=torch.zeros((R, D // 32), dtype=torch.float16, device=dev),
                    zero=torch.zeros((R, D // 32), dtype=torch.float16, device=dev))
        b0, n0 = qjl.quantize_keys(P, keys)
        c0, s0, z0 = qjl.quantize_values_2bit(vals)
        for k, v in (("bits", b0), ("norms", n0), ("codes", c0), ("scale", s0), ("zero", z0)):
            pool[k][rows] = v
        del b0, n0, c0, s0, z0, rows
        seq = torch.full((G,), Nd, dtype=torch.int32, device=dev)
        cache = qjl.PagedCache(T, table, seq, pool["bits"], pool["norms"], pool["codes"], pool["scale"],
                               pool["zero"])
        pos = torch.full((G,), Nd - 1, dtype=torch.int32, device=dev)
        newk = wl.normal((G, D), 511, dev, torch.bfloat16)
        newv = wl.normal((G, D), 512, dev, torch.bfloat16)
        q = wl.decode_queries(dev, B=Bd, H=Hd, d=D).reshape(-1, D)
        sq = torch.empty((G, m), dtype=torch.float32, device=dev)
        out = torch.empty((G, D), dtype=torch.float32, device=dev)
        ws = torch.empty((qjl.decode_paged_workspace_bytes(G, Nd, D),), dtype=torch.uint8, device=dev)
        smx = 1.0 / math.sqrt(D)
        stages = [
            Stage("append_keys", lambda: qjl.append_keys(P, cache, newk, pos), G, 2 * D + m // 8 + 4,
                  fqjl_flops_per_key(D, m), bound="launch"),
            Stage("append_values", lambda: qjl.append_values_2bit(cache, newv, pos), G, 2 * D + D // 4 + D // 8,
                  bound="launch"),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), G, 4 * D + 4 * m, bound="launch"),
            Stage("decode_attention_paged", lambda: qjl.decode_attention_paged(P, cache, sq, Nd, smx, out=out,
                                                                               workspace=ws), G * Nd,
                  m // 8 + 4 + D // 4 + D // 8, 0, "decode_stream_kernel", "decode.cu", launches=2),
        ]
        W.update(units=G * Nd, unit="tokens/s", inputs=[newk, newv, q], outputs=[out], dtype="bf16",
                 desc="%s: D-FQJL sigma_rel 0.5, B=32, 32 heads, N=16384 in 256-token pages (shuffled block "
                      "table), d=128, m=256; append 1 key + 2-bit value per head, project queries, fused paged "
                      "decode" % name)
    elif name == "prefill_causal":
        # causal prefill of 32 heads x 4096 tokens (d=128, m=256 dense): sketch the keys, quantize the values,
        # project every position's query, then the fused causal attention; units are query-key pairs
        Gp, Lp, m = 32, 4096, 256
        P = qjl.Projection(2, D, m, "dense", s_bf16=True)
        keys, vals = wl.decode_kv(dev, B=1, H=Gp, N=Lp, d=D)
        keys, vals = keys.reshape(-1, D), vals.reshape(-1, D)
        q = wl.normal((Gp * Lp, D), 407, dev)
        bits = torch.empty((Gp * Lp, m // 32), dtype=torch.int32, device=dev)
        norms = torch.empty((Gp * Lp,), dtype=torch.float32, device=dev)
        codes = torch.empty((Gp * Lp, D // 16), dtype=torch.int32, device=dev)
        sc = torch.empty((Gp * Lp, D // 32), dtype=torch.float16, device=dev)
        zr = torch.empty((Gp * Lp, D // 32), dtype=torch.float16, device=dev)
        sq = torch.empty((Gp * Lp, m), dtype=torch.float32, device=dev)
        out = torch.empty((Gp, Lp, D), dtype=torch.float32, device=dev)
        pairs = Gp * Lp * (Lp + 1) // 2
        stages = [
            Stage("quantize_keys", lambda: qjl.quantize_keys(P, keys, bits=bits, norms=norms), Gp * Lp,
                  2 * D + m // 8 + 4, 2 * D * m, "dense_tc_kernel", "dense_tc.cu"),
            Stage("quantize_values", lambda: qjl.quantize_values_2bit(vals, codes=codes, scale=sc, zero=zr), Gp * Lp,
                  2 * D + D // 4 + D // 8),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), Gp * Lp, 4 * D + 4 * m,
                  kernel="project_mma_kernel", src="project_mma.cu"),
            # work per (query, key) pair: 2 d flops of P.V plus 2 m of sign-dot multiply-adds
            Stage("prefill_attention", lambda: qjl.prefill_attention(
                P, bits.view(Gp, Lp, -1), norms.view(Gp, Lp), codes.view(Gp, Lp, -1), sc.view(Gp, Lp, -1),
                zr.view(Gp, Lp, -1), sq.view(Gp, Lp, m), 1.0 / math.sqrt(D), out=out), pairs, 0, 2 * D + 2 * m,
                "prefill_tc_kernel", "prefill.cu", "tensor"),
        ]
        W.update(units=pairs, unit="query-key pairs/s", inputs=[keys, vals, q], outputs=[out], dtype="bf16",
                 desc="%s: 32 heads x 4096 tokens, d=128, m=256 dense bf16 S; quantize keys and 2-bit values, project "
                      "all queries, fused causal attention" % name)
    elif name == "kivi_keys_decode":
        # the KIVI per-channel 2-bit key baseline on the decode_llama7b keys: quantize every key per
        # channel (32-token blocks) and score one query per head; "accuracy" compares its scores and the
        # QJL sketch's (dense, m=256) with the exact inner products on sampled heads
        G = B * H
        keys = wl.llama_keys(dev, B=B, H=H, N=N, d=D).reshape(G, N, D)
        q = wl.llama_queries(dev, B=B, H=H, d=D).reshape(G, 1, D)
        nb = (N + 31) // 32
        codes = torch.empty((G, N, D // 16), dtype=torch.int32, device=dev)
        sc = torch.empty((G, nb, D), dtype=torch.float16, device=dev)
        zr = torch.empty((G, nb, D), dtype=torch.float16, device=dev)
        out = torch.empty((G, 1, N), dtype=torch.float32, device=dev)
        stages = [
            Stage("kivi_quantize_keys", lambda: qjl.kivi_quantize_keys_2bit(keys, codes, sc, zr), G * N,
                  2 * D + D // 4 + 4 * D // 32, 0, "kivi_keys_quantize_kernel", "kivi_keys.cu"),
            Stage("kivi_key_scores", lambda: qjl.kivi_key_scores(codes, sc, zr, q, out=out), G * N,
                  D // 4 + 4 * D // 32 + 4, 0, "kivi_key_scores_kernel", "kivi_keys.cu"),
        ]
        W.update(units=G * N, unit="keys/s", inputs=[keys, q], outputs=[out], dtype="bf16",
                 desc="%s: KIVI per-channel 2-bit keys (32-token blocks, fp16 scale/zero, 48 B/key) on B=8, "
                      "heads=32, N=32768, d=128; quantize all keys, score 1 query/head" % name)

        def accuracy(heads=(0, 37, 101, 255)):
            import numpy as np
            Pq = qjl.Projection(2, D, M, "dense", s_bf16=True)
            res = {"sampled_heads": len(heads), "keys_per_head": N}
            errs = {"kivi_2bit_per_channel": [], "qjl_dense_m256": []}
            exact_all = []
            for g in heads:
                kh = keys[g].double().cpu().numpy()
                qh = q[g, 0].double().cpu().numpy()
                exact = kh @ qh
                bits, nrm = qjl.quantize_keys(Pq, keys[g])
                sqh = qjl.project_queries(Pq, q[g])
                est = qjl.scores(Pq, bits.view(1, N, M // 32), nrm.view(1, N), sqh.view(1, 1, M))
                errs["qjl_dense_m256"].append(est[0, 0].double().cpu().numpy() - exact)
                errs["kivi_2bit_per_channel"].append(out[g, 0].double().cpu().numpy() - exact)
                exact_all.append(exact)
            ex = np.concatenate(exact_all)
            for k, e in errs.items():
                e = np.concatenate(e)
                res[k] = {"rel_rms_error": float(np.sqrt((e * e).mean() / (ex * ex).mean())),
                          "bytes_per_key": 48 if k.startswith("kivi") else M // 8 + 4}
            return res
        W["accuracy"] = accuracy
    else:
        raise SystemExit("unknown workload %s" % name)
    W["stages"] = stages
    return W


PER_CONFIG = ["dense_1head", "gqa_decode", "pfqjl_bulk_m256", "pfqjl_bulk_m1024", "dfqjl_decode"]


def stage_roof(st, ms, pk):
    """A stage's achieved rate on its binding roof: HBM bytes, bf16 tensor flops or fp32 lane operations."""
    t = ms * 1e-3
    gbs = st.units * st.bytes_per_unit / t / 1e9
    e = {"ms": ms, "units_per_s": st.units / t, "gbs": gbs, "frac_hbm_measured": gbs / pk["hbm_gbs"],
         "frac_8tbs": gbs / 8000.0, "bytes_per_unit": st.bytes_per_unit, "bound": st.bound}
    if st.flops_per_unit:
        e["flops_per_unit"] = st.flops_per_unit
        e["tflops"] = st.units * st.flops_per_unit / t / 1e12
    if st.alu_ops_per_unit:
        e["alu_ops_per_unit"] = st.alu_ops_per_unit
        e["alu_tops"] = st.units * st.alu_ops_per_unit / t / 1e12
        e["alu_frac"] = e["alu_tops"] / FP32_TFLOPS
    if st.bound == "tensor":
        e["frac"] = e["tflops"] / (st.peak_scale * pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))
        e["frac_of"] = ("bf16 tensor peak (sustained, measured)" if st.peak_scale == 1.0 else
                        "int8 tensor peak: measured bf16 (sustained) x 2, the nominal int8 : bf16 ratio")
        e["frac_burst"] = e["tflops"] / (st.peak_scale * pk["bf16_tflops"])
    elif st.bound == "alu":
        e["frac"] = e["tflops"] / FP32_TFLOPS
        e["frac_of"] = "FP32 lane ceiling (derived: 148 SMs x 128 lanes x 1.965 GHz)"
    elif st.bound == "launch":
        e["frac"] = None
        e["frac_of"] = "launch-bound (microseconds of work)"
    else:
        e["frac"] = e["frac_hbm_measured"]
        e["frac_of"] = "HBM copy bandwidth (measured)"
    return e


def time_region(stages, steps, stream, torch, world, local, period_ms=50):
    """Time `steps` whole steps (events around every stage) between barriers, with clocks sampled."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local, period_ms) as clk:
        clk.mark()
        t_start.record(stream)
        for i in range(steps):
            for j, st in enumerate(stages):
                evs[i][j].record(stream)
                st.fn()
            evs[i][len(stages)].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        clk.mark()
    barrier(world)
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), world)
    k_ms = [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i in range(len(stages))]
    return ms_total / steps, k_ms, clk.summary()


def analyse(Wk, k_ms, pk, workload):
    stages = Wk["stages"]
    kernels = {st.name: stage_roof(st, ms, pk) for st, ms in zip(stages, k_ms)}
    dom = max(range(len(stages)), key=lambda i: k_ms[i])
    ds = stages[dom]
    e = kernels[ds.name]
    roof = {"bound": "hbm", "kernel": "%s (%s)" % (ds.kernel, ds.name), "achieved": e["gbs"],
            "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": e["frac_hbm_measured"], "peak_kind": pk["kind"],
            "traffic": ncu_traffic(ds.kernel, workload, ds.src) if ds.src else None,
            "bytes_per_launch": ds.units * ds.bytes_per_unit}
    if ds.bound == "alu":
        roof.update({"bound": "alu", "achieved": e["tflops"], "peak": FP32_TFLOPS, "unit": "TFLOP/s",
                     "frac": e["frac"], "peak_kind": "derived: 148 SMs x 128 FP32 lanes x 1.965 GHz",
                     "flops_per_launch": ds.units * ds.flops_per_unit, "hbm_gbs": e["gbs"],
                     "hbm_frac": e["frac_hbm_measured"]})
    elif ds.bound == "tensor":
        roof.update({"bound": "tensor", "achieved": e["tflops"],
                     "peak": ds.peak_scale * pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                     "unit": "TFLOP/s", "frac": e["frac"], "peak_kind": pk["kind"] + " (bf16, sustained)",
                     "flops_per_launch": ds.units * ds.flops_per_unit // ds.launches, "hbm_gbs": e["gbs"],
                     "hbm_frac": e["frac_hbm_measured"]})
        if ds.alu_ops_per_unit:
            roof.update({"alu_tops": e["alu_tops"], "alu_frac": e["alu_frac"]})
    elif ds.flops_per_unit:
        roof["tensor_tflops"] = e["tflops"]
        roof["tensor_frac_of_sustained"] = e["tflops"] / pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    return kernels, roof


def cold_leg(stage, torch, stream, reps=20):
    """One stage timed alone, L2 flushed before every call by reading a 256 MB buffer. A read flush
    leaves L2 full of clean lines: a write flush would leave dirty ones whose write-back the timed
    call would pay for (and the earlier calls' own dirty outputs are written back during the flush)."""
    flush = torch.ones((64 << 20,), dtype=torch.float32, device=torch.cuda.current_device())
    ts = []
    for r in range(reps + 3):
        flush.sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        stage.fn()
        b.record(stream)
        torch.cuda.synchronize()
        if r >= 3:
            ts.append(a.elapsed_time(b))
    del flush
    return statistics.median(ts), statistics.mean(ts), reps


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["decode_llama7b", "gqa_decode", "dense_1head", "pfqjl_bulk_m256", "pfqjl_bulk_m1024",
                             "dfqjl_decode", "paged_decode", "kivi_keys_decode", "prefill_causal"])
    ap.add_argument("--ref-sample", type=int, default=4096)
    ap.add_argument("--profile-case", default=None,
                    choices=["quantize", "scores", "fqjl", "fqjl1024", "dfqjl", "values", "decode", "prefill",
                             "many256", "many1024"],
                    help="run one small case of a single kernel (3 launches after 2 warm-ups) for ncu")
    ap.add_argument("--profile-keys", type=int, default=1 << 20)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--sustained-seconds", type=float, default=2.5,
                    help="length of the sustained leg (the headline step repeated under the power cap)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the other configs (single-GPU runs only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_case:
        return profile_case(args.profile_case, args.profile_keys)

    import torch
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import bit_kv_cache_qjl_b200 as qjl
    from bit_kv_cache_qjl_b200 import workloads as wl

    pk, pk_kind = peaks()
    pk = dict(pk, kind=pk_kind)
    stream = torch.cuda.current_stream()

    Wk = build_workload(args.workload, dev, qjl, wl, torch)
    stages = Wk["stages"]

    def step():
        for st in stages:
            st.fn()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ms_step, k_ms, clocks = time_region(stages, args.steps, stream, torch, world, local)
    units = Wk["units"]
    value = job_throughput(units, world, ms_step)
    kernels, roof = analyse(Wk, k_ms, pk, args.workload)

    # the score stage alone, L2 flushed before every call: its HBM fraction without any L2-resident
    # tail of the bits that the quantize stage has just written
    cold = None
    sc_stage = next((st for st in stages if st.name == "scores"), None)
    if sc_stage is not None:
        med, mean, reps = cold_leg(sc_stage, torch, stream)
        cold = dict(stage_roof(sc_stage, med, pk), kernel=sc_stage.kernel, reps=reps, ms_mean=mean,
                    rule="median of %d calls, each after a 256 MB read that flushes L2 (clean lines)" % reps)

    # sustained: the same step repeated for a few seconds, long enough for the 1 kW power cap to act
    n_sus = max(args.steps, int(math.ceil(args.sustained_seconds * 1e3 / ms_step)))
    s_ms, s_k, s_clk = time_region(stages, n_sus, stream, torch, world, local, period_ms=100)
    s_kern, s_roof = analyse(Wk, s_k, pk, args.workload)
    sustained = {"steps": n_sus, "ms_per_step": s_ms, "value": job_throughput(units, world, s_ms),
                 "kernels": {k: {"ms": v["ms"], "frac": v["frac"], "frac_of": v["frac_of"]} for k, v in s_kern.items()},
                 "roofline_frac": s_roof["frac"], "clocks": s_clk}

    # end to end through the same calls with host buffers (pinned), copies inside the timed region
    h_in = []
    for t in Wk["inputs"]:
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        h_in.append(h)
    h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in Wk["outputs"]]
    torch.cuda.synchronize()

    def e2e_step():
        for t, h in zip(Wk["inputs"], h_in):
            t.copy_(h, non_blocking=True)
        step()
        for t, h in zip(Wk["outputs"], h_out):
            h.copy_(t, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world)
    h2d = sum(h.numel() * h.element_size() for h in h_in)
    d2h = sum(h.numel() * h.element_size() for h in h_out)
    accuracy = Wk["accuracy"]() if "accuracy" in Wk and rank == 0 else None
    w_unit, w_dtype, w_desc = Wk["unit"], Wk["dtype"], Wk["desc"]
    launches = sum(st.launches for st in stages) * args.steps
    del Wk, stages, h_in, h_out
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and args.workload in ORACLE_UNIT:
        cpu = cpu_baseline(args.workload)

    # the other configs, each timed the same way in this process, with the oracle beside it
    per_config = None
    if world == 1 and not args.no_per_config:
        per_config = {}
        for name in PER_CONFIG:
            if name == args.workload:
                continue
            W2 = build_workload(name, dev, qjl, wl, torch)
            st2 = W2["stages"]
            for _ in range(args.warmup):
                for st in st2:
                    st.fn()
            torch.cuda.synchronize()
            ms2, k2, clk2 = time_region(st2, args.steps, stream, torch, world, local)
            kern2, roof2 = analyse(W2, k2, pk, name)
            q = kern2.get("quantize_keys")
            per_config[name] = {
                "workload": W2["desc"], "value": W2["units"] / (ms2 * 1e-3), "unit": W2["unit"],
                "ms_per_step": ms2, "steps": args.steps, "kernels": kern2, "roofline": roof2,
                "quantize_vectors_per_s": q["units_per_s"] if q else None, "clocks": clk2,
                "cpu_baseline": None if args.no_cpu else cpu_baseline(name)}
            del W2, st2
            torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": w_unit,
        "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w_dtype, "data": "synthetic",
        "config": run_config(w_desc, units, world),
        "roofline": roof,
        "kernels": kernels,
        "scores_cold": cold,
        "sustained": sustained,
        "e2e": {"value": world * units / (e2e_ms * 1e-3), "unit": w_unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "per_config": per_config,
    }
    if accuracy is not None:
        line["accuracy"] = accuracy
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

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


def source_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel, workload, src):
    """Per-launch DRAM bytes from profiles/traffic.txt, valid only for the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    h = source_hash(os.path.join(ROOT, "bit_kv_cache_qjl_b200", "csrc", src))
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == kernel and f[1] == workload and f[3] == h:
            return float(f[2])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


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


def cpu_oracle_rate(sample_keys, seconds_hint=None):
    """Time the oracle (as it stands) on `sample_keys` keys of the workload: keys/s, threads."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle
    from bit_kv_cache_qjl_b200 import workloads as wl
    O = oracle.params.make_projection(2, D, M, oracle.params.KIND_DENSE, s_bf16=True)
    heads = max(1, sample_keys // N)
    per = min(N, sample_keys)
    keys = wl.llama_keys("cpu", B=1, H=heads, N=per).reshape(heads, per, D).to("cpu").float().numpy()
    q = wl.llama_queries("cpu", B=1, H=heads).reshape(heads, D).numpy()
    t0 = time.perf_counter()
    for h in range(heads):
        words, norms, _ = oracle.qjl.quantize_keys(O, keys[h].astype(np.float64))
        sq = oracle.qjl.project_queries(O, q[h:h + 1].astype(np.float64))
        oracle.qjl.scores(O, words[None], norms[None], sq[None])
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return heads * per / dt, dt, threads, heads * per


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
    sample = args.ref_sample
    for _ in range(args.warmup):
        cpu_oracle_rate(sample)
    total_keys, total_t = 0, 0.0
    threads = 1
    for _ in range(args.steps):
        rate, dt, threads, k = cpu_oracle_rate(sample)
        total_keys += k
        total_t += dt
    value = total_keys / total_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": run_config(default_desc(), B * H * N, world),
            "cpu_baseline": {"value": value, "unit": "keys/s", "cores": threads, "kind": "oracle",
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
                 launches=1):
        self.name, self.fn, self.units, self.launches = name, fn, units, launches
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
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), G, 4 * D + 4 * M),
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
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), G * J, 4 * D + 4 * m),
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
                  2 * D * M, "dense_simt_kernel", "dense_simt.cu"),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), J, 4 * D + 4 * M),
            Stage("scores", lambda: qjl.scores(P, bits.view(1, n, M // 32), norms.view(1, n), sq.view(1, J, M), out=out),
                  n, M // 8 + 4 + 4 * J, 0, "scores_stream_kernel", "scores.cu"),
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
            Stage("quantize_keys", lambda: qjl.quantize_keys(P, keys, bits=bits, norms=norms), n,
                  2 * d + m // 8 + 4, fqjl_flops_per_key(d, m), "fqjl_keys_kernel", "fqjl_keys.cu", "alu"),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), J, 4 * d + 4 * m),
            Stage("scores", lambda: qjl.scores(P, bits[:ns].view(1, ns, m // 32), norms[:ns].view(1, ns),
                                               sq.view(1, J, m), out=out), ns, m // 8 + 4 + 4 * J, 0,
                  "scores_stream_kernel", "scores.cu"),
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
            Stage("quantize_keys", lambda: qjl.quantize_keys(P, keys, bits=bits, norms=norms), G * Nd,
                  2 * D + m // 8 + 4, fqjl_flops_per_key(D, m), "fqjl_keys_kernel", "fqjl_keys.cu", "alu"),
            Stage("quantize_values", lambda: qjl.quantize_values_2bit(vals, codes=codes, scale=sc, zero=zr), G * Nd,
                  2 * D + D // 4 + D // 8, 0, "values_2bit_kernel", "values.cu"),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), G, 4 * D + 4 * m),
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
                  fqjl_flops_per_key(D, m)),
            Stage("append_values", lambda: qjl.append_values_2bit(cache, newv, pos), G, 2 * D + D // 4 + D // 8),
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), G, 4 * D + 4 * m),
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
            Stage("project_queries", lambda: qjl.project_queries(P, q, out=sq), Gp * Lp, 4 * D + 4 * m),
            # work per (query, key) pair: 2 d flops of P.V plus 2 m of sign-dot multiply-adds
            Stage("prefill_attention", lambda: qjl.prefill_attention(
                P, bits.view(Gp, Lp, -1), norms.view(Gp, Lp), codes.view(Gp, Lp, -1), sc.view(Gp, Lp, -1),
                zr.view(Gp, Lp, -1), sq.view(Gp, Lp, m), 1.0 / math.sqrt(D), out=out), pairs, 0, 2 * D + 2 * m,
                "prefill_kernel", "prefill.cu", "tensor"),
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["decode_llama7b", "gqa_decode", "dense_1head", "pfqjl_bulk_m256", "pfqjl_bulk_m1024",
                             "dfqjl_decode", "paged_decode", "kivi_keys_decode", "prefill_causal"])
    ap.add_argument("--ref-sample", type=int, default=4096)
    ap.add_argument("--cpu-sample", type=int, default=1 << 21)
    ap.add_argument("--profile-case", default=None,
                    choices=["quantize", "scores", "fqjl", "fqjl1024", "dfqjl", "values", "decode", "prefill"],
                    help="run one small case of a single kernel (3 launches after 2 warm-ups) for ncu")
    ap.add_argument("--profile-keys", type=int, default=1 << 20)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu", action="store_true")
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

    Wk = build_workload(args.workload, dev, qjl, wl, torch)
    stages = Wk["stages"]
    stream = torch.cuda.current_stream()

    def step(ev=None):
        for i, st in enumerate(stages):
            if ev is not None:
                ev[i].record(stream)
            st.fn()
        if ev is not None:
            ev[len(stages)].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), world)
    ms_step = ms_total / args.steps
    k_ms = [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i in range(len(stages))]
    units = Wk["units"]
    value = job_throughput(units, world, ms_step)

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

    pk, pk_kind = peaks()
    hbm = pk["hbm_gbs"]
    tf = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    kernels = {}
    for st, ms in zip(stages, k_ms):
        gbs = st.units * st.bytes_per_unit / (ms * 1e-3) / 1e9
        e = {"ms": ms, "units_per_s": st.units / (ms * 1e-3), "gbs": gbs, "frac_hbm_measured": gbs / hbm,
             "frac_8tbs": gbs / 8000.0, "bytes_per_unit": st.bytes_per_unit}
        if st.flops_per_unit:
            e["tflops"] = st.units * st.flops_per_unit / (ms * 1e-3) / 1e12
        kernels[st.name] = e
    dom = max(range(len(stages)), key=lambda i: k_ms[i])
    ds = stages[dom]
    d_gbs = kernels[ds.name]["gbs"]
    roof = {"bound": "hbm", "kernel": "%s (%s)" % (ds.kernel, ds.name), "achieved": d_gbs, "peak": hbm,
            "unit": "GB/s", "frac": d_gbs / hbm, "peak_kind": pk_kind,
            "traffic": ncu_traffic(ds.kernel, args.workload, ds.src) if ds.src else None,
            "bytes_per_launch": ds.units * ds.bytes_per_unit}
    if ds.bound == "alu":
        # the Walsh-Hadamard transform is bound by fp32 issue, not by HBM: report its fp32 operation
        # rate against the FP32 lane ceiling, and keep the HBM fraction beside it
        tfl = kernels[ds.name]["tflops"]
        roof.update({"bound": "alu", "achieved": tfl, "peak": FP32_TFLOPS, "unit": "TFLOP/s",
                     "frac": tfl / FP32_TFLOPS, "peak_kind": "derived: 148 SMs x 128 FP32 lanes x 1.965 GHz",
                     "flops_per_launch": ds.units * ds.flops_per_unit, "hbm_gbs": d_gbs, "hbm_frac": d_gbs / hbm})
    elif ds.bound == "tensor":
        tfl = kernels[ds.name]["tflops"]
        roof.update({"bound": "tensor", "achieved": tfl, "peak": tf, "unit": "TFLOP/s", "frac": tfl / tf,
                     "peak_kind": pk_kind + " (bf16, sustained)", "flops_per_launch": ds.units * ds.flops_per_unit,
                     "hbm_gbs": d_gbs, "hbm_frac": d_gbs / hbm})
    elif ds.flops_per_unit:
        roof["tensor_tflops"] = kernels[ds.name]["tflops"]
        roof["tensor_frac_of_sustained"] = kernels[ds.name]["tflops"] / tf
    clocks = clk.summary()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and args.workload == WORKLOAD:
        rate, dt, threads, k = cpu_oracle_rate(args.cpu_sample)
        cpu = {"value": rate, "unit": "keys/s", "cores": threads, "kind": "oracle",
               "sample": "%d keys of the workload (%d head slices of %d keys): oracle quantize + project + "
                         "score, %.1f s" % (k, max(1, k // N), min(N, k), dt)}

    line = {
        "metric": METRIC, "value": value, "unit": Wk["unit"], "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": Wk["dtype"], "data": "synthetic",
        "config": run_config(Wk["desc"], units, world),
        "roofline": roof,
        "kernels": kernels,
        "e2e": {"value": world * units / (e2e_ms * 1e-3), "unit": Wk["unit"], "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": sum(st.launches for st in stages) * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if "accuracy" in Wk and rank == 0:
        line["accuracy"] = Wk["accuracy"]()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

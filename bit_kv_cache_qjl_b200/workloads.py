"""Seeded synthetic inputs for the five workloads (input generation only).

This module holds none of the method's arithmetic. It draws keys, values and
queries with the shapes and value distributions of the workloads below and
returns torch tensors. Tests pass the same tensors to the CUDA library and,
as host copies, to the oracle. The pages name no dataset or benchmark, so
every input is synthetic by definition.

Workloads (sizes as run by bench.py; tests shrink N or n and keep the rest):
  dense_1head     d=128, m=256, fp32 S (seed 1); 4096 keys and 16 queries iid
                  N(0,1) fp32 (seed 101).
  decode_llama7b  B=8, 32 heads, d=128, m=256, bf16 S (seed 2), N=32768; bf16
                  keys N(0,1) with 4 outlier channels per head scaled x10
                  (channels from randperm(128) under seed 202+h); 1 fp32
                  query per head (seed 203).
  gqa_decode      B=16, 32 query heads over 8 KV heads, d=128, m=512 (seed 3),
                  N=131072; bf16 keys N(0,1) times a per-(KV head, channel)
                  scale exp(U[ln 0.5, ln 8]) (seed 303); queries fp32 (seed 304).
  pfqjl_bulk      P-FQJL (seed 4), 2^24 keys d=256 bf16 N(0,1) (seed 404),
                  m=256 and m=1024; the first 2^20 keys scored against 64
                  queries (seed 405).
  dfqjl_decode    D-FQJL (seed 5, sigma_rel 0.5), B=32, 32 heads, d=128, m=256,
                  N=16384; keys and values bf16 N(0,1) (seeds 505, 506);
                  queries fp32 (seed 507).
"""

import math

import torch

WORKLOADS = {
    "dense_1head": dict(kind="dense", d=128, m=256, proj_seed=1, s_bf16=False, n=4096, nq=16,
                        key_seed=101, key_dtype=torch.float32),
    "decode_llama7b": dict(kind="dense", d=128, m=256, proj_seed=2, s_bf16=True, B=8, H=32, N=32768,
                           key_seed=202, query_seed=203, key_dtype=torch.bfloat16),
    "gqa_decode": dict(kind="dense", d=128, m=512, proj_seed=3, s_bf16=True, B=16, Hq=32, Hkv=8, N=131072,
                       key_seed=303, query_seed=304, key_dtype=torch.bfloat16),
    "pfqjl_bulk": dict(kind="pfqjl", d=256, ms=(256, 1024), proj_seed=4, n=1 << 24, n_score=1 << 20, nq=64,
                       key_seed=404, query_seed=405, key_dtype=torch.bfloat16),
    "dfqjl_decode": dict(kind="dfqjl", d=128, m=256, proj_seed=5, sigma_rel=0.5, B=32, H=32, N=16384,
                         key_seed=505, value_seed=506, query_seed=507, key_dtype=torch.bfloat16),
}


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, seed, device="cpu", dtype=torch.float32):
    """iid N(0,1) of ``shape`` drawn in fp32 under ``seed``, cast to ``dtype``."""
    x = torch.randn(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.to(dtype)


def dense_1head(device="cpu", n=4096, nq=16):
    w = WORKLOADS["dense_1head"]
    keys = normal((n, w["d"]), w["key_seed"], device)
    queries = normal((nq, w["d"]), w["key_seed"] + 1000, device)
    return keys, queries


def llama_keys(device="cpu", B=8, H=32, N=32768, d=128, seed=202, outliers=4, factor=10.0):
    """[B, H, N, d] bf16 keys N(0,1) with `outliers` channels per head scaled by `factor`."""
    keys = normal((B, H, N, d), seed, device)
    for h in range(H):
        ch = torch.randperm(d, generator=_gen(seed + h, "cpu"))[:outliers].to(device)
        keys[:, h, :, ch] *= factor
    return keys.to(torch.bfloat16)


def llama_queries(device="cpu", B=8, H=32, d=128, seed=203):
    return normal((B, H, d), seed, device)


def gqa_keys(device="cpu", B=16, Hkv=8, N=131072, d=128, seed=303):
    """[B, Hkv, N, d] bf16 keys N(0,1) times per-(KV head, channel) log-uniform scales in [0.5, 8]."""
    g = _gen(seed, "cpu")
    u = torch.rand((Hkv, d), generator=g)
    scale = torch.exp(math.log(0.5) + u * (math.log(8.0) - math.log(0.5))).to(device)
    keys = normal((B, Hkv, N, d), seed + 1, device)
    keys *= scale[None, :, None, :]
    return keys.to(torch.bfloat16)


def gqa_queries(device="cpu", B=16, Hq=32, d=128, seed=304):
    return normal((B, Hq, d), seed, device)


def bulk_keys(device="cpu", n=1 << 24, d=256, seed=404):
    return normal((n, d), seed, device, torch.bfloat16)


def bulk_queries(device="cpu", nq=64, d=256, seed=405):
    return normal((nq, d), seed, device)


def decode_kv(device="cpu", B=32, H=32, N=16384, d=128, key_seed=505, value_seed=506):
    keys = normal((B, H, N, d), key_seed, device, torch.bfloat16)
    values = normal((B, H, N, d), value_seed, device, torch.bfloat16)
    return keys, values


def decode_queries(device="cpu", B=32, H=32, d=128, seed=507):
    return normal((B, H, d), seed, device)

"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle runs.

This module only draws random numbers and lays them out; it holds none of the
attention method's arithmetic (no RoPE, no windows, no softmax).

Recipe: every (tensor, batch, head) slab comes from its own numpy PCG64 stream
seeded with ``[seed, workload_id, tensor_id, b, head]``; values are standard
normal fp32 and are rounded to bf16 (round-to-nearest-even, by torch) where the
workload is bf16.  The "pair energy" variant multiplies both components of
frequency pair i of every token by ``1 + 0.5*sin(phase)`` with one uniform
phase per (tensor, head, pair), drawn from its own stream.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

DEFAULT_SEED = 20260803

T_Q, T_K, T_V = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtype and the method's parameters."""

    name: str
    wid: int                 # workload id, part of every RNG seed
    batch: int
    q_heads: int
    kv_heads: int
    d: int
    seq: int                 # prefill: sequence length; decode: cache length
    dtype: torch.dtype
    theta: float
    alphas: tuple
    pair_energy: bool = False
    q_chunk: int = 0         # >0: causal prefill in query chunks of this size
    decode: bool = False


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 1, 1, 1, 64, 512, torch.float32, 1e4, (1.0,)),
    "layer_8k": Workload("layer_8k", 2, 1, 28, 4, 128, 8192, torch.bfloat16, 1e7,
                         (0.5, 1.0, 2.0, math.inf)),
    "layer_32k_pair_energy": Workload("layer_32k_pair_energy", 3, 1, 28, 4, 128, 32768, torch.bfloat16,
                                      1e7, (1.0,), pair_energy=True),
    "layer_128k_chunked": Workload("layer_128k_chunked", 4, 1, 28, 4, 128, 131072, torch.bfloat16, 1e7,
                                   (0.5, 1.0), q_chunk=8192),
    "decode_1m": Workload("decode_1m", 5, 4, 28, 4, 128, 1 << 20, torch.bfloat16, 1e7, (1.0,),
                          decode=True),
}


def _slab(seed, wid, tensor_id, b, head, n, d) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64([seed, wid, tensor_id, b, head]))
    return rng.standard_normal((n, d), dtype=np.float32)


def _pair_scale(seed, wid, tensor_id, head, d) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64([seed, wid, 100 + tensor_id, head]))
    phase = rng.uniform(0.0, 2.0 * math.pi, size=d // 2)
    s = (1.0 + 0.5 * np.sin(phase)).astype(np.float32)
    return np.repeat(s, 2)  # both components of a pair share the factor


def token_major(seed, wid, tensor_id, batch, n, heads, d, dtype=torch.bfloat16, pair_energy=False,
                threads: int = 8) -> torch.Tensor:
    """A [batch][n][heads][d] CPU tensor of seeded N(0,1) values in ``dtype``."""
    out = torch.empty((batch, n, heads, d), dtype=dtype)

    def fill(bh):
        b, h = bh
        x = _slab(seed, wid, tensor_id, b, h, n, d)
        if pair_energy:
            x *= _pair_scale(seed, wid, tensor_id, h, d)[None, :]
        out[b, :, h, :] = torch.from_numpy(x).to(dtype)

    jobs = [(b, h) for b in range(batch) for h in range(heads)]
    if threads > 1 and len(jobs) > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(fill, jobs))
    else:
        for j in jobs:
            fill(j)
    return out


def prefill_inputs(w: Workload, seed: int = DEFAULT_SEED, seq: int | None = None):
    """(q, k, v) CPU tensors for a prefill workload, token-major [B][S][H][d]."""
    S = w.seq if seq is None else seq
    q = token_major(seed, w.wid, T_Q, w.batch, S, w.q_heads, w.d, w.dtype, w.pair_energy)
    k = token_major(seed, w.wid, T_K, w.batch, S, w.kv_heads, w.d, w.dtype, w.pair_energy)
    v = token_major(seed, w.wid, T_V, w.batch, S, w.kv_heads, w.d, w.dtype, False)
    return q, k, v


def decode_inputs(w: Workload, seed: int = DEFAULT_SEED, n_cache: int | None = None):
    """(q [B][Hq][d], k_rot [B][N][Hkv][d], v [B][N][Hkv][d]) CPU tensors.

    The key cache values are used as already-rotated keys (the workload's cache
    holds keys after RoPE); q is the raw new query of each sequence."""
    N = w.seq if n_cache is None else n_cache
    q = token_major(seed, w.wid, T_Q, w.batch, 1, w.q_heads, w.d, w.dtype)[:, 0].contiguous()
    k = token_major(seed, w.wid, T_K, w.batch, N, w.kv_heads, w.d, w.dtype)
    v = token_major(seed, w.wid, T_V, w.batch, N, w.kv_heads, w.d, w.dtype)
    return q, k, v


def random_prefill(batch, q_len, kv_len, q_heads, kv_heads, d, dtype, seed, wid=900):
    """Small seeded (q, k, v) for tests: q [B][q_len][Hq][d], k/v [B][kv_len][Hkv][d]."""
    q = token_major(seed, wid, T_Q, batch, q_len, q_heads, d, dtype, threads=1)
    k = token_major(seed, wid, T_K, batch, kv_len, kv_heads, d, dtype, threads=1)
    v = token_major(seed, wid, T_V, batch, kv_len, kv_heads, d, dtype, threads=1)
    return q, k, v

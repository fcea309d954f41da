"""Split-KV decode across devices: each rank holds a contiguous range of every
sequence's key positions, decodes the query against its range
(atf_decode_partial), the ranks exchange their partials with one all-gather over
the process group (NCCL over NVLink between GPUs), and every rank merges them
(atf_decode_merge) into the full output.

The exchange is the only communication: B x Hq x (d + 2) fp32 per rank
(58 KB for 4 sequences x 28 heads x d = 128), independent of the cache length.
Ranges are balanced by decode traffic rather than by key count: a key near the
query reads more of its 8-pair chunks (more pairs still inside their windows) than
a far one, so the ranges near the query are shorter.
"""
from __future__ import annotations

import contextlib
import math

import numpy as np

from . import atf


def key_traffic(distance: np.ndarray, W: np.ndarray, d: int) -> np.ndarray:
    """Decode traffic of keys at the given distances from the query, in 32-byte
    units: the value row (d/16 units) plus each 8-pair key chunk whose highest
    pair's window still reaches the key (chunk c is read while distance <= W[8c+7])."""
    wc = np.asarray(W, dtype=np.int64)[7::8]  # W of each chunk's last (widest) pair
    live = (np.asarray(distance, dtype=np.int64)[:, None] <= wc[None, :]).sum(axis=1)
    return d // 16 + live


def shard_ranges(n_keys: int, world: int, d: int, theta: float, alpha: float) -> list[tuple[int, int]]:
    """Contiguous key-position ranges [lo, hi) of one sequence of n_keys keys (its
    query at position n_keys - 1), one per rank, with near-equal decode traffic.
    Every key is in exactly one range; ranges may be empty when world > n_keys."""
    if world < 1 or n_keys < 0:
        raise ValueError("world >= 1 and n_keys >= 0 required")
    if n_keys == 0:
        return [(0, 0)] * world
    W = atf.atf_windows(d, theta, alpha) if not math.isinf(alpha) else np.full(d // 2, 2**62, dtype=np.int64)
    dist = (n_keys - 1) - np.arange(n_keys, dtype=np.int64)
    cum = np.concatenate([[0], np.cumsum(key_traffic(dist, W, d))])
    total = int(cum[-1])
    cuts = [0]
    for r in range(1, world):
        cuts.append(int(np.searchsorted(cum, total * r / world, side="left")))
    cuts.append(n_keys)  # non-decreasing: cum is, and so are the targets
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def _gpu_partial(q, kc, v, n_keys, key_pos0, q_pos, theta, alpha, pairing, stream):
    import torch

    B, Hq, d = q.shape
    _, Hkv, _, N, _ = kc.shape
    part = torch.empty((B, Hq, d + 2), dtype=torch.float32, device=q.device)
    need = atf.atf_decode_workspace_bytes(B, Hq, Hkv, int(max(max(n_keys), 1)), d)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    atf.atf_decode_partial(q, kc, v, part, B, n_keys, key_pos0, q_pos, N, Hq, Hkv, d, theta, alpha, ws, need,
                           None, stream, pairing)
    return part


def _torch_stream(stream, device):
    """The torch stream object for a stream argument of the binding (None: torch's
    current stream, an int: a raw cudaStream_t handle, else a torch stream)."""
    import torch

    if stream is None:
        return None
    if isinstance(stream, int):
        return torch.cuda.ExternalStream(stream, device=device)
    return stream


def _gpu_merge(parts, world, B, Hq, d, stream):
    import torch

    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=parts.device)
    atf.atf_decode_merge(parts, world, B, Hq, d, out, stream)
    return out


def decode_split_kv(q, kc_local, v_local, n_keys_local, key_pos0, q_pos, theta, alpha, group=None,
                    pairing=atf.ATF_PAIRS_INTERLEAVED, stream=None, partial_fn=None, merge_fn=None):
    """One decode step of sequences whose caches are split across the ranks of
    `group` (torch.distributed).  This rank's cache holds, for sequence b,
    n_keys_local[b] rotated keys at positions key_pos0[b] .. (chunk-major
    kc_local [B][Hkv][d/16][N][16], values v_local [B][N][Hkv][d]); the query q
    [B][Hq][d] (raw, rotated here at q_pos[b]) is the same on every rank.
    Returns the merged output [B][Hq][d] on every rank.

    partial_fn / merge_fn replace the GPU partial and merge (same arguments and
    layouts); the exchange and the bookkeeping are the same either way."""
    import torch
    import torch.distributed as dist

    B, Hq, d = q.shape
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    part = (partial_fn or _gpu_partial)(q, kc_local, v_local, list(n_keys_local), list(key_pos0), list(q_pos),
                                       theta, alpha, pairing, stream)
    if world > 1:
        # the partial was written on `stream`: issue the exchange on that stream too,
        # so the gather reads the partial only after the kernel that writes it, and
        # the merge (also on `stream`) reads the gathered parts only after the gather
        ts = _torch_stream(stream, part.device) if part.is_cuda else None
        with (torch.cuda.stream(ts) if ts is not None else contextlib.nullcontext()):
            if dist.get_backend(group) == "nccl":
                gathered = torch.empty((world,) + tuple(part.shape), dtype=part.dtype, device=part.device)
                dist.all_gather_into_tensor(gathered, part.contiguous(), group=group)
            else:
                pieces = [torch.empty_like(part) for _ in range(world)]
                dist.all_gather(pieces, part.contiguous(), group=group)
                gathered = torch.stack(pieces)
    else:
        gathered = part[None]
    return (merge_fn or _gpu_merge)(gathered, world, B, Hq, d, stream)

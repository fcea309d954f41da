"""Split-KV decode on the CPU: the oracle's partial/merge pinned against the C
decode oracle, the traffic-balanced shard ranges, and the two-rank exchange of
decode_split_kv over gloo with oracle partials and merge."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from oracle import splitkv as osk
from rope_frequency_sparse_b200 import splitkv, synth


def _inputs(B, N, Hq, Hkv, d, seed):
    q = synth.token_major(seed, 950, 0, B, 1, Hq, d, torch.bfloat16, threads=1)[:, 0].contiguous()
    k = synth.token_major(seed, 950, 1, B, N, Hkv, d, torch.bfloat16, threads=1)
    v = synth.token_major(seed, 950, 2, B, N, Hkv, d, torch.bfloat16, threads=1)
    return q, k, v


@pytest.mark.parametrize("alpha", [1.0, 0.5, math.inf])
def test_merged_partials_equal_the_decode_oracle(alpha):
    B, N, Hq, Hkv, d, theta = 2, 300, 4, 2, 64, 1e4
    q, k, v = _inputs(B, N, Hq, Hkv, d, seed=81)
    want, _ = oracle.decode(q, k, v, [N, N], theta, alpha)
    for cuts in ([0, 300], [0, 1, 299, 300], [0, 150, 150, 300], [0, 17, 40, 222, 300]):
        parts = np.stack([osk.partial(q, k, v, [lo] * B, [hi] * B, [N - 1] * B, theta, alpha)
                          for lo, hi in zip(cuts[:-1], cuts[1:])])
        assert np.abs(osk.merge(parts) - want).max() < 1e-12, cuts


@pytest.mark.parametrize("alpha", [1.0, math.inf])
def test_partial_at_far_key_positions_equals_the_near_one(alpha):
    """Only distances enter the logits: keys rotated at key_pos0 + n with the query
    at key_pos0 + q_pos give the partial of keys at n with the query at q_pos (up to
    the fp64 error of angles near 2^31 * omega).  Ignoring key_pos0 would put every
    key about 2^31 away, outside every finite window."""
    B, N, Hq, Hkv, d, theta = 1, 400, 4, 2, 64, 1e4
    q, k, v = _inputs(B, N, Hq, Hkv, d, seed=83)
    P = (1 << 31) + 12345
    near = osk.partial(q, oracle.rope(k, theta), v, [0], [N], [N + 6], theta, alpha)
    far = osk.partial(q, oracle.rope(k, theta, pos0=P), v, [0], [N], [P + N + 6], theta, alpha, key_pos0=[P])
    assert np.abs(far - near).max() < 1e-5


def test_empty_range_merges_as_nothing():
    B, N, Hq, Hkv, d, theta = 1, 64, 2, 1, 64, 1e4
    q, k, v = _inputs(B, N, Hq, Hkv, d, seed=82)
    empty = osk.partial(q, k, v, [10], [10], [N - 1], theta, 1.0)
    assert np.all(np.isneginf(empty[..., d])) and np.all(empty[..., d + 1] == 0)
    full = osk.partial(q, k, v, [0], [N], [N - 1], theta, 1.0)
    assert np.array_equal(osk.merge(np.stack([empty, full])), osk.merge(full[None]))


@pytest.mark.parametrize("n,world,alpha", [(1 << 20, 8, 1.0), (5000, 3, 0.5), (100, 4, math.inf), (3, 5, 1.0)])
def test_shard_ranges_cover_and_balance(n, world, alpha):
    d, theta = 128, 1e7
    r = splitkv.shard_ranges(n, world, d, theta, alpha)
    assert len(r) == world and r[0][0] == 0 and r[-1][1] == n
    assert all(a[1] == b[0] for a, b in zip(r[:-1], r[1:])) and all(lo <= hi for lo, hi in r)
    W = np.full(d // 2, 2**62) if math.isinf(alpha) else oracle.windows(d, theta, alpha)[0]
    t = splitkv.key_traffic((n - 1) - np.arange(n), W, d)
    per = [int(t[lo:hi].sum()) for lo, hi in r]
    if n >= world:
        assert max(per) - min(per) <= 2 * int(t.max())  # equal up to the keys at the cuts
    if math.isinf(alpha) and n >= world:
        sizes = [hi - lo for lo, hi in r]
        assert max(sizes) - min(sizes) <= 1


def test_key_traffic_counts_live_chunks():
    W = np.array([3, 5, 7, 9, 11, 13, 15, 17] + [100] * 8)  # d = 32: two chunks, last pairs 17 and 100
    assert splitkv.key_traffic(np.array([0, 17, 18, 100, 101]), W, 32).tolist() == [4, 4, 3, 3, 2]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, N, Hq, Hkv, d, theta, alpha = 2, 700, 4, 2, 64, 1e4, 1.0
        q, k, v = _inputs(B, N, Hq, Hkv, d, seed=83)
        lens = [700, 411]  # the second sequence is shorter
        lo, hi = zip(*[splitkv.shard_ranges(L, world, d, theta, alpha)[rank] for L in lens])

        def partial_fn(q_, kc, v_, n_keys, key_pos0, q_pos, th, al, pairing, stream):
            his = [p0 + n for p0, n in zip(key_pos0, n_keys)]
            return torch.from_numpy(osk.partial(q_, kc, v_, key_pos0, his, q_pos, th, al))

        def merge_fn(parts, w, B_, Hq_, d_, stream):
            assert parts.shape == (w, B_, Hq_, d_ + 2)
            return osk.merge(parts.numpy())

        out = splitkv.decode_split_kv(q, k, v, [h - l for l, h in zip(lo, hi)], list(lo), [L - 1 for L in lens],
                                      theta, alpha, partial_fn=partial_fn, merge_fn=merge_fn)
        want, _ = oracle.decode(q, k, v, lens, theta, alpha)
        result_q.put((rank, float(np.abs(out - want).max())))
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_over_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    result_q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, result_q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    errs = dict(result_q.get(timeout=10) for _ in range(world))
    assert sorted(errs) == [0, 1] and max(errs.values()) < 1e-12

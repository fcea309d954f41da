"""The figures bench.py reports are computed on the host from closed forms; each
is checked here against a brute-force count over every (query, key, pair) or
(key, chunk) of small workloads, with the oracle's window table."""
import dataclasses
import itertools

import numpy as np
import pytest

import bench
import oracle
from rope_frequency_sparse_b200 import synth

TINY = dataclasses.replace(synth.WORKLOADS["layer_8k"], name="tiny", batch=2, seq=61, q_heads=3, kv_heads=1, d=16,
                           theta=50.0)


def _windows(d, theta, alpha):
    return oracle.windows(d, theta, alpha)[0]


@pytest.mark.parametrize("alpha", [0.25, 1.0, 3.0])
def test_prefill_flops_and_skipped_pairs_match_brute_force(alpha):
    w = TINY
    W = [int(x) for x in _windows(w.d, w.theta, alpha)]
    active = skipped = 0
    for m in range(w.seq):
        for n in range(m + 1):
            for i in range(w.d // 2):
                if m - n <= W[i]:
                    active += 1
                else:
                    skipped += 1
    P = w.seq * (w.seq + 1) // 2
    eff, dense, sk = bench.prefill_flops(w, alpha, windows=_windows)
    assert sk == w.batch * w.q_heads * skipped
    assert eff == w.batch * w.q_heads * (4 * active + 2 * w.d * P)  # 2 flops per dim of the active pairs, P.V
    assert dense == w.batch * w.q_heads * (4 * (w.d // 2) * P + 2 * w.d * P)
    assert bench.causal_elements(w) == w.batch * w.q_heads * P
    for m in (0, 1, 17, w.seq - 1):
        act_m = sum(1 for n in range(m + 1) for i in range(w.d // 2) if m - n <= W[i])
        assert bench.row_flops(w, alpha, m, windows=_windows) == 4 * act_m + 2 * w.d * (m + 1)


def test_prefill_flops_at_infinite_alpha_count_every_pair():
    eff, dense, sk = bench.prefill_flops(TINY, float("inf"), windows=_windows)
    assert sk == 0 and eff == dense


DEC = dataclasses.replace(synth.WORKLOADS["decode_1m"], name="tiny_decode", batch=3, seq=700, q_heads=4,
                          kv_heads=2, d=32, theta=300.0)


@pytest.mark.parametrize("alpha", [0.5, 1.0, float("inf")])
def test_decode_byte_counts_match_brute_force(alpha, monkeypatch):
    w = DEC
    monkeypatch.setattr(bench, "window_table", lambda d, th, a, windows=None: [int(x) for x in _windows(d, th, a)])
    W = [int(x) for x in _windows(w.d, w.theta, alpha)]
    N = w.seq
    # active: (key, pair) with the query's distance to the key within the pair's window
    a = sum(1 for n in range(N) for i in range(w.d // 2) if N - 1 - n <= W[i])
    qo = 2 * w.batch * w.q_heads * w.d * 2
    act, dense = bench.decode_bytes(w, alpha)
    assert act == w.batch * w.kv_heads * (4 * a + 2 * w.d * N) + qo
    assert dense == w.batch * w.kv_heads * 4 * N * w.d + qo
    # moved: per 128-key tile, a 32-byte chunk row of every key of the tile when
    # some key of the tile needs some pair of the chunk; every value row
    rows = 0
    for t0 in range(0, N, 128):
        tile = range(t0, min(N, t0 + 128))
        for c in range(w.d // 16):
            if any(N - 1 - n <= W[i] for n, i in itertools.product(tile, range(8 * c, 8 * c + 8))):
                rows += len(tile)
    assert bench.decode_moved_bytes(w, alpha) == w.batch * w.kv_heads * (32 * rows + N * w.d * 2) + qo


def test_recorded_traffic_requires_the_profiled_source():
    # the decode profile states the sha256 of the source it measured: it is current
    assert bench.recorded_traffic("decode.cu", "decode_1m.md") == pytest.approx(5896968668)
    # the same figure is not offered for another kernel's source
    assert bench.recorded_traffic("fasa.cu", "decode_1m.md") is None
    assert bench.recorded_traffic("decode.cu", "no_such_profile.md") is None

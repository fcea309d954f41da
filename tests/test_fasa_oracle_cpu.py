"""Pins of the FASA-style decode oracle (oracle/fasa.py) against facts that do
not come from the oracle itself: closed forms, brute force, planted inputs and
the dense decode oracle."""
import math

import numpy as np
import torch

import oracle
from oracle import fasa


def _bf16(shape, seed):
    g = np.random.default_rng(seed)
    return torch.from_numpy(g.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)


def test_all_pairs_score_is_the_full_dot_product():
    q = _bf16((1, 4, 128), 1)
    k = _bf16((1, 50, 2, 128), 2)
    sc = fasa.tip_scores(q, k, [50], (1 << 64) - 1)
    qd, kd = q.double().numpy(), k.double().numpy()
    for h in range(4):
        exact = kd[0, :, h // 2, :] @ qd[0, h]
        bound = 128 * 2.0 ** -24 * (np.abs(kd[0, :, h // 2, :]) @ np.abs(qd[0, h]))  # one rounding per dim
        assert np.all(np.abs(sc[0, h] - exact) <= bound)


def test_one_pair_score_is_that_pairs_product_sum():
    q = _bf16((2, 2, 64), 3)
    k = _bf16((2, 30, 1, 64), 4)
    i = 9
    sc = fasa.tip_scores(q, k, [30, 17], 1 << i)
    qd, kd = q.double().numpy(), k.double().numpy()
    for b, L in ((0, 30), (1, 17)):
        for h in range(2):
            want = (qd[b, h, 2 * i] * kd[b, :L, 0, 2 * i] + qd[b, h, 2 * i + 1] * kd[b, :L, 0, 2 * i + 1])
            assert np.array_equal(sc[b, h, :L], want.astype(np.float32))  # products exact, one rounding
            assert np.all(np.isneginf(sc[b, h, L:]))


def test_scores_ignore_pairs_outside_the_mask():
    q = _bf16((1, 1, 128), 5)
    k = _bf16((1, 40, 1, 128), 6).clone()
    mask = (1 << 3) | (1 << 40)
    before = fasa.tip_scores(q, k, [40], mask)
    k[..., 10:20] = 7.0  # pairs 5..9, not in the mask
    assert np.array_equal(fasa.tip_scores(q, k, [40], mask), before)
    k[..., 80] = 7.0  # pair 40, in the mask
    assert not np.array_equal(fasa.tip_scores(q, k, [40], mask), before)


def test_planted_monotone_scores_select_the_last_keys():
    N, budget = 64, 10
    q = torch.zeros(1, 1, 64)
    q[0, 0, 2 * 5] = 1.0
    k = torch.zeros(1, N, 1, 64)
    k[0, :, 0, 2 * 5] = torch.arange(N, dtype=torch.float32) / 8  # exact in bf16
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    sel = fasa.select(fasa.tip_scores(q, k, [N], 1 << 5), [N], budget)
    assert sel[0, 0].tolist() == list(range(N - budget, N))


def test_equal_scores_select_the_lowest_indices_and_pad():
    q = _bf16((1, 2, 64), 7)
    k = torch.zeros(1, 20, 1, 64, dtype=torch.bfloat16)  # every score is 0 (and -0 counts as +0)
    sel = fasa.select(fasa.tip_scores(q, k, [20], (1 << 32) - 1), [20], 8)
    assert sel[0, 0].tolist() == list(range(8)) and sel[0, 1].tolist() == list(range(8))
    short = fasa.select(fasa.tip_scores(q, k, [5], (1 << 32) - 1), [5], 8)
    assert short[0, 0].tolist() == [0, 1, 2, 3, 4, -1, -1, -1]


def test_selection_equals_brute_force_sort():
    q = _bf16((2, 4, 64), 8)
    k = _bf16((2, 300, 2, 64), 9)
    kv_len, mask, budget = [300, 123], 0xF0F0_0000_0000_00FF & ((1 << 32) - 1), 37
    sc = fasa.tip_scores(q, k, kv_len, mask)
    sel = fasa.select(sc, kv_len, budget)
    for b in range(2):
        for h in range(4):
            brute = sorted(range(kv_len[b]), key=lambda n: (-float(sc[b, h, n]), n))[:budget]
            assert sel[b, h].tolist() == sorted(brute)


def test_focused_attention_over_every_token_is_the_dense_decode():
    B, N, Hq, Hkv, d, theta = 2, 90, 4, 2, 64, 1e4
    q = _bf16((B, Hq, d), 10)
    k_rot = _bf16((B, N, Hkv, d), 11)
    v = _bf16((B, N, Hkv, d), 12)
    want, _ = oracle.decode(q, k_rot, v, [N, N], theta, math.inf)
    q_rot = oracle.rope(q[:, None], theta, pos0=N - 1)[:, 0]  # fp64, as the decode oracle rotates it
    sel = np.tile(np.arange(N, dtype=np.int32), (B, Hq, 1))
    got = fasa.focused_attention(q_rot, k_rot, v, sel)
    assert np.abs(got - want).max() < 1e-12


def test_focused_attention_over_one_token_returns_its_value():
    q = _bf16((1, 3, 64), 13)
    k = _bf16((1, 10, 1, 64), 14)
    v = _bf16((1, 10, 1, 64), 15)
    sel = np.array([[[4, -1], [7, -1], [0, -1]]], dtype=np.int32)
    got = fasa.focused_attention(q, k, v, sel)
    vd = v.double().numpy()
    for h, n in enumerate((4, 7, 0)):
        assert np.array_equal(got[0, h], vd[0, n, 0])

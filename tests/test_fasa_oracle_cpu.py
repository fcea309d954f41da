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
    # the full dot product from torch's own fp64 contraction, heads mapped by GQA
    full = torch.einsum("bngd,bhd->bhng", k.double(), q.double())  # [b][q head][key][kv head]
    for h in range(4):
        want = full[0, h, :, h // 2].numpy()
        assert np.allclose(sc[0, h], want, rtol=0, atol=1e-12 * (1 + np.abs(want).max()))


def test_one_pair_score_is_that_pairs_product_sum():
    q = _bf16((2, 2, 64), 3)
    k = _bf16((2, 30, 1, 64), 4)
    i = 9
    sc = fasa.tip_scores(q, k, [30, 17], 1 << i)
    qd, kd = q.double().numpy(), k.double().numpy()
    for b, L in ((0, 30), (1, 17)):
        for h in range(2):
            want = qd[b, h, 2 * i] * kd[b, :L, 0, 2 * i] + qd[b, h, 2 * i + 1] * kd[b, :L, 0, 2 * i + 1]
            assert np.array_equal(sc[b, h, :L], want)  # two bf16 products and one sum, exact in fp64
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


def _fp32_sum(q, k, dims):
    """fp32 sequential sums of the products over `dims` in that order (products of
    bf16 numbers are exact in fp32; each addition rounds once)."""
    acc = np.zeros(k.shape[0], dtype=np.float32)
    for j in dims:
        acc = (acc + (np.float32(q[j]) * k[:, j].astype(np.float32)).astype(np.float32)).astype(np.float32)
    return acc.astype(np.float64)


def test_score_bound_holds_for_fp32_sums_in_any_order():
    """The bound n 2^-24 sum|q_j k_j| covers an fp32 evaluation in any summation
    order, on random and on cancellation-heavy inputs (large terms that cancel)."""
    g = np.random.default_rng(20)
    mask = (1 << 64) - 1
    for big in (False, True):
        qf = g.standard_normal((1, 1, 128)).astype(np.float32)
        kf = g.standard_normal((1, 400, 1, 128)).astype(np.float32)
        if big:
            kf[..., 0::2] *= 1e3
            kf[..., 1::2] = -kf[..., 0::2] * qf[..., None, None, 0::2][0] / np.where(qf[..., 1::2] == 0, 1, qf[..., 1::2])[0, 0]
        q = torch.from_numpy(qf).to(torch.bfloat16)
        k = torch.from_numpy(kf).to(torch.bfloat16)
        exact = fasa.tip_scores(q, k, [400], mask)[0, 0]
        bound = fasa.score_bound(q, k, [400], mask)[0, 0]
        qd, kd = q.float().numpy()[0, 0], k.float().numpy()[0, :, 0]
        dims = np.arange(128)
        for order in (dims, dims[::-1], g.permutation(128)):
            got = _fp32_sum(qd, kd, order)
            assert np.all(np.abs(got - exact) <= bound), (big, np.abs(got - exact).max(), bound.min())


def _chunk_step_sum(qd, kd, chunks):
    """A model of a 16-dim chunk step: the running sum and the chunk's products
    aligned to the largest of them, each truncated (toward zero) below that one's
    24th significant bit, added exactly, the result truncated to fp32."""
    from fractions import Fraction

    out = np.empty(kd.shape[0], dtype=np.float64)
    for n in range(kd.shape[0]):
        run = 0.0
        for c in chunks:
            terms = [run] + [float(qd[j]) * float(kd[n, j]) for j in range(16 * c, 16 * c + 16)]
            big = max(abs(x) for x in terms)
            if big == 0.0:
                continue
            unit = Fraction(2) ** (math.frexp(big)[1] - 24)  # the largest term's 24th significant bit
            tot = sum(Fraction(math.trunc(Fraction(x) / unit)) * unit for x in terms)
            run = float(np.float32(float(tot)))  # exact result to fp32; then toward zero
            if abs(run) > abs(float(tot)):
                run = float(np.nextafter(np.float32(run), np.float32(0.0)))
        out[n] = run
    return out


def test_tensor_bound_holds_for_a_truncating_chunk_step_adder():
    """The "tensor" bound covers the simulated chunk-step adder on random and on
    cancellation-heavy keys, and is not looser than needed by orders of magnitude."""
    g = np.random.default_rng(23)
    mask = (0xFF << 8) | (0x0F << 48)  # one whole and one half chunk
    chunks = [1, 6]
    for big in (False, True):
        qf = g.standard_normal((1, 1, 128)).astype(np.float32)
        kf = g.standard_normal((1, 120, 1, 128)).astype(np.float32)
        if big:
            kf[..., 16:32:2] *= 1e4
            kf[..., 17:32:2] = -kf[..., 16:32:2] * (qf[0, 0, 16:32:2] / np.where(qf[0, 0, 17:32:2] == 0, 1,
                                                                                 qf[0, 0, 17:32:2]))
        q = torch.from_numpy(qf).to(torch.bfloat16)
        k = torch.from_numpy(kf).to(torch.bfloat16)
        qd, kd = q.float().numpy()[0, 0].copy(), k.float().numpy()[0, :, 0].copy()
        dims = [j for i in fasa.pair_list(mask, 128) for j in (2 * i, 2 * i + 1)]
        keep = np.zeros(128, dtype=bool)
        keep[dims] = True
        qd[~keep] = 0.0  # the kernel's B operand is zero outside the dominant pairs
        exact = fasa.tip_scores(q, k, [120], mask)[0, 0]
        bound = fasa.score_bound(q, k, [120], mask, model="tensor")[0, 0]
        got = _chunk_step_sum(qd, kd, chunks)
        err = np.abs(got - exact)
        assert np.all(err <= bound), (big, err.max(), bound.min())
        mag = fasa.score_bound(q, k, [120], mask, model="fma")[0, 0] / (len(dims) * 2.0 ** -24)
        assert np.all(bound <= 18 * 2.0 ** -23 * 2 * 1.01 * mag + 1e-30)


def test_check_selection_accepts_correct_and_rejects_wrong_selections():
    q = _bf16((1, 2, 64), 21)
    k = _bf16((1, 500, 1, 64), 22)
    kv_len, mask, budget = [500], 0xFF00FF, 40
    exact = fasa.tip_scores(q, k, kv_len, mask)
    bound = fasa.score_bound(q, k, kv_len, mask)
    sel = fasa.select(exact, kv_len, budget)
    fasa.check_selection(sel, k, kv_len, budget, exact, bound, mask)  # the oracle's own selection

    def rejects(bad):
        try:
            fasa.check_selection(bad, k, kv_len, budget, exact, bound, mask)
        except AssertionError:
            return True
        return False

    # the lowest kept key swapped for the lowest-scoring dropped key
    bad = sel.copy()
    kept = bad[0, 0]
    drop = np.setdiff1d(np.arange(500), kept)
    worst = kept[np.argmin(exact[0, 0, kept])]
    loser = drop[np.argmin(exact[0, 0, drop])]
    bad[0, 0] = np.sort(np.where(kept == worst, loser, kept))
    assert rejects(bad)
    # unsorted, duplicated, out of range, wrong padding
    bad = sel.copy()
    bad[0, 1, :2] = bad[0, 1, 1::-1]
    assert rejects(bad)
    bad = sel.copy()
    bad[0, 1, 1] = bad[0, 1, 0]
    assert rejects(bad)
    bad = sel.copy()
    bad[0, 1, -1] = 500
    assert rejects(bad)
    short = fasa.select(exact, [30], budget)
    fasa.check_selection(short, k, [30], budget, fasa.tip_scores(q, k, [30], mask), fasa.score_bound(q, k, [30], mask),
                         mask)
    short[0, 0, 35] = 3
    try:
        fasa.check_selection(short, k, [30], budget, fasa.tip_scores(q, k, [30], mask),
                             fasa.score_bound(q, k, [30], mask), mask)
        raise RuntimeError("padding not checked")
    except AssertionError:
        pass


def test_check_selection_enforces_the_lower_index_among_identical_keys():
    q = torch.zeros(1, 1, 64)
    q[0, 0, 2 * 5] = 1.0
    k = torch.zeros(1, 10, 1, 64)
    k[0, :, 0, 2 * 5] = torch.tensor([3.0, 1, 1, 1, 0, 0, 1, 2, 0, 1])
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    mask, budget = 1 << 5, 4  # keys 0 (3), 7 (2), then two of the five keys scoring 1
    exact = fasa.tip_scores(q, k, [10], mask)
    bound = fasa.score_bound(q, k, [10], mask)
    good = np.array([[[0, 1, 2, 7]]], dtype=np.int32)
    assert np.array_equal(fasa.select(exact, [10], budget), good)
    fasa.check_selection(good, k, [10], budget, exact, bound, mask)
    bad = np.array([[[0, 1, 6, 7]]], dtype=np.int32)  # key 6 kept while the identical key 2 is dropped
    try:
        fasa.check_selection(bad, k, [10], budget, exact, bound, mask)
        raise RuntimeError("tie rule not checked")
    except AssertionError:
        pass

"""Pins for the fp64 oracle: each check ties it to something other than itself
(closed forms, an independent library routine, invariants of the mathematics).

Method: "ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57 Prozent"
(sudo-ai.de), section "Was ATFlash anders macht" -- every RoPE frequency pair
gets its own distance window proportional to its wavelength; outside it the
pair's query-key product is left out, and the rest of attention (online
softmax, P.V) is unchanged (section "Die Zahlen - und ihre Grenze").
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from rope_frequency_sparse_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, val = line.split(":", 1)
                rows[key.strip()] = val.strip()
    return rows


def _rotate_complex(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """RoPE written as complex multiplication: pair i of a token at position p is
    the complex number x_{2i} + j x_{2i+1}, multiplied by exp(j p omega_i).
    x [B][S][H][d] fp64, pos [S]."""
    d = x.shape[-1]
    omega = np.exp(-(2.0 * np.arange(d // 2) / d) * np.log(theta))
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * pos[None, :, None, None] * omega[None, None, None, :])
    y = np.empty_like(x)
    y[..., 0::2] = z.real
    y[..., 1::2] = z.imag
    return y


def _tri(x):
    return x * (x + 1) // 2 if x > 0 else 0


# --------------------------------------------------------------------------- windows

def test_windows_exact_powers_golden():
    """theta=16, d=4: omega = (1, 1/4) exactly, so lambda = (2 pi, 8 pi)."""
    g = _read_golden("windows_d4_theta16.txt")
    for alpha_s in ("1", "0.5", "3"):
        W, om = oracle.windows(4, 16.0, float(alpha_s))
        assert om.tolist() == [1.0, 0.25]
        want = [int(t) for t in g[f"alpha={alpha_s}"].split(",")]
        assert W.tolist() == want
    W, _ = oracle.windows(4, 16.0, math.inf)
    assert W.tolist() == [2**63 - 1] * 2


@pytest.mark.parametrize("d,theta", [(64, 1e4), (128, 1e7), (128, 5e5), (16, 100.0)])
@pytest.mark.parametrize("alpha", [0.25, 0.5, 1.0, 2.0, 7.3])
def test_windows_bracket_wavelength(d, theta, alpha):
    """W_i is the smallest integer >= alpha*lambda_i; lambda_0 = 2 pi for every theta;
    wavelengths grow with i, so W is non-decreasing (the active set is a suffix)."""
    W, om = oracle.windows(d, theta, alpha)
    assert W[0] == math.ceil(alpha * 2 * math.pi)
    for i in range(d // 2):
        lam = 2 * math.pi * math.exp((2 * i / d) * math.log(theta))  # exp-log, not pow
        assert W[i] - 1 < alpha * lam * (1 + 1e-12) and alpha * lam * (1 - 1e-12) <= W[i]
    assert (np.diff(W) >= 0).all()


def test_windows_tiny_fp32_workload_table():
    """d=64, theta=1e4, alpha=1: the first pairs' windows, by hand:
    2 pi * 1e4^(2i/64) for i = 0..3 is 6.283, 8.378, 11.17, 14.90."""
    W, _ = oracle.windows(64, 1e4, 1.0)
    assert W[:4].tolist() == [7, 9, 12, 15]


# --------------------------------------------------------------------------- skip count

@pytest.mark.parametrize("S,d,theta,alpha", [(40, 4, 16.0, 1.0), (97, 8, 100.0, 0.5), (150, 16, 1e4, 1.0),
                                               (1, 8, 1e4, 1.0), (64, 16, 1e4, math.inf)])
def test_skip_count_closed_form(S, d, theta, alpha):
    """Skipped (query, key, pair) triples = sum_i sum_{m<S} max(0, m - W_i)
    = sum_i T(S-1-W_i) with T(x) = x(x+1)/2."""
    q, k, v = synth.random_prefill(1, S, S, 2, 1, d, torch.float32, seed=3)
    _, skipped = oracle.prefill(q, k, v, theta, alpha)
    W, _ = oracle.windows(d, theta, alpha)
    want = 2 * sum(_tri(S - 1 - int(w)) if w < 2**62 else 0 for w in W)
    assert skipped == want


def test_skip_count_golden_d4():
    g = _read_golden("windows_d4_theta16.txt")
    q, k, v = synth.random_prefill(1, 40, 40, 1, 1, 4, torch.float32, seed=1)
    _, skipped = oracle.prefill(q, k, v, 16.0, 1.0)
    assert skipped == int(g["skipped_S40_alpha=1"])


def test_skip_count_tiny_fp32_workload():
    """The 512-token fp32 workload: sum_i T(511 - W_i) over its window table."""
    w = synth.WORKLOADS["tiny_fp32"]
    q, k, v = synth.prefill_inputs(w)
    _, skipped = oracle.prefill(q, k, v, w.theta, 1.0)
    W = [math.ceil(2 * math.pi * math.exp((2 * i / 64) * math.log(1e4))) for i in range(32)]
    assert skipped == sum(_tri(511 - x) for x in W) == 1389990


def test_skip_count_chunked_and_decode():
    S, d, theta, alpha = 130, 8, 50.0, 1.0
    W, _ = oracle.windows(d, theta, alpha)
    q, k, v = synth.random_prefill(1, S, S, 1, 1, d, torch.float32, seed=5)
    _, sk = oracle.prefill(q[:, 70:100], k, v, theta, alpha, q_offset=70)
    assert sk == sum(max(0, m - int(w)) for m in range(70, 100) for w in W)
    kr = torch.from_numpy(oracle.rope(k, theta)).float()
    _, skd = oracle.decode(q[:, 0], kr, v, [S], theta, alpha)
    assert skd == sum(max(0, S - 1 - int(w)) for w in W)


# --------------------------------------------------------------------------- RoPE

def test_rope_unit_vectors():
    """A unit vector in pair i at position p rotates to (cos p omega_i, sin p omega_i)
    (the standard counter-clockwise 2-D rotation)."""
    d, theta = 8, 100.0
    pos = [0, 1, 5, 1000, 2**20 - 1]
    y = np.concatenate([oracle.rope(np.zeros((1, 1, 1, d), np.float32) + np.eye(d, dtype=np.float32)[2 * i]
                                    .reshape(1, 1, 1, d), theta, pos0=p) for i in range(d // 2) for p in pos],
                       axis=1)
    r = 0
    for i in range(d // 2):
        om = theta ** (-2 * i / d)
        for p in pos:
            vec = y[0, r, 0]
            assert abs(vec[2 * i] - math.cos(p * om)) < 1e-12
            assert abs(vec[2 * i + 1] - math.sin(p * om)) < 1e-12
            assert np.abs(np.delete(vec, [2 * i, 2 * i + 1])).max() == 0
            r += 1


def test_rope_matches_complex_form_and_is_relative():
    q, k, _ = synth.random_prefill(2, 33, 33, 3, 3, 16, torch.float32, seed=11)
    y = oracle.rope(q, 1e4, pos0=7)
    want = _rotate_complex(q.double().numpy(), np.arange(7, 40, dtype=np.float64), 1e4)
    assert np.abs(y - want).max() < 1e-12
    # <R(m) q, R(n) k> depends only on m - n
    a = (oracle.rope(q, 1e4, pos0=0) * oracle.rope(k, 1e4, pos0=3)).sum(-1)
    b = (oracle.rope(q, 1e4, pos0=100) * oracle.rope(k, 1e4, pos0=103)).sum(-1)
    assert np.abs(a - b).max() < 1e-9


# --------------------------------------------------------------------------- special cases

@pytest.mark.parametrize("alpha", [math.inf, 1e9])
def test_dense_case_equals_sdpa(alpha):
    """Every window >= the sequence: plain causal RoPE attention, checked against
    torch's fp64 scaled_dot_product_attention with GQA."""
    B, S, Hq, Hkv, d, theta = 2, 37, 4, 2, 16, 100.0
    q, k, v = synth.random_prefill(B, S, S, Hq, Hkv, d, torch.float32, seed=7)
    out, skipped = oracle.prefill(q, k, v, theta, alpha)
    assert skipped == 0
    pos = np.arange(S, dtype=np.float64)
    qr = torch.from_numpy(_rotate_complex(q.double().numpy(), pos, theta))
    kr = torch.from_numpy(_rotate_complex(k.double().numpy(), pos, theta))
    ref = torch.nn.functional.scaled_dot_product_attention(
        qr.transpose(1, 2), kr.transpose(1, 2), v.double().transpose(1, 2), is_causal=True, enable_gqa=True)
    assert np.abs(out - ref.transpose(1, 2).numpy()).max() < 1e-12


def test_all_pairs_inactive_gives_logit_zero():
    """theta = 1.0001, alpha = 0.1: alpha*lambda_i < 1 for all i, so every W_i = 1.
    Keys at distance 0 and 1 see all pairs; every farther key has an EMPTY active
    set and logit 0 (kept in the softmax):
      out_m = (e^{s0} v_m + e^{s1} v_{m-1} + sum_{n<=m-2} v_n) / (e^{s0} + e^{s1} + m - 1)."""
    S, d, theta, alpha = 9, 8, 1.0001, 0.1
    W, _ = oracle.windows(d, theta, alpha)
    assert W.tolist() == [1] * (d // 2)
    q, k, v = synth.random_prefill(1, S, S, 1, 1, d, torch.float32, seed=13)
    out, _ = oracle.prefill(q, k, v, theta, alpha)
    pos = np.arange(S, dtype=np.float64)
    qr = _rotate_complex(q.double().numpy(), pos, theta)[0, :, 0]
    kr = _rotate_complex(k.double().numpy(), pos, theta)[0, :, 0]
    vv = v.double().numpy()[0, :, 0]
    for m in range(S):
        s0 = qr[m] @ kr[m] / math.sqrt(d)
        if m == 0:
            want = vv[0]
        else:
            s1 = qr[m] @ kr[m - 1] / math.sqrt(d)
            num = math.exp(s0) * vv[m] + math.exp(s1) * vv[m - 1] + vv[: m - 1].sum(0)
            want = num / (math.exp(s0) + math.exp(s1) + (m - 1))
        assert np.abs(out[0, m, 0] - want).max() < 1e-12


def test_single_active_pair_window_boundary():
    """q and k nonzero only in pair j: the logit is |z_q||z_k| cos((m-n) omega_j + arg z_q - arg z_k)/sqrt d
    while m-n <= W_j and exactly 0 beyond; the boundary is inclusive."""
    S, d, theta, j = 60, 8, 30.0, 2
    om_j = theta ** (-2 * j / d)
    alpha = 17.5 / (2 * math.pi / om_j)  # alpha*lambda_j = 17.5 -> W_j = 18
    W, _ = oracle.windows(d, theta, alpha)
    assert W[j] == 18
    q, k, v = synth.random_prefill(1, S, S, 1, 1, d, torch.float32, seed=17)
    mask = torch.zeros(d)
    mask[2 * j: 2 * j + 2] = 1
    q, k = q * mask, k * mask
    out, _ = oracle.prefill(q, k, v, theta, alpha)
    zq = q[0, :, 0, 2 * j].double().numpy() + 1j * q[0, :, 0, 2 * j + 1].double().numpy()
    zk = k[0, :, 0, 2 * j].double().numpy() + 1j * k[0, :, 0, 2 * j + 1].double().numpy()
    vv = v.double().numpy()[0, :, 0]
    for m in range(S):
        n = np.arange(m + 1)
        dl = m - n
        s = np.abs(zq[m]) * np.abs(zk[n]) * np.cos(dl * om_j + np.angle(zq[m]) - np.angle(zk[n])) / math.sqrt(d)
        s = np.where(dl <= 18, s, 0.0)
        p = np.exp(s - s.max())
        want = (p[:, None] * vv[: m + 1]).sum(0) / p.sum()
        assert np.abs(out[0, m, 0] - want).max() < 1e-12


# --------------------------------------------------------------------------- invariants

def test_constant_v_gives_constant_out():
    q, k, v = synth.random_prefill(1, 50, 50, 2, 1, 16, torch.float32, seed=19)
    v = torch.full_like(v, 0.375)
    out, _ = oracle.prefill(q, k, v, 1e4, 0.7)
    assert np.abs(out - 0.375).max() < 1e-14


def test_chunked_equals_unchunked():
    S, theta, alpha = 96, 1e3, 0.8
    q, k, v = synth.random_prefill(1, S, S, 4, 2, 16, torch.float32, seed=23)
    full, sk_full = oracle.prefill(q, k, v, theta, alpha)
    parts, sk = [], 0
    for c0 in range(0, S, 32):
        o, s = oracle.prefill(q[:, c0:c0 + 32], k[:, : c0 + 32], v[:, : c0 + 32], theta, alpha, q_offset=c0)
        parts.append(o)
        sk += s
    assert np.abs(np.concatenate(parts, axis=1) - full).max() < 1e-13
    assert sk == sk_full


def test_decode_equals_last_prefill_row():
    S, theta, alpha = 77, 1e4, 1.0
    q, k, v = synth.random_prefill(2, S, S, 4, 2, 16, torch.float32, seed=29)
    full, _ = oracle.prefill(q, k, v, theta, alpha)
    kr = torch.from_numpy(oracle.rope(k, theta)).float()
    dec, _ = oracle.decode(q[:, -1], kr, v, [S, S], theta, alpha)
    assert np.abs(dec - full[:, -1]).max() < 1e-5  # cache rounded to fp32 after rotation


def test_decode_ragged_lengths_match_prefill_rows():
    S, theta, alpha = 40, 1e4, 0.6
    q, k, v = synth.random_prefill(1, S, S, 2, 1, 16, torch.float32, seed=31)
    full, _ = oracle.prefill(q, k, v, theta, alpha)
    kr = torch.from_numpy(oracle.rope(k, theta)).float()
    for L in (1, 2, 17, 40):
        dec, _ = oracle.decode(q[:, L - 1], kr, v, [L], theta, alpha)
        assert np.abs(dec[0] - full[0, L - 1]).max() < 1e-5


def test_head_permutation_equivariance():
    S, Hq, Hkv = 30, 6, 3
    q, k, v = synth.random_prefill(1, S, S, Hq, Hkv, 16, torch.float32, seed=37)
    out, _ = oracle.prefill(q, k, v, 1e4, 1.0)
    perm_kv = [2, 0, 1]
    perm_q = [2 * g + r for g in perm_kv for r in range(2)]
    out_p, _ = oracle.prefill(q[:, :, perm_q], k[:, :, perm_kv], v[:, :, perm_kv], 1e4, 1.0)
    assert np.abs(out_p - out[:, :, perm_q]).max() < 1e-14


def test_bf16_inputs_widen_exactly():
    q, k, v = synth.random_prefill(1, 20, 20, 2, 1, 16, torch.bfloat16, seed=41)
    o1, s1 = oracle.prefill(q, k, v, 1e4, 1.0)
    o2, s2 = oracle.prefill(q.float(), k.float(), v.float(), 1e4, 1.0)
    assert s1 == s2 and np.abs(o1 - o2).max() == 0.0


def test_sampled_rows_match_full():
    q, k, v = synth.random_prefill(1, 64, 64, 2, 1, 16, torch.float32, seed=43)
    full, _ = oracle.prefill(q, k, v, 1e4, 1.0)
    rows = [0, 5, 63]
    part, _ = oracle.prefill(q, k, v, 1e4, 1.0, rows=rows)
    assert np.abs(part[:, rows] - full[:, rows]).max() == 0.0
    assert np.isnan(part[:, 1]).all()


# --------------------------------------------------------------------------- rotate-half pairing

def _half_to_interleaved(x):
    """Reorder the last axis so that rotate-half pair i = dims (i, i + d/2) lands on
    dims (2i, 2i+1)."""
    d = x.shape[-1]
    perm = np.empty(d, dtype=np.int64)
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    return x[..., perm]


def _rotate_half_complex(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE as complex multiplication: pair i is x_i + j x_{i+d/2}."""
    d = x.shape[-1]
    omega = np.exp(-(2.0 * np.arange(d // 2) / d) * np.log(theta))
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    z = z * np.exp(1j * pos[None, :, None, None] * omega[None, None, None, :])
    return np.concatenate([z.real, z.imag], axis=-1)


def test_rotate_half_rope_unit_vectors():
    """A unit vector in dim i (< d/2) at position p rotates to cos p omega_i in dim i
    and sin p omega_i in dim i + d/2; a unit vector in dim i + d/2 to -sin, cos."""
    d, theta = 8, 100.0
    eye = np.eye(d, dtype=np.float32)
    for i in range(d // 2):
        om = theta ** (-2 * i / d)
        for p in (0, 1, 7, 2**20 - 1):
            a = oracle.rope(eye[i].reshape(1, 1, 1, d), theta, pos0=p, pairing=oracle.ROTATE_HALF)[0, 0, 0]
            b = oracle.rope(eye[i + d // 2].reshape(1, 1, 1, d), theta, pos0=p, pairing=oracle.ROTATE_HALF)[0, 0, 0]
            assert abs(a[i] - math.cos(p * om)) < 1e-12 and abs(a[i + d // 2] - math.sin(p * om)) < 1e-12
            assert abs(b[i] + math.sin(p * om)) < 1e-12 and abs(b[i + d // 2] - math.cos(p * om)) < 1e-12
            assert np.abs(np.delete(a, [i, i + d // 2])).max() == 0
            assert np.abs(np.delete(b, [i, i + d // 2])).max() == 0


def test_rotate_half_rope_matches_complex_form():
    q, _, _ = synth.random_prefill(2, 21, 21, 3, 3, 16, torch.float32, seed=13)
    y = oracle.rope(q, 1e4, pos0=5, pairing=oracle.ROTATE_HALF)
    want = _rotate_half_complex(q.double().numpy(), np.arange(5, 26, dtype=np.float64), 1e4)
    assert np.abs(y - want).max() < 1e-12


@pytest.mark.parametrize("alpha", [0.5, 1.0, math.inf])
def test_rotate_half_equals_interleaved_on_reordered_dims(alpha):
    """Pair i of the rotate-half convention is pair i of the interleaved one once
    dims (i, i+d/2) are moved to (2i, 2i+1) in q and k (v untouched): the same
    windows, logits, outputs and skipped pairs."""
    B, S, Hq, Hkv, d, theta = 1, 70, 4, 2, 16, 100.0
    q, k, v = synth.random_prefill(B, S, S, Hq, Hkv, d, torch.float32, seed=17)
    out_h, sk_h = oracle.prefill(q, k, v, theta, alpha, pairing=oracle.ROTATE_HALF)
    qi = torch.from_numpy(np.ascontiguousarray(_half_to_interleaved(q.numpy())))
    ki = torch.from_numpy(np.ascontiguousarray(_half_to_interleaved(k.numpy())))
    out_i, sk_i = oracle.prefill(qi, ki, v, theta, alpha, pairing=oracle.INTERLEAVED)
    assert sk_h == sk_i
    assert np.abs(out_h - out_i).max() < 1e-12
    W, _ = oracle.windows(d, theta, alpha)
    assert sk_h == Hq * sum(_tri(S - 1 - int(w)) for w in W)


def test_rotate_half_dense_case_equals_sdpa():
    B, S, Hq, Hkv, d, theta = 2, 29, 4, 2, 16, 100.0
    q, k, v = synth.random_prefill(B, S, S, Hq, Hkv, d, torch.float32, seed=19)
    out, skipped = oracle.prefill(q, k, v, theta, math.inf, pairing=oracle.ROTATE_HALF)
    assert skipped == 0
    pos = np.arange(S, dtype=np.float64)
    qr = torch.from_numpy(_rotate_half_complex(q.double().numpy(), pos, theta))
    kr = torch.from_numpy(_rotate_half_complex(k.double().numpy(), pos, theta))
    ref = torch.nn.functional.scaled_dot_product_attention(
        qr.transpose(1, 2), kr.transpose(1, 2), v.double().transpose(1, 2), is_causal=True, enable_gqa=True)
    assert np.abs(out - ref.transpose(1, 2).numpy()).max() < 1e-12


def test_rotate_half_decode_equals_last_prefill_row():
    B, S, Hq, Hkv, d, theta = 1, 45, 4, 2, 16, 100.0
    q, k, v = synth.random_prefill(B, S, S, Hq, Hkv, d, torch.float32, seed=23)
    out_p, _ = oracle.prefill(q, k, v, theta, 1.0, pairing=oracle.ROTATE_HALF)
    k_rot = torch.from_numpy(oracle.rope(k, theta, pairing=oracle.ROTATE_HALF).astype(np.float32))
    out_d, _ = oracle.decode(q[:, -1], k_rot, v, [S], theta, 1.0, pairing=oracle.ROTATE_HALF)
    # the decode path reads k rotated once to fp32; compare at fp32 rounding of k~
    assert np.abs(out_d - out_p[:, -1]).max() < 1e-5

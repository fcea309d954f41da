"""Prefill kernels (fp32 CUDA-core and bf16 tcgen05) against the fp64 oracle.

Tolerances: max-abs 1e-4 for fp32 inputs, 2e-2 for bf16 inputs; the skipped
pair counter must equal the oracle's brute-force count exactly.  Every case also
reports how far the windowed result is from the dense one, so a test whose
tolerance could not tell the two apart would show up.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
TOL_FP32 = 1e-4


def run_gpu(q, k, v, theta, alpha, q_offset=0):
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    out = atf.prefill(q.cuda(), k.cuda(), v.cuda(), theta, alpha, q_offset=q_offset, skipped=cnt)
    atf.atf_check()
    return out.cpu().double().numpy(), int(cnt.item())


def check_case(q, k, v, theta, alpha, tol, q_offset=0, rows=None):
    got, cnt = run_gpu(q, k, v, theta, alpha, q_offset)
    want, skipped = oracle.prefill(q, k, v, theta, alpha, q_offset=q_offset, rows=rows)
    if rows is not None:
        got, want = got[:, rows], want[:, rows]
    err = np.abs(got - want).max()
    assert np.isfinite(got).all()
    assert err <= tol, f"max abs err {err}"
    if rows is None:
        assert cnt == skipped, (cnt, skipped)
    return err, cnt


def test_tiny_fp32_workload():
    """512 tokens, one head, d=64, theta=1e4, alpha=1, fp32."""
    w = synth.WORKLOADS["tiny_fp32"]
    q, k, v = synth.prefill_inputs(w)
    err, cnt = check_case(q, k, v, w.theta, 1.0, TOL_FP32)
    assert cnt == 1389990
    dense, _ = run_gpu(q, k, v, w.theta, math.inf)
    sparse, _ = run_gpu(q, k, v, w.theta, 1.0)
    assert np.abs(dense - sparse).max() > 100 * TOL_FP32  # the windows change the answer


@pytest.mark.parametrize("S,d,G", [(1, 128, 1), (17, 64, 1), (64, 128, 7), (300, 128, 1)])
def test_fp32_small(S, d, G):
    q, k, v = synth.random_prefill(1, S, S, G, 1, d, torch.float32, seed=S)
    check_case(q, k, v, 1e4, 0.7, TOL_FP32)


# ---------------------------------------------------------------- bf16, tensor cores

BF16_CASES = [
    # B, S, Hq, Hkv, d, theta, alpha
    (1, 1, 1, 1, 128, 1e7, 1.0),
    (1, 17, 2, 1, 128, 1e7, 1.0),
    (1, 128, 1, 1, 128, 1e4, 1.0),
    (1, 129, 7, 1, 128, 1e7, 1.0),
    (1, 255, 2, 2, 64, 1e4, 1.0),
    (1, 256, 7, 1, 64, 1e4, 0.5),
    (2, 300, 14, 2, 128, 1e7, 1.0),
    (1, 700, 7, 1, 128, 1e7, 0.5),
    (1, 700, 7, 1, 128, 1e7, 2.0),
    (1, 700, 7, 1, 128, 1e7, math.inf),
    (1, 1000, 4, 2, 64, 1e4, 1.0),
    (1, 1500, 2, 1, 128, 500.0, 0.3),   # many windows inside the sequence
    (1, 640, 2, 1, 128, 1e7, 127 / (2 * math.pi) - 1e-6),  # W_0 = 127: boundary on a tile edge
    (1, 640, 2, 1, 128, 1e7, 128 / (2 * math.pi) - 1e-6),  # W_0 = 128
    (1, 640, 2, 1, 128, 1e7, 255 / (2 * math.pi) - 1e-6),  # W_0 = 255
]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,theta,alpha", BF16_CASES)
def test_bf16_against_oracle(B, S, Hq, Hkv, d, theta, alpha):
    q, k, v = synth.random_prefill(B, S, S, Hq, Hkv, d, torch.bfloat16, seed=1000 + S)
    err, _ = check_case(q, k, v, theta, alpha, TOL_BF16)
    if not math.isinf(alpha) and S > 200:
        dense, _ = run_gpu(q, k, v, theta, math.inf)
        sparse, _ = run_gpu(q, k, v, theta, alpha)
        assert np.abs(dense - sparse).max() > 2 * TOL_BF16


def test_bf16_all_pairs_inactive():
    """theta=1.0001, alpha=0.1: every W_i = 1, so keys beyond distance 1 have no
    active pair (logit 0) and most tiles issue no QK MMA at all."""
    q, k, v = synth.random_prefill(1, 400, 400, 2, 1, 128, torch.bfloat16, seed=5)
    check_case(q, k, v, 1.0001, 0.1, TOL_BF16)


def test_bf16_dense_alpha_matches_huge_alpha():
    q, k, v = synth.random_prefill(1, 513, 513, 4, 1, 128, torch.bfloat16, seed=6)
    a, c1 = run_gpu(q, k, v, 1e7, math.inf)
    b, c2 = run_gpu(q, k, v, 1e7, 1e12)
    assert c1 == 0 and c2 == 0
    assert np.abs(a - b).max() <= 1e-2


@pytest.mark.parametrize("q_offset,q_len,alpha", [(256, 128, 1.0), (100, 77, 1.0), (512, 300, 1.0), (1, 1, 1.0),
                                                  (700, 300, 0.5), (640, 384, 2.0)])
def test_bf16_query_offset_chunk(q_offset, q_len, alpha):
    kv_len = q_offset + q_len
    q, k, v = synth.random_prefill(1, q_len, kv_len, 7, 1, 128, torch.bfloat16, seed=q_offset)
    check_case(q, k, v, 1e7, alpha, TOL_BF16, q_offset=q_offset)


@pytest.mark.parametrize("alpha", [0.5, 1.0, 2.0])
def test_bf16_chunked_equals_unchunked(alpha):
    """Query chunks against all earlier keys give the unchunked result and count,
    and match the oracle (the 128k workload's structure at a size the oracle
    finishes in seconds)."""
    S, C = 1024, 256
    q, k, v = synth.random_prefill(1, S, S, 7, 1, 128, torch.bfloat16, seed=9)
    full, cnt_full = run_gpu(q, k, v, 1e7, alpha)
    parts, cnt = [], 0
    for c0 in range(0, S, C):
        o, c = run_gpu(q[:, c0:c0 + C], k[:, : c0 + C], v[:, : c0 + C], 1e7, alpha, q_offset=c0)
        parts.append(o)
        cnt += c
    assert cnt == cnt_full
    got = np.concatenate(parts, axis=1)
    assert np.abs(got - full).max() <= 1e-2
    want, skipped = oracle.prefill(q, k, v, 1e7, alpha)
    assert np.abs(got - want).max() <= TOL_BF16
    assert cnt == skipped
    dense, _ = oracle.prefill(q, k, v, 1e7, math.inf)
    assert np.abs(want - dense).max() > 2 * TOL_BF16


def test_bf16_batch_rows_independent():
    q, k, v = synth.random_prefill(3, 200, 200, 7, 1, 128, torch.bfloat16, seed=11)
    all3, _ = run_gpu(q, k, v, 1e7, 1.0)
    one, _ = run_gpu(q[1:2], k[1:2], v[1:2], 1e7, 1.0)
    assert np.abs(all3[1:2] - one).max() == 0.0


# ---------------------------------------------------------------- full-size workloads, sampled rows
#
# Outputs at these lengths are averages over thousands of keys, and far rows of
# the windowed and the dense result differ by little more than the tolerance.  So
# every sampled test also runs the oracle with every window open on the same rows
# and checks that the rows it samples separate the two by more than twice the
# tolerance, and that wherever a row separates them clearly (by more than four
# times the tolerance) the GPU is within a quarter of that separation of the
# windowed result: a kernel with a wrong window would fail there.

def _sample_rows(S, n, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 1000, S // 2, S - 129, S - 128, S - 1]
    return sorted(set(fixed) | set(rng.integers(0, S, n).tolist()))


def _closed_form_skipped(w, alpha):
    W, _ = oracle.windows(w.d, w.theta, alpha)
    return w.q_heads * sum(max(0, x) * (max(0, x) + 1) // 2 for x in (w.seq - 1 - W.astype(object)))


def _check_sampled(got, q, k, v, theta, alpha, rows):
    """got: GPU output rows [B][len(rows)][Hq][d] (fp64)."""
    want, _ = oracle.prefill(q, k, v, theta, alpha, rows=rows)
    dense, _ = oracle.prefill(q, k, v, theta, math.inf, rows=rows)
    want, dense = want[:, rows], dense[:, rows]
    err_row = np.abs(got - want).max(axis=(0, 2, 3))
    sep_row = np.abs(want - dense).max(axis=(0, 2, 3))
    assert err_row.max() <= TOL_BF16, err_row.max()
    assert sep_row.max() > 2 * TOL_BF16, sep_row.max()
    clear = sep_row > 4 * TOL_BF16
    assert clear.any()
    assert (err_row[clear] <= 0.25 * sep_row[clear]).all(), (err_row[clear], sep_row[clear])


@pytest.mark.parametrize("alpha", [0.5, 1.0, 2.0, math.inf])
def test_layer_8k_sampled(alpha):
    w = synth.WORKLOADS["layer_8k"]
    q, k, v = synth.prefill_inputs(w)
    rows = _sample_rows(w.seq, 16, 1)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    out = atf.prefill(q.cuda(), k.cuda(), v.cuda(), w.theta, alpha, skipped=cnt)
    atf.atf_check()
    got = out[:, rows].cpu().double().numpy()
    if math.isinf(alpha):
        want, _ = oracle.prefill(q, k, v, w.theta, alpha, rows=rows)
        assert np.abs(got - want[:, rows]).max() <= TOL_BF16
    else:
        _check_sampled(got, q, k, v, w.theta, alpha, rows)
    assert int(cnt.item()) == _closed_form_skipped(w, alpha)


def test_layer_32k_pair_energy_sampled():
    w = synth.WORKLOADS["layer_32k_pair_energy"]
    q, k, v = synth.prefill_inputs(w)
    rows = _sample_rows(w.seq, 8, 2)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    out = atf.prefill(q.cuda(), k.cuda(), v.cuda(), w.theta, 1.0, skipped=cnt)
    atf.atf_check()
    _check_sampled(out[:, rows].cpu().double().numpy(), q, k, v, w.theta, 1.0, rows)
    assert int(cnt.item()) == _closed_form_skipped(w, 1.0) == 428871773932


@pytest.fixture(scope="module")
def layer_128k():
    w = synth.WORKLOADS["layer_128k_chunked"]
    return w, synth.prefill_inputs(w)


@pytest.mark.parametrize("alpha,closed", [(1.0, 8185992614072), (0.5, 8847662256216)])
def test_layer_128k_chunked_sampled(layer_128k, alpha, closed):
    """131072 tokens prefilled in 16 query chunks of 8192 against all earlier keys:
    keys rotated once into a cache, each chunk's queries rotated at their offset,
    the launches the benchmark times."""
    w, (q, k, v) = layer_128k
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    k_rot, _ = atf.rope_layout(kd, w.theta)
    out = torch.empty_like(qd)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    C = w.q_chunk
    for c0 in range(0, w.seq, C):
        q_rot, _ = atf.rope_layout(qd[:, c0:c0 + C].contiguous(), w.theta, pos_offset=c0)
        o = atf.prefill(q_rot, k_rot[:, : c0 + C], vd[:, : c0 + C], w.theta, alpha, q_offset=c0, rotated=True,
                        skipped=cnt)
        out[:, c0:c0 + C] = o
    atf.atf_check()
    rows = [0, 127, 128, 1000, 8191, 8192, 65535, 65536 + 4097, 122880, w.seq - 1]
    _check_sampled(out[:, rows].cpu().double().numpy(), q, k, v, w.theta, alpha, rows)
    assert int(cnt.item()) == _closed_form_skipped(w, alpha) == closed

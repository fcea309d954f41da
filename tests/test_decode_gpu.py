"""Decode kernel (split-KV over the pair-chunk-major key cache) against the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _gpu_decode(q, k_rot, v, kv_len, theta, alpha):
    qd, kd, vd = q.cuda(), k_rot.cuda(), v.cuda()
    _, kc = atf.rope_layout(kd, theta, rotate=False, rotated_out=False, chunked_out=True)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    out = atf.decode(qd, kc, vd, kv_len, theta, alpha, skipped=cnt)
    atf.atf_check()
    return out.cpu().double().numpy(), int(cnt.item())


@pytest.mark.parametrize("B,N,kv_len,Hq,Hkv,d,theta,alpha", [
    (2, 300, [300, 129], 28, 4, 128, 1e7, 1.0),
    (1, 1, [1], 7, 1, 128, 1e7, 1.0),
    (3, 5000, [5000, 4097, 33], 14, 2, 128, 1e4, 0.5),
    (2, 2048, [2048, 1000], 4, 4, 64, 1e4, 1.0),
    (1, 3000, [3000], 8, 1, 128, 1.0001, 0.1),  # every W_i = 1: far keys have no active pair
    (1, 4000, [4000], 7, 1, 128, 1e7, math.inf),
])
def test_decode_against_oracle(B, N, kv_len, Hq, Hkv, d, theta, alpha):
    q = synth.token_major(7, 501, 0, B, 1, Hq, d, torch.bfloat16, threads=1)[:, 0].contiguous()
    k = synth.token_major(7, 501, 1, B, N, Hkv, d, torch.bfloat16, threads=1)
    v = synth.token_major(7, 501, 2, B, N, Hkv, d, torch.bfloat16, threads=1)
    got, cnt = _gpu_decode(q, k, v, kv_len, theta, alpha)
    want, skipped = oracle.decode(q, k, v, kv_len, theta, alpha)
    assert np.abs(got - want).max() <= TOL
    assert cnt == skipped


def test_decode_equals_last_prefill_row():
    """Decode at kv_len = L reproduces row L-1 of the prefill on the same inputs."""
    L, theta, alpha = 777, 1e7, 1.0
    q, k, v = synth.random_prefill(1, L, L, 7, 1, 128, torch.bfloat16, seed=21)
    pre = atf.prefill(q.cuda(), k.cuda(), v.cuda(), theta, alpha).cpu().double().numpy()
    k_rot, kc = atf.rope_layout(k.cuda(), theta, chunked_out=True)
    out = atf.decode(q[:, -1].contiguous().cuda(), kc, v.cuda(), [L], theta, alpha)
    atf.atf_check()
    assert np.abs(out.cpu().double().numpy() - pre[:, -1]).max() <= TOL


def test_decode_1m_cache():
    """4 sequences x 1,048,576 cached keys, 28/4 heads, d=128, theta=1e7, alpha=1."""
    w = synth.WORKLOADS["decode_1m"]
    q, k, v = synth.decode_inputs(w)
    kv_len = [w.seq] * w.batch
    got, cnt = _gpu_decode(q, k, v, kv_len, w.theta, 1.0)
    want, skipped = oracle.decode(q, k, v, kv_len, w.theta, 1.0)
    assert np.abs(got - want).max() <= TOL
    assert cnt == skipped == 5200191024

"""Rotate-half (NeoX-style) pairing end to end on the GPU against the oracle.

The oracle follows the rotate-half definition directly (pair i = dims i, i+d/2);
the library rotates rotate-half pairs and writes pair i to dims (2i, 2i+1), the
order its attention kernels read.  These tests feed both the same raw inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu

TOL = 2e-2
HALF = atf.ATF_PAIRS_ROTATE_HALF


def _interleave(x: np.ndarray) -> np.ndarray:
    """dims (i, i + d/2) -> (2i, 2i+1) along the last axis."""
    d = x.shape[-1]
    perm = np.empty(d, dtype=np.int64)
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    return x[..., perm]


@pytest.mark.parametrize("S,H,d,theta,pos0", [(33, 4, 128, 1e7, 0), (257, 7, 128, 1e7, 4096),
                                              (19, 2, 64, 1e4, (1 << 20) - 19)])
def test_rope_rotate_half_matches_oracle(S, H, d, theta, pos0):
    x = synth.token_major(3, 601, 0, 2, S, H, d, torch.bfloat16, threads=1)
    want = torch.from_numpy(_interleave(oracle.rope(x, theta, pos0=pos0, pairing=oracle.ROTATE_HALF)))
    want = want.to(torch.bfloat16)
    xr, xc = atf.rope_layout(x.cuda(), theta, pos_offset=pos0, chunked_out=True, pairing=HALF)
    got = xr.cpu()
    assert (got.view(torch.int16) == want.view(torch.int16)).float().mean() > 0.999
    assert (got.float() - want.float()).abs().max().item() <= 2.0 ** -7 * want.float().abs().max().item()
    B = x.shape[0]
    assert torch.equal(xc.cpu(), got.view(B, S, H, d // 16, 16).permute(0, 2, 3, 1, 4).contiguous())
    # rotate = 3: the reordering alone, for caches already rotated
    xo, _ = atf.rope_layout(x.cuda(), theta, rotate=False, pairing=HALF)
    assert torch.equal(xo.cpu(), torch.from_numpy(_interleave(x.view(torch.int16).numpy())).view(torch.bfloat16))


@pytest.mark.parametrize("B,S,Hq,Hkv,d,theta,alpha", [
    (1, 300, 7, 1, 128, 1e7, 1.0),
    (2, 517, 8, 2, 128, 1e4, 0.5),
    (1, 640, 4, 4, 64, 1e4, 1.0),
    (1, 384, 7, 1, 128, 1e7, math.inf),
])
def test_prefill_rotate_half_against_oracle(B, S, Hq, Hkv, d, theta, alpha):
    q, k, v = synth.random_prefill(B, S, S, Hq, Hkv, d, torch.bfloat16, seed=31)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    got = atf.prefill(q.cuda(), k.cuda(), v.cuda(), theta, alpha, skipped=cnt, pairing=HALF)
    atf.atf_check()
    want, skipped = oracle.prefill(q, k, v, theta, alpha, pairing=oracle.ROTATE_HALF)
    assert np.abs(got.cpu().double().numpy() - want).max() <= TOL
    assert int(cnt.item()) == skipped
    # the pairing matters: the interleaved reading of the same inputs differs
    other, _ = oracle.prefill(q, k, v, theta, alpha, pairing=oracle.INTERLEAVED)
    assert np.abs(other - want).max() > 2 * TOL


def test_prefill_rotate_half_chunk_with_offset():
    """A query chunk at an offset against the full preceding keys (chunked prefill)."""
    q_offset, q_len, theta = 1024, 256, 1e7
    q, k, v = synth.random_prefill(1, q_len, q_offset + q_len, 7, 1, 128, torch.bfloat16, seed=37)
    got = atf.prefill(q.cuda(), k.cuda(), v.cuda(), theta, 1.0, q_offset=q_offset, pairing=HALF)
    atf.atf_check()
    want, _ = oracle.prefill(q, k, v, theta, 1.0, q_offset=q_offset, pairing=oracle.ROTATE_HALF)
    assert np.abs(got.cpu().double().numpy() - want).max() <= TOL


@pytest.mark.parametrize("B,N,kv_len,Hq,Hkv,d,theta,alpha", [
    (2, 3000, [3000, 1337], 28, 4, 128, 1e7, 1.0),
    (1, 2048, [2048], 4, 4, 64, 1e4, 0.5),
])
def test_decode_rotate_half_against_oracle(B, N, kv_len, Hq, Hkv, d, theta, alpha):
    q = synth.token_major(9, 602, 0, B, 1, Hq, d, torch.bfloat16, threads=1)[:, 0].contiguous()
    k = synth.token_major(9, 602, 1, B, N, Hkv, d, torch.bfloat16, threads=1)
    v = synth.token_major(9, 602, 2, B, N, Hkv, d, torch.bfloat16, threads=1)
    # the cache holds rotate-half-rotated keys (rounded to bf16, as a model's cache would)
    k_rot = torch.from_numpy(oracle.rope(k, theta, pairing=oracle.ROTATE_HALF)).to(torch.bfloat16)
    _, kc = atf.rope_layout(k_rot.cuda(), theta, rotate=False, rotated_out=False, chunked_out=True, pairing=HALF)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    got = atf.decode(q.cuda(), kc, v.cuda(), kv_len, theta, alpha, skipped=cnt, pairing=HALF)
    atf.atf_check()
    want, skipped = oracle.decode(q, k_rot, v, kv_len, theta, alpha, pairing=oracle.ROTATE_HALF)
    assert np.abs(got.cpu().double().numpy() - want).max() <= TOL
    assert int(cnt.item()) == skipped

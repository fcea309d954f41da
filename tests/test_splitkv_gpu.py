"""Split-KV decode on one GPU: the key ranges of emulated ranks decoded one after
the other (atf_decode_partial on each rank's own cache) and merged
(atf_decode_merge), against the oracle and the single-cache decode."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import splitkv as osk
from rope_frequency_sparse_b200 import atf, splitkv, synth

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _setup(B, N, Hq, Hkv, d, theta, seed):
    q = synth.token_major(seed, 960, 0, B, 1, Hq, d, torch.bfloat16, threads=1)[:, 0].contiguous()
    k = synth.token_major(seed, 960, 1, B, N, Hkv, d, torch.bfloat16, threads=1)
    v = synth.token_major(seed, 960, 2, B, N, Hkv, d, torch.bfloat16, threads=1)
    k_rot = torch.from_numpy(oracle.rope(k, theta)).to(torch.bfloat16)  # keys rotated at their positions
    return q, k_rot, v


def _rank_cache(k_rot, v, ranges):
    """A rank's own cache: sequence b's keys ranges[b] = (lo, hi) in slots 0 .. hi-lo-1."""
    B, _, Hkv, d = k_rot.shape
    n_loc = max(1, max(hi - lo for lo, hi in ranges))
    kl = torch.zeros(B, n_loc, Hkv, d, dtype=torch.bfloat16)
    vl = torch.zeros(B, n_loc, Hkv, d, dtype=torch.bfloat16)
    for b, (lo, hi) in enumerate(ranges):
        kl[b, : hi - lo] = k_rot[b, lo:hi]
        vl[b, : hi - lo] = v[b, lo:hi]
    _, kc = atf.rope_layout(kl.cuda(), 1e4, rotate=False, rotated_out=False, chunked_out=True)
    return kc, vl.cuda()


def _partial(q, kc, vl, ranges, lens, theta, alpha, cnt=None):
    B, Hq, d = q.shape
    _, Hkv, _, N, _ = kc.shape
    part = torch.empty(B, Hq, d + 2, dtype=torch.float32, device="cuda")
    n_keys = [hi - lo for lo, hi in ranges]
    need = atf.atf_decode_workspace_bytes(B, Hq, Hkv, max(max(n_keys), 1), d)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    atf.atf_decode_partial(q.cuda(), kc, vl, part, B, n_keys, [lo for lo, _ in ranges], [L - 1 for L in lens], N, Hq,
                           Hkv, d, theta, alpha, ws, need, cnt)
    return part


@pytest.mark.parametrize("world,alpha", [(3, 1.0), (2, 0.5), (5, math.inf)])
def test_merged_ranks_match_oracle_and_full_decode(world, alpha):
    B, N, Hq, Hkv, d, theta = 2, 3000, 28, 4, 128, 1e7
    lens = [3000, 1337]
    q, k_rot, v = _setup(B, N, Hq, Hkv, d, theta, seed=91)
    per_seq = [splitkv.shard_ranges(L, world, d, theta, alpha) for L in lens]
    parts, cnt = [], torch.zeros(1, dtype=torch.int64, device="cuda")
    for r in range(world):
        ranges = [per_seq[b][r] for b in range(B)]
        kc, vl = _rank_cache(k_rot, v, ranges)
        parts.append(_partial(q, kc, vl, ranges, lens, theta, alpha, cnt))
    stacked = torch.stack(parts).contiguous()
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    atf.atf_decode_merge(stacked, world, B, Hq, d, out)
    atf.atf_check()
    want, skipped = oracle.decode(q, k_rot, v, lens, theta, alpha)
    assert np.abs(out.cpu().double().numpy() - want).max() <= TOL
    assert int(cnt.item()) == skipped
    # against the single-cache decode on the same rotated keys
    _, kc_full = atf.rope_layout(k_rot.cuda(), 1e4, rotate=False, rotated_out=False, chunked_out=True)
    full = atf.decode(q.cuda(), kc_full, v.cuda(), lens, theta, alpha)
    atf.atf_check()
    assert (out.float() - full.float()).abs().max().item() <= TOL


def test_one_part_is_the_decode_bit_for_bit():
    B, N, Hq, Hkv, d, theta = 2, 2000, 8, 2, 64, 1e4
    lens = [2000, 777]
    q, k_rot, v = _setup(B, N, Hq, Hkv, d, theta, seed=92)
    _, kc = atf.rope_layout(k_rot.cuda(), 1e4, rotate=False, rotated_out=False, chunked_out=True)
    part = _partial(q, kc, v.cuda(), [(0, L) for L in lens], lens, theta, 1.0)
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    atf.atf_decode_merge(part, 1, B, Hq, d, out)
    full = atf.decode(q.cuda(), kc, v.cuda(), lens, theta, 1.0)
    atf.atf_check()
    assert torch.equal(out, full)
    # decode_split_kv without a process group is the same partial and merge
    sk = splitkv.decode_split_kv(q.cuda(), kc, v.cuda(), lens, [0, 0], [L - 1 for L in lens], theta, 1.0)
    atf.atf_check()
    assert torch.equal(sk, full)


def test_an_empty_range_contributes_nothing():
    B, N, Hq, Hkv, d, theta = 1, 1500, 7, 1, 128, 1e7
    q, k_rot, v = _setup(B, N, Hq, Hkv, d, theta, seed=93)
    kc0, vl0 = _rank_cache(k_rot, v, [(0, N)])
    kce, vle = _rank_cache(k_rot, v, [(N, N)])
    p0 = _partial(q, kc0, vl0, [(0, N)], [N], theta, 1.0)
    pe = _partial(q, kce, vle, [(N, N)], [N], theta, 1.0)
    assert torch.isneginf(pe[..., d]).all() and (pe[..., d + 1] == 0).all()
    a = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    b = torch.empty_like(a)
    atf.atf_decode_merge(torch.stack([pe, p0]).contiguous(), 2, B, Hq, d, a)
    atf.atf_decode_merge(p0, 1, B, Hq, d, b)
    atf.atf_check()
    assert torch.equal(a, b)


@pytest.mark.parametrize("alpha", [1.0, math.inf])
def test_partial_beyond_position_2_31(alpha):
    """Keys at positions past 2^31 (the query a few positions after the last key):
    positions are 64-bit, distances stay below 2^31, and with alpha = inf every
    key keeps every pair (the 32-bit window clamp is exact)."""
    B, N, Hq, Hkv, d, theta = 1, 3000, 28, 4, 128, 1e7
    P = (1 << 31) + 12345
    q = synth.token_major(94, 960, 0, B, 1, Hq, d, torch.bfloat16, threads=1)[:, 0].contiguous()
    k = synth.token_major(94, 960, 1, B, N, Hkv, d, torch.bfloat16, threads=1)
    v = synth.token_major(94, 960, 2, B, N, Hkv, d, torch.bfloat16, threads=1)
    k_rot = torch.from_numpy(oracle.rope(k, theta, pos0=P)).to(torch.bfloat16)  # key n at position P + n
    _, kc = atf.rope_layout(k_rot.cuda(), 1e4, rotate=False, rotated_out=False, chunked_out=True)
    q_pos = P + N + 6
    part = torch.empty(B, Hq, d + 2, dtype=torch.float32, device="cuda")
    need = atf.atf_decode_workspace_bytes(B, Hq, Hkv, N, d)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    atf.atf_decode_partial(q.cuda(), kc, v.cuda(), part, B, [N], [P], [q_pos], N, Hq, Hkv, d, theta, alpha, ws,
                           need, None)
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    atf.atf_decode_merge(part, 1, B, Hq, d, out)
    atf.atf_check()
    want = osk.merge(osk.partial(q, k_rot, v, [0], [N], [q_pos], theta, alpha, key_pos0=[P])[None])
    assert np.abs(out.cpu().double().numpy() - want).max() <= TOL

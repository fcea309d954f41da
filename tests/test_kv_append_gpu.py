"""KV-cache append (new tokens rotated into the chunk-major key cache, values
copied) against the one-shot layout and the oracle, and decode on appended caches."""
import numpy as np
import pytest
import torch

import oracle
from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _empty_caches(B, N, Hkv, d, fill=0.0):
    kc = torch.full((B, Hkv, d // 16, N, 16), fill, dtype=torch.bfloat16, device="cuda")
    vc = torch.full((B, N, Hkv, d), fill, dtype=torch.bfloat16, device="cuda")
    return kc, vc


def _packed(x, counts, starts):
    """rows starts[b] .. starts[b] + counts[b] - 1 of every sequence b of x [B][S][H][d], packed."""
    return torch.cat([x[b, starts[b]: starts[b] + counts[b]] for b in range(x.shape[0])], dim=0).contiguous()


@pytest.mark.parametrize("pairing", [atf.ATF_PAIRS_INTERLEAVED, atf.ATF_PAIRS_ROTATE_HALF])
def test_append_in_pieces_equals_one_shot_layout(pairing):
    B, S, Hkv, d, theta = 2, 700, 4, 128, 1e7
    k = synth.token_major(5, 701, 0, B, S, Hkv, d, torch.bfloat16, threads=1).cuda()
    v = synth.token_major(5, 701, 1, B, S, Hkv, d, torch.bfloat16, threads=1).cuda()
    _, want = atf.rope_layout(k, theta, rotated_out=False, chunked_out=True, pairing=pairing)
    kc, vc = _empty_caches(B, S, Hkv, d)
    pos = [0, 0]
    for piece in ([300, 1], [1, 450], [399, 249]):  # ragged pieces, all tokens in the end
        atf.atf_kv_append(_packed(k, piece, pos), _packed(v, piece, pos), kc, vc, B, piece, pos, S, Hkv, d, theta,
                          pairing)
        pos = [p + n for p, n in zip(pos, piece)]
    atf.atf_check()
    assert pos == [S, S]
    assert torch.equal(kc, want)
    assert torch.equal(vc, v)


def test_append_varlen_leaves_other_slots_alone():
    B, N, Hkv, d, theta = 3, 4096, 2, 64, 1e4
    counts, starts = [5, 0, 1000], [100, 7, 3000]
    k = synth.token_major(6, 702, 0, B, N, Hkv, d, torch.bfloat16, threads=1).cuda()
    v = synth.token_major(6, 702, 1, B, N, Hkv, d, torch.bfloat16, threads=1).cuda()
    sentinel = 1234.0
    kc, vc = _empty_caches(B, N, Hkv, d, fill=sentinel)
    atf.atf_kv_append(_packed(k, counts, starts), _packed(v, counts, starts), kc, vc, B, counts, starts, N, Hkv, d,
                      theta)
    atf.atf_check()
    _, full = atf.rope_layout(k, theta, rotated_out=False, chunked_out=True)
    for b in range(B):
        lo, hi = starts[b], starts[b] + counts[b]
        assert torch.equal(kc[b, :, :, lo:hi], full[b, :, :, lo:hi])
        assert torch.equal(vc[b, lo:hi], v[b, lo:hi])
        untouched_k = torch.cat([kc[b, :, :, :lo].flatten(), kc[b, :, :, hi:].flatten()])
        untouched_v = torch.cat([vc[b, :lo].flatten(), vc[b, hi:].flatten()])
        assert (untouched_k == sentinel).all() and (untouched_v == sentinel).all()


def test_appended_keys_match_oracle_rotation():
    B, S, Hkv, d, theta, p0 = 1, 64, 4, 128, 1e7, (1 << 20) - 64
    k = synth.token_major(7, 703, 0, B, S, Hkv, d, torch.bfloat16, threads=1)
    kc, vc = _empty_caches(B, 1 << 20, Hkv, d)
    atf.atf_kv_append(k[0].contiguous().cuda(), k[0].contiguous().cuda(), kc, vc, 1, [S], [p0], 1 << 20, Hkv, d,
                      theta)
    atf.atf_check()
    want = torch.from_numpy(oracle.rope(k, theta, pos0=p0)).to(torch.bfloat16)  # [1][S][H][d]
    got = kc[0, :, :, p0:].permute(2, 0, 1, 3).reshape(S, Hkv, d).cpu()
    assert (got.view(torch.int16) == want[0].view(torch.int16)).float().mean() > 0.999
    assert (got.float() - want[0].float()).abs().max().item() <= 2.0 ** -7 * want.float().abs().max().item()


def test_decode_serving_loop_on_appended_cache():
    """Prefix appended at once, then one token per sequence and step, decoding after
    each append, against the oracle on the same keys."""
    B, N, Hq, Hkv, d, theta, alpha = 2, 1536, 14, 2, 128, 1e7, 1.0
    prefix, steps = [1000, 517], 4
    q = synth.token_major(8, 704, 0, B, steps, Hq, d, torch.bfloat16, threads=1)
    k = synth.token_major(8, 704, 1, B, N, Hkv, d, torch.bfloat16, threads=1)
    v = synth.token_major(8, 704, 2, B, N, Hkv, d, torch.bfloat16, threads=1)
    kd, vd = k.cuda(), v.cuda()
    kc, vc = _empty_caches(B, N, Hkv, d)
    atf.atf_kv_append(_packed(kd, prefix, [0, 0]), _packed(vd, prefix, [0, 0]), kc, vc, B, prefix, [0, 0], N,
                      Hkv, d, theta)
    k_rot = torch.from_numpy(oracle.rope(k, theta)).to(torch.bfloat16)  # the cache the oracle reads
    lens = list(prefix)
    for s in range(steps):
        one = [1] * B
        atf.atf_kv_append(_packed(kd, one, lens), _packed(vd, one, lens), kc, vc, B, one, lens, N, Hkv, d, theta)
        lens = [n + 1 for n in lens]
        qs = q[:, s].contiguous()
        got = atf.decode(qs.cuda(), kc, vc, lens, theta, alpha)
        atf.atf_check()
        want, _ = oracle.decode(qs, k_rot, v, lens, theta, alpha)
        assert np.abs(got.cpu().double().numpy() - want).max() <= TOL, s

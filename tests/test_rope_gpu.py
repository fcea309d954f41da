"""RoPE + pair-chunk-major layout kernel against the oracle's fp64 rotation."""
import numpy as np
import pytest
import torch

import oracle
from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu


def _bf16_round(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("S,H,d,theta,pos0", [(33, 4, 128, 1e7, 0), (300, 28, 128, 1e7, 1000),
                                              (17, 2, 64, 1e4, (1 << 20) - 17), (5, 1, 128, 1e7, (1 << 21))])
def test_rope_bf16_matches_oracle(S, H, d, theta, pos0):
    x = synth.token_major(1, 77, 0, 2, S, H, d, torch.bfloat16, threads=1)
    want = _bf16_round(oracle.rope(x, theta, pos0=pos0))
    xr, xc = atf.rope_layout(x.cuda(), theta, pos_offset=pos0, chunked_out=True)
    got = xr.cpu()
    diff = (got.float() - want.float()).abs()
    # one rounding of an fp64 value to bf16 on both sides: identical except at
    # exact rounding ties of differently rounded fp64 inputs
    assert (got.view(torch.int16) == want.view(torch.int16)).float().mean() > 0.999
    assert diff.max().item() <= 2.0 ** -7 * want.float().abs().max().item()
    # chunk-major copy holds exactly the rotated values: [B][H][d/16][S][16]
    B = x.shape[0]
    ref = got.view(B, S, H, d // 16, 16).permute(0, 2, 3, 1, 4).contiguous()
    assert torch.equal(xc.cpu(), ref)


def test_rope_fp32_matches_oracle():
    x = synth.token_major(2, 78, 0, 1, 512, 1, 64, torch.float32, threads=1)
    want = oracle.rope(x, 1e4, pos0=0)
    xr, _ = atf.rope_layout(x.cuda(), 1e4)
    assert np.abs(xr.cpu().double().numpy() - want).max() < 1e-6


def test_layout_only_copy_is_exact():
    x = synth.token_major(3, 79, 0, 2, 130, 4, 128, torch.bfloat16, threads=1).cuda()
    xr, xc = atf.rope_layout(x, 1e7, rotate=False, chunked_out=True)
    assert torch.equal(xr, x)
    ref = x.view(2, 130, 4, 8, 16).permute(0, 2, 3, 1, 4).contiguous()
    assert torch.equal(xc, ref)

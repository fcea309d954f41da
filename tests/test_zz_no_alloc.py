"""atf_decode_noalloc: the decode entry point for callers that cannot allocate
device memory on the decode path (a host application whose memory manager owns
all device memory, or a latency-critical loop where an allocation could
synchronise the device).  Its scratch is a fixed device array inside the
library.  It runs the same kernels with the same key-range splits as atf_decode
(which uses a caller workspace), so its output must be bit-identical to
atf_decode's, on two calls in a row (the second call sees the array as the first
left it).  Collected last on purpose."""
import numpy as np
import pytest
import torch

from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode_twice():
    B, N, Hq, Hkv, d, theta, alpha = 3, 5000, 28, 4, 128, 1e7, 1.0
    kv_len = [5000, 4097, 777]
    q = synth.token_major(11, 601, 0, B, 1, Hq, d, torch.bfloat16, threads=1)[:, 0].contiguous().cuda()
    k = synth.token_major(11, 601, 1, B, N, Hkv, d, torch.bfloat16, threads=1).cuda()
    v = synth.token_major(11, 601, 2, B, N, Hkv, d, torch.bfloat16, threads=1).cuda()
    _, kc = atf.rope_layout(k, theta, rotate=False, rotated_out=False, chunked_out=True)

    cnt_ref = torch.zeros(1, dtype=torch.int64, device="cuda")
    ref = atf.decode(q, kc, v, kv_len, theta, alpha, skipped=cnt_ref)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
        atf.atf_decode_noalloc(q, kc, v, out, B, kv_len, N, Hq, Hkv, d, theta, alpha, cnt)
        atf.atf_check()
        assert torch.equal(out, ref), (call, (out.float() - ref.float()).abs().max().item())
        assert int(cnt.item()) == int(cnt_ref.item())


def test_noalloc_rejects_calls_beyond_its_fixed_scratch():
    cap = atf.atf_decode_noalloc_scratch_bytes()
    # one partial per (sequence, query head, split): 400 x 64 x 130 floats > 8 MiB
    B, Hq, Hkv, d = 400, 64, 8, 128
    assert atf.atf_decode_workspace_bytes(B, Hq, Hkv, 1 << 20, d) > cap
    fake = 1 << 20  # never dereferenced: the call is rejected before any work
    with pytest.raises(atf.AtfError) as e:
        atf.atf_decode_noalloc(fake, fake, fake, fake, B, np.full(B, 1 << 20), 1 << 20, Hq, Hkv, d, 1e7, 1.0)
    assert e.value.status == atf.ATF_ERR_UNSUPPORTED
    assert "scratch" in atf.atf_last_error()

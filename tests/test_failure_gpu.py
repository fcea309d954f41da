"""Failure detection without a GPU fault: a kernel whose barrier is never
completed gives up after a short bounded wait, records the expiry in the device
error word, and returns; the host reads it back as ATF_ERR_TIMEOUT and the
context stays usable."""
import pytest
import torch

from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_expiry_is_reported_and_context_survives():
    atf.atf_check()  # clean state
    atf.atf_selftest_timeout(2_000_000)  # ~1 ms of SM clocks
    with pytest.raises(atf.AtfError) as e:
        atf.atf_check()
    assert e.value.status == atf.ATF_ERR_TIMEOUT
    atf.atf_check()  # the error word was cleared
    # the context still runs real work afterwards
    q, k, v = synth.random_prefill(1, 64, 64, 2, 1, 128, torch.bfloat16, seed=3)
    out = atf.prefill(q.cuda(), k.cuda(), v.cuda(), 1e7, 1.0)
    atf.atf_check()
    assert torch.isfinite(out.float()).all()

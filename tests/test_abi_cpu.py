"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/atf.h declares, computes the window table like the oracle, and
rejects bad arguments before touching a device."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle
from rope_frequency_sparse_b200 import atf, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return atf.load_library()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "atf.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(atf_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("d,theta", [(64, 1e4), (128, 1e7), (128, 5e5), (64, 1.0001)])
@pytest.mark.parametrize("alpha", [0.1, 0.5, 1.0, 2.0, math.inf])
def test_windows_match_oracle(lib, d, theta, alpha):
    W_lib = atf.atf_windows(d, theta, alpha)
    W_or, _ = oracle.windows(d, theta, alpha)
    assert W_lib.tolist() == W_or.tolist()


def _status(fn):
    try:
        fn()
    except atf.AtfError as e:
        return e.status
    return atf.ATF_OK


def test_rejects_bad_arguments_before_any_device_call(lib):
    fake = 1 << 20  # a 16-byte aligned address; never dereferenced
    P = atf.atf_prefill_ex
    assert _status(lambda: P(fake, fake, fake, fake, 1, 128, 128, 28, 4, 96, 0, 0, 1, 1e7, 1.0)) == \
        atf.ATF_ERR_UNSUPPORTED
    assert _status(lambda: P(fake, fake, fake, fake, 1, 128, 128, 28, 5, 128, 0, 0, 1, 1e7, 1.0)) == \
        atf.ATF_ERR_INVALID_ARG
    assert _status(lambda: P(fake, fake, fake, fake, 1, 128, 100, 28, 4, 128, 0, 0, 1, 1e7, 1.0)) == \
        atf.ATF_ERR_INVALID_ARG  # kv_len < q_offset + q_len
    assert _status(lambda: P(None, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1, 1e7, 1.0)) == \
        atf.ATF_ERR_INVALID_ARG
    assert _status(lambda: P(fake + 8, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1, 1e7, 1.0)) == \
        atf.ATF_ERR_INVALID_ARG  # misaligned
    assert _status(lambda: P(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1, 0.5, 1.0)) == \
        atf.ATF_ERR_INVALID_ARG  # theta <= 1
    assert _status(lambda: P(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1, 1e7, -1.0)) == \
        atf.ATF_ERR_INVALID_ARG  # alpha <= 0
    assert _status(lambda: P(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 0, 1e7, 1.0)) == \
        atf.ATF_ERR_INVALID_ARG  # unrotated inputs need a workspace
    assert "workspace" in atf.atf_last_error()
    D = atf.atf_decode
    assert _status(lambda: D(fake, fake, fake, fake, 2, [5, 0], 8, 28, 4, 128, 1e7, 1.0, fake, 1 << 20)) == \
        atf.ATF_ERR_INVALID_ARG  # kv_len 0
    assert _status(lambda: D(fake, fake, fake, fake, 1, [9], 8, 28, 4, 128, 1e7, 1.0, fake, 1 << 20)) == \
        atf.ATF_ERR_INVALID_ARG  # kv_len > n_cache
    assert _status(lambda: D(fake, fake, fake, fake, 1, [8], 8, 36, 4, 128, 1e7, 1.0, fake, 1 << 20)) == \
        atf.ATF_ERR_UNSUPPORTED  # 9 query heads per kv head
    assert _status(lambda: D(fake, fake, fake, fake, 1, [8], 8, 28, 4, 128, 1e7, 1.0, fake, 4)) == \
        atf.ATF_ERR_INVALID_ARG  # workspace too small
    assert _status(lambda: atf.atf_rope_layout(fake, None, fake, 1, 8, 4, 128, 0, 1e7, 1, atf.ATF_FP32)) == \
        atf.ATF_ERR_UNSUPPORTED  # chunk-major is bf16 only
    assert _status(lambda: atf.atf_rope_layout(fake, fake, None, 1, 8, 4, 128, 0, 1e7, 4, atf.ATF_BF16)) == \
        atf.ATF_ERR_INVALID_ARG  # no such rotate mode
    assert _status(lambda: D(fake, fake, fake, fake, 1, [8], 8, 28, 4, 128, 1e7, 1.0, fake, 1 << 20,
                             pairing=2)) == atf.ATF_ERR_INVALID_ARG  # no such pairing
    A = atf.atf_kv_append
    assert _status(lambda: A(fake, fake, fake, fake, 2, [3, 4], [0, 5], 8, 4, 128, 1e7)) == \
        atf.ATF_ERR_INVALID_ARG  # 5 + 4 > 8 slots
    assert _status(lambda: A(fake, fake, fake, fake, 1, [-1], [0], 8, 4, 128, 1e7)) == atf.ATF_ERR_INVALID_ARG
    assert _status(lambda: A(fake + 8, fake, fake, fake, 1, [1], [0], 8, 4, 128, 1e7)) == \
        atf.ATF_ERR_INVALID_ARG  # misaligned
    assert _status(lambda: A(fake, fake, fake, fake, 1, [1], [0], 8, 4, 96, 1e7)) == atf.ATF_ERR_UNSUPPORTED
    DP = atf.atf_decode_partial
    assert _status(lambda: DP(fake, fake, fake, fake, 1, [5], [10], [13], 8, 28, 4, 128, 1e7, 1.0, fake,
                              1 << 20)) == atf.ATF_ERR_INVALID_ARG  # query before the last key (14)
    assert _status(lambda: DP(fake, fake, fake, fake, 1, [9], [0], [100], 8, 28, 4, 128, 1e7, 1.0, fake,
                              1 << 20)) == atf.ATF_ERR_INVALID_ARG  # more keys than slots
    assert _status(lambda: DP(fake, fake, fake, fake, 1, [2], [-1], [100], 8, 28, 4, 128, 1e7, 1.0, fake,
                              1 << 20)) == atf.ATF_ERR_INVALID_ARG  # negative position
    # distances of 2^31 or more would overflow the kernels' 32-bit windows
    assert _status(lambda: DP(fake, fake, fake, fake, 1, [4], [5], [5 + (1 << 31)], 8, 28, 4, 128, 1e7,
                              math.inf, fake, 1 << 20)) == atf.ATF_ERR_UNSUPPORTED
    assert _status(lambda: DP(fake, fake, fake, fake, 1, [4], [(1 << 32) + 5], [(1 << 32) + 8], 8, 28, 4, 128,
                              1e7, math.inf, fake, 1)) == atf.ATF_ERR_INVALID_ARG  # far positions pass that check
    assert _status(lambda: atf.atf_decode_merge(fake, 0, 1, 28, 128, fake)) == atf.ATF_ERR_INVALID_ARG
    assert _status(lambda: atf.atf_decode_merge(fake, 2, 1, 28, 96, fake)) == atf.ATF_ERR_UNSUPPORTED
    assert _status(lambda: atf.atf_decode_merge(fake + 4, 2, 1, 28, 128, fake)) == atf.ATF_ERR_INVALID_ARG
    F = atf.atf_fasa_decode
    fws = atf.atf_fasa_workspace_bytes(1, 28, 64, 16, 128)
    ok_args = dict(batch=1, kv_len=[64], n_cache=64, heads=28, kv_heads=4, d=128, pair_mask=0xFF, budget=16)

    def fasa(**kw):
        a = dict(ok_args, **kw)
        return _status(lambda: F(fake, fake, fake, fake, a["batch"], a["kv_len"], a["n_cache"], a["heads"],
                                 a["kv_heads"], a["d"], a["pair_mask"], a["budget"], workspace=kw.get("ws", fake),
                                 workspace_bytes=kw.get("wsb", fws)))

    assert fasa(pair_mask=0) == atf.ATF_ERR_INVALID_ARG
    assert fasa(d=64, pair_mask=1 << 32) == atf.ATF_ERR_INVALID_ARG  # pair past d/2
    assert fasa(budget=0) == atf.ATF_ERR_UNSUPPORTED
    assert fasa(budget=4097) == atf.ATF_ERR_UNSUPPORTED
    assert fasa(kv_len=[0]) == atf.ATF_ERR_INVALID_ARG
    assert fasa(kv_len=[65]) == atf.ATF_ERR_INVALID_ARG
    assert fasa(heads=36) == atf.ATF_ERR_UNSUPPORTED  # 9 query heads per kv head
    assert fasa(heads=30) == atf.ATF_ERR_INVALID_ARG  # heads % kv_heads
    assert fasa(d=96) == atf.ATF_ERR_UNSUPPORTED
    assert fasa(wsb=fws - 1) == atf.ATF_ERR_INVALID_ARG and "workspace" in atf.atf_last_error()
    assert fasa(ws=fake + 8) == atf.ATF_ERR_INVALID_ARG  # misaligned
    assert fasa(ws=None) == atf.ATF_ERR_INVALID_ARG
    H = atf.atf_prefill_host
    need = atf.atf_prefill_host_workspace_bytes(1, 128, 128, 28, 4, 128, 0)
    assert _status(lambda: H(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1e7, 1.0, fake, need - 1)) == \
        atf.ATF_ERR_INVALID_ARG  # workspace too small
    assert "workspace" in atf.atf_last_error()
    assert _status(lambda: H(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1e7, 1.0, fake + 8, need)) == \
        atf.ATF_ERR_INVALID_ARG  # misaligned workspace
    assert _status(lambda: H(fake, fake, fake, fake, 1, 128, 100, 28, 4, 128, 0, 0, 1e7, 1.0, fake, need)) == \
        atf.ATF_ERR_INVALID_ARG  # kv_len < q_offset + q_len
    assert _status(lambda: H(fake, fake, fake, fake, 1, 128, 128, 28, 4, 96, 0, 0, 1e7, 1.0, fake, need)) == \
        atf.ATF_ERR_UNSUPPORTED
    assert _status(lambda: H(fake, fake, fake, fake, 1, 128, 128, 28, 5, 128, 0, 0, 1e7, 1.0, fake, need)) == \
        atf.ATF_ERR_INVALID_ARG  # heads % kv_heads
    assert _status(lambda: H(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1e7, 1.0, fake, need,
                             chunk_rows=-1)) == atf.ATF_ERR_INVALID_ARG
    assert _status(lambda: H(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1e7, 1.0, fake, need,
                             pairing=2)) == atf.ATF_ERR_INVALID_ARG
    assert _status(lambda: H(fake, None, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1e7, 1.0, fake, need)) == \
        atf.ATF_ERR_INVALID_ARG
    assert _status(lambda: H(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 0.5, 1.0, fake, need)) == \
        atf.ATF_ERR_INVALID_ARG  # theta <= 1


def test_empty_inputs_are_no_ops(lib):
    atf.atf_prefill_ex(None, None, None, None, 1, 0, 0, 28, 4, 128, 0, 0, 1, 1e7, 1.0)
    atf.atf_prefill_ex(None, None, None, None, 0, 16, 16, 28, 4, 128, 0, 0, 1, 1e7, 1.0)
    atf.atf_decode(None, None, None, None, 0, [], 8, 28, 4, 128, 1e7, 1.0, None, 0)
    atf.atf_rope_layout(None, None, None, 0, 8, 4, 128, 0, 1e7, 1, 0)
    atf.atf_kv_append(None, None, None, None, 0, [], [], 8, 4, 128, 1e7)
    atf.atf_kv_append(None, None, None, None, 2, [0, 0], [3, 8], 8, 4, 128, 1e7)  # nothing to append
    atf.atf_prefill_host(None, None, None, None, 1, 0, 0, 28, 4, 128, 0, 0, 1e7, 1.0, None, 0)
    atf.atf_fasa_decode(None, None, None, None, 0, [], 8, 28, 4, 128, 0xFF, 16)


def test_workspace_sizes(lib):
    assert atf.atf_prefill_workspace_bytes(1, 8192, 8192, 28, 4, 128, 0, 1) == 0
    ws = atf.atf_prefill_workspace_bytes(1, 8192, 8192, 28, 4, 128, 0, 0)
    assert ws >= 8192 * 28 * 128 * 2 + 8192 * 4 * 128 * 2
    # host path: device copies of q, k, v, rotated q and k, and the output
    hws = atf.atf_prefill_host_workspace_bytes(2, 1000, 1500, 28, 4, 128, 0)
    qb, kb = 2 * 1000 * 28 * 128 * 2, 2 * 1500 * 4 * 128 * 2
    assert hws == 3 * qb + 3 * kb
    assert atf.atf_prefill_host_workspace_bytes(2, 1000, 1500, 28, 4, 128, 1) == 2 * qb + 2 * kb
    assert atf.atf_prefill_host_workspace_bytes(0, 1000, 1500, 28, 4, 128, 0) == 0
    # FASA: candidate indices and scores per (sequence, query head, key slot of the 1024-key warp segments),
    # a count per segment, 4096-bin sample histograms, the thresholds (padded to 256 bytes), the selected
    # indices and their scores, a flag per row, attention partials (128 selected keys per split)
    fws = atf.atf_fasa_workspace_bytes(4, 28, 1 << 20, 2048, 128)
    rows = 4 * 28
    assert fws == (rows * (1 << 20) * 8 + rows * 1024 * 4 + rows * 4096 * 4 + 512 + 2 * rows * 2048 * 4 + 512
                   + rows * 16 * 130 * 4)
    # a cache that is not a whole number of segments rounds up to one
    assert atf.atf_fasa_workspace_bytes(1, 1, 1000, 10, 64) == (1024 * 8 + 256 + 4096 * 4 + 256 + 256 + 256 + 256
                                                                 + 512)
    dws = atf.atf_decode_workspace_bytes(4, 28, 4, 1 << 20, 128)
    assert dws % (4 * 28 * 130 * 4) == 0 and dws > 0


def test_valid_call_without_gpu_fails_loudly(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    fake = 1 << 20
    st = _status(lambda: atf.atf_prefill_ex(fake, fake, fake, fake, 1, 128, 128, 28, 4, 128, 0, 0, 1, 1e7, 1.0))
    assert st == atf.ATF_ERR_CUDA

"""Prefill from host buffers (atf_prefill_host): the chunked, copy-overlapped
pipeline gives the result of one prefill over all rows, against the device-path
prefill and the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _inputs(B, q_len, kv_len, Hq, Hkv, d, seed, pinned=True):
    q, k, v = synth.random_prefill(B, q_len, kv_len, Hq, Hkv, d, torch.bfloat16, seed=seed)
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    return q, k, v


@pytest.mark.parametrize("chunk_rows", [256, 512, 0, 4096])
def test_host_pipeline_equals_device_prefill_bitwise(chunk_rows):
    """Chunks that start on 256-row boundaries keep every query tile where the
    one-shot prefill has it, so the outputs agree bit for bit."""
    B, S, Hq, Hkv, d, theta, alpha = 2, 1000, 8, 2, 128, 1e7, 1.0
    q, k, v = _inputs(B, S, S, Hq, Hkv, d, seed=41)
    cnt_h = torch.zeros(1, dtype=torch.int64, device="cuda")
    got = atf.prefill_host(q, k, v, theta, alpha, skipped=cnt_h, chunk_rows=chunk_rows)
    cnt_d = torch.zeros(1, dtype=torch.int64, device="cuda")
    want = atf.prefill(q.cuda(), k.cuda(), v.cuda(), theta, alpha, skipped=cnt_d)
    atf.atf_check()
    assert got.device.type == "cpu" and got.is_pinned()
    assert torch.equal(got, want.cpu())
    assert int(cnt_h.item()) == int(cnt_d.item())


@pytest.mark.parametrize("B,q_len,kv_len,q_offset,Hq,Hkv,d,theta,alpha,chunk_rows,pairing", [
    (1, 700, 700, 0, 7, 1, 128, 1e7, 1.0, 300, atf.ATF_PAIRS_INTERLEAVED),      # ragged chunks
    (2, 384, 1024, 640, 8, 2, 128, 1e4, 0.5, 128, atf.ATF_PAIRS_INTERLEAVED),   # chunk at an offset
    (1, 517, 517, 0, 4, 4, 64, 1e4, 1.0, 200, atf.ATF_PAIRS_ROTATE_HALF),
    (3, 256, 256, 0, 8, 1, 128, 1e7, math.inf, 64, atf.ATF_PAIRS_INTERLEAVED),  # dense, many chunks
])
def test_host_pipeline_against_oracle(B, q_len, kv_len, q_offset, Hq, Hkv, d, theta, alpha, chunk_rows, pairing):
    q, k, v = _inputs(B, q_len, kv_len, Hq, Hkv, d, seed=43)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    got = atf.prefill_host(q, k, v, theta, alpha, q_offset=q_offset, skipped=cnt, chunk_rows=chunk_rows,
                           pairing=pairing)
    opair = oracle.ROTATE_HALF if pairing == atf.ATF_PAIRS_ROTATE_HALF else oracle.INTERLEAVED
    want, skipped = oracle.prefill(q, k, v, theta, alpha, q_offset=q_offset, pairing=opair)
    assert np.abs(got.double().numpy() - want).max() <= TOL
    assert int(cnt.item()) == skipped


def test_host_pipeline_prerotated_and_pageable():
    """rotated = 1 uploads straight into the rotated buffers; pageable host memory
    gives the same output as pinned."""
    B, S, Hq, Hkv, d, theta, alpha = 1, 640, 8, 2, 128, 1e7, 1.0
    q, k, v = _inputs(B, S, S, Hq, Hkv, d, seed=47, pinned=False)
    qr, _ = atf.rope_layout(q.cuda(), theta)
    kr, _ = atf.rope_layout(k.cuda(), theta)
    qr, kr = qr.cpu(), kr.cpu()
    got_rot = atf.prefill_host(qr, kr, v, theta, alpha, rotated=True, chunk_rows=256)
    got_raw = atf.prefill_host(q, k, v, theta, alpha, chunk_rows=256)
    got_pin = atf.prefill_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), theta, alpha, chunk_rows=256)
    assert torch.equal(got_rot, got_raw)
    assert torch.equal(got_raw, got_pin)


def test_host_pipeline_orders_with_the_callers_stream():
    """Work queued on the caller's stream before the call finishes before the
    uploads land, and work queued after it sees the whole output."""
    B, S, Hq, Hkv, d, theta, alpha = 1, 1024, 8, 2, 128, 1e7, 1.0
    q, k, v = _inputs(B, S, S, Hq, Hkv, d, seed=53)
    need = atf.atf_prefill_host_workspace_bytes(B, S, S, Hq, Hkv, d, 0)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q).pin_memory()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        ws.fill_(0xFF)  # garbage in every device buffer, on the same stream, just before the call
        atf.atf_prefill_host(q, k, v, out, B, S, S, Hq, Hkv, d, 0, 0, theta, alpha, ws, need, chunk_rows=256,
                             stream=side)
        after = torch.empty(B, S, Hq, d, dtype=torch.bfloat16, device="cuda")
        after.copy_(out, non_blocking=True)  # queued after the call on the same stream
    side.synchronize()
    want = atf.prefill(q.cuda(), k.cuda(), v.cuda(), theta, alpha)
    atf.atf_check()
    assert torch.equal(out, want.cpu())
    assert torch.equal(after.cpu(), want.cpu())

"""FASA-style decode (atf_fasa_decode) against the oracle.

The oracle's scores are exact (fp64); the kernel's are fp32 sums on the tensor
cores (16-dim cache chunks, one accumulation step each), so each kernel score
must lie within the oracle's "tensor" bound of the exact one, the kernel's
selection must be a correct one for the exact scores (oracle check_selection:
count and order, no dropped key ahead of a kept one by more than their bounds,
lower index first among identical keys), and the output must match the oracle's
focused attention over the kernel's own selection within the bf16 tolerance.

On small-integer inputs every product and partial sum is an exact integer, so
any summation order gives the exact score: there the kernel's scores must equal
the oracle's bit for bit and its selection must be the oracle's own (this pins
which dims, pairs and heads the kernel pairs up, independently of rounding)."""
import numpy as np
import pytest
import torch

from oracle import fasa as ofasa
from rope_frequency_sparse_b200 import atf, synth

pytestmark = pytest.mark.gpu

TOL = 2e-2
LOW16 = 0xFFFF << 48  # the 16 lowest-frequency pairs of d = 128 (two cache chunks)


def _inputs(B, N, Hq, Hkv, d, seed):
    q = synth.token_major(seed, 901, 0, B, 1, Hq, d, torch.bfloat16, threads=1)[:, 0].contiguous()
    k = synth.token_major(seed, 901, 1, B, N, Hkv, d, torch.bfloat16, threads=1)
    v = synth.token_major(seed, 901, 2, B, N, Hkv, d, torch.bfloat16, threads=1)
    return q, k, v


def _chunked(k_rot):
    """The chunk-major copy of already-rotated keys (a pure re-layout)."""
    _, kc = atf.rope_layout(k_rot.cuda(), 1e4, rotate=False, rotated_out=False, chunked_out=True)
    return kc


def _run(q, k, v, kv_len, mask, budget):
    B, Hq, d = q.shape
    N = k.shape[1]
    sel = torch.full((B, Hq, budget), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    out = atf.fasa_decode(q.cuda(), _chunked(k), v.cuda(), kv_len, mask, budget, selected=sel, scores=sc)
    atf.atf_check()
    return out.cpu(), sel.cpu().numpy(), sc.cpu().numpy()


def _check(q, k, v, kv_len, mask, budget):
    out, sel, sc = _run(q, k, v, kv_len, mask, budget)
    exact = ofasa.tip_scores(q, k, kv_len, mask)
    bound = ofasa.score_bound(q, k, kv_len, mask, model="tensor")
    for b, L in enumerate(kv_len):
        assert np.all(np.abs(sc[b, :, :L].astype(np.float64) - exact[b, :, :L]) <= bound[b, :, :L]), b
    ofasa.check_selection(sel, k, kv_len, budget, exact, bound, mask)
    want = ofasa.focused_attention(q, k, v, sel)
    assert np.abs(out.double().numpy() - want).max() <= TOL
    return sel


@pytest.mark.parametrize("B,N,kv_len,Hq,Hkv,d,mask,budget", [
    (2, 3000, [3000, 1337], 28, 4, 128, LOW16, 256),
    (1, 5000, [4999], 7, 1, 128, (1 << 3) | (0xFF << 20) | (1 << 63), 1000),
    (3, 700, [700, 1, 333], 4, 4, 64, 0b1010_0000_1111_0000_0000_0000_0000_0001, 100),
    (1, 2048, [2048], 8, 1, 64, (1 << 32) - 1, 4096),  # budget above kv_len: every key
])
def test_fasa_matches_oracle(B, N, kv_len, Hq, Hkv, d, mask, budget):
    q, k, v = _inputs(B, N, Hq, Hkv, d, seed=61)
    _check(q, k, v, kv_len, mask, budget)


@pytest.mark.parametrize("d,mask", [
    (128, (0x0F << 8) | (0xFF << 40) | (1 << 63)),  # part of a chunk, a whole chunk, one pair
    (64, (1 << 32) - 1),                            # every pair
])
def test_fasa_scores_are_exact_on_small_integers(d, mask):
    B, N, Hq, Hkv = 2, 3000, 8, 2
    kv_len, budget = [3000, 2222], 500
    g = np.random.default_rng(17)
    q = torch.from_numpy(g.integers(-8, 9, (B, Hq, d)).astype(np.float32)).to(torch.bfloat16)
    k = torch.from_numpy(g.integers(-8, 9, (B, N, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(g.standard_normal((B, N, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    out, sel, sc = _run(q, k, v, kv_len, mask, budget)
    exact = ofasa.tip_scores(q, k, kv_len, mask)
    for b, L in enumerate(kv_len):
        assert np.array_equal(sc[b, :, :L].astype(np.float64), exact[b, :, :L]), b
    assert np.array_equal(sel, ofasa.select(exact, kv_len, budget))  # many equal scores: the index decides
    assert np.abs(out.double().numpy() - ofasa.focused_attention(q, k, v, sel)).max() <= TOL


def test_fasa_heavy_ties_use_every_radix_pass():
    """Scores with five distinct values over 20000 keys: the budget boundary falls
    inside a block of equal scores, decided by the key index alone."""
    B, N, Hq, Hkv, d = 1, 20000, 2, 1, 64
    g = np.random.default_rng(5)
    q = torch.zeros(B, Hq, d)
    q[:, :, 2 * 7] = 1.0
    q[:, 1, 2 * 7] = -1.0
    k = torch.zeros(B, N, Hkv, d)
    k[..., 2 * 7] = torch.from_numpy(g.integers(-2, 3, size=(B, N, Hkv)).astype(np.float32))
    v = torch.from_numpy(g.standard_normal((B, N, Hkv, d)).astype(np.float32))
    q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    sel = _check(q, k, v, [N], 1 << 7, 3001)
    assert (sel >= 0).all()


def test_fasa_lists_longer_than_a_scan_block_stages():
    """65536 keys, 2048 per scan block: head 0 scores every key alike (all are
    candidates), head 1 scores keys 0..2999 high (they are all above the threshold
    bin, 2048 of them in one block), so both lists overflow a block's shared-memory
    stage and spill to the global append."""
    B, N, Hq, Hkv, d = 1, 1 << 16, 2, 1, 64
    g = np.random.default_rng(9)
    q = torch.zeros(B, Hq, d)
    q[:, :, 2 * 7] = 1.0
    k = torch.zeros(B, N, Hkv, d)
    k[0, :, 0, 2 * 7] = 1.0
    k[0, :3000, 0, 2 * 7 + 1] = 2.0
    q[:, 1, 2 * 7 + 1] = 1.0
    v = torch.from_numpy(g.standard_normal((B, N, Hkv, d)).astype(np.float32))
    q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    sel = _check(q, k, v, [N], 1 << 7, 4000)
    assert (sel[0, 0] == np.arange(4000)).all() and (sel[0, 1] == np.arange(4000)).all()


def test_fasa_unrepresentative_sample_falls_back_to_every_key():
    """The threshold comes from sampled keys (the first 32 of every 1024).  Here
    only the sampled keys score high, so fewer keys than the budget reach the
    threshold and the selection is redone over every key's score: the sampled
    keys plus the best of the rest, and the output from those."""
    B, N, Hq, Hkv, d = 1, 20000, 3, 1, 64
    g = np.random.default_rng(13)
    q = torch.zeros(B, Hq, d)
    q[:, :, 2 * 5] = 1.0
    q[:, 1, 2 * 5 + 1] = 0.25
    q[:, 2, 2 * 5] = -1.0
    k = torch.from_numpy(0.1 * g.standard_normal((B, N, Hkv, d)).astype(np.float32))
    sampled = (np.arange(N) % 1024) < 32
    k[0, sampled, 0, 2 * 5] = 4.0
    v = torch.from_numpy(g.standard_normal((B, N, Hkv, d)).astype(np.float32))
    q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    budget = 2048
    sel = _check(q, k, v, [N], 1 << 5, budget)
    n_sampled = int(sampled.sum())
    assert n_sampled < budget
    for h in (0, 1):  # every sampled key is kept, and budget - n_sampled others
        assert np.isin(np.nonzero(sampled)[0], sel[0, h]).all()
    assert not np.isin(np.nonzero(sampled)[0], sel[0, 2]).any()  # head 2 scores them lowest


def test_fasa_without_optional_outputs_gives_the_same_result():
    q, k, v = _inputs(2, 4096, 8, 2, 128, seed=67)
    kv_len, budget = [4096, 2500], 300
    out1, _, _ = _run(q, k, v, kv_len, LOW16, budget)
    out2 = atf.fasa_decode(q.cuda(), _chunked(k), v.cuda(), kv_len, LOW16, budget).cpu()
    atf.atf_check()
    assert torch.equal(out1, out2)


def test_fasa_more_sequences_than_chain_streams():
    """Each sequence's scoring, selection and attention run as one chain on the
    library's streams, round robin over four: six sequences of mixed lengths reuse
    two of them."""
    q, k, v = _inputs(6, 2600, 8, 2, 128, seed=73)
    _check(q, k, v, [2600, 1, 1300, 2600, 700, 2599], LOW16, 300)


def test_fasa_captured_in_a_graph_matches_direct_calls():
    """The call forks its chains from the caller's stream and joins them back, so
    it captures into a CUDA graph; replays give the direct call's output and
    selection bit for bit."""
    B, N, Hq, Hkv, d, budget = 5, 3000, 28, 4, 128, 256
    q, k, v = _inputs(B, N, Hq, Hkv, d, seed=79)
    kv_len = [3000, 2999, 1000, 2048, 77]
    qd, kd, vd = q.cuda(), _chunked(k), v.cuda()
    wsb = atf.atf_fasa_workspace_bytes(B, Hq, N, budget, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(qd)
    sel = torch.empty((B, Hq, budget), dtype=torch.int32, device="cuda")

    def call():
        atf.atf_fasa_decode(qd, kd, vd, out, B, kv_len, N, Hq, Hkv, d, LOW16, budget, sel, None, ws, wsb, None)

    call()
    torch.cuda.synchronize()
    atf.atf_check()
    out_ref, sel_ref = out.clone(), sel.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for _ in range(2):
        out.zero_()
        sel.fill_(-3)
        graph.replay()
        torch.cuda.synchronize()
        atf.atf_check()
        assert torch.equal(out, out_ref) and torch.equal(sel, sel_ref)


def test_fasa_full_size_cache():
    """One sequence of the 4 x 2^20-token decode workload, 28 query heads, budget 2048."""
    N, budget = 1 << 20, 2048
    q = synth.token_major(71, 902, 0, 1, 1, 28, 128, torch.bfloat16, threads=4)[:, 0].contiguous()
    k = synth.token_major(71, 902, 1, 1, N, 4, 128, torch.bfloat16, threads=4)
    v = synth.token_major(71, 902, 2, 1, N, 4, 128, torch.bfloat16, threads=4)
    _check(q, k, v, [N], LOW16, budget)

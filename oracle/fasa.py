"""Oracle for the FASA-style decode: token scoring on dominant frequency pairs
(Token Importance Predictor, TIP), top-k selection, then attention over the
selected tokens only (Focused Attention Computation, FAC).  Page "FASA", section
"Das FASA-Framework arbeitet in zwei Hauptphasen" (the two phases) and section
"Funktionale Sparsitaet auf Frequenz-Chunk-Ebene" (the dominant frequency chunks).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU legs, never by the CUDA library.  Plain numpy, one step per
phase, in the pages' order.

Readings of what the page leaves open:
- The dominant set is given (calibrating it needs model weights) as a set of
  RoPE frequency pairs; pair i = rotated dims (2i, 2i+1).
- A token's importance for query head h is the partial dot product of the
  rotated query and key over the dominant pairs only.
- Every query head selects its own ``budget`` tokens among keys 0..kv_len-1:
  highest score first, equal scores by lower key index.
- FAC is plain softmax attention, (1/sqrt d) q.k over all d dims, on the selected
  keys and their values.

The scores here are the exact partial dot products, in fp64 (a bf16 x bf16
product is exact in fp64, and so is the sum of at most 128 of them whose
magnitudes stay within 2^29 of each other -- below that the error is far under
any fp32 rounding).  A GPU computes them in fp32, so its selection is one of
possibly several correct ones where scores lie within rounding of each other:
``check_selection`` states which selections are correct (count and order; no
dropped key scoring above a kept one by more than the two keys' fp32 bounds;
the lower index first among keys whose dominant dims are identical), and
``score_bound`` gives the bound for one of two ways of summing in fp32:
- "fma": the n products added one at a time, each with one rounding: within
  n * 2^-24 * sum |q_j k_j| of the exact sum, in any order;
- "tensor": the dominant dims grouped by 16-dim cache chunk (pairs 8c .. 8c+7),
  each chunk's products added to the running fp32 sum in one step.  Assumed of
  such a step (a hardware adder that aligns its 17 addends to the largest one
  and keeps at least 24 bits of each): its result is within 18 * 2^-23 of the
  largest addend's magnitude of the exact step result.  Over C chunks this gives
  18 * 2^-23 * C * sum |q_j k_j| (times 1 + 2^-16 for the running sum's own
  error), plus C * 2^-120 for products below fp32's normal range.  This is a
  stated model, not a documented property: the GPU tests check every kernel
  score against it.
FAC is fp64.

Pins (tests/test_fasa_oracle_cpu.py): the all-pairs score is the full dot
product; a one-pair score is that pair's product sum; pairs outside the mask do
not change a score; a planted monotone score selects the last keys; all-equal
scores select the first keys; the selection equals a brute-force sort; the
"fma" bound holds for fp32 sums taken in any order, and the "tensor" bound for
a simulated chunk-step adder that truncates every addend below the largest
one's 24th bit; check_selection accepts the
oracle's selection and rejects planted wrong ones; FAC over every token equals
the oracle's dense decode; FAC over one token returns its value.
"""
from __future__ import annotations

import numpy as np


def _f32(x) -> np.ndarray:
    """bf16 / fp32 torch tensor or array -> float32 numpy array (exact)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float32).numpy()
    except ImportError:
        pass
    return np.asarray(x, dtype=np.float32)


def _f64(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:
        pass
    return np.asarray(x, dtype=np.float64)


def pair_list(mask: int, d: int) -> list[int]:
    """The pairs i < d/2 whose bit i is set in `mask`, ascending."""
    return [i for i in range(d // 2) if (mask >> i) & 1]


def _masked_dims(mask: int, d: int) -> np.ndarray:
    return np.array([j for i in pair_list(mask, d) for j in (2 * i, 2 * i + 1)], dtype=np.int64)


def tip_scores(q_rot, k_rot, kv_len, mask: int) -> np.ndarray:
    """Exact TIP scores, float64 [B][Hq][N]; entries at n >= kv_len[b] are -inf.

    q_rot [B][Hq][d] and k_rot [B][N][Hkv][d] are rotated (interleaved pairs);
    query head h reads kv head h // (Hq / Hkv)."""
    q = _f64(q_rot)
    k = _f64(k_rot)
    B, Hq, d = q.shape
    _, N, Hkv, _ = k.shape
    G = Hq // Hkv
    kl = np.asarray(kv_len, dtype=np.int64).reshape(-1)
    out = np.full((B, Hq, N), -np.inf, dtype=np.float64)
    dims = _masked_dims(mask, d)
    for b in range(B):
        L = int(kl[b])
        for h in range(Hq):
            out[b, h, :L] = k[b, :L, h // G][:, dims] @ q[b, h, dims]
    return out


def score_bound(q_rot, k_rot, kv_len, mask: int, model: str = "fma") -> np.ndarray:
    """Per-key bound [B][Hq][N] on |fp32 score - exact score| (0 past kv_len) for
    the summation `model` ("fma" or "tensor", described above)."""
    q = _f64(q_rot)
    k = _f64(k_rot)
    B, Hq, d = q.shape
    _, N, Hkv, _ = k.shape
    G = Hq // Hkv
    kl = np.asarray(kv_len, dtype=np.int64).reshape(-1)
    dims = _masked_dims(mask, d)
    if model == "fma":
        rel, absolute = dims.size * 2.0 ** -24, 0.0
    elif model == "tensor":
        chunks = len({int(i) // 8 for i in pair_list(mask, d)})
        rel, absolute = 18 * 2.0 ** -23 * chunks * (1 + 2.0 ** -16), chunks * 2.0 ** -120
    else:
        raise ValueError(model)
    out = np.zeros((B, Hq, N), dtype=np.float64)
    for b in range(B):
        L = int(kl[b])
        for h in range(Hq):
            out[b, h, :L] = rel * (np.abs(k[b, :L, h // G][:, dims]) @ np.abs(q[b, h, dims])) + absolute
    return out


def select(scores: np.ndarray, kv_len, budget: int) -> np.ndarray:
    """Top-`budget` key indices per (b, h), ascending, padded with -1: highest
    score first, equal scores by lower index.  int32 [B][Hq][budget]."""
    B, Hq, _ = scores.shape
    kl = np.asarray(kv_len, dtype=np.int64).reshape(-1)
    out = np.full((B, Hq, budget), -1, dtype=np.int32)
    for b in range(B):
        L = int(kl[b])
        n = np.arange(L)
        for h in range(Hq):
            order = np.lexsort((n, -np.asarray(scores[b, h, :L], dtype=np.float64)))  # primary: score desc
            keep = np.sort(order[: min(budget, L)])
            out[b, h, : len(keep)] = keep
    return out


def focused_attention(q_rot, k_rot, v, sel: np.ndarray) -> np.ndarray:
    """FAC in fp64: softmax((1/sqrt d) q.k) over the selected keys, times their
    values.  [B][Hq][d] float64."""
    q = _f64(q_rot)
    k = _f64(k_rot)
    vv = _f64(v)
    B, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            idx = sel[b, h][sel[b, h] >= 0]
            if idx.size == 0:
                continue
            kk = k[b, idx, h // G, :]
            s = kk @ q[b, h] / np.sqrt(d)
            p = np.exp(s - s.max())
            out[b, h] = (p / p.sum()) @ vv[b, idx, h // G, :]
    return out


def check_selection(sel, k_rot, kv_len, budget: int, exact: np.ndarray, bound: np.ndarray, mask: int) -> None:
    """Raises AssertionError unless `sel` [B][Hq][budget] (int) is a correct
    selection for the exact scores: per (b, h), the first min(budget, kv_len)
    entries are distinct key indices in [0, kv_len) in ascending order and the
    rest are -1; no dropped key's exact score exceeds a kept key's by more than
    the two keys' bounds (bound[b][h][n]); and where a dropped key's dominant
    dims equal a kept key's exactly (so any evaluation scores them alike), the
    kept one has the lower index."""
    sel = np.asarray(sel)
    k = _f64(k_rot)
    B, Hq, _ = sel.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    kl = np.asarray(kv_len, dtype=np.int64).reshape(-1)
    dims = _masked_dims(mask, k.shape[3])
    for b in range(B):
        L = int(kl[b])
        c = min(budget, L)
        for h in range(Hq):
            row = sel[b, h]
            kept = row[:c].astype(np.int64)
            assert (row[c:] == -1).all(), (b, h, "padding")
            assert (kept >= 0).all() and (kept < L).all(), (b, h, "range")
            assert (np.diff(kept) > 0).all(), (b, h, "ascending and distinct")
            if c == L:
                continue
            is_kept = np.zeros(L, dtype=bool)
            is_kept[kept] = True
            e, bd = exact[b, h, :L], bound[b, h, :L]
            # the kernel keeps k over d only if its fp32 score of k is at least that
            # of d, so e_d - bd_d <= fp32_d <= fp32_k <= e_k + bd_k for every pair
            drop = np.nonzero(~is_kept)[0]
            best_drop = drop[np.argmax(e[drop] - bd[drop])]
            worst_kept = kept[np.argmin(e[kept] + bd[kept])]
            assert e[best_drop] - bd[best_drop] <= e[worst_kept] + bd[worst_kept], \
                (b, h, "dropped key", int(best_drop), "outscores kept key", int(worst_kept))
            # keys with identical dominant dims score identically in any evaluation:
            # among them, the kept ones must be the lowest indices
            tie = drop[np.isin(e[drop], e[kept])]
            if tie.size:
                kd = k[b, :L, h // G][:, dims]
                first_drop = {}
                for n in tie:
                    first_drop.setdefault(kd[n].tobytes(), int(n))
                for n in kept[np.isin(e[kept], e[tie])]:
                    fd = first_drop.get(kd[n].tobytes())
                    assert fd is None or fd > n, (b, h, "identical keys: kept", int(n), "after dropped", fd)


def fasa_decode(q_rot, k_rot, v, kv_len, mask: int, budget: int):
    """The whole path on exact scores: (output fp64 [B][Hq][d], selected int32
    [B][Hq][budget], exact scores float64 [B][Hq][N])."""
    sc = tip_scores(q_rot, k_rot, kv_len, mask)
    sel = select(sc, kv_len, budget)
    return focused_attention(q_rot, k_rot, v, sel), sel, sc

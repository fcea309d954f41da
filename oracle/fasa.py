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

The selection is an integer decision taken on floating-point scores, so both
sides take it on the same fp32 numbers: starting from +0, the dims of the
dominant pairs are taken in ascending order (2i, then 2i+1, pairs ascending)
and each adds its product with one fused multiply-add in fp32,
s <- fl(q_j * k_j + s).  Here that rounding is reproduced in fp64: q_j * k_j (a
bf16 x bf16 product, 16 significant bits) and s (24 bits) sum exactly in fp64
whenever their exponents are within 28 of each other; otherwise the smaller
term is below a quarter of an fp32 ulp of the larger, which is itself an fp32
number, and both roundings return it.  So fp32(fp64(s) + fp64(q_j) * fp64(k_j))
is exactly the fused result.  FAC itself is fp64.

Pins (tests/test_fasa_oracle_cpu.py): the all-pairs score equals the full dot
product within fp32 summation error; a one-pair score equals that pair's
product sum; a planted monotone score selects the last keys; all-equal scores
select the first keys; the selection equals a brute-force sort; FAC over every
token equals the oracle's dense decode; FAC over one token returns its value.
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


def tip_scores(q_rot, k_rot, kv_len, mask: int) -> np.ndarray:
    """TIP scores, float32 [B][Hq][N]; entries at n >= kv_len[b] are -inf.

    q_rot [B][Hq][d] and k_rot [B][N][Hkv][d] are rotated (interleaved pairs);
    query head h reads kv head h // (Hq / Hkv)."""
    q = _f32(q_rot)
    k = _f32(k_rot)
    B, Hq, d = q.shape
    _, N, Hkv, _ = k.shape
    G = Hq // Hkv
    kl = np.asarray(kv_len, dtype=np.int64).reshape(-1)
    out = np.full((B, Hq, N), -np.inf, dtype=np.float32)
    pairs = pair_list(mask, d)
    for b in range(B):
        L = int(kl[b])
        for h in range(Hq):
            kk = k[b, :L, h // G, :]  # [L][d]
            s = np.zeros(L, dtype=np.float32)
            for i in pairs:
                for j in (2 * i, 2 * i + 1):  # one fused multiply-add per dim
                    s = (s.astype(np.float64) + np.float64(q[b, h, j]) * kk[:, j].astype(np.float64)).astype(np.float32)
            out[b, h, :L] = s + np.float32(0.0)  # -0 and +0 score alike
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
            order = np.lexsort((n, -scores[b, h, :L].astype(np.float64)))  # primary: score desc
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


def fasa_decode(q_rot, k_rot, v, kv_len, mask: int, budget: int):
    """The whole path: (output fp64 [B][Hq][d], selected int32 [B][Hq][budget],
    scores float32 [B][Hq][N])."""
    sc = tip_scores(q_rot, k_rot, kv_len, mask)
    sel = select(sc, kv_len, budget)
    return focused_attention(q_rot, k_rot, v, sel), sel, sc

"""Oracle for the split-KV decode: the windowed decode of one query against a
range of key positions, as a partial (softmax numerator, maximum, row sum), and
the log-sum-exp merge of partials.  Definitions as in the decode oracle (page
"ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57 Prozent", section
"Was ATFlash anders macht": logit = (1/sqrt d) sum of the products of the pairs
whose window W_i reaches the distance; no active pair gives logit 0), restricted
to keys lo .. hi-1 with the query at q_pos.  Interleaved pairs.

TEST INFRASTRUCTURE ONLY (tests/, never the CUDA library).  numpy, fp64.

Partial layout, [B][Hq][d + 2]: sum_n e^(s_n - m) v_n (d entries), m * log2(e)
(the maximum logit in log2 units; -inf for an empty range), sum_n e^(s_n - m).

Pin (tests/test_splitkv_cpu.py): merging the partials of any partition of the
keys equals the C decode oracle over all keys; an empty range merges as nothing.
"""
from __future__ import annotations

import numpy as np

from . import rope, windows

LOG2E = 1.4426950408889634


def _f64(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:
        pass
    return np.asarray(x, dtype=np.float64)


def partial(q, k_rot, v, lo, hi, q_pos, theta: float, alpha: float, key_pos0=None) -> np.ndarray:
    """Partials [B][Hq][d + 2] of raw queries q [B][Hq][d] (rotated here at
    q_pos[b]) against keys lo[b] .. hi[b]-1 of k_rot / v [B][N][Hkv][d]: key n
    sits at position key_pos0[b] + n (key_pos0 None: position n) and was rotated
    there."""
    qq = _f64(q)
    k = _f64(k_rot)
    vv = _f64(v)
    B, Hq, d = qq.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    W = np.asarray(windows(d, theta, alpha)[0], dtype=np.float64)
    out = np.zeros((B, Hq, d + 2))
    for b in range(B):
        qr = rope(q[b:b + 1][:, None], theta, pos0=int(q_pos[b]))[0, 0]  # [Hq][d], from q's own bits
        n = np.arange(int(lo[b]), int(hi[b]))
        if n.size == 0:
            out[b, :, d] = -np.inf
            continue
        p0 = 0 if key_pos0 is None else int(key_pos0[b])
        delta = int(q_pos[b]) - (p0 + n)
        active = W[None, :] >= delta[:, None]  # [keys][pairs]
        for h in range(Hq):
            kk = k[b, n, h // G, :]
            pp = qr[h, 0::2] * kk[:, 0::2] + qr[h, 1::2] * kk[:, 1::2]  # pair products [keys][pairs]
            s = (pp * active).sum(axis=1) / np.sqrt(d)
            m = s.max()
            e = np.exp(s - m)
            out[b, h, :d] = e @ vv[b, n, h // G, :]
            out[b, h, d] = m * LOG2E
            out[b, h, d + 1] = e.sum()
    return out


def merge(parts: np.ndarray) -> np.ndarray:
    """Merge partials [R][B][Hq][d + 2] into the output [B][Hq][d] (fp64)."""
    parts = np.asarray(parts, dtype=np.float64)
    d = parts.shape[-1] - 2
    m = parts[..., d]
    M = m.max(axis=0)
    f = np.where(np.isneginf(m), 0.0, np.exp2(m - M[None]))
    num = (parts[..., :d] * f[..., None]).sum(axis=0)
    den = (parts[..., d + 1] * f).sum(axis=0)
    return num / np.where(den > 0, den, 1.0)[..., None]

"""fp64 CPU oracle for causal GQA attention with one distance window per RoPE
frequency pair (ATFlash, "Was ATFlash anders macht" on the sudo-ai.de page
"ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57 Prozent").

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library never imports it and shares no code with it.

The arithmetic lives in ``atf_oracle.c`` (plain C, fp64, pthreads over rows);
this module only marshals numpy/torch arrays into it.  ``build()`` compiles the
C file with gcc into ``liboracle.so`` next to it.

Parity pins (what this oracle is checked against, in ``tests/test_oracle_pins.py``):
closed-form window values, the closed-form skipped pair count, the dense case
against torch's fp64 ``scaled_dot_product_attention``, the all-inactive case
in closed form, a single-pair planted case in closed form, and invariants
(constant V, chunked == unchunked, decode == last prefill row, head
permutation, RoPE rotation of unit vectors).  Nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "atf_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F32 = 1
BF16 = 0
INTERLEAVED = 0   # frequency pair i = dims (2i, 2i+1), as the method's formula is written
ROTATE_HALF = 1   # pair i = dims (i, i + d/2), NeoX-style checkpoints


def build(force: bool = False) -> str:
    """Compile atf_oracle.c into liboracle.so (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm", "-lpthread"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        c_p = ctypes.c_void_p
        lib.oracle_windows.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_double, c_p, c_p]
        lib.oracle_windows.restype = None
        lib.oracle_rope.argtypes = [c_p, ctypes.c_int, c_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_longlong, ctypes.c_double, ctypes.c_int]
        lib.oracle_rope.restype = None
        lib.oracle_prefill.argtypes = [c_p, c_p, c_p, ctypes.c_int, c_p, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_double, ctypes.c_double, c_p, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int]
        lib.oracle_prefill.restype = ctypes.c_ulonglong
        lib.oracle_decode.argtypes = [c_p, c_p, c_p, ctypes.c_int, c_p, ctypes.c_int, ctypes.c_longlong,
                                      c_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.oracle_decode.restype = ctypes.c_ulonglong
        _lib = lib
    return _lib


def _as_raw(x):
    """Return (contiguous numpy array, dtype code) holding x's exact bits.

    fp32 arrays pass as float32; bf16 tensors pass as their raw uint16 patterns
    (widened exactly to fp64 inside the C code)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            raise TypeError(f"oracle: unsupported tensor dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle: unsupported array dtype {x.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def windows(d: int, theta: float, alpha: float):
    """(W[d/2] int64, omega[d/2] fp64) of the method's window table."""
    W = np.zeros(d // 2, dtype=np.int64)
    om = np.zeros(d // 2, dtype=np.float64)
    _load().oracle_windows(d, float(theta), float(alpha), _ptr(W), _ptr(om))
    return W, om


def rope(x, theta: float, pos0: int = 0, pairing: int = INTERLEAVED) -> np.ndarray:
    """RoPE of x[batch][seq][heads][d] at positions pos0 + t, in fp64 (same layout)."""
    a, code = _as_raw(x)
    B, S, H, d = a.shape
    y = np.zeros((B, S, H, d), dtype=np.float64)
    _load().oracle_rope(_ptr(a), code, _ptr(y), B, S, H, d, int(pos0), float(theta), int(pairing))
    return y


def prefill(q, k, v, theta: float, alpha: float, q_offset: int = 0, rows=None, nthreads: int = 0,
            pairing: int = INTERLEAVED):
    """Causal windowed attention.  q [B][q_len][Hq][d], k/v [B][kv_len][Hkv][d].

    Returns (out fp64 [B][q_len][Hq][d], skipped pair count).  With ``rows``
    (indices t into q_len) only those rows are computed; the others are NaN."""
    qa, code = _as_raw(q)
    ka, code_k = _as_raw(k)
    va, code_v = _as_raw(v)
    assert code == code_k == code_v, "q, k, v must share a dtype"
    B, q_len, Hq, d = qa.shape
    Bk, kv_len, Hkv, dk = ka.shape
    assert Bk == B and dk == d and va.shape == ka.shape and Hq % Hkv == 0
    out = np.full((B, q_len, Hq, d), np.nan, dtype=np.float64)
    if rows is None:
        rp, nr = None, 0
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        assert r.size == 0 or (r.min() >= 0 and r.max() < q_len)
        rp, nr = _ptr(r), int(r.size)
    skipped = _load().oracle_prefill(_ptr(qa), _ptr(ka), _ptr(va), code, _ptr(out), B, q_len, kv_len,
                                     int(q_offset), Hq, Hkv, d, float(theta), float(alpha), rp, nr,
                                     int(nthreads), int(pairing))
    return out, int(skipped)


def decode(q, k_rot, v, kv_len, theta: float, alpha: float, nthreads: int = 0, pairing: int = INTERLEAVED):
    """One query per sequence at position kv_len[b]-1 against an already rotated
    key cache.  q [B][Hq][d] (unrotated), k_rot/v [B][n_cache][Hkv][d].

    Returns (out fp64 [B][Hq][d], skipped pair count)."""
    qa, code = _as_raw(q)
    ka, code_k = _as_raw(k_rot)
    va, code_v = _as_raw(v)
    assert code == code_k == code_v
    B, Hq, d = qa.shape
    Bk, n_cache, Hkv, dk = ka.shape
    assert Bk == B and dk == d and va.shape == ka.shape
    kl = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int64).reshape(B))
    assert (kl >= 1).all() and (kl <= n_cache).all()
    out = np.zeros((B, Hq, d), dtype=np.float64)
    skipped = _load().oracle_decode(_ptr(qa), _ptr(ka), _ptr(va), code, _ptr(out), B, int(n_cache),
                                    _ptr(kl), Hq, Hkv, d, float(theta), float(alpha), int(nthreads),
                                    int(pairing))
    return out, int(skipped)

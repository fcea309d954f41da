"""Thin Python binding of the C ABI in include/atf.h (libatf.so).

Argument marshalling only: every step of the attention path runs in the CUDA
kernels of libatf.so.  Functions keep the C names; tensors are passed as torch
tensors (their device pointers) or raw integer addresses.  There is no CPU
fallback: if the library is missing, importing a function raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libatf.so")

ATF_OK, ATF_ERR_INVALID_ARG, ATF_ERR_UNSUPPORTED, ATF_ERR_CUDA, ATF_ERR_TIMEOUT = range(5)
ATF_BF16, ATF_FP32 = 0, 1
ATF_PAIRS_INTERLEAVED, ATF_PAIRS_ROTATE_HALF = 0, 1
STATUS_NAMES = {0: "ATF_OK", 1: "ATF_ERR_INVALID_ARG", 2: "ATF_ERR_UNSUPPORTED", 3: "ATF_ERR_CUDA",
                4: "ATF_ERR_TIMEOUT"}


class AtfError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class PrefillArgs(ctypes.Structure):
    """Mirror of atf_prefill_args."""

    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("batch", ctypes.c_int), ("q_len", ctypes.c_int), ("kv_len", ctypes.c_int), ("heads", ctypes.c_int),
        ("kv_heads", ctypes.c_int), ("d", ctypes.c_int),
        ("q_offset", ctypes.c_longlong),
        ("dtype", ctypes.c_int), ("rotated", ctypes.c_int),
        ("theta", ctypes.c_double), ("alpha", ctypes.c_double),
        ("skipped_pairs", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("pairing", ctypes.c_int),
    ]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libatf.so (built by rope_frequency_sparse_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is not built; run __graft_entry__.build() "
                           "(or python -m rope_frequency_sparse_b200.build)")
    lib = ctypes.CDLL(path)
    vp, i, d, ll, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_longlong, ctypes.c_size_t
    sigs = {
        "atf_windows": ([i, d, d, vp], i),
        "atf_rope_layout": ([vp, vp, vp, i, i, i, i, ll, d, i, i, vp], i),
        "atf_prefill_workspace_bytes": ([i, i, i, i, i, i, i, i], sz),
        "atf_prefill_ex": ([ctypes.POINTER(PrefillArgs), vp], i),
        "atf_prefill": ([vp, vp, vp, vp, i, i, i, i, d, d, vp], i),
        "atf_prefill_host_workspace_bytes": ([i, i, i, i, i, i, i], sz),
        "atf_prefill_host": ([ctypes.POINTER(PrefillArgs), i, vp], i),
        "atf_decode": ([vp, vp, vp, vp, i, vp, ll, i, i, i, d, d, i, vp, sz, vp, vp], i),
        "atf_decode_workspace_bytes": ([i, i, i, ll, i], sz),
        "atf_decode_partial": ([vp, vp, vp, vp, i, vp, vp, vp, ll, i, i, i, d, d, i, vp, sz, vp, vp], i),
        "atf_decode_merge": ([vp, i, i, i, i, vp, vp], i),
        "atf_decode_noalloc": ([vp, vp, vp, vp, i, vp, ll, i, i, i, d, d, i, vp, vp], i),
        "atf_decode_noalloc_scratch_bytes": ([], sz),
        "atf_kv_append": ([vp, vp, vp, vp, i, vp, vp, ll, i, i, d, i, vp], i),
        "atf_fasa_decode": ([vp, vp, vp, vp, i, vp, ll, i, i, i, ctypes.c_ulonglong, i, vp, vp, vp, sz, vp], i),
        "atf_fasa_workspace_bytes": ([i, i, ll, i, i], sz),
        "atf_check": ([vp], i),
        "atf_selftest_timeout": ([ll, vp], i),
        "atf_last_error": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def atf_last_error() -> str:
    return load_library().atf_last_error().decode()


def _check(st: int):
    if st != ATF_OK:
        raise AtfError(st, atf_last_error())


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return ATF_BF16
    if t.dtype == torch.float32:
        return ATF_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------ C entry points

def atf_windows(d: int, theta: float, alpha: float) -> np.ndarray:
    W = np.zeros(d // 2, dtype=np.int64)
    _check(load_library().atf_windows(d, float(theta), float(alpha), W.ctypes.data_as(ctypes.c_void_p)))
    return W


def atf_rope_layout(x, x_rot, x_chunked, batch, seq, heads, d, pos_offset, theta, rotate, dtype, stream=None):
    _check(load_library().atf_rope_layout(_ptr(x), _ptr(x_rot), _ptr(x_chunked), batch, seq, heads, d,
                                          int(pos_offset), float(theta), int(rotate), int(dtype), _stream(stream)))


def atf_prefill_workspace_bytes(batch, q_len, kv_len, heads, kv_heads, d, dtype, rotated) -> int:
    return int(load_library().atf_prefill_workspace_bytes(batch, q_len, kv_len, heads, kv_heads, d, dtype, rotated))


def atf_prefill_ex(q, k, v, out, batch, q_len, kv_len, heads, kv_heads, d, q_offset, dtype, rotated, theta, alpha,
                   skipped_pairs=None, workspace=None, workspace_bytes=0, stream=None, pairing=ATF_PAIRS_INTERLEAVED):
    a = PrefillArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(out), batch, q_len, kv_len, heads, kv_heads, d, int(q_offset),
                    int(dtype), int(rotated), float(theta), float(alpha), _ptr(skipped_pairs), _ptr(workspace),
                    int(workspace_bytes), int(pairing))
    _check(load_library().atf_prefill_ex(ctypes.byref(a), _stream(stream)))


def atf_prefill_host_workspace_bytes(batch, q_len, kv_len, heads, kv_heads, d, rotated) -> int:
    return int(load_library().atf_prefill_host_workspace_bytes(batch, q_len, kv_len, heads, kv_heads, d, rotated))


def atf_prefill_host(q, k, v, out, batch, q_len, kv_len, heads, kv_heads, d, q_offset, rotated, theta, alpha,
                     workspace, workspace_bytes, chunk_rows=0, skipped_pairs=None, stream=None,
                     pairing=ATF_PAIRS_INTERLEAVED):
    """q, k, v, out are host buffers (CPU tensors, pinned for overlap); workspace is device memory."""
    a = PrefillArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(out), batch, q_len, kv_len, heads, kv_heads, d, int(q_offset),
                    ATF_BF16, int(rotated), float(theta), float(alpha), _ptr(skipped_pairs), _ptr(workspace),
                    int(workspace_bytes), int(pairing))
    _check(load_library().atf_prefill_host(ctypes.byref(a), int(chunk_rows), _stream(stream)))


def atf_prefill(q, k, v, out, seq, heads, kv_heads, d, theta, alpha, stream=None):
    _check(load_library().atf_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), seq, heads, kv_heads, d, float(theta),
                                      float(alpha), _stream(stream)))


def atf_decode(q, k_chunked, v, out, batch, kv_len, n_cache, heads, kv_heads, d, theta, alpha, workspace,
               workspace_bytes, skipped_pairs=None, stream=None, pairing=ATF_PAIRS_INTERLEAVED):
    kl = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int64).reshape(-1))
    _check(load_library().atf_decode(_ptr(q), _ptr(k_chunked), _ptr(v), _ptr(out), batch,
                                     kl.ctypes.data_as(ctypes.c_void_p), int(n_cache), heads, kv_heads, d,
                                     float(theta), float(alpha), int(pairing), _ptr(workspace),
                                     int(workspace_bytes), _ptr(skipped_pairs), _stream(stream)))


def atf_decode_partial(q, k_chunked, v, partial, batch, n_keys, key_pos0, q_pos, n_cache, heads, kv_heads, d, theta,
                       alpha, workspace, workspace_bytes, skipped_pairs=None, stream=None,
                       pairing=ATF_PAIRS_INTERLEAVED):
    """Decode over a key range (slots 0.. at positions key_pos0..; query at q_pos): the merged partial."""
    arrs = [np.ascontiguousarray(np.asarray(x, dtype=np.int64).reshape(-1)) for x in (n_keys, key_pos0, q_pos)]
    _check(load_library().atf_decode_partial(_ptr(q), _ptr(k_chunked), _ptr(v), _ptr(partial), batch,
                                             *[a.ctypes.data_as(ctypes.c_void_p) for a in arrs], int(n_cache),
                                             heads, kv_heads, d, float(theta), float(alpha), int(pairing),
                                             _ptr(workspace), int(workspace_bytes), _ptr(skipped_pairs),
                                             _stream(stream)))


def atf_decode_merge(partials, n_parts, batch, heads, d, out, stream=None):
    _check(load_library().atf_decode_merge(_ptr(partials), int(n_parts), batch, heads, d, _ptr(out),
                                           _stream(stream)))


def atf_decode_noalloc(q, k_chunked, v, out, batch, kv_len, n_cache, heads, kv_heads, d, theta, alpha,
                       skipped_pairs=None, stream=None, pairing=ATF_PAIRS_INTERLEAVED):
    """atf_decode with its scratch in the library's fixed device array (no allocation)."""
    kl = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int64).reshape(-1))
    _check(load_library().atf_decode_noalloc(_ptr(q), _ptr(k_chunked), _ptr(v), _ptr(out), batch,
                                             kl.ctypes.data_as(ctypes.c_void_p), int(n_cache), heads, kv_heads, d,
                                             float(theta), float(alpha), int(pairing), _ptr(skipped_pairs),
                                             _stream(stream)))


def atf_decode_noalloc_scratch_bytes() -> int:
    return int(load_library().atf_decode_noalloc_scratch_bytes())


def atf_decode_workspace_bytes(batch, heads, kv_heads, max_kv_len, d) -> int:
    return int(load_library().atf_decode_workspace_bytes(batch, heads, kv_heads, int(max_kv_len), d))


def atf_kv_append(k_new, v_new, k_cache_chunked, v_cache, batch, n_new, pos, n_cache, kv_heads, d, theta,
                  pairing=ATF_PAIRS_INTERLEAVED, stream=None):
    nn = np.ascontiguousarray(np.asarray(n_new, dtype=np.int32).reshape(-1))
    ps = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    _check(load_library().atf_kv_append(_ptr(k_new), _ptr(v_new), _ptr(k_cache_chunked), _ptr(v_cache), batch,
                                        nn.ctypes.data_as(ctypes.c_void_p), ps.ctypes.data_as(ctypes.c_void_p),
                                        int(n_cache), kv_heads, d, float(theta), int(pairing), _stream(stream)))


def atf_fasa_workspace_bytes(batch, heads, n_cache, budget, d) -> int:
    return int(load_library().atf_fasa_workspace_bytes(batch, heads, int(n_cache), budget, d))


def atf_fasa_decode(q_rot, k_chunked, v, out, batch, kv_len, n_cache, heads, kv_heads, d, pair_mask, budget,
                    selected=None, scores=None, workspace=None, workspace_bytes=0, stream=None):
    kl = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int64).reshape(-1))
    _check(load_library().atf_fasa_decode(_ptr(q_rot), _ptr(k_chunked), _ptr(v), _ptr(out), batch,
                                          kl.ctypes.data_as(ctypes.c_void_p), int(n_cache), heads, kv_heads, d,
                                          int(pair_mask) & ((1 << 64) - 1), int(budget), _ptr(selected),
                                          _ptr(scores), _ptr(workspace), int(workspace_bytes), _stream(stream)))


def atf_check(stream=None):
    _check(load_library().atf_check(_stream(stream)))


def atf_selftest_timeout(limit_cycles: int, stream=None):
    _check(load_library().atf_selftest_timeout(int(limit_cycles), _stream(stream)))


# ------------------------------------------------------------------ torch conveniences (allocation only)

def rope_layout(x, theta, pos_offset=0, rotated_out=True, chunked_out=False, rotate=True, stream=None,
                pairing=ATF_PAIRS_INTERLEAVED):
    """Rotate x [B][S][H][d] (torch, CUDA); returns (x_rot or None, x_chunked or None).
    With rotate-half pairing the outputs hold pair i in dims (2i, 2i+1)."""
    import torch

    B, S, H, d = x.shape
    xr = torch.empty_like(x) if rotated_out else None
    xc = torch.empty((B, H, d // 16, S, 16), dtype=x.dtype, device=x.device) if chunked_out else None
    mode = (2 if rotate else 3) if pairing == ATF_PAIRS_ROTATE_HALF else (1 if rotate else 0)
    atf_rope_layout(x, xr, xc, B, S, H, d, pos_offset, theta, mode, dtype_code(x), stream)
    return xr, xc


def prefill(q, k, v, theta, alpha, q_offset=0, rotated=False, skipped=None, out=None, workspace=None, stream=None,
            pairing=ATF_PAIRS_INTERLEAVED):
    """Windowed causal prefill; q [B][q_len][Hq][d], k/v [B][kv_len][Hkv][d] (torch, CUDA)."""
    import torch

    B, q_len, Hq, d = q.shape
    _, kv_len, Hkv, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    dt = dtype_code(q)
    need = atf_prefill_workspace_bytes(B, q_len, kv_len, Hq, Hkv, d, dt, int(rotated))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    atf_prefill_ex(q, k, v, out, B, q_len, kv_len, Hq, Hkv, d, q_offset, dt, int(rotated), theta, alpha,
                   skipped, workspace, need, stream, pairing)
    return out


def prefill_host(q, k, v, theta, alpha, q_offset=0, rotated=False, skipped=None, out=None, workspace=None,
                 chunk_rows=0, stream=None, pairing=ATF_PAIRS_INTERLEAVED, device=None):
    """Windowed causal prefill of host tensors (CPU, bf16; pinned for overlapped
    copies): q [B][q_len][Hq][d], k/v [B][kv_len][Hkv][d].  Returns the host
    output once the stream has finished (this call synchronises the stream)."""
    import torch

    B, q_len, Hq, d = q.shape
    _, kv_len, Hkv, _ = k.shape
    for t in (q, k, v):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise TypeError("prefill_host takes contiguous bf16 CPU tensors")
    if out is None:
        out = torch.empty_like(q, pin_memory=q.is_pinned())
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    need = atf_prefill_host_workspace_bytes(B, q_len, kv_len, Hq, Hkv, d, int(rotated))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    atf_prefill_host(q, k, v, out, B, q_len, kv_len, Hq, Hkv, d, q_offset, int(rotated), theta, alpha, workspace,
                     need, chunk_rows, skipped, stream, pairing)
    atf_check(stream)
    return out


def decode(q, k_chunked, v, kv_len, theta, alpha, skipped=None, out=None, workspace=None, stream=None,
           pairing=ATF_PAIRS_INTERLEAVED):
    """Decode step; q [B][Hq][d], k_chunked [B][Hkv][d/16][N][16], v [B][N][Hkv][d] (torch, CUDA)."""
    import torch

    B, Hq, d = q.shape
    _, Hkv, _, N, _ = k_chunked.shape
    kl = np.asarray(kv_len, dtype=np.int64).reshape(-1)
    need = atf_decode_workspace_bytes(B, Hq, Hkv, int(kl.max()) if kl.size else 1, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    atf_decode(q, k_chunked, v, out, B, kl, N, Hq, Hkv, d, theta, alpha, workspace, need, skipped, stream, pairing)
    return out


def fasa_decode(q_rot, k_chunked, v, kv_len, pair_mask, budget, selected=None, scores=None, out=None,
                workspace=None, stream=None):
    """FASA-style decode; q_rot [B][Hq][d] (rotated), k_chunked [B][Hkv][d/16][N][16],
    v [B][N][Hkv][d] (torch, CUDA, bf16).  Returns out [B][Hq][d]."""
    import torch

    B, Hq, d = q_rot.shape
    _, Hkv, _, N, _ = k_chunked.shape
    if out is None:
        out = torch.empty_like(q_rot)
    need = atf_fasa_workspace_bytes(B, Hq, N, budget, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q_rot.device)
    atf_fasa_decode(q_rot, k_chunked, v, out, B, kv_len, N, Hq, Hkv, d, pair_mask, budget, selected, scores,
                    workspace, need, stream)
    return out


def is_dense(alpha: float) -> bool:
    return math.isinf(alpha)

"""B200 (sm_100a) causal GQA attention with one distance window per RoPE
frequency pair.  The compute runs in libatf.so (see include/atf.h); this
package holds its thin ctypes binding (``atf``), the build step (``build``)
and the seeded synthetic inputs (``synth``)."""
from .atf import (  # noqa: F401
    ATF_BF16, ATF_FP32, AtfError, atf_check, atf_decode, atf_decode_workspace_bytes, atf_last_error, atf_prefill,
    atf_prefill_ex, atf_prefill_workspace_bytes, atf_rope_layout, atf_selftest_timeout, atf_windows, decode,
    load_library, prefill, rope_layout,
)

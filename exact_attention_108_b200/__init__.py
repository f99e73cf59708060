"""B200-native exact attention: Python binding over the C-ABI library ``libfattn.so``.

Importing the package loads nothing; the shared library is opened on first use
and a missing library is a hard error (there is no fallback path).

    from exact_attention_108_b200 import fwd, bwd
    o, lse = fwd(q, k, v, causal=True)
    dq, dk, dv = bwd(q, k, v, o, lse, do, causal=True)
"""
from .binding import (  # noqa: F401
    FattnError,
    bwd,
    bwd_ex,
    decode,
    device_status,
    fwd,
    fwd_ex,
    load,
    status_string,
    workspace_size,
)

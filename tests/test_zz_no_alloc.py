"""fattn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers have no way to give the library a workspace -- a plugin inside a
host application that owns all device memory, or a serving loop that forbids
allocations on its request path.  For them fattn_bwd_noalloc takes its scratch
from one fixed 32 MiB array kept in device memory.  This file checks, through
the C ABI, that two calls in a row give what fattn_bwd gives with a workspace
(the array keeps the previous call's contents, which must not leak into the next
call), and that a shape needing more scratch than the array holds is refused
before anything runs.  It is collected last so that a failure here cannot stop
the other GPU tests from running first.
"""
import ctypes
import math

import pytest
import torch

from exact_attention_108_b200 import binding
from gpu_common import assert_device_ok, check_grad, gpu_inputs


@pytest.mark.gpu
def test_noalloc_backward_matches_workspace_backward_on_two_calls():
    # Two different problems back to back: the second call must not see the first's scratch.
    for (B, H, N, d, causal, seed) in [(1, 2, 512, 128, True, 41), (2, 1, 384, 64, False, 42)]:
        _, (q, k, v, do) = gpu_inputs(B, H, N, d, seed)
        scale = 1.0 / math.sqrt(d)
        o, lse = binding.fwd(q, k, v, causal=causal, scale=scale)
        ref = binding.bwd(q, k, v, o, lse, do, causal=causal, scale=scale)
        got = binding.bwd_noalloc(q, k, v, o, lse, do, causal=causal, scale=scale)
        assert_device_ok()
        for g, r, name in zip(got, ref, ("dQ", "dK", "dV")):
            check_grad(g.double().cpu().numpy(), r.double().cpu().numpy(), name, "noalloc vs workspace")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = binding.load()
    fake = 1 << 20  # 16-byte aligned; rejected before any device work, never dereferenced
    B, H, N, d = 1, 1, 65536, 128  # needs 65536 * 130 * 4 bytes > 32 MiB of scratch
    assert lib.fattn_bwd_workspace_size(B, H, N, d) > binding.NOALLOC_SCRATCH_BYTES
    rc = lib.fattn_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake,
                               B, H, N, d, 1, ctypes.c_float(0.088), None)
    assert rc == binding.FATTN_ERR_SCRATCH_TOO_SMALL
    assert "scratch" in binding.status_string(rc)

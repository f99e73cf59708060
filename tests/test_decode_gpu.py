"""GPU parity of split-KV decoding (fattn_decode) with the fp64 oracle: a few query
rows against a long key/value cache, grouped key/value heads packed into one
tile, several key splits merged by their log-sum-exp."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_108_b200 import binding
from exact_attention_108_b200.workloads import to_f64
from gpu_common import assert_device_ok, check_o

pytestmark = pytest.mark.gpu


def _inputs(B, H, H_kv, N_q, N_k, cap, d, seed, tail_fill=float("nan")):
    """q and a cache of capacity cap whose rows past N_k hold tail_fill (never to be read)."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, H, N_q, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, H_kv, N_k, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, H_kv, N_k, d), generator=g).to(torch.bfloat16)
    kc = torch.full((B, H_kv, cap, d), tail_fill, dtype=torch.bfloat16)
    vc = torch.full((B, H_kv, cap, d), tail_fill, dtype=torch.bfloat16)
    kc[:, :, :N_k] = k
    vc[:, :, :N_k] = v
    return (q, k, v), (q.cuda(), kc.cuda(), vc.cuda())


def _check_lse(lse, ref):
    g = lse.double().cpu().numpy()
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), empty)
    assert np.abs(g[~empty] - ref[~empty]).max() <= 1e-3


CASES = [
    # B, H, H_kv, N_q, N_k, cap, d, splits
    (2, 8, 2, 1, 4096, 4096, 128, 0),      # one new token, groups of four heads, library-chosen splits
    (2, 8, 2, 1, 4096, 4200, 128, 1),      # one split: the CTA writes O itself
    (2, 8, 2, 1, 4096, 4096, 128, 7),      # splits of uneven length (32 tiles in 7)
    (1, 4, 4, 5, 1000, 1024, 64, 3),       # ragged cache, five new rows
    (1, 32, 1, 8, 2048, 2048, 128, 0),     # 256 packed rows: two row tiles
    (3, 6, 3, 16, 777, 800, 64, 0),        # sixteen new rows, ragged
    (1, 8, 2, 1, 3000, 3072, 256, 0),      # d = 256, library-chosen splits, ragged cache
    (2, 4, 1, 3, 1500, 1600, 96, 0),       # d = 96, one key/value head, three new rows
    (1, 6, 3, 2, 2500, 2500, 32, 4),       # d = 32, four splits
]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,cap,d,splits", CASES)
def test_decode_matches_oracle(B, H, H_kv, N_q, N_k, cap, d, splits, causal):
    (q, k, v), (qg, kc, vc) = _inputs(B, H, H_kv, N_q, N_k, cap, d, 300 + N_k + splits)
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.decode(qg, kc, vc, n_k=N_k, causal=causal, scale=scale, num_splits=splits)
    assert_device_ok()
    o_ref, lse_ref = oracle.ref_fwd_general(to_f64(q), to_f64(k), to_f64(v), causal, scale)
    check_o(o, o_ref, f"decode splits={splits}")
    _check_lse(lse, lse_ref)


def test_decode_more_queries_than_keys_causal():
    """N_q > N_k, causal: the first N_q - N_k rows see no key (O = 0, LSE = -inf)."""
    (q, k, v), (qg, kc, vc) = _inputs(1, 2, 1, 20, 8, 8, 64, 5)
    o, lse = binding.decode(qg, kc, vc, causal=True, num_splits=1)
    assert_device_ok()
    o_ref, lse_ref = oracle.ref_fwd_general(to_f64(q), to_f64(k), to_f64(v), True, 0.125)
    assert torch.count_nonzero(o[:, :, :12]).item() == 0
    check_o(to_f64(o[:, :, 12:]), o_ref[:, :, 12:])
    _check_lse(lse, lse_ref)


def test_decode_equals_forward_on_the_same_problem():
    """Decoding computes the forward's function: compare with fattn_fwd_ex."""
    (q, k, v), (qg, kc, vc) = _inputs(2, 8, 4, 3, 1500, 1500, 128, 6)
    o1, l1 = binding.decode(qg, kc, vc, causal=True)
    o2, l2 = binding.fwd_ex(qg, kc, vc, causal=True)
    assert_device_ok()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_decode_full_size_grouped_heads():
    """B=8, H=32, H_kv=8, one new token against 32768 cached keys; every head checked."""
    B, H, H_kv, N_q, N_k, d = 8, 32, 8, 1, 32768, 128
    (q, k, v), (qg, kc, vc) = _inputs(B, H, H_kv, N_q, N_k, N_k, d, 7)
    o, lse = binding.decode(qg, kc, vc, causal=True)
    assert_device_ok()
    o_ref, lse_ref = oracle.ref_fwd_general(to_f64(q), to_f64(k), to_f64(v), True, 1.0 / math.sqrt(d))
    check_o(o, o_ref, "decode 8x32/8 heads, N_k = 32768")
    _check_lse(lse, lse_ref)

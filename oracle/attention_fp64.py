"""CPU fp64 oracle for exact scaled-dot-product attention (test infrastructure).

This module is TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it.  The CUDA library never calls it and shares no code with it.

What it computes (the plain definition, written out):

* Standard attention, page 1 "二、算子融合 1. 传统注意力计算流程" and page 3 "3.
  从CUDA原理理解注意力机制的计算瓶颈": S = Q K^T, P = softmax(S), O = P V, with
  Q, K, V each N x d per head.
* The op chain of page 2 "传统注意力为何容易受 IO 限制": the product Q K^T is
  scaled, masked, passed through softmax and multiplied by V.  Dropout is not
  modelled (rate 0).  The mask is causal: query i sees keys 0..i inclusive.
* The saved statistic of page 2 "三、融合算子" / "四、反向传播": the per-row
  log-sum-exp of the scaled, masked scores, natural log.
* The backward pass is the softmax Jacobian written out by hand (page 2 "四、
  反向传播选择重计算" says only that P is recomputed; the gradient itself is the
  textbook chain rule, see ``ref_bwd``).

Every array is float64.  Inputs arrive as float64 copies of the bf16 tensors the
GPU consumes (bf16 -> fp64 is exact), shaped [B, H, N, d].

Memory: S and P are materialised one block of query rows at a time (rows are
independent), so a 32768-key head needs ``row_block * N * 8`` bytes, not N^2*8.

Parity status: every public function here is pinned by ``tests/test_oracle.py``
(brute force, finite differences, closed forms, library softmax, invariants).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "scores",
    "causal_keep",
    "softmax_rows",
    "ref_probs",
    "ref_fwd",
    "ref_fwd_rows",
    "ref_bwd",
    "ref_bwd_head",
    "ref_dq_rows",
    "softmax_grad",
    "brute_fwd",
    "finite_diff_grads",
    "softmax_rows_masked",
    "kv_head_of",
    "philox4x32_10",
    "dropout_threshold",
    "dropout_multiplier",
    "ref_fwd_general",
    "ref_fwd_general_rows",
    "ref_bwd_general",
    "ref_dq_general_rows",
    "brute_fwd_general",
    "finite_diff_grads_general",
]


# --------------------------------------------------------------------------
# Steps of the definition (kept as separate functions so that a reader can
# check each against the pages, and so that tests can plant a mistake in one).
# --------------------------------------------------------------------------

def scores(q_rows: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """Scaled scores s_ij = scale * <q_i, k_j> for a block of query rows.

    Page 3 section 3: S = Q K^T costs O(N^2 d); page 2: the product is scaled.
    ``q_rows`` is [R, d], ``k`` is [N, d]; returns [R, N].
    """
    return scale * (q_rows @ k.T)


def causal_keep(row_ids: np.ndarray, n_keys: int, offset: int = 0) -> np.ndarray:
    """Boolean [R, N] mask: True where key j may be attended by query i.

    Causal (lower-triangular, diagonal included): key j is visible to query i
    iff j <= i + offset.  Page 2 lists a mask in the op chain without fixing its
    form; the causal reading is the one the workloads name.  With as many
    queries as keys the offset is 0.  With N_q queries and N_k keys the mask is
    aligned at the bottom right, offset = N_k - N_q: the last query sees every
    key, as it would if the queries were the last N_q positions of the sequence.
    """
    cols = np.arange(n_keys)
    return cols[None, :] <= np.asarray(row_ids)[:, None] + offset


def softmax_rows(s: np.ndarray):
    """Row softmax with max subtraction; returns (P, LSE) for scores ``s``.

    Masked entries are -inf on entry.  m_i = max_j s_ij; P_ij =
    exp(s_ij - m_i) / sum_j exp(s_ij - m_i); LSE_i = m_i + ln sum_j exp(s_ij -
    m_i).  Max subtraction for stability: page 1 "二、2" (数值稳定性) and page 3
    "6.2" (softmax kept in high precision).
    """
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=1, keepdims=True)
    p = e / z
    lse = (m + np.log(z))[:, 0]
    return p, lse


def _head_probs(qh, kh, causal, scale, r0, r1):
    """P and LSE for query rows [r0, r1) of one head."""
    s = scores(qh[r0:r1], kh, scale)
    if causal:
        keep = causal_keep(np.arange(r0, r1), kh.shape[0])
        s = np.where(keep, s, -np.inf)
    return softmax_rows(s)


def _row_blocks(n: int, row_block: int | None):
    rb = n if row_block is None else max(1, min(n, row_block))
    for r0 in range(0, n, rb):
        yield r0, min(n, r0 + rb)


def _auto_block(n: int) -> int:
    # keep one block of S (plus P and a temporary) near 256 MiB
    return max(1, min(n, (256 << 20) // (8 * 3 * max(n, 1))))


# --------------------------------------------------------------------------
# Forward
# --------------------------------------------------------------------------

def ref_probs(q: np.ndarray, k: np.ndarray, causal: bool, scale: float) -> np.ndarray:
    """Full probability tensor P [B, H, N, N] (small shapes only)."""
    B, H, N, _ = q.shape
    out = np.empty((B, H, N, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            out[b, h], _ = _head_probs(q[b, h], k[b, h], causal, scale, 0, N)
    return out


def ref_fwd(q, k, v, causal: bool, scale: float, row_block: int | None = None):
    """Exact attention forward: returns (O [B,H,N,d], LSE [B,H,N]) in fp64.

    O = softmax(scale * Q K^T + mask) V per (b, h), page 3 section 3 and page 2.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, H, N, d = q.shape
    o = np.empty((B, H, N, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, H, N), dtype=np.float64)
    rb = row_block if row_block is not None else _auto_block(N)
    for b in range(B):
        for h in range(H):
            for r0, r1 in _row_blocks(N, rb):
                p, l_ = _head_probs(q[b, h], k[b, h], causal, scale, r0, r1)
                o[b, h, r0:r1] = p @ v[b, h]
                lse[b, h, r0:r1] = l_
    return o, lse


def ref_fwd_rows(qh, kh, vh, rows, causal: bool, scale: float):
    """O and LSE for selected query rows of ONE head ([N,d] arrays).

    Each output row depends only on its own query row, so this is the same
    definition evaluated at O(len(rows) * N * d) cost (used for full-size
    sampled checks).
    """
    qh, kh, vh = (np.asarray(t, dtype=np.float64) for t in (qh, kh, vh))
    rows = np.asarray(rows, dtype=np.int64)
    s = scores(qh[rows], kh, scale)
    if causal:
        s = np.where(causal_keep(rows, kh.shape[0]), s, -np.inf)
    p, lse = softmax_rows(s)
    return p @ vh, lse


# --------------------------------------------------------------------------
# Backward (hand-derived from the softmax Jacobian)
#
# Loss L = sum(dO * O).  With O = P V:        dV = P^T dO,   dP = dO V^T.
# Softmax Jacobian dP_ij/ds_ik = P_ij (delta_jk - P_ik) gives
#       ds_ij = P_ij (dP_ij - sum_k P_ik dP_ik).
# With s = scale * Q K^T (masked entries are constants):
#       dQ = scale * ds K,   dK = scale * ds^T Q.
# The row term sum_k P_ik dP_ik is computed from this module's own P.
# --------------------------------------------------------------------------

def softmax_grad(p: np.ndarray, dp: np.ndarray) -> np.ndarray:
    """ds_ij = P_ij (dP_ij - sum_k P_ik dP_ik): the softmax Jacobian applied to dP."""
    row_term = np.sum(p * dp, axis=1, keepdims=True)
    return p * (dp - row_term)


def ref_bwd_head(qh, kh, vh, doh, causal: bool, scale: float, row_block: int | None = None):
    """dQ, dK, dV for ONE head ([N, d] arrays), S/P recomputed per row block."""
    qh, kh, vh, doh = (np.asarray(t, dtype=np.float64) for t in (qh, kh, vh, doh))
    N = qh.shape[0]
    dq = np.zeros_like(qh)
    dk = np.zeros_like(kh)
    dv = np.zeros_like(vh)
    rb = row_block if row_block is not None else _auto_block(N)
    for r0, r1 in _row_blocks(N, rb):
        p, _ = _head_probs(qh, kh, causal, scale, r0, r1)
        dv += p.T @ doh[r0:r1]
        dp = doh[r0:r1] @ vh.T
        ds = softmax_grad(p, dp)
        dq[r0:r1] = scale * (ds @ kh)
        dk += scale * (ds.T @ qh[r0:r1])
    return dq, dk, dv


def ref_bwd(q, k, v, do, causal: bool, scale: float, row_block: int | None = None):
    """Gradients (dQ, dK, dV) of L = sum(dO * O) for all heads, fp64."""
    B, H = q.shape[:2]
    dq = np.empty(q.shape, dtype=np.float64)
    dk = np.empty(k.shape, dtype=np.float64)
    dv = np.empty(v.shape, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h] = ref_bwd_head(
                q[b, h], k[b, h], v[b, h], do[b, h], causal, scale, row_block)
    return dq, dk, dv


def ref_dq_rows(qh, kh, vh, doh, rows, causal: bool, scale: float):
    """dQ for selected query rows of one head: each row needs only its own P row."""
    qh, kh, vh, doh = (np.asarray(t, dtype=np.float64) for t in (qh, kh, vh, doh))
    rows = np.asarray(rows, dtype=np.int64)
    s = scores(qh[rows], kh, scale)
    if causal:
        s = np.where(causal_keep(rows, kh.shape[0]), s, -np.inf)
    p, _ = softmax_rows(s)
    dp = doh[rows] @ vh.T
    return scale * (softmax_grad(p, dp) @ kh)


# --------------------------------------------------------------------------
# Independent cross-checks used only to pin the functions above
# --------------------------------------------------------------------------

def brute_fwd(q, k, v, causal: bool, scale: float):
    """Pure-Python triple loop with math.exp (no BLAS, no numpy reductions).

    Written separately from ``ref_fwd`` so that a mistake in one is caught by
    the other; tiny shapes only.  Returns nested lists O[b][h][i][c], LSE[b][h][i].
    """
    B, H, N, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    dv_ = len(v[0][0][0])
    O = [[[[0.0] * dv_ for _ in range(N)] for _ in range(H)] for _ in range(B)]
    L = [[[0.0] * N for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(N):
                visible = range(i + 1) if causal else range(N)
                logits = []
                for j in visible:
                    acc = 0.0
                    for c in range(d):
                        acc += float(q[b][h][i][c]) * float(k[b][h][j][c])
                    logits.append((j, scale * acc))
                top = max(x for _, x in logits)
                weights = [(j, math.exp(x - top)) for j, x in logits]
                total = sum(w for _, w in weights)
                for c in range(dv_):
                    O[b][h][i][c] = sum(w * float(v[b][h][j][c]) for j, w in weights) / total
                L[b][h][i] = top + math.log(total)
    return O, L


def finite_diff_grads(q, k, v, do, causal: bool, scale: float, eps: float = 1e-6):
    """Central differences of L = sum(dO * O) w.r.t. every element of Q, K, V."""
    q, k, v, do = (np.array(t, dtype=np.float64) for t in (q, k, v, do))

    def loss(qq, kk, vv):
        o, _ = ref_fwd(qq, kk, vv, causal, scale)
        return float(np.sum(do * o))

    grads = []
    for which in range(3):
        base = [q, k, v]
        g = np.zeros_like(base[which])
        it = np.nditer(base[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [t.copy() for t in base]
            minus = [t.copy() for t in base]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * eps)
        grads.append(g)
    return tuple(grads)


# --------------------------------------------------------------------------
# General shapes: N_q queries against N_k keys, grouped key/value heads, dropout
#
# Page 3 section 3 states Q, K, V each as an N x d matrix; the readings here
# take the queries and the keys/values to have their own lengths (N_q, N_k) and
# let several query heads share one key/value head (H query heads, H_kv key/value
# heads, H a multiple of H_kv; query head h reads key/value head h // (H / H_kv)).
# Page 2's op chain (传统注意力为何容易受 IO 限制) puts Dropout between the
# softmax and the product with V: each weight P_ij is kept with probability
# 1 - p and then divided by 1 - p, or dropped (set to 0).  The normaliser of the
# softmax (and so the LSE) is that of the undropped weights.
# --------------------------------------------------------------------------

def softmax_rows_masked(s: np.ndarray):
    """softmax_rows, where a row may have no visible key at all (every entry -inf).

    Such a row (possible only with causal and N_q > N_k) has an empty softmax:
    it gets P = 0, hence O = 0, and LSE = -inf (the log of an empty sum).
    """
    empty = np.all(np.isneginf(s), axis=1)
    p = np.zeros_like(s)
    lse = np.full(s.shape[0], -np.inf)
    if (~empty).any():
        p[~empty], lse[~empty] = softmax_rows(s[~empty])
    return p, lse


def kv_head_of(h: int, H: int, H_kv: int) -> int:
    """Key/value head read by query head h: consecutive groups of H / H_kv query heads share one."""
    return h // (H // H_kv)


_PHILOX_M0, _PHILOX_M1 = 0xD2511F53, 0xCD9E8D57   # round multipliers
_PHILOX_W0, _PHILOX_W1 = 0x9E3779B9, 0xBB67AE85   # key schedule increments
_U32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
    1, 2, 3", SC'11): a counter-based generator.  ``ctr`` is four uint32 arrays (any
    common shape), ``key`` two uint32 scalars; returns four uint32 arrays.

    Each of the 10 rounds multiplies words 0 and 2 by the two round constants
    (64-bit products split into high and low halves) and mixes:
        (c0, c1, c2, c3) <- (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)),
    and between rounds the key is advanced by the Weyl increments (W0, W1).
    """
    c = [np.asarray(x, dtype=np.uint64) & _U32 for x in ctr]
    k0, k1 = np.uint64(int(key[0]) & 0xFFFFFFFF), np.uint64(int(key[1]) & 0xFFFFFFFF)
    for rnd in range(10):
        if rnd > 0:
            k0 = np.uint64((int(k0) + _PHILOX_W0) & 0xFFFFFFFF)
            k1 = np.uint64((int(k1) + _PHILOX_W1) & 0xFFFFFFFF)
        p0 = np.uint64(_PHILOX_M0) * c[0]   # < 2^64: exact in uint64
        p1 = np.uint64(_PHILOX_M1) * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _U32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _U32
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return [x.astype(np.uint32) for x in c]


def dropout_threshold(p: float) -> int:
    """The 32-bit draw r keeps a weight iff r >= t, t = floor(p * 2^32) (at most 2^32 - 1)."""
    return min(int(math.floor(float(p) * 4294967296.0)), 4294967295)


def dropout_multiplier(bh: int, rows, n_k: int, p: float, seed: int, offset: int) -> np.ndarray:
    """Dropout factor [R, N_k] for query rows ``rows`` of flattened head bh = b*H + h:
    0 where the weight is dropped, 1 / (1 - p) where it is kept.

    The draw for (bh, i, j) is word j mod 4 of Philox4x32-10 with counter
    (i, floor(j / 4), bh, offset) and key (seed mod 2^32, floor(seed / 2^32)):
    one generator call covers four consecutive keys of a row, so the forward and
    the backward regenerate the same mask from the indices alone.
    """
    rows = np.asarray(rows, dtype=np.int64)
    if p == 0.0:
        return np.ones((rows.size, n_k))
    cols = np.arange(n_k, dtype=np.int64)
    shape = (rows.size, n_k)
    ctr = (np.broadcast_to(rows[:, None], shape), np.broadcast_to(cols[None, :] >> 2, shape),
           np.full(shape, bh), np.full(shape, offset & 0xFFFFFFFF))
    words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    r = np.choose(np.broadcast_to(cols[None, :] & 3, shape), words)
    keep = r.astype(np.int64) >= dropout_threshold(p)
    return np.where(keep, 1.0 / (1.0 - p), 0.0)


def _general_shapes(q, k):
    B, H, N_q, _ = q.shape
    H_kv, N_k = k.shape[1], k.shape[2]
    assert H % H_kv == 0, "H must be a multiple of H_kv"
    return B, H, H_kv, N_q, N_k


def _general_probs(qh, kh, rows, causal, scale, n_q):
    """P (undropped) and LSE for query rows ``rows`` of one head against all of its keys."""
    s = scores(qh[rows], kh, scale)
    if causal:
        s = np.where(causal_keep(rows, kh.shape[0], kh.shape[0] - n_q), s, -np.inf)
    return softmax_rows_masked(s)


def ref_fwd_general(q, k, v, causal: bool, scale: float, dropout_p: float = 0.0, seed: int = 0,
                    offset: int = 0, row_block: int | None = None):
    """Forward for q [B,H,N_q,d] against k, v [B,H_kv,N_k,d]: (O [B,H,N_q,d], LSE [B,H,N_q]).

    O = (P o Z) V with P = softmax(scale Q K^T + mask) and Z the dropout factor;
    LSE is that of the undropped scores.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, H, H_kv, N_q, N_k = _general_shapes(q, k)
    o = np.empty((B, H, N_q, v.shape[-1]))
    lse = np.empty((B, H, N_q))
    rb = row_block if row_block is not None else _auto_block(N_k)
    for b in range(B):
        for h in range(H):
            g = kv_head_of(h, H, H_kv)
            for r0, r1 in _row_blocks(N_q, rb):
                rows = np.arange(r0, r1)
                p, l_ = _general_probs(q[b, h], k[b, g], rows, causal, scale, N_q)
                z = dropout_multiplier(b * H + h, rows, N_k, dropout_p, seed, offset)
                o[b, h, r0:r1] = (p * z) @ v[b, g]
                lse[b, h, r0:r1] = l_
    return o, lse


def ref_fwd_general_rows(q, k, v, b: int, h: int, rows, causal: bool, scale: float,
                         dropout_p: float = 0.0, seed: int = 0, offset: int = 0):
    """O and LSE of selected query rows of head (b, h) (each row needs only its own P row)."""
    B, H, H_kv, N_q, N_k = _general_shapes(q, k)
    g = kv_head_of(h, H, H_kv)
    rows = np.asarray(rows, dtype=np.int64)
    qh, kh, vh = (np.asarray(t, dtype=np.float64) for t in (q[b, h], k[b, g], v[b, g]))
    p, lse = _general_probs(qh, kh, rows, causal, scale, N_q)
    z = dropout_multiplier(b * H + h, rows, N_k, dropout_p, seed, offset)
    return (p * z) @ vh, lse


def ref_bwd_general(q, k, v, do, causal: bool, scale: float, dropout_p: float = 0.0, seed: int = 0,
                    offset: int = 0, row_block: int | None = None):
    """Gradients (dQ, dK, dV) of L = sum(dO * O) for ref_fwd_general.

    With O = (P o Z) V:   dV = (P o Z)^T dO,   dP = (dO V^T) o Z,
    ds = P o (dP - rowsum(P o dP)) (softmax Jacobian, as in ref_bwd),
    dQ = scale ds K,  dK = scale ds^T Q.  A key/value head's dK and dV add up
    the contributions of every query head in its group.
    """
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    B, H, H_kv, N_q, N_k = _general_shapes(q, k)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rb = row_block if row_block is not None else _auto_block(N_k)
    for b in range(B):
        for h in range(H):
            g = kv_head_of(h, H, H_kv)
            for r0, r1 in _row_blocks(N_q, rb):
                rows = np.arange(r0, r1)
                p, _ = _general_probs(q[b, h], k[b, g], rows, causal, scale, N_q)
                z = dropout_multiplier(b * H + h, rows, N_k, dropout_p, seed, offset)
                dv[b, g] += (p * z).T @ do[b, h, r0:r1]
                dp = (do[b, h, r0:r1] @ v[b, g].T) * z
                ds = softmax_grad(p, dp)
                dq[b, h, r0:r1] = scale * (ds @ k[b, g])
                dk[b, g] += scale * (ds.T @ q[b, h, r0:r1])
    return dq, dk, dv


def ref_dq_general_rows(q, k, v, do, b: int, h: int, rows, causal: bool, scale: float,
                        dropout_p: float = 0.0, seed: int = 0, offset: int = 0):
    """dQ of selected query rows of head (b, h)."""
    B, H, H_kv, N_q, N_k = _general_shapes(q, k)
    g = kv_head_of(h, H, H_kv)
    rows = np.asarray(rows, dtype=np.int64)
    qh, kh, vh = (np.asarray(t, dtype=np.float64) for t in (q[b, h], k[b, g], v[b, g]))
    doh = np.asarray(do[b, h], dtype=np.float64)
    p, _ = _general_probs(qh, kh, rows, causal, scale, N_q)
    z = dropout_multiplier(b * H + h, rows, N_k, dropout_p, seed, offset)
    dp = (doh[rows] @ vh.T) * z
    return scale * (softmax_grad(p, dp) @ kh)


def brute_fwd_general(q, k, v, causal: bool, scale: float, mult=None):
    """Pure-Python loops for the general forward (tiny shapes): explicit key/value
    head mapping h // (H / H_kv), the bottom-right causal test j <= i + N_k - N_q,
    O = 0 and LSE = -inf for a row with no visible key, and the dropout factor
    ``mult[b][h][i][j]`` (1 when None) applied to the weights of O only."""
    B, H, N_q, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    H_kv, N_k, dv_ = len(k[0]), len(k[0][0]), len(v[0][0][0])
    G = H // H_kv
    O = [[[[0.0] * dv_ for _ in range(N_q)] for _ in range(H)] for _ in range(B)]
    L = [[[0.0] * N_q for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            g = h // G
            for i in range(N_q):
                visible = [j for j in range(N_k) if (not causal) or j <= i + (N_k - N_q)]
                if not visible:
                    L[b][h][i] = -math.inf
                    continue
                logits = []
                for j in visible:
                    acc = 0.0
                    for c in range(d):
                        acc += float(q[b][h][i][c]) * float(k[b][g][j][c])
                    logits.append((j, scale * acc))
                top = max(x for _, x in logits)
                weights = [(j, math.exp(x - top)) for j, x in logits]
                total = sum(w for _, w in weights)
                for c in range(dv_):
                    acc = 0.0
                    for j, w in weights:
                        f = 1.0 if mult is None else float(mult[b][h][i][j])
                        acc += w * f * float(v[b][g][j][c])
                    O[b][h][i][c] = acc / total
                L[b][h][i] = top + math.log(total)
    return O, L


def finite_diff_grads_general(q, k, v, do, causal: bool, scale: float, dropout_p: float = 0.0,
                              seed: int = 0, offset: int = 0, eps: float = 1e-6):
    """Central differences of L = sum(dO * O) for ref_fwd_general (dropout mask fixed)."""
    q, k, v, do = (np.array(t, dtype=np.float64) for t in (q, k, v, do))

    def loss(qq, kk, vv):
        o, _ = ref_fwd_general(qq, kk, vv, causal, scale, dropout_p, seed, offset)
        return float(np.sum(do * o))

    grads = []
    for which in range(3):
        base = [q, k, v]
        g = np.zeros_like(base[which])
        it = np.nditer(base[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [t.copy() for t in base]
            minus = [t.copy() for t in base]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * eps)
        grads.append(g)
    return tuple(grads)

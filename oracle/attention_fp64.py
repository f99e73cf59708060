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


def causal_keep(row_ids: np.ndarray, n_keys: int) -> np.ndarray:
    """Boolean [R, N] mask: True where key j may be attended by query i.

    Causal (lower-triangular, diagonal included): key j is visible to query i
    iff j <= i.  Page 2 lists a mask in the op chain without fixing its form;
    the causal reading is the one the workloads name.
    """
    cols = np.arange(n_keys)
    return cols[None, :] <= row_ids[:, None]


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

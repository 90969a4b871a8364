"""Plain fp64 CPU oracle for exact scaled dot-product attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: only the
test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may call it.  It shares no code with the CUDA library.

What it computes, and where the pages fix it
--------------------------------------------
* "FlashAttention" (interactiveprimer.com), introduction and "The bottleneck is memory,
  not multiplication": the method computes *exactly* scaled dot-product attention over N
  tokens per head; only the memory traffic changes.  "FlashAttention, simplified", "The
  trick", and "What FlashAttention actually buys", "The actual problem", say the same: the
  result is identical to the standard pipeline.  So the oracle for the forward is that
  standard pipeline written out: form S = scale * Q K^T, take a row softmax, multiply by V.
* The per-row log-sum-exp (LSE) that the forward also returns is the natural-log
  normaliser of the scaled, masked logits: LSE_i = log sum_j exp(S_ij).
* Causal masking (query i sees keys j <= i, same length for queries and keys) is not on
  the pages; it is the plain reading used throughout this library.  With fewer queries
  than keys (Nq < Nk: a chunk of new tokens whose keys follow those of earlier tokens)
  the queries are the last Nq tokens of the sequence, query i at position i + Nk - Nq
  (``chunk_positions``), so under causal masking it sees keys j <= i + Nk - Nq
  (bottom-right alignment); with Nq == Nk this is the rule above.
* ``attention_head_tiled`` is a second, independent route to the same numbers: the
  online-softmax recurrence of "FlashAttention, simplified", "The trick" (running max m,
  running sum l, accumulator acc, rescale by alpha = exp(m - m_new), one division by l at
  the end), with the scale, the causal mask and the LSE added.
* The backward pass: "What FlashAttention actually buys", "Why the distinction matters
  downstream", says only that the backward recomputes the score tiles instead of storing
  them.  The gradients themselves are the textbook derivative of softmax attention:
  dV = P^T dO, dP = dO V^T, D_i = sum_k dO_ik O_ik, dS = P * (dP - D), dQ = scale dS K,
  dK = scale dS^T Q.

Everything is float64.  Inputs of lower precision (bf16, fp32) are upcast exactly.
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _rows(n_q: int, q_index) -> np.ndarray:
    return np.arange(n_q) if q_index is None else np.asarray(q_index, dtype=np.int64)


def chunk_positions(n_q: int, n_k: int) -> np.ndarray:
    """Positions of n_q queries that are the last n_q tokens of an n_k-token sequence:
    query i sits at i + n_k - n_q (0..n-1 when n_q == n_k).  Needs n_q <= n_k."""
    if n_q > n_k:
        raise ValueError(f"{n_q} queries cannot be the last tokens of {n_k} keys")
    return np.arange(n_q) + (n_k - n_q)


def scores(Q, K, scale: float, causal: bool, q_index=None) -> np.ndarray:
    """S = scale * Q K^T for one head, with -inf where a causal query may not look.

    Q is [n_q, d] (rows may be any subset of the head's queries; ``q_index`` gives their
    positions, default 0..n_q-1), K is [N, d].  Under ``causal`` query i sees keys j <= i.
    """
    Q = _f64(Q)
    K = _f64(K)
    S = scale * (Q @ K.T)
    if causal:
        i = _rows(Q.shape[0], q_index)
        j = np.arange(K.shape[0])
        S = np.where(j[None, :] > i[:, None], -np.inf, S)
    return S


def softmax_rows(S: np.ndarray):
    """Row softmax of S and the natural-log normaliser of each row.

    Returns (P, LSE) with P_ij = exp(S_ij - LSE_i) and LSE_i = log sum_j exp(S_ij).
    The row max is subtracted before exponentiating so that large logits do not overflow.
    """
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    Z = E.sum(axis=1, keepdims=True)
    P = E / Z
    LSE = m[:, 0] + np.log(Z[:, 0])
    return P, LSE


def attention_head(Q, K, V, scale: float, causal: bool, q_index=None):
    """Standard (materialising) attention for one head: returns (O, LSE, P).

    O = softmax(scale Q K^T [masked]) V, LSE as in ``softmax_rows``.  Q may be a subset
    of rows (see ``scores``); K and V are the head's full [N, d] keys and values.
    """
    S = scores(Q, K, scale, causal, q_index)
    P, LSE = softmax_rows(S)
    O = P @ _f64(V)
    return O, LSE, P


def attention_head_tiled(Q, K, V, scale: float, causal: bool, block_q: int, block_k: int,
                         q_index=None):
    """Online-softmax tiled attention for one head: returns (O, LSE).

    Follows the recurrence of "FlashAttention, simplified", "The trick": per block of
    queries, walk the key/value blocks in order keeping a running row max m, a running
    sum l of exponentials and an unnormalised accumulator acc; when a larger max arrives,
    rescale l and acc by alpha = exp(m - m_new); divide by l once at the end.

    A row whose keys seen so far are all masked has m_new = -inf; exp(-inf - (-inf)) is
    undefined, so for such a row the exponentials are taken relative to 0 instead (they
    are all exp(-inf) = 0 and l, acc stay 0).  Every causal row has at least its own key,
    so no finished row has l = 0.
    """
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    n_q, d = Q.shape
    N = K.shape[0]
    rows = _rows(n_q, q_index)
    O = np.empty((n_q, V.shape[1]))
    LSE = np.empty(n_q)
    for q0 in range(0, n_q, block_q):
        Qb = Q[q0:q0 + block_q]
        ib = rows[q0:q0 + block_q]
        m = np.full(Qb.shape[0], -np.inf)
        l = np.zeros(Qb.shape[0])
        acc = np.zeros((Qb.shape[0], V.shape[1]))
        for k0 in range(0, N, block_k):
            Kb = K[k0:k0 + block_k]
            Vb = V[k0:k0 + block_k]
            S = scale * (Qb @ Kb.T)
            if causal:
                jb = np.arange(k0, k0 + Kb.shape[0])
                S = np.where(jb[None, :] > ib[:, None], -np.inf, S)
            m_new = np.maximum(m, S.max(axis=1))
            ref = np.where(np.isneginf(m_new), 0.0, m_new)
            alpha = np.exp(m - ref)
            E = np.exp(S - ref[:, None])
            l = alpha * l + E.sum(axis=1)
            acc = alpha[:, None] * acc + E @ Vb
            m = m_new
        O[q0:q0 + block_q] = acc / l[:, None]
        LSE[q0:q0 + block_q] = m + np.log(l)
    return O, LSE


def attention_bwd_head(Q, K, V, dO, scale: float, causal: bool, O_given=None, q_index=None):
    """Analytic gradients of O = softmax(scale Q K^T [masked]) V for one head.

    Returns (dQ, dK, dV, D) where D_i = sum_k dO_ik O_ik.  Masked entries have P = 0 and
    so contribute nothing to any gradient.

    By default D uses the exact O.  A backward pass that is handed the forward's output
    (as the recompute-based backward is) forms D from that stored O instead; pass it as
    ``O_given`` to get exactly that computation.  With O_given equal to the exact O the
    two agree.  ``q_index`` gives the query rows' positions as in ``scores`` (default
    0..n_q-1).
    """
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    dO = _f64(dO)
    O, _, P = attention_head(Q, K, V, scale, causal, q_index)
    if O_given is not None:
        O = _f64(O_given)
    dV = P.T @ dO
    dP = dO @ V.T
    D = (dO * O).sum(axis=1)
    dS = P * (dP - D[:, None])
    dQ = scale * (dS @ K)
    dK = scale * (dS.T @ Q)
    return dQ, dK, dV, D


def attention_bwd_dq_rows(Q_rows, K, V, dO_rows, scale: float, causal: bool, q_index):
    """dQ (and D) for a subset of query rows of one head.

    dQ_i needs only q_i, dO_i and the head's full K and V: with P_i the row of
    probabilities and O_i = P_i V, D_i = dO_i . O_i, dS_i = P_i * (dO_i V^T - D_i) and
    dQ_i = scale dS_i K.  Returns (dQ_rows, D_rows).
    """
    K = _f64(K)
    V = _f64(V)
    dO_rows = _f64(dO_rows)
    O, _, P = attention_head(Q_rows, K, V, scale, causal, q_index)
    dP = dO_rows @ V.T
    D = (dO_rows * O).sum(axis=1)
    dS = P * (dP - D[:, None])
    dQ = scale * (dS @ K)
    return dQ, D


def attention_fwd(Q, K, V, scale: float, causal: bool):
    """Forward over Q [B, H, Nq, d], K and V [B, H, Nk, d] (Nq <= Nk when causal; the
    queries are the last Nq tokens, see ``chunk_positions``): returns (O [B,H,Nq,d],
    LSE [B,H,Nq]), float64."""
    Q = _f64(Q)
    B, H, N, _ = Q.shape
    pos = chunk_positions(N, np.shape(K)[2]) if causal else None
    O = np.empty(Q.shape[:3] + (np.shape(V)[3],))
    LSE = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            O[b, h], LSE[b, h], _ = attention_head(Q[b, h], np.asarray(K)[b, h],
                                                   np.asarray(V)[b, h], scale, causal, pos)
    return O, LSE


def attention_bwd(Q, K, V, dO, scale: float, causal: bool):
    """Backward over Q, dO [B, H, Nq, d], K, V [B, H, Nk, d] (as ``attention_fwd``):
    returns (dQ, dK, dV, D), float64."""
    Q = _f64(Q)
    B, H, N, d = Q.shape
    pos = chunk_positions(N, np.shape(K)[2]) if causal else None
    dQ = np.empty(Q.shape)
    dK = np.empty(np.shape(K))
    dV = np.empty(np.shape(V))
    D = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            dQ[b, h], dK[b, h], dV[b, h], D[b, h] = attention_bwd_head(
                Q[b, h], np.asarray(K)[b, h], np.asarray(V)[b, h], np.asarray(dO)[b, h],
                scale, causal, q_index=pos)
    return dQ, dK, dV, D

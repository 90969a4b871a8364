"""Pins for the fp64 oracle, and a check that the pins have teeth.

Each pin checks the oracle against something other than itself: a value derived by hand
(tests/golden), a closed form, an invariant of softmax attention, brute force in plain
Python, a second algorithm (the online-softmax recurrence of "FlashAttention,
simplified", "The trick"), or central finite differences for the backward.

``test_mutant_is_caught`` plants one plausible mistake at a time in a copy of the
oracle's source (a dropped scale, a flipped mask, a transposed operand, a wrong sign...)
and requires that at least one pin fails on it.
"""
import inspect
import json
import math
import os
import types

import numpy as np
import pytest

import oracle.attention as ORACLE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _bhnd(rng, B, H, N, d, sigma=1.0):
    return rng.standard_normal((B, H, N, d)) * sigma


# --------------------------------------------------------------------------- pins
def pin_golden_forward(A):
    g = json.load(open(os.path.join(GOLDEN, "hand_example_fwd.json")))
    Q, K, V = (np.array(g[k]) for k in ("Q", "K", "V"))
    O, LSE, _ = A.attention_head(Q, K, V, g["scale"], False)
    np.testing.assert_allclose(O, g["O"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(LSE, g["LSE"], rtol=0, atol=1e-13)
    O, LSE, _ = A.attention_head(Q, K, V, g["scale"], True)
    np.testing.assert_allclose(O, g["O_causal"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(LSE, g["LSE_causal"], rtol=0, atol=1e-13)
    # the same problem with the logits' factor moved into the scale argument
    O, LSE, _ = A.attention_head(Q * 2.0, K, V, 0.5, False)
    np.testing.assert_allclose(O, g["O"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(LSE, g["LSE"], rtol=0, atol=1e-13)
    Ob, LSEb = A.attention_fwd(Q[None, None], K[None, None], V[None, None], g["scale"], True)
    np.testing.assert_allclose(Ob[0, 0], g["O_causal"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(LSEb[0, 0], g["LSE_causal"], rtol=0, atol=1e-13)


def pin_golden_backward(A):
    g = json.load(open(os.path.join(GOLDEN, "hand_example_bwd.json")))
    Q, K, V, dO = (np.array(g[k]) for k in ("Q", "K", "V", "dO"))
    dQ, dK, dV, D = A.attention_bwd_head(Q, K, V, dO, g["scale"], False)
    for got, key in ((dQ, "dQ"), (dK, "dK"), (dV, "dV"), (D, "D")):
        np.testing.assert_allclose(got, g[key], rtol=0, atol=1e-13, err_msg=key)
    dQr, Dr = A.attention_bwd_dq_rows(Q, K, V, dO, g["scale"], False, [0])
    np.testing.assert_allclose(dQr, g["dQ"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(Dr, g["D"], rtol=0, atol=1e-13)


def pin_rows_sum_to_one(A):
    rng = _rng(1)
    for causal in (False, True):
        Q = rng.standard_normal((33, 8))
        K = rng.standard_normal((33, 8))
        S = A.scores(Q, K, 0.7, causal)
        P, _ = A.softmax_rows(S)
        np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        assert (P >= 0).all()
        _, _, P2 = A.attention_head(Q, K, K, 0.7, causal)
        np.testing.assert_allclose(P2.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        if causal:
            assert (np.triu(P2, 1) == 0).all()


def pin_identical_keys_mean_of_values(A):
    rng = _rng(2)
    B, H, N, d = 2, 3, 19, 4
    Q = _bhnd(rng, B, H, N, d)
    V = _bhnd(rng, B, H, N, 5)
    k = rng.standard_normal((B, H, 1, d))
    K = np.repeat(k, N, axis=2)      # one key per head, repeated N times
    O, LSE = A.attention_fwd(Q, K, V, 0.9, False)
    np.testing.assert_allclose(O, np.broadcast_to(V.mean(axis=2, keepdims=True), O.shape),
                               rtol=0, atol=1e-13)
    logit = 0.9 * np.einsum("bhnd,bhd->bhn", Q, k[:, :, 0])
    np.testing.assert_allclose(LSE, logit + math.log(N), rtol=0, atol=1e-12)
    O, LSE = A.attention_fwd(Q, K, V, 0.9, True)
    prefix_mean = np.cumsum(V, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    np.testing.assert_allclose(O, prefix_mean, rtol=0, atol=1e-13)
    np.testing.assert_allclose(LSE, logit + np.log(np.arange(1, N + 1)), rtol=0, atol=1e-12)


def pin_single_key(A):
    rng = _rng(3)
    Q = _bhnd(rng, 2, 2, 1, 6)
    K = _bhnd(rng, 2, 2, 1, 6)
    V = _bhnd(rng, 2, 2, 1, 6)
    for causal in (False, True):
        O, LSE = A.attention_fwd(Q, K, V, 0.25, causal)
        np.testing.assert_allclose(O, V, rtol=0, atol=1e-15)
        np.testing.assert_allclose(LSE, 0.25 * (Q * K).sum(-1), rtol=0, atol=1e-14)


def pin_causal_first_row(A):
    rng = _rng(4)
    Q = _bhnd(rng, 2, 2, 11, 5)
    K = _bhnd(rng, 2, 2, 11, 5)
    V = _bhnd(rng, 2, 2, 11, 5)
    O, LSE = A.attention_fwd(Q, K, V, 0.3, True)
    np.testing.assert_allclose(O[:, :, 0], V[:, :, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(LSE[:, :, 0], 0.3 * (Q[:, :, 0] * K[:, :, 0]).sum(-1),
                               rtol=0, atol=1e-14)
    # the last causal row sees every key, so it equals the non-causal last row
    On, LSEn = A.attention_fwd(Q, K, V, 0.3, False)
    np.testing.assert_allclose(O[:, :, -1], On[:, :, -1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(LSE[:, :, -1], LSEn[:, :, -1], rtol=0, atol=1e-13)


def pin_lse_bounds(A):
    rng = _rng(5)
    Q = rng.standard_normal((40, 8)) * 2
    K = rng.standard_normal((40, 8)) * 2
    for causal in (False, True):
        _, LSE, _ = A.attention_head(Q, K, K, 0.5, causal)
        S = 0.5 * Q @ K.T
        if causal:
            S = np.where(np.tri(40, dtype=bool), S, -np.inf)
        smax = S.max(axis=1)
        visible = np.isfinite(S).sum(axis=1)
        assert (LSE >= smax - 1e-12).all()
        assert (LSE <= smax + np.log(visible) + 1e-12).all()


def pin_shift_invariance(A):
    """Adding c_i to every logit of row i leaves O unchanged and adds c_i to LSE.  The
    shift is made through the inputs: one extra feature, c_i / scale on the query and
    1 on every key."""
    rng = _rng(6)
    N, d, scale = 23, 6, 0.4
    Q = rng.standard_normal((N, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, 3))
    c = rng.standard_normal(N) * 5
    Qa = np.concatenate([Q, (c / scale)[:, None]], axis=1)
    Ka = np.concatenate([K, np.ones((N, 1))], axis=1)
    for causal in (False, True):
        O, LSE, _ = A.attention_head(Q, K, V, scale, causal)
        Oa, LSEa, _ = A.attention_head(Qa, Ka, V, scale, causal)
        np.testing.assert_allclose(Oa, O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(LSEa, LSE + c, rtol=0, atol=1e-12)


def pin_large_logits(A):
    """Logits near +-1000 overflow exp() unless the row max is taken out first; the
    result must stay finite and equal the shifted small-logit problem."""
    rng = _rng(7)
    N, d = 17, 4
    Q = rng.standard_normal((N, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    shift = 1000.0
    Qa = np.concatenate([Q, np.full((N, 1), shift)], axis=1)
    Ka = np.concatenate([K, np.ones((N, 1))], axis=1)
    for causal in (False, True):
        O, LSE, _ = A.attention_head(Q, K, V, 1.0, causal)
        Oa, LSEa, _ = A.attention_head(Qa, Ka, V, 1.0, causal)
        assert np.isfinite(Oa).all() and np.isfinite(LSEa).all()
        np.testing.assert_allclose(Oa, O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(LSEa, LSE + shift, rtol=0, atol=1e-9)
        Ot, LSEt = A.attention_head_tiled(Qa, Ka, V, 1.0, causal, 5, 4)
        np.testing.assert_allclose(Ot, O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(LSEt, LSE + shift, rtol=0, atol=1e-9)


def _brute_force_head(Q, K, V, scale, causal, first_pos=0):
    """Softmax attention with Python scalars and loops, one entry at a time.  Query i
    stands at position first_pos + i of the key sequence (causal: it sees keys up to
    there)."""
    n, dv = len(Q), len(V[0])
    O = [[0.0] * dv for _ in range(n)]
    LSE = [0.0] * n
    for i in range(n):
        logits = []
        for j in range(len(K)):
            if causal and j > first_pos + i:
                continue
            logits.append((j, scale * sum(Q[i][t] * K[j][t] for t in range(len(Q[i])))))
        big = max(s for _, s in logits)
        weights = [(j, math.exp(s - big)) for j, s in logits]
        total = sum(w for _, w in weights)
        for j, w in weights:
            for t in range(dv):
                O[i][t] += w / total * V[j][t]
        LSE[i] = big + math.log(total)
    return np.array(O), np.array(LSE)


def pin_brute_force_small(A):
    rng = _rng(8)
    for N in (1, 2, 3, 4):
        for d in (1, 3):
            Q = rng.standard_normal((N, d))
            K = rng.standard_normal((N, d))
            V = rng.standard_normal((N, 2))
            for causal in (False, True):
                O, LSE, _ = A.attention_head(Q, K, V, 0.8, causal)
                Ob, LSEb = _brute_force_head(Q.tolist(), K.tolist(), V.tolist(), 0.8, causal)
                np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-14)
                np.testing.assert_allclose(LSE, LSEb, rtol=0, atol=1e-14)


def pin_chunk_brute_force(A):
    """Fewer queries than keys: the [B, H, N, d] wrapper treats the queries as the last
    tokens of the key sequence (bottom-right causal alignment), checked entry by entry
    against Python loops."""
    rng = _rng(14)
    for nq, nk in ((1, 3), (2, 3), (2, 5), (3, 4)):
        Q = rng.standard_normal((nq, 2))
        K = rng.standard_normal((nk, 2))
        V = rng.standard_normal((nk, 3))
        for causal in (False, True):
            O, LSE = A.attention_fwd(Q[None, None], K[None, None], V[None, None], 0.9, causal)
            Ob, LSEb = _brute_force_head(Q.tolist(), K.tolist(), V.tolist(), 0.9, causal,
                                         first_pos=nk - nq)
            np.testing.assert_allclose(O[0, 0], Ob, rtol=0, atol=1e-14)
            np.testing.assert_allclose(LSE[0, 0], LSEb, rtol=0, atol=1e-14)


def pin_chunk_is_tail_of_full_sequence(A):
    """Attention of the last Nq queries against all Nk keys equals the last Nq rows of
    causal attention over the whole sequence; with the gradient of the earlier rows set
    to zero, the whole sequence's dK, dV and last dQ rows equal the chunk's."""
    rng = _rng(15)
    nk, nq, d, scale = 11, 4, 3, 0.8
    Qf, K, V = (rng.standard_normal((nk, d)) for _ in range(3))
    G = np.zeros((nk, d))
    G[nk - nq:] = rng.standard_normal((nq, d))
    Of, LSEf, _ = A.attention_head(Qf, K, V, scale, True)
    O, LSE = A.attention_fwd(Qf[None, None, nk - nq:], K[None, None], V[None, None], scale,
                             True)
    np.testing.assert_allclose(O[0, 0], Of[nk - nq:], rtol=0, atol=1e-14)
    np.testing.assert_allclose(LSE[0, 0], LSEf[nk - nq:], rtol=0, atol=1e-14)
    dQf, dKf, dVf, _ = A.attention_bwd_head(Qf, K, V, G, scale, True)
    dQ, dK, dV, _ = A.attention_bwd(Qf[None, None, nk - nq:], K[None, None], V[None, None],
                                    G[None, None, nk - nq:], scale, True)
    np.testing.assert_allclose(dQ[0, 0], dQf[nk - nq:], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dK[0, 0], dKf, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dV[0, 0], dVf, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(A.chunk_positions(nq, nk), np.arange(nk - nq, nk))
    with pytest.raises(ValueError):
        A.chunk_positions(nk + 1, nk)


def pin_tiled_matches_naive(A):
    rng = _rng(9)
    N, d = 200, 8
    Q = rng.standard_normal((N, d)) * 2
    K = rng.standard_normal((N, d)) * 2
    V = rng.standard_normal((N, d))
    for causal in (False, True):
        O, LSE, _ = A.attention_head(Q, K, V, 0.35, causal)
        for bq, bk in ((16, 37), (50, 64), (200, 128), (7, 1)):
            Ot, LSEt = A.attention_head_tiled(Q, K, V, 0.35, causal, bq, bk)
            np.testing.assert_allclose(Ot, O, rtol=0, atol=1e-12)
            np.testing.assert_allclose(LSEt, LSE, rtol=0, atol=1e-12)
    # a subset of rows, as the row-sampled checks use it
    rows = np.array([0, 3, 127, 128, 199])
    O, LSE, _ = A.attention_head(Q[rows], K, V, 0.35, True, q_index=rows)
    Ot, LSEt = A.attention_head_tiled(Q[rows], K, V, 0.35, True, 2, 64, q_index=rows)
    np.testing.assert_allclose(Ot, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSEt, LSE, rtol=0, atol=1e-12)


def _fd_grad(f, X, h=1e-6):
    G = np.zeros_like(X)
    it = np.nditer(X, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        Xp = X.copy()
        Xm = X.copy()
        Xp[idx] += h
        Xm[idx] -= h
        G[idx] = (f(Xp) - f(Xm)) / (2 * h)
    return G


def pin_finite_differences(A):
    """Central differences of L = sum(O * G) confirm dQ, dK, dV (dO = G)."""
    rng = _rng(10)
    for N, d in ((1, 2), (3, 2), (7, 4)):
        for causal in (False, True):
            Q = rng.standard_normal((N, d))
            K = rng.standard_normal((N, d))
            V = rng.standard_normal((N, d))
            G = rng.standard_normal((N, d))
            scale = 0.7
            dQ, dK, dV, _ = A.attention_bwd_head(Q, K, V, G, scale, causal)

            def loss(Qx, Kx, Vx):
                return float((A.attention_head(Qx, Kx, Vx, scale, causal)[0] * G).sum())

            for got, fd in (
                (dQ, _fd_grad(lambda X: loss(X, K, V), Q)),
                (dK, _fd_grad(lambda X: loss(Q, X, V), K)),
                (dV, _fd_grad(lambda X: loss(Q, K, X), V)),
            ):
                np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-8)


def pin_chunk_finite_differences(A):
    """Central differences confirm the backward for queries placed at later positions
    (fewer queries than keys, causal)."""
    rng = _rng(16)
    nq, nk, d, scale = 3, 6, 2, 0.7
    pos = A.chunk_positions(nq, nk)
    Q = rng.standard_normal((nq, d))
    K = rng.standard_normal((nk, d))
    V = rng.standard_normal((nk, d))
    G = rng.standard_normal((nq, d))
    dQ, dK, dV, _ = A.attention_bwd_head(Q, K, V, G, scale, True, q_index=pos)

    def loss(Qx, Kx, Vx):
        return float((A.attention_head(Qx, Kx, Vx, scale, True, pos)[0] * G).sum())

    for got, fd in ((dQ, _fd_grad(lambda X: loss(X, K, V), Q)),
                    (dK, _fd_grad(lambda X: loss(Q, X, V), K)),
                    (dV, _fd_grad(lambda X: loss(Q, K, X), V))):
        np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-8)


def pin_dq_rows_finite_differences(A):
    rng = _rng(11)
    N, d, scale = 9, 3, 0.6
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    rows = np.array([0, 4, 8])
    Qr = rng.standard_normal((3, d))
    G = rng.standard_normal((3, d))
    for causal in (False, True):
        dQr, Dr = A.attention_bwd_dq_rows(Qr, K, V, G, scale, causal, rows)

        def loss(X):
            return float((A.attention_head(X, K, V, scale, causal, rows)[0] * G).sum())

        np.testing.assert_allclose(dQr, _fd_grad(loss, Qr), rtol=1e-6, atol=1e-8)
        O = A.attention_head(Qr, K, V, scale, causal, rows)[0]
        np.testing.assert_allclose(Dr, (G * O).sum(1), rtol=0, atol=1e-13)


def pin_batched_backward(A):
    """The [B, H, N, d] wrapper routes every head to its own inputs: heads are made
    independent by giving each a different single-key problem."""
    rng = _rng(12)
    B, H, N, d = 2, 3, 5, 2
    Q, K, V, dO = (_bhnd(rng, B, H, N, d) for _ in range(4))
    dQ, dK, dV, D = A.attention_bwd(Q, K, V, dO, 0.5, True)
    for b in range(B):
        for h in range(H):
            def loss(Qx, Kx, Vx, b=b, h=h):
                return float((A.attention_head(Qx, Kx, Vx, 0.5, True)[0] * dO[b, h]).sum())
            np.testing.assert_allclose(dQ[b, h], _fd_grad(lambda X: loss(X, K[b, h], V[b, h]),
                                                          Q[b, h]), rtol=1e-6, atol=1e-8)
            np.testing.assert_allclose(dK[b, h], _fd_grad(lambda X: loss(Q[b, h], X, V[b, h]),
                                                          K[b, h]), rtol=1e-6, atol=1e-8)
            np.testing.assert_allclose(dV[b, h], _fd_grad(lambda X: loss(Q[b, h], K[b, h], X),
                                                          V[b, h]), rtol=1e-6, atol=1e-8)


def pin_backward_with_given_output(A):
    """The stored-output variant: with the exact O it equals the default; with another
    O it forms D from that O, and only dQ and dK move (dV = P^T dO does not use D)."""
    rng = _rng(13)
    N, d, scale = 6, 3, 0.9
    Q, K, V, dO = (rng.standard_normal((N, d)) for _ in range(4))
    for causal in (False, True):
        base = A.attention_bwd_head(Q, K, V, dO, scale, causal)
        O = A.attention_head(Q, K, V, scale, causal)[0]
        same = A.attention_bwd_head(Q, K, V, dO, scale, causal, O_given=O)
        for x, y in zip(base, same):
            np.testing.assert_allclose(x, y, rtol=0, atol=1e-14)
        Ob = O + 0.01 * rng.standard_normal(O.shape)
        got = A.attention_bwd_head(Q, K, V, dO, scale, causal, O_given=Ob)
        np.testing.assert_allclose(got[3], (dO * Ob).sum(1), rtol=0, atol=1e-14)
        np.testing.assert_allclose(got[2], base[2], rtol=0, atol=1e-14)
        assert np.abs(got[0] - base[0]).max() > 1e-6


PINS = [
    pin_golden_forward,
    pin_golden_backward,
    pin_rows_sum_to_one,
    pin_identical_keys_mean_of_values,
    pin_single_key,
    pin_causal_first_row,
    pin_lse_bounds,
    pin_shift_invariance,
    pin_large_logits,
    pin_brute_force_small,
    pin_chunk_brute_force,
    pin_chunk_is_tail_of_full_sequence,
    pin_tiled_matches_naive,
    pin_finite_differences,
    pin_chunk_finite_differences,
    pin_dq_rows_finite_differences,
    pin_batched_backward,
    pin_backward_with_given_output,
]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(ORACLE)


# ------------------------------------------------------------------ planted mistakes
MUTANTS = [
    ("scores", "S = scale * (Q @ K.T)", "S = (Q @ K.T)"),
    ("scores", "j[None, :] > i[:, None]", "j[None, :] < i[:, None]"),
    ("scores", "j[None, :] > i[:, None]", "j[None, :] >= i[:, None]"),
    ("softmax_rows", "E = np.exp(S - m)", "E = np.exp(S)"),
    ("softmax_rows", "Z = E.sum(axis=1, keepdims=True)", "Z = E.sum(axis=0, keepdims=True)"),
    ("softmax_rows", "P = E / Z", "P = E"),
    ("softmax_rows", "LSE = m[:, 0] + np.log(Z[:, 0])", "LSE = m[:, 0] + Z[:, 0]"),
    ("softmax_rows", "LSE = m[:, 0] + np.log(Z[:, 0])", "LSE = np.log(Z[:, 0])"),
    ("attention_head", "O = P @ _f64(V)", "O = P.T @ _f64(V)"),
    ("attention_head_tiled", "l = alpha * l + E.sum(axis=1)", "l = l + E.sum(axis=1)"),
    ("attention_head_tiled", "acc = alpha[:, None] * acc + E @ Vb", "acc = acc + E @ Vb"),
    ("attention_head_tiled", "m = m_new", "m = m"),
    ("attention_head_tiled", "jb = np.arange(k0, k0 + Kb.shape[0])",
     "jb = np.arange(0, Kb.shape[0])"),
    ("attention_head_tiled", "S = scale * (Qb @ Kb.T)", "S = (Qb @ Kb.T)"),
    ("attention_head_tiled", "LSE[q0:q0 + block_q] = m + np.log(l)",
     "LSE[q0:q0 + block_q] = m"),
    ("attention_bwd_head", "dV = P.T @ dO", "dV = P @ dO"),
    ("attention_bwd_head", "dP = dO @ V.T", "dP = dO @ K.T"),
    ("attention_bwd_head", "D = (dO * O).sum(axis=1)", "D = (dO * O).sum(axis=0)"),
    ("attention_bwd_head", "dS = P * (dP - D[:, None])", "dS = P * (D[:, None] - dP)"),
    ("attention_bwd_head", "dS = P * (dP - D[:, None])", "dS = P * dP"),
    ("attention_bwd_head", "dQ = scale * (dS @ K)", "dQ = (dS @ K)"),
    ("attention_bwd_head", "dK = scale * (dS.T @ Q)", "dK = scale * (dS @ Q)"),
    ("attention_bwd_head", "dK = scale * (dS.T @ Q)", "dK = (dS.T @ Q)"),
    ("attention_bwd_head", "        O = _f64(O_given)", "        O = O"),
    ("attention_bwd_dq_rows", "dQ = scale * (dS @ K)", "dQ = (dS @ K)"),
    ("attention_bwd_dq_rows", "D = (dO_rows * O).sum(axis=1)", "D = (dO_rows * dO_rows).sum(axis=1)"),
    ("attention_fwd", "O[b, h], LSE[b, h], _ = attention_head(Q[b, h], np.asarray(K)[b, h],",
     "O[b, h], LSE[b, h], _ = attention_head(Q[b, h], np.asarray(K)[b, 0],"),
    ("attention_bwd", "Q[b, h], np.asarray(K)[b, h], np.asarray(V)[b, h], np.asarray(dO)[b, h],",
     "Q[b, h], np.asarray(K)[b, h], np.asarray(V)[0, h], np.asarray(dO)[b, h],"),
    ("chunk_positions", "return np.arange(n_q) + (n_k - n_q)", "return np.arange(n_q)"),
    ("chunk_positions", "return np.arange(n_q) + (n_k - n_q)",
     "return np.arange(n_q) + (n_q - n_k)"),
    ("attention_bwd_head", "O, _, P = attention_head(Q, K, V, scale, causal, q_index)",
     "O, _, P = attention_head(Q, K, V, scale, causal)"),
    ("attention_bwd", "scale, causal, q_index=pos)", "scale, causal)"),
    ("attention_fwd", "np.asarray(V)[b, h], scale, causal, pos)",
     "np.asarray(V)[b, h], scale, causal)"),
]


def _mutant_module(func_name, old, new):
    src = inspect.getsource(ORACLE)
    fsrc = inspect.getsource(getattr(ORACLE, func_name))
    assert fsrc.count(old) == 1, (func_name, old)
    assert src.count(fsrc) == 1
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(fsrc, fsrc.replace(old, new)), "oracle_mutant", "exec"),
         mod.__dict__)
    return mod


@pytest.mark.parametrize("func_name,old,new", MUTANTS,
                         ids=[f"{m[0]}:{i}" for i, m in enumerate(MUTANTS)])
def test_mutant_is_caught(func_name, old, new):
    mod = _mutant_module(func_name, old, new)
    caught = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin(mod)
            except Exception as e:  # an assertion, a shape error or a NaN all count
                caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin caught the planted mistake {old!r} -> {new!r}"

"""The largest shapes: a 131,072-token context and more heads than a grid's y extent.

At N = 131072 the oracle cannot form whole heads, so the test compares rows the oracle
computes one by one (O, LSE and dQ of sampled rows: each needs only its own query row and
all keys) and checks dV and dK through properties that hold at any size: every row of
probabilities sums to one, so the key rows of dV = P^T dO sum to the sum of the dO rows;
and every row of dS = P * (dP - D) sums to zero (D_i = sum_j P_ij dP_ij), so the key rows
of dK = scale dS^T Q sum to zero.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, inputs
from parity import assert_bf16_close, assert_lse_close, to64

pytestmark = pytest.mark.gpu


def test_long_context_131072():
    B, H, N, d = 1, 1, 131072, 128
    scale = d ** -0.5
    ins = inputs.make_inputs(B, H, N, d, seed=131, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=True)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=True)
    binding.check_device_error()
    rows = np.array(inputs.sample_rows(N, 48, seed=17))
    Q, K, V, dOh = (to64(ins[n][0, 0]) for n in ("Q", "K", "V", "dO"))
    rO, rL, _ = oracle.attention_head(Q[rows], K, V, scale, True, q_index=rows)
    assert_bf16_close(to64(O[0, 0, rows]), rO, "N=131072 O rows")
    assert_lse_close(to64(LSE[0, 0, rows]), rL, "N=131072 LSE rows")
    rdQ, _ = oracle.attention_bwd_dq_rows(Q[rows], K, V, dOh[rows], scale, True, rows)
    assert_bf16_close(to64(dQ[0, 0, rows]), rdQ, "N=131072 dQ rows")
    # sum_j dV_j = sum_j sum_i P_ij dO_i = sum_i dO_i.  The kernel rounds P to bf16 before
    # the product and rounds dV to bf16 (relative errors up to 2^-9 each, unbiased), so
    # the difference is a sum of independent errors with standard deviation at most
    # 2^-9 / sqrt(3) * sqrt(sum_i dO_i^2 + sum_j dV_j^2) per column; allow six of them.
    gv = to64(dV[0, 0])
    diff = np.abs(gv.sum(axis=0) - dOh.sum(axis=0))
    sigma = 2.0 ** -9 / math.sqrt(3) * np.sqrt((dOh ** 2).sum(axis=0) + (gv ** 2).sum(axis=0))
    assert (diff <= 6 * sigma).all(), f"sum of dV rows: max diff {diff.max():.3e}, 6 sigma {6 * sigma.min():.3e}"
    gk = to64(dK[0, 0])
    assert np.isfinite(to64(dQ)).all() and np.isfinite(gk).all() and np.isfinite(gv).all()
    # sum_j dK_j = scale sum_i (sum_j dS_ij) Q_i = 0.  What rounding leaves, per column c,
    # is a sum of independent unbiased errors (relative variance 2^-18 / 3 each) from
    #   (a) dS rounded to bf16 before the dK product: scale^2 sum_i Q_ic^2 sum_j dS_ij^2
    #   (c) dK rounded to bf16: sum_j dK_jc^2
    # and one that is not a rounding of the product itself:
    #   (b) D formed from the forward's bf16 output: row i's dS then sums to
    #       e_i = dO_i . (O_i - O_i^bf16) instead of zero, adding scale sum_i e_i Q_ic.
    # (a) and (b) need row quantities the oracle gives row by row (each row needs only its
    # query and all keys): sum_j dS_ij^2, and e_i from the exact O and the forward's O.
    # Both fall like 1/i along a causal head, so their sums are estimated from every row
    # of the first tile and 24 rows drawn in each stratum [2^k, 2^(k+1)), and doubled for
    # the sampling error.  Allow six standard deviations.
    u = 2.0 ** -18 / 3.0
    O64 = to64(O[0, 0])
    var_c = u * (gk ** 2).sum(axis=0)
    rng = np.random.default_rng(2024)
    strata = [(0, 128, 128)] + [(1 << k, 1 << (k + 1), 24) for k in range(7, 17)]
    var_a = np.zeros(d)
    var_b = np.zeros(d)
    for lo, hi, m in strata:
        rs = np.arange(lo, hi) if m >= hi - lo else np.sort(rng.choice(np.arange(lo, hi), m, replace=False))
        for c0 in range(0, len(rs), 32):
            r = rs[c0:c0 + 32]
            rO_, _, P = oracle.attention_head(Q[r], K, V, scale, True, q_index=r)
            Dr = (dOh[r] * rO_).sum(axis=1)
            dS = P * (dOh[r] @ V.T - Dr[:, None])
            s_i = (dS ** 2).sum(axis=1)
            e_i = Dr - (dOh[r] * O64[r]).sum(axis=1)
            w = (hi - lo) / len(rs)
            var_a += w * ((Q[r] ** 2) * s_i[:, None]).sum(axis=0)
            var_b += w * ((Q[r] ** 2) * (e_i ** 2)[:, None]).sum(axis=0)
    var_a *= 2.0 * u * scale ** 2
    var_b *= 2.0 * scale ** 2
    sigma_k = np.sqrt(var_a + var_b + var_c)
    diff_k = np.abs(gk.sum(axis=0))
    assert (diff_k <= 6 * sigma_k).all(), (
        f"sum of dK rows: max {diff_k.max():.3e} at column {int(diff_k.argmax())}, "
        f"6 sigma there {6 * sigma_k[int(diff_k.argmax())]:.3e}")


def test_more_heads_than_a_grid_dimension():
    """B*H = 81,920 heads of 40 tokens (one ragged tile each): work units are numbered
    flat, so nothing depends on a 65,535 grid extent; heads checked across the range."""
    B, H, N, d = 512, 160, 40, 64
    scale = 0.125
    ins = inputs.make_inputs(B, H, N, d, seed=160, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=True)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=True)
    binding.check_device_error()
    for b, h in ((0, 0), (255, 80), (511, 159), (409, 7)):
        Qh, Kh, Vh, dOh = (to64(ins[n][b, h]) for n in ("Q", "K", "V", "dO"))
        rO, rL, _ = oracle.attention_head(Qh, Kh, Vh, scale, True)
        assert_bf16_close(to64(O[b, h]), rO, f"O b={b} h={h}")
        assert_lse_close(to64(LSE[b, h]), rL, f"LSE b={b} h={h}")
        ref = oracle.attention_bwd_head(Qh, Kh, Vh, dOh, scale, True, O_given=to64(O[b, h]))
        for got, r, name in zip((dQ, dK, dV), ref[:3], ("dQ", "dK", "dV")):
            assert_bf16_close(to64(got[b, h]), r, f"{name} b={b} h={h}")

"""The largest shapes: a 131,072-token context and more heads than a grid's y extent.

At N = 131072 the oracle cannot form whole heads, so the test compares rows the oracle
computes one by one (O, LSE and dQ of sampled rows: each needs only its own query row and
all keys) and checks dV through a property that holds at any size: every row of
probabilities sums to one, so the key rows of dV = P^T dO sum to the sum of the dO rows.
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

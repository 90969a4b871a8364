"""Parity for fewer queries than keys (fa_fwd_qk, fa_bwd_qk) against the fp64 oracle.

The queries are the last Nq of the Nk tokens: under causal masking query i sees keys
j <= i + Nk - Nq.  Shapes cover ragged tiles on both sides, offsets Nk - Nq that are and
are not multiples of the 128-row tile, and non-causal Nq > Nk.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, inputs
from parity import (EXACT_MIN_ROWS, assert_bf16_close, assert_bf16_close_scaled,
                    assert_bwd_exact, assert_lse_close,
                    bf16_max_abs_bound, errors, to64)

pytestmark = pytest.mark.gpu


def _inputs(B, H, Nq, Nk, d, seed, sigma_qk=1.0):
    """Q and dO with Nq rows, K and V with Nk rows, drawn like make_inputs."""
    a = inputs.make_inputs(B, H, Nq, d, seed=seed, sigma_qk=sigma_qk, with_dO=True)
    b = inputs.make_inputs(B, H, Nk, d, seed=seed + 1, sigma_qk=sigma_qk)
    return {"Q": a["Q"], "dO": a["dO"], "K": b["K"], "V": b["V"]}


def _positions(Nq, Nk, causal):
    return oracle.chunk_positions(Nq, Nk) if causal else None


SHAPES = [(1, 5), (100, 300), (128, 256), (129, 200), (256, 1000), (77, 77), (300, 1)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nq,Nk", SHAPES)
def test_qk_forward(Nq, Nk, d, causal):
    if causal and Nq > Nk:
        pytest.skip("causal needs Nq <= Nk")
    ins = _inputs(1, 2, Nq, Nk, d, seed=Nq * 7 + Nk)
    scale = d ** -0.5
    q, k, v = (ins[n].cuda() for n in ("Q", "K", "V"))
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=causal)
    binding.check_device_error()
    pos = _positions(Nq, Nk, causal)
    for h in range(2):
        rO, rL, _ = oracle.attention_head(to64(ins["Q"][0, h]), to64(ins["K"][0, h]),
                                          to64(ins["V"][0, h]), scale, causal, pos)
        assert_bf16_close(to64(O[0, h]), rO, f"O Nq={Nq} Nk={Nk} d={d} causal={causal}")
        assert_lse_close(to64(LSE[0, h]), rL, f"LSE Nq={Nq} Nk={Nk}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nq,Nk", SHAPES)
def test_qk_backward(Nq, Nk, d, causal):
    """With many more queries than keys, dK and dV sum over many rows and are far from
    order one (Nq=300 against one key: dV is the sum of 300 dO rows, |dV| ~ 34), so the
    absolute bound scales with the largest value (``bf16_max_abs_bound``); rel-L2 keeps
    the stated 5e-3.  Shapes with at least EXACT_MIN_ROWS queries and keys are held to
    the exact gradient; smaller ones to the gradient with the handed-over bf16 O (and to
    the max-abs bound against the exact one)."""
    if causal and Nq > Nk:
        pytest.skip("causal needs Nq <= Nk")
    ins = _inputs(1, 2, Nq, Nk, d, seed=Nq * 11 + Nk)
    scale = d ** -0.5
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=causal)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=causal)
    binding.check_device_error()
    assert dQ.shape == q.shape and dK.shape == k.shape and dV.shape == v.shape
    pos = _positions(Nq, Nk, causal)
    for h in range(2):
        args = [to64(ins[n][0, h]) for n in ("Q", "K", "V", "dO")]
        exact = oracle.attention_bwd_head(*args, scale, causal, q_index=pos)
        # D formed with the bf16 output the backward is handed (see test_bwd_gpu)
        given = oracle.attention_bwd_head(*args, scale, causal, O_given=to64(O[0, h]),
                                          q_index=pos)
        for k_, name, got in ((0, "dQ", dQ), (1, "dK", dK), (2, "dV", dV)):
            g = to64(got[0, h])
            what = f"{name} Nq={Nq} Nk={Nk} d={d} causal={causal}"
            if min(Nq, Nk) >= EXACT_MIN_ROWS:
                assert_bwd_exact(g, exact[k_], what)
                continue
            assert_bf16_close_scaled(g, given[k_], what)
            max_abs, _ = errors(g, exact[k_])
            bound = bf16_max_abs_bound(exact[k_])
            assert max_abs <= bound, f"{name} vs exact: max_abs={max_abs:.3e} > {bound:.3e}"


def test_qk_prefill_chunk():
    """A 1024-token chunk against 8192 keys (B=1, H=8, d=128, causal): the prefill
    shape the Nq != Nk entry points exist for; two heads checked in full, forward and
    backward, against the exact gradient."""
    B, H, Nq, Nk, d = 1, 8, 1024, 8192, 128
    ins = _inputs(B, H, Nq, Nk, d, seed=91)
    scale = d ** -0.5
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=True)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=True)
    binding.check_device_error()
    pos = oracle.chunk_positions(Nq, Nk)
    for h in (0, 5):
        args = [to64(ins[n][0, h]) for n in ("Q", "K", "V", "dO")]
        rO, rL, _ = oracle.attention_head(args[0], args[1], args[2], scale, True, pos)
        assert_bf16_close(to64(O[0, h]), rO, f"prefill O h={h}")
        assert_lse_close(to64(LSE[0, h]), rL, f"prefill LSE h={h}")
        ref = oracle.attention_bwd_head(*args, scale, True, q_index=pos)
        for k_, name, got in ((0, "dQ", dQ), (1, "dK", dK), (2, "dV", dV)):
            assert_bf16_close(to64(got[0, h]), ref[k_], f"prefill {name} h={h}")


def test_qk_equal_lengths_match_square_entry_points():
    """fa_fwd_qk / fa_bwd_qk with Nq == Nk are the square calls: same bits."""
    ins = inputs.make_inputs(1, 3, 300, 128, seed=5, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O1, L1 = binding.fwd(q, k, v, causal=True)
    O2 = torch.empty_like(O1)
    L2 = torch.empty_like(L1)
    st = binding.lib().fa_fwd_qk(q.data_ptr(), k.data_ptr(), v.data_ptr(), O2.data_ptr(),
                                 L2.data_ptr(), 1, 3, 300, 300, 128, 128 ** -0.5, 1,
                                 torch.cuda.current_stream().cuda_stream)
    assert st == binding.FA_OK
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)

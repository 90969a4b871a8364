"""Parity for padded batches of different lengths (fa_fwd_varlen, fa_bwd_varlen).

Each sequence is checked against the oracle on its own rows (its queries aligned with
the end of its keys), the padding of every input is filled with finite values that
must not leak into the result, and every output row past a sequence's length must keep
the value it had before the call.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, inputs
from parity import (EXACT_MIN_ROWS, assert_bf16_close_scaled, assert_bwd_exact,
                    assert_lse_close, bf16_max_abs_bound, errors,
                    to64)

pytestmark = pytest.mark.gpu

SENTINEL = 7.0


def _padded_inputs(B, H, Nq, Nk, d, seed):
    a = inputs.make_inputs(B, H, Nq, d, seed=seed, with_dO=True)
    b = inputs.make_inputs(B, H, Nk, d, seed=seed + 1)
    return {"Q": a["Q"], "dO": a["dO"], "K": b["K"], "V": b["V"]}


def _run(ins, lq, lk, d, causal, with_bwd):
    B, H, Nq, _ = ins["Q"].shape
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    sq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    sk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    O = torch.full_like(q, SENTINEL)
    LSE = torch.full((B, H, Nq), SENTINEL, device="cuda")
    binding.fwd_varlen(q, k, v, sq, sk, causal=causal, O=O, LSE=LSE)
    binding.check_device_error()
    grads = None
    if with_bwd:
        grads = [torch.full_like(t, SENTINEL) for t in (q, k, v)]
        binding.bwd_varlen(q, k, v, O, do, LSE, sq, sk, causal=causal, dQ=grads[0],
                           dK=grads[1], dV=grads[2])
        binding.check_device_error()
    return O, LSE, grads


def _check(ins, lq, lk, d, causal, O, LSE, grads):
    B, H = ins["Q"].shape[:2]
    scale = d ** -0.5
    for b in range(B):
        for h in range(H):
            nq, nk = lq[b], lk[b]
            # rows past the sequence keep their old values
            assert bool((O[b, h, nq:] == SENTINEL).all()), f"O padding written b={b}"
            assert bool((LSE[b, h, nq:] == SENTINEL).all()), f"LSE padding written b={b}"
            if grads is not None:
                assert bool((grads[0][b, h, nq:] == SENTINEL).all()), f"dQ padding b={b}"
                assert bool((grads[1][b, h, nk:] == SENTINEL).all()), f"dK padding b={b}"
                assert bool((grads[2][b, h, nk:] == SENTINEL).all()), f"dV padding b={b}"
            if grads is not None and nq == 0 and nk > 0:
                # keys no query sees: their gradients are exactly zero
                assert bool((grads[1][b, h, :nk] == 0).all()), f"dK of keys without queries b={b}"
                assert bool((grads[2][b, h, :nk] == 0).all()), f"dV of keys without queries b={b}"
            if nq == 0 or nk == 0:
                continue
            Q = to64(ins["Q"][b, h, :nq])
            K = to64(ins["K"][b, h, :nk])
            V = to64(ins["V"][b, h, :nk])
            dO = to64(ins["dO"][b, h, :nq])
            pos = oracle.chunk_positions(nq, nk) if causal else None
            rO, rL, _ = oracle.attention_head(Q, K, V, scale, causal, pos)
            what = f"b={b} h={h} lq={nq} lk={nk} causal={causal}"
            assert_bf16_close_scaled(to64(O[b, h, :nq]), rO, "O " + what)
            assert_lse_close(to64(LSE[b, h, :nq]), rL, "LSE " + what)
            if grads is None:
                continue
            given = oracle.attention_bwd_head(Q, K, V, dO, scale, causal,
                                              O_given=to64(O[b, h, :nq]), q_index=pos)
            exact = oracle.attention_bwd_head(Q, K, V, dO, scale, causal, q_index=pos)
            for k_, name, n in ((0, "dQ", nq), (1, "dK", nk), (2, "dV", nk)):
                got = to64(grads[k_][b, h, :n])
                if min(nq, nk) >= EXACT_MIN_ROWS:
                    assert_bwd_exact(got, exact[k_], f"{name} {what}")
                    continue
                assert_bf16_close_scaled(got, given[k_], f"{name} {what}")
                max_abs, _ = errors(got, exact[k_])
                assert max_abs <= bf16_max_abs_bound(exact[k_]), f"{name} vs exact {what}"


CASES = [
    # (Nq, Nk, lengths_q, lengths_k): ragged, empty, single-row and full sequences
    (300, 300, [300, 1, 129, 0, 77, 256], [300, 1, 129, 5, 200, 256]),
    (256, 640, [256, 100, 1, 200], [640, 100, 33, 513]),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_varlen_forward_backward(case, d, causal):
    Nq, Nk, lq, lk = CASES[case]
    if causal:
        lq = [min(a, b) for a, b in zip(lq, lk)]
    ins = _padded_inputs(len(lq), 2, Nq, Nk, d, seed=500 + case)
    O, LSE, grads = _run(ins, lq, lk, d, causal, with_bwd=True)
    _check(ins, lq, lk, d, causal, O, LSE, grads)


def test_varlen_full_lengths_match_padded_call():
    """With every length equal to the padded one, the padded-batch calls give the same
    bits as fa_fwd / fa_bwd."""
    B, H, N, d = 3, 2, 333, 128
    ins = inputs.make_inputs(B, H, N, d, seed=8, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O1, L1 = binding.fwd(q, k, v, causal=True)
    g1 = binding.bwd(q, k, v, O1, do, L1, causal=True)
    full = torch.full((B,), N, dtype=torch.int32, device="cuda")
    O2, L2 = binding.fwd_varlen(q, k, v, full, full, causal=True)
    g2 = binding.bwd_varlen(q, k, v, O1, do, L1, full, full, causal=True)
    binding.check_device_error()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_varlen_bad_length_is_reported_and_skipped():
    """A length above the padded one is caught on the device: that sequence is skipped,
    the others are computed, and fa_check_device_error reports FA_ERR_INVALID_ARG."""
    B, H, N, d = 2, 1, 256, 64
    ins = _padded_inputs(B, H, N, N, d, seed=77)
    lq, lk = [N + 1, 200], [N, 200]
    q, k, v = (ins[n].cuda() for n in ("Q", "K", "V"))
    sq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    sk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    O = torch.full_like(q, SENTINEL)
    LSE = torch.full((B, H, N), SENTINEL, device="cuda")
    binding.fwd_varlen(q, k, v, sq, sk, causal=False, O=O, LSE=LSE)
    with pytest.raises(binding.FAError) as e:
        binding.check_device_error()
    assert e.value.status == binding.FA_ERR_INVALID_ARG
    binding.check_device_error()  # the report clears the error word
    assert bool((O[0] == SENTINEL).all())
    _check({n: t[1:] for n, t in ins.items()}, lq[1:], lk[1:], d, False, O[1:], LSE[1:], None)

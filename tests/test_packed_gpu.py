"""Parity for packed batches (fa_fwd_packed, fa_bwd_packed): the tokens of all sequences
one after another, [tokens, H, d], delimited by start arrays.  Each sequence and head is
compared with the oracle on its own rows (queries aligned with the end of its keys);
query rows of a sequence without keys must keep their old values."""
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


def _packed(total, H, d, seed, with_dO=False):
    """[total, H, d] bf16 tensors drawn like make_inputs (head-major draw, then packed)."""
    x = inputs.make_inputs(1, H, total, d, seed=seed, with_dO=with_dO)
    return {n: t[0].transpose(0, 1).contiguous() for n, t in x.items()}


def _cu(lengths):
    return torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32,
                        device="cuda")


CASES = [
    ([300, 1, 129, 0, 77, 256], [300, 1, 129, 5, 200, 256]),
    ([256, 100, 1, 200, 0], [640, 100, 33, 513, 0]),
    # lengths around the 32-row groups the output stores work in: a group of rows that
    # ends inside a sequence is written whole, one that crosses its end row by row (the
    # rows after it belong to the next sequence)
    ([31, 32, 33, 95, 96, 97, 160], [31, 32, 33, 95, 96, 97, 160]),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_packed_forward_backward(case, d, causal):
    lq, lk = CASES[case]
    if causal:
        lq = [min(a, b) for a, b in zip(lq, lk)]
    H, scale = 2, d ** -0.5
    tq, tk = sum(lq), sum(lk)
    a = _packed(tq, H, d, seed=700 + case, with_dO=True)
    b = _packed(tk, H, d, seed=710 + case)
    q, do = a["Q"].cuda(), a["dO"].cuda()
    k, v = b["K"].cuda(), b["V"].cuda()
    cq, ck = _cu(lq), _cu(lk)
    O = torch.full_like(q, SENTINEL)
    LSE = torch.full((H, tq), SENTINEL, device="cuda")
    binding.fwd_packed(q, k, v, cq, ck, max(lq), max(lk), scale=scale, causal=causal, O=O,
                       LSE=LSE)
    binding.check_device_error()
    dQ, dK, dV = (torch.full_like(t, SENTINEL) for t in (q, k, v))
    binding.bwd_packed(q, k, v, O, do, LSE, cq, ck, max(lq), max(lk), scale=scale,
                       causal=causal, dQ=dQ, dK=dK, dV=dV)
    binding.check_device_error()
    q0s, k0s = np.cumsum([0] + lq), np.cumsum([0] + lk)
    for s, (nq, nk) in enumerate(zip(lq, lk)):
        qs, ks = slice(q0s[s], q0s[s] + nq), slice(k0s[s], k0s[s] + nk)
        if nk == 0:
            assert bool((O[qs] == SENTINEL).all()) and bool((dQ[qs] == SENTINEL).all())
            continue
        if nq == 0:
            # keys no query sees: their gradients are exactly zero
            assert bool((dK[ks] == 0).all()) and bool((dV[ks] == 0).all()), f"seq {s}"
            continue
        pos = oracle.chunk_positions(nq, nk) if causal else None
        for h in range(H):
            Qh, Kh, Vh, Gh = (to64(t[sl, h]) for t, sl in ((a["Q"], qs), (b["K"], ks),
                                                            (b["V"], ks), (a["dO"], qs)))
            rO, rL, _ = oracle.attention_head(Qh, Kh, Vh, scale, causal, pos)
            what = f"seq {s} h={h} lq={nq} lk={nk} causal={causal}"
            assert_bf16_close_scaled(to64(O[qs, h]), rO, "O " + what)
            assert_lse_close(to64(LSE[h, qs]), rL, "LSE " + what)
            given = oracle.attention_bwd_head(Qh, Kh, Vh, Gh, scale, causal,
                                              O_given=to64(O[qs, h]), q_index=pos)
            exact = oracle.attention_bwd_head(Qh, Kh, Vh, Gh, scale, causal, q_index=pos)
            for k_, name, got, sl in ((0, "dQ", dQ, qs), (1, "dK", dK, ks), (2, "dV", dV, ks)):
                g = to64(got[sl, h])
                if min(nq, nk) >= EXACT_MIN_ROWS:
                    assert_bwd_exact(g, exact[k_], f"{name} {what}")
                    continue
                assert_bf16_close_scaled(g, given[k_], f"{name} {what}")
                max_abs, _ = errors(g, exact[k_])
                assert max_abs <= bf16_max_abs_bound(exact[k_]), f"{name} vs exact {what}"


def test_packed_bad_starts_are_reported():
    """A start array that decreases is caught on the device: that sequence is skipped
    and fa_check_device_error reports FA_ERR_INVALID_ARG; the others are computed."""
    H, d = 1, 64
    a = _packed(300, H, d, seed=720)
    q, k, v = a["Q"].cuda(), a["K"].cuda(), a["V"].cuda()
    # sequence 1 runs backwards (200 -> 100), sequence 2 is empty
    cu = torch.tensor([0, 200, 100, 100], dtype=torch.int32, device="cuda")
    O = torch.full_like(q, SENTINEL)
    binding.fwd_packed(q, k, v, cu, cu, 200, 200, O=O)
    with pytest.raises(binding.FAError) as e:
        binding.check_device_error()
    assert e.value.status == binding.FA_ERR_INVALID_ARG
    rO, _, _ = oracle.attention_head(to64(a["Q"][:200, 0]), to64(a["K"][:200, 0]),
                                     to64(a["V"][:200, 0]), 0.125, False)
    assert_bf16_close_scaled(to64(O[:200, 0]), rO, "sequence 0")
    assert bool((O[200:] == SENTINEL).all())

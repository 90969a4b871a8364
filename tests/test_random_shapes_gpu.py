"""Seeded random shapes: forward and backward against the oracle on problems drawn at
random (query and key counts with offsets that are not multiples of the tile, both head
sizes and masks, logit scales from flat to peaked; bf16 and float32), so that no mask or
tail rule is only exercised at hand-picked sizes.  Every case is fixed by its seed."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, inputs
from parity import (EXACT_MIN_ROWS, assert_bf16_close, assert_bf16_close_scaled,
                    assert_bwd_exact, assert_f32_close,
                    assert_lse_close, bf16_max_abs_bound, errors, to64)

pytestmark = pytest.mark.gpu


def _case(seed):
    rng = np.random.default_rng(seed)
    d = int(rng.choice([64, 128]))
    causal = bool(rng.integers(2))
    Nk = int(rng.integers(1, 900))
    Nq = int(rng.integers(1, Nk + 1)) if (causal or rng.random() < 0.5) else int(rng.integers(1, 900))
    H = int(rng.integers(1, 4))
    sigma = float(rng.choice([0.5, 1.0, 2.0]))
    return d, causal, Nq, Nk, H, sigma


@pytest.mark.parametrize("seed", range(24))
def test_random_shape(seed):
    d, causal, Nq, Nk, H, sigma = _case(seed)
    a = inputs.make_inputs(1, H, Nq, d, seed=9000 + seed, sigma_qk=sigma, with_dO=True)
    b = inputs.make_inputs(1, H, Nk, d, seed=9500 + seed, sigma_qk=sigma)
    scale = d ** -0.5
    q, do = a["Q"].cuda(), a["dO"].cuda()
    k, v = b["K"].cuda(), b["V"].cuda()
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=causal)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=causal)
    binding.check_device_error()
    pos = oracle.chunk_positions(Nq, Nk) if causal else None
    what = f"seed={seed} d={d} causal={causal} Nq={Nq} Nk={Nk} sigma={sigma}"
    for h in range(H):
        Qh, Gh = to64(a["Q"][0, h]), to64(a["dO"][0, h])
        Kh, Vh = to64(b["K"][0, h]), to64(b["V"][0, h])
        rO, rL, _ = oracle.attention_head(Qh, Kh, Vh, scale, causal, pos)
        assert_bf16_close(to64(O[0, h]), rO, "O " + what)
        assert_lse_close(to64(LSE[0, h]), rL, "LSE " + what)
        given = oracle.attention_bwd_head(Qh, Kh, Vh, Gh, scale, causal,
                                          O_given=to64(O[0, h]), q_index=pos)
        exact = oracle.attention_bwd_head(Qh, Kh, Vh, Gh, scale, causal, q_index=pos)
        for k_, name, got in ((0, "dQ", dQ), (1, "dK", dK), (2, "dV", dV)):
            g = to64(got[0, h])
            assert_bf16_close_scaled(g, given[k_], f"{name} {what}")
            max_abs, rel_l2 = errors(g, exact[k_])
            if sigma <= 1.0 and min(Nq, Nk) >= EXACT_MIN_ROWS:
                assert_bwd_exact(g, exact[k_], f"{name} {what}")
            elif sigma > 1.0:
                # peaked logits: rounding O to bf16 alone moves D far enough that dQ and dK
                # leave the max-abs bound against the exact gradient (seed 10: 0.030 against
                # a bound of 0.028, with no kernel error at all); the given-O check above
                # keeps the full bound and the exact one keeps rel-L2, as for sigma 3
                assert rel_l2 <= 1e-2, f"{name} vs exact {what}: rel_l2={rel_l2:.3e}"
            else:
                assert max_abs <= bf16_max_abs_bound(exact[k_]), f"{name} vs exact {what}"


@pytest.mark.parametrize("seed", range(8))
def test_random_shape_f32(seed):
    """The float32 path at random query and key counts, heads and masks."""
    rng = np.random.default_rng(20000 + seed)
    d = int(rng.choice([64, 128]))
    causal = bool(rng.integers(2))
    Nk = int(rng.integers(1, 400))
    Nq = int(rng.integers(1, Nk + 1)) if causal else int(rng.integers(1, 400))
    H = int(rng.integers(1, 3))
    a = inputs.make_inputs(1, H, Nq, d, seed=9900 + seed, dtype=torch.float32, with_dO=True)
    b = inputs.make_inputs(1, H, Nk, d, seed=9950 + seed, dtype=torch.float32)
    scale = d ** -0.5
    q, do = a["Q"].cuda(), a["dO"].cuda()
    k, v = b["K"].cuda(), b["V"].cuda()
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=causal)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=causal)
    binding.check_device_error()
    assert O.dtype == torch.float32 and dQ.dtype == torch.float32
    pos = oracle.chunk_positions(Nq, Nk) if causal else None
    what = f"f32 seed={seed} d={d} causal={causal} Nq={Nq} Nk={Nk}"
    for h in range(H):
        Qh, Gh = to64(a["Q"][0, h]), to64(a["dO"][0, h])
        Kh, Vh = to64(b["K"][0, h]), to64(b["V"][0, h])
        rO, rL, _ = oracle.attention_head(Qh, Kh, Vh, scale, causal, pos)
        assert_f32_close(to64(O[0, h]), rO, "O " + what)
        assert_lse_close(to64(LSE[0, h]), rL, "LSE " + what)
        ref = oracle.attention_bwd_head(Qh, Kh, Vh, Gh, scale, causal, q_index=pos)
        for k_, name, got in ((0, "dQ", dQ), (1, "dK", dK), (2, "dV", dV)):
            assert_f32_close(to64(got[0, h]), ref[k_], f"{name} {what}")

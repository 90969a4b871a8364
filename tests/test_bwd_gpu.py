"""Backward parity: fa_bwd through the C ABI against the analytic fp64 oracle.

The CUDA forward provides O and LSE (as a user would run it); the oracle recomputes
everything from Q, K, V, dO in float64.  Small problems are compared in full; the named
workload (B=2, H=16, N=8192, d=128, causal) in full on two seeded (batch, head) pairs and
on a seeded subset of dQ rows in every head.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, inputs
from parity import (BF16_MAX_ABS, EXACT_MIN_ROWS, assert_bf16_close, assert_f32_close, errors,
                    to64)

pytestmark = pytest.mark.gpu


def _fwd_bwd(ins, scale, causal):
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=causal)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=causal)
    binding.check_device_error()
    return dQ, dK, dV, O


def _check_head(ins, grads, b, h, scale, causal, what=""):
    """Against the exact gradient, within the bf16 tolerance."""
    Q, K, V, dO = (to64(ins[n][b, h]) for n in ("Q", "K", "V", "dO"))
    rQ, rK, rV, _ = oracle.attention_bwd_head(Q, K, V, dO, scale, causal)
    for got, ref, name in zip(grads, (rQ, rK, rV), ("dQ", "dK", "dV")):
        assert_bf16_close(to64(got[b, h]), ref, f"{what} {name} b={b} h={h} causal={causal}")


def _check_head_given_O(ins, grads, O, b, h, scale, causal, what=""):
    """For fewer than EXACT_MIN_ROWS rows only: against the gradient formed with the bf16
    forward output that fa_bwd was handed (D = rowsum(dO * O)).  For a handful of keys
    the bf16 rounding of O alone moves dQ by about 1% relative L2 (the difference dP - D
    is then small), so tiny problems are held to the bf16 tolerance on this reference,
    and to the max-abs bound against the exact gradient."""
    Q, K, V, dO = (to64(ins[n][b, h]) for n in ("Q", "K", "V", "dO"))
    exact = oracle.attention_bwd_head(Q, K, V, dO, scale, causal)
    given = oracle.attention_bwd_head(Q, K, V, dO, scale, causal, O_given=to64(O[b, h]))
    for k, name in enumerate(("dQ", "dK", "dV")):
        got = to64(grads[k][b, h])
        assert_bf16_close(got, given[k], f"{what} {name} b={b} h={h} causal={causal}")
        max_abs, _ = errors(got, exact[k])
        assert max_abs <= BF16_MAX_ABS, f"{what} {name} vs exact: max_abs={max_abs:.3e}"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 2, 100, 128, 129, 256, 300, 513])
def test_bwd_full_small(N, d, causal):
    """Whole heads against the exact gradient within the stated bf16 tolerance from
    EXACT_MIN_ROWS rows on; below that against the gradient with the handed-over O."""
    ins = inputs.make_inputs(1, 3, N, d, seed=2000 + N, with_dO=True)
    scale = 1.0 / np.sqrt(d)
    *grads, O = _fwd_bwd(ins, scale, causal)
    for h in range(3):
        if N >= EXACT_MIN_ROWS:
            _check_head(ins, grads, 0, h, scale, causal, f"N={N} d={d}")
        else:
            _check_head_given_O(ins, grads, O, 0, h, scale, causal, f"N={N} d={d}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_many_units_per_cta(causal):
    # 2 * 40 heads * 8 tiles = 640 units per kernel > 148 SMs
    B, H, N, d = 2, 40, 1000, 64
    ins = inputs.make_inputs(B, H, N, d, seed=31, with_dO=True)
    *grads, _ = _fwd_bwd(ins, 0.125, causal)
    for b, h in ((0, 0), (1, 39), (0, 17)):
        _check_head(ins, grads, b, h, 0.125, causal, "many units")


def test_workload_n8192_backward():
    w = inputs.WORKLOADS["n8192_d128_causal_bwd"]
    ins = inputs.make_workload_inputs(w)
    *grads, _ = _fwd_bwd(ins, w.scale, w.causal)
    rng = np.random.default_rng(1234)
    pairs = {(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(2)}
    for b, h in sorted(pairs):
        _check_head(ins, grads, b, h, w.scale, w.causal, w.name)
    dQ = to64(grads[0])
    rows = np.array(inputs.sample_rows(w.N, 256, seed=99))
    for b in range(w.B):
        for h in range(w.H):
            Q, K, V, dO = (to64(ins[n][b, h]) for n in ("Q", "K", "V", "dO"))
            rQ, _ = oracle.attention_bwd_dq_rows(Q[rows], K, V, dO[rows], w.scale, w.causal,
                                                 rows)
            assert_bf16_close(dQ[b, h, rows], rQ, f"{w.name} dQ rows b={b} h={h}")


def test_bwd_deterministic_and_in_bounds():
    B, H, N, d = 1, 6, 777, 128
    ins = inputs.make_inputs(B, H, N, d, seed=8, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, causal=True)
    guard = 4096
    n = B * H * N * d
    bufs = [torch.full((2 * guard + n,), 5.0, device="cuda", dtype=torch.bfloat16)
            for _ in range(3)]
    views = [b[guard:guard + n].view(B, H, N, d) for b in bufs]
    ws_bytes = binding.workspace_bytes(B, H, N, d)
    wsbuf = torch.full((ws_bytes + 2 * guard,), 0xAB, device="cuda", dtype=torch.uint8)
    ws = wsbuf[guard:guard + ws_bytes]
    outs = []
    for _ in range(2):
        binding.bwd(q, k, v, O, do, LSE, causal=True, dQ=views[0], dK=views[1], dV=views[2],
                    workspace=ws)
        binding.check_device_error()
        outs.append([t.clone() for t in views])
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    for b in bufs:
        assert bool((b[:guard] == 5.0).all()) and bool((b[-guard:] == 5.0).all())
    assert bool((wsbuf[:guard] == 0xAB).all()) and bool((wsbuf[-guard:] == 0xAB).all())


@pytest.mark.parametrize("d", [64, 128])
def test_outputs_at_16_byte_offsets(d):
    """Outputs that start 16 bytes past a 32-byte boundary (the least alignment the calls
    accept) get the same bits as outputs at aligned addresses: O, dQ, dK and dV, whose
    stores use wider or bulk forms where the address allows."""
    B, H, N = 1, 3, 300
    ins = inputs.make_inputs(B, H, N, d, seed=21, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, causal=True)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, causal=True)
    n = B * H * N * d
    bufs = [torch.full((n + 64,), 3.0, device="cuda", dtype=torch.bfloat16) for _ in range(4)]
    views = [b[8:8 + n].view(B, H, N, d) for b in bufs]  # 16 bytes past the allocation
    assert all(t.data_ptr() % 32 == 16 for t in views)
    O2, _ = binding.fwd(q, k, v, causal=True, O=views[0])
    binding.bwd(q, k, v, O, do, LSE, causal=True, dQ=views[1], dK=views[2], dV=views[3])
    binding.check_device_error()
    for got, want in zip(views, (O, dQ, dK, dV)):
        assert torch.equal(got, want)
    for b in bufs:
        assert bool((b[:8] == 3.0).all()) and bool((b[8 + n:] == 3.0).all())


def test_bwd_rejects_small_workspace():
    ins = inputs.make_inputs(1, 2, 256, 64, seed=1, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v)
    small = torch.empty(64, device="cuda", dtype=torch.uint8)
    with pytest.raises(binding.FAError) as e:
        binding.bwd(q, k, v, O, do, LSE, workspace=small)
    assert e.value.status == binding.FA_ERR_INVALID_ARG


def _head_and_rows(ins, grads, w_scale, causal, heads, rows_count, seed, what):
    B, H, N, d = ins["Q"].shape
    for b, h in heads:
        _check_head(ins, grads, b, h, w_scale, causal, what)
    dQ = to64(grads[0])
    rows = np.array(inputs.sample_rows(N, rows_count, seed=seed))
    for b in range(B):
        for h in range(H):
            Q, K, V, dO = (to64(ins[n][b, h]) for n in ("Q", "K", "V", "dO"))
            rQ, _ = oracle.attention_bwd_dq_rows(Q[rows], K, V, dO[rows], w_scale, causal, rows)
            assert_bf16_close(dQ[b, h, rows], rQ, f"{what} dQ rows b={b} h={h}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_n4096_d128(causal):
    ins = inputs.make_inputs(1, 4, 4096, 128, seed=41, with_dO=True)
    scale = 128 ** -0.5
    *grads, _ = _fwd_bwd(ins, scale, causal)
    _head_and_rows(ins, grads, scale, causal, ((0, 3),), 128, 7, f"N=4096 d=128 causal={causal}")


def test_bwd_n4096_d64_causal():
    ins = inputs.make_inputs(2, 4, 4096, 64, seed=42, with_dO=True)
    *grads, _ = _fwd_bwd(ins, 0.125, True)
    _head_and_rows(ins, grads, 0.125, True, ((1, 2),), 128, 8, "N=4096 d=64")


def test_bwd_ragged_n10000():
    # the 10,000-token length: a ragged last tile in every kernel of the backward
    ins = inputs.make_inputs(1, 2, 10000, 128, seed=43, with_dO=True)
    scale = 128 ** -0.5
    *grads, _ = _fwd_bwd(ins, scale, True)
    _head_and_rows(ins, grads, scale, True, ((0, 1),), 64, 9, "N=10000")


def test_bwd_large_logits():
    """Logits of std 9 (sigma_qk = 3): probabilities far from uniform and gradients up to
    ~13 in magnitude.  Two references, with bounds derived from the arithmetic:
    * the gradient formed with the bf16 forward output the backward is handed
      (D = rowsum(dO * O)): rel-L2 <= 5e-3 as stated, max-abs <= 4 * 2^-9 * max|ref|
      (the stated absolute 2e-2 is for O(1) values; one bf16 rounding of a value near 13
      is already 0.025, and both dS and the result are rounded);
    * the exact gradient: rel-L2 <= 1e-2.  With peaked probabilities dP - D is small, so
      the bf16 rounding of O inside D moves dQ and dK by ~3e-3 on its own (an fp64 model
      of the rounding gives 4.6e-3 before the output is rounded)."""
    ins = inputs.make_inputs(1, 2, 2048, 128, seed=44, sigma_qk=3.0, with_dO=True)
    scale = 128 ** -0.5
    *grads, O = _fwd_bwd(ins, scale, True)
    for h in range(2):
        Q, K, V, dO = (to64(ins[n][0, h]) for n in ("Q", "K", "V", "dO"))
        exact = oracle.attention_bwd_head(Q, K, V, dO, scale, True)
        given = oracle.attention_bwd_head(Q, K, V, dO, scale, True, O_given=to64(O[0, h]))
        for k, name in enumerate(("dQ", "dK", "dV")):
            got = to64(grads[k][0, h])
            max_abs, rel_l2 = errors(got, given[k])
            bound = 4 * 2.0 ** -9 * float(np.abs(given[k]).max())
            assert rel_l2 <= 5e-3 and max_abs <= bound, (
                f"sigma 3 {name} h={h} vs given-O: max_abs={max_abs:.3e} (bound {bound:.3e}) "
                f"rel_l2={rel_l2:.3e}")
            _, rel_exact = errors(got, exact[k])
            assert rel_exact <= 1e-2, f"sigma 3 {name} h={h} vs exact: rel_l2={rel_exact:.3e}"


# ------------------------------------------------------------------ float32 backward
def _fwd_bwd_f32(ins, scale, causal):
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=causal)
    dQ, dK, dV = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=causal)
    binding.check_device_error()
    assert dQ.dtype == torch.float32
    return dQ, dK, dV


def _check_head_f32(ins, grads, b, h, scale, causal, what=""):
    """fa_bwd_f32 against the exact fp64 gradient within the float32 tolerance (every
    step of both the forward that supplies O and LSE and the backward is float32)."""
    Q, K, V, dO = (to64(ins[n][b, h]) for n in ("Q", "K", "V", "dO"))
    ref = oracle.attention_bwd_head(Q, K, V, dO, scale, causal)
    for got, r, name in zip(grads, ref[:3], ("dQ", "dK", "dV")):
        assert_f32_close(to64(got[b, h]), r, f"{what} {name} b={b} h={h} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_f32_tiny_workload(causal):
    # B=1 H=1 N=256 d=64 float32: the configuration the float32 path exists for
    w = inputs.WORKLOADS["tiny_f32"]
    ins = inputs.make_inputs(w.B, w.H, w.N, w.d, seed=w.seed, dtype=torch.float32,
                             with_dO=True)
    grads = _fwd_bwd_f32(ins, w.scale, causal)
    _check_head_f32(ins, grads, 0, 0, w.scale, causal, w.name)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 31, 32, 33, 100, 300])
def test_bwd_f32_small(N, d, causal):
    ins = inputs.make_inputs(1, 2, N, d, seed=3000 + N, dtype=torch.float32, with_dO=True)
    scale = 1.0 / np.sqrt(d)
    grads = _fwd_bwd_f32(ins, scale, causal)
    for h in range(2):
        _check_head_f32(ins, grads, 0, h, scale, causal, f"f32 N={N} d={d}")


def test_bwd_f32_many_heads_and_large_logits():
    # blocks are numbered flat over (head, row block): 3 * 7 heads of 3 row blocks; logits
    # of std 9 exercise the exponentials far from the row maximum
    B, H, N, d = 3, 7, 70, 128
    ins = inputs.make_inputs(B, H, N, d, seed=77, sigma_qk=3.0, dtype=torch.float32,
                             with_dO=True)
    scale = d ** -0.5
    grads = _fwd_bwd_f32(ins, scale, True)
    for b, h in ((0, 0), (1, 3), (2, 6)):
        _check_head_f32(ins, grads, b, h, scale, True, "f32 many heads")


def test_bwd_f32_deterministic_and_in_bounds():
    B, H, N, d = 1, 3, 333, 64
    ins = inputs.make_inputs(B, H, N, d, seed=9, dtype=torch.float32, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, causal=False)
    guard = 1024
    n = B * H * N * d
    bufs = [torch.full((2 * guard + n,), 7.0, device="cuda") for _ in range(3)]
    views = [b[guard:guard + n].view(B, H, N, d) for b in bufs]
    ws_bytes = binding.workspace_bytes(B, H, N, d)
    wsbuf = torch.full((ws_bytes + 2 * guard,), 0xCD, device="cuda", dtype=torch.uint8)
    ws = wsbuf[guard:guard + ws_bytes]
    outs = []
    for _ in range(2):
        binding.bwd(q, k, v, O, do, LSE, dQ=views[0], dK=views[1], dV=views[2], workspace=ws)
        binding.check_device_error()
        outs.append([t.clone() for t in views])
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    for b in bufs:
        assert bool((b[:guard] == 7.0).all()) and bool((b[-guard:] == 7.0).all())
    assert bool((wsbuf[:guard] == 0xCD).all()) and bool((wsbuf[-guard:] == 0xCD).all())

"""Forward parity: fa_fwd / fa_fwd_f32 through the C ABI against the fp64 oracle.

Small problems are compared in full (several 128-row tiles and ragged tails); the named
workloads are compared on every head for a seeded subset of rows (each output row
depends only on its own query and the head's keys and values) and in full on one head.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, inputs
from parity import (assert_bf16_close, assert_f32_close, assert_lse_close, to64)

pytestmark = pytest.mark.gpu


def _run(ins, scale, causal):
    q, k, v = (ins[n].cuda() for n in ("Q", "K", "V"))
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=causal)
    binding.check_device_error()
    return O, LSE


def _full_check(ins, scale, causal, f32=False):
    O, LSE = _run(ins, scale, causal)
    Q, K, V = (to64(ins[n]) for n in ("Q", "K", "V"))
    B, H = Q.shape[:2]
    for b in range(B):
        for h in range(H):
            Or, LSEr, _ = oracle.attention_head(Q[b, h], K[b, h], V[b, h], scale, causal)
            what = f"b={b} h={h} causal={causal}"
            if f32:
                assert_f32_close(to64(O[b, h]), Or, what)
                assert_f32_close(to64(LSE[b, h]), LSEr, what + " LSE")
            else:
                assert_bf16_close(to64(O[b, h]), Or, what)
                assert_lse_close(to64(LSE[b, h]), LSEr, what)
    return O, LSE


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_f32_workload(causal):
    w = inputs.WORKLOADS["tiny_f32"]
    ins = inputs.make_workload_inputs(w)
    assert ins["Q"].dtype == torch.float32
    _full_check(ins, w.scale, causal, f32=True)


@pytest.mark.parametrize("N", [1, 7, 200, 300])
@pytest.mark.parametrize("d", [64, 128])
def test_f32_ragged(N, d):
    ins = inputs.make_inputs(2, 2, N, d, seed=N + d, dtype=torch.float32)
    for causal in (False, True):
        _full_check(ins, 1.0 / np.sqrt(d), causal, f32=True)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 2, 64, 127, 128, 129, 255, 256, 257, 383, 600])
def test_bf16_full_small(N, d, causal):
    ins = inputs.make_inputs(1, 3, N, d, seed=1000 + N)
    _full_check(ins, 1.0 / np.sqrt(d), causal)


@pytest.mark.parametrize("causal", [False, True])
def test_bf16_many_units_per_cta(causal):
    # 2 * 40 heads * 4 units = 320 units > 148 SMs: every CTA walks several units
    ins = inputs.make_inputs(2, 40, 1000, 64, seed=77)
    _full_check(ins, 0.125, causal)


def _rows_check(w, rows_per_head=256, full_heads=((0, 0),), check_lse=True, extra_rows=()):
    ins = inputs.make_workload_inputs(w)
    O, LSE = _run(ins, w.scale, w.causal)
    Q, K, V = (to64(ins[n]) for n in ("Q", "K", "V"))
    O64, LSE64 = to64(O), to64(LSE)
    rows = np.array(sorted(set(inputs.sample_rows(w.N, rows_per_head, seed=1234)) |
                           set(extra_rows)))
    for b in range(w.B):
        for h in range(w.H):
            Or, LSEr, _ = oracle.attention_head(Q[b, h, rows], K[b, h], V[b, h], w.scale,
                                                w.causal, q_index=rows)
            assert_bf16_close(O64[b, h, rows], Or, f"{w.name} b={b} h={h} rows")
            if check_lse:
                assert_lse_close(LSE64[b, h, rows], LSEr, f"{w.name} b={b} h={h}")
    for b, h in full_heads:
        Or, LSEr, _ = oracle.attention_head(Q[b, h], K[b, h], V[b, h], w.scale, w.causal)
        assert_bf16_close(O64[b, h], Or, f"{w.name} b={b} h={h} full head")
        if check_lse:
            assert_lse_close(LSE64[b, h], LSEr, f"{w.name} b={b} h={h} full head")


@pytest.mark.parametrize("name", ["n4096_d64", "n4096_d64_causal"])
def test_workload_n4096_d64(name):
    w = inputs.WORKLOADS[name]
    _rows_check(w, rows_per_head=256, full_heads=((0, 0), (3, 15)))


def test_workload_n10000_ragged_tail():
    # 512 seeded rows per head, the tile boundaries and the ragged last tile (16 rows),
    # in all 32 heads; one head in full
    w = inputs.WORKLOADS["n10000_d128_causal"]
    _rows_check(w, rows_per_head=512, full_heads=((0, 31),))


def test_workload_n32768_large_logits():
    # 512 seeded rows per head plus the whole first and last 128-row tiles, all 8 heads,
    # with LSE (a full 32K x 32K head is left to the row checks: each row is exact alone)
    w = inputs.WORKLOADS["n32768_d128_causal_sigma3"]
    _rows_check(w, rows_per_head=512, full_heads=(), extra_rows=range(128))


def test_workload_n8192_forward():
    # the benchmark workload's forward: O and LSE on 256 seeded rows of every head and
    # one head in full
    w = inputs.WORKLOADS["n8192_d128_causal_bwd"]
    _rows_check(w, rows_per_head=256, full_heads=((1, 7),))


def test_deterministic_and_in_bounds():
    """Two runs give identical bits, and nothing is written outside O and LSE."""
    B, H, N, d = 2, 8, 1500, 128
    ins = inputs.make_inputs(B, H, N, d, seed=5)
    q, k, v = (ins[n].cuda() for n in ("Q", "K", "V"))
    guard = 4096
    obuf = torch.full((2 * guard + B * H * N * d,), 7.0, device="cuda", dtype=torch.bfloat16)
    lbuf = torch.full((2 * guard + B * H * N,), -3.0, device="cuda", dtype=torch.float32)
    O = obuf[guard:guard + B * H * N * d].view(B, H, N, d)
    LSE = lbuf[guard:guard + B * H * N].view(B, H, N)
    outs = []
    for _ in range(2):
        binding.fwd(q, k, v, causal=True, O=O, LSE=LSE)
        binding.check_device_error()
        outs.append((O.clone(), LSE.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    for buf, val in ((obuf, 7.0), (lbuf, -3.0)):
        assert bool((buf[:guard] == val).all()) and bool((buf[-guard:] == val).all())


def test_identical_keys_give_mean_of_values():
    """All keys equal -> every visible key gets the same weight (a closed form)."""
    B, H, N, d = 1, 2, 700, 64
    ins = inputs.make_inputs(B, H, N, d, seed=9)
    k = ins["K"][:, :, :1].expand(B, H, N, d).contiguous()
    q, v = ins["Q"].cuda(), ins["V"].cuda()
    O, _ = binding.fwd(q, k.cuda(), v, causal=False)
    ref = to64(ins["V"]).mean(axis=2, keepdims=True)
    assert_bf16_close(to64(O), np.broadcast_to(ref, O.shape), "non-causal mean")
    O, _ = binding.fwd(q, k.cuda(), v, causal=True)
    ref = np.cumsum(to64(ins["V"]), axis=2) / np.arange(1, N + 1)[None, None, :, None]
    assert_bf16_close(to64(O), ref, "causal prefix mean")


def test_empty_and_lse_optional():
    q = torch.zeros((1, 1, 0, 64), device="cuda", dtype=torch.bfloat16)
    O, LSE = binding.fwd(q, q, q)
    assert O.shape == (1, 1, 0, 64)
    ins = inputs.make_inputs(1, 2, 333, 128, seed=3)
    q, k, v = (ins[n].cuda() for n in ("Q", "K", "V"))
    O1, LSE1 = binding.fwd(q, k, v, causal=True)
    O2, LSE2 = binding.fwd(q, k, v, causal=True, want_lse=False)
    assert LSE2 is None and torch.equal(O1, O2)


def test_trace_events_bracket_each_kernel():
    """fa_trace_events: one boundary before and after the forward kernel, four around the
    backward's three kernels, all in stream order."""
    ins = inputs.make_inputs(1, 4, 2048, 128, seed=21, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    with binding.trace_kernels(ev[0:2]):
        O, LSE = binding.fwd(q, k, v, causal=True)
    with binding.trace_kernels(ev[2:6]):
        binding.bwd(q, k, v, O, do, LSE, causal=True)
    torch.cuda.synchronize()
    spans = [ev[0].elapsed_time(ev[1])] + [ev[i].elapsed_time(ev[i + 1]) for i in range(2, 5)]
    assert all(t > 0 for t in spans), spans
    # outside the context nothing is recorded any more
    before = ev[1].elapsed_time(ev[2])
    binding.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert ev[1].elapsed_time(ev[2]) == before

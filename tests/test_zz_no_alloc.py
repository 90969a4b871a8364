"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Some callers have no allocator to draw a workspace from (a plugin host that hands over
only tensors, a framework step whose memory plan is fixed, a loop that must not enter
cudaMalloc).  fa_bwd_noalloc serves them from a fixed scratch array inside the library.
These tests call it through the C ABI and hold it to what fa_bwd (caller-provided
workspace) gives on the same inputs, over consecutive calls of different sizes, since
every call reuses the same scratch.

The file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_64_b200 import binding, inputs
from parity import assert_bf16_close, to64


def _problem(B, H, N, d, causal, seed):
    ins = inputs.make_inputs(B, H, N, d, seed=seed, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = binding.fwd(q, k, v, causal=causal)
    return q, k, v, do, O, LSE


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_on_consecutive_calls():
    cases = [(2, 4, 1000, 128, True, 11), (1, 3, 513, 64, False, 12), (2, 4, 1000, 128, True, 11)]
    for B, H, N, d, causal, seed in cases:
        q, k, v, do, O, LSE = _problem(B, H, N, d, causal, seed)
        ref = binding.bwd(q, k, v, O, do, LSE, causal=causal)
        outs = [torch.full_like(q, float("nan")) for _ in range(3)]
        got = binding.bwd_noalloc(q, k, v, O, do, LSE, causal=causal, dQ=outs[0], dK=outs[1],
                                  dV=outs[2])
        binding.check_device_error()
        for g, r, name in zip(got, ref, ("dQ", "dK", "dV")):
            assert_bf16_close(to64(g), to64(r), f"noalloc {name} N={N} d={d} causal={causal}")
            assert torch.equal(g, r), f"noalloc {name} differs from fa_bwd bitwise"


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = binding.lib()
    cap = int(lib.fa_bwd_noalloc_max_scratch_bytes())
    assert cap == 8 << 20
    A = 0x100000
    args = [A + i * 0x100000 for i in range(9)]
    # 2^20 padded rows fit exactly; one more 128-row tile does not
    rows_ok = (1 << 20) // 128 * 128
    assert binding.workspace_bytes(1, 1, rows_ok, 128) == cap
    st = lib.fa_bwd_noalloc(*args, 1, 1, rows_ok + 1, 128, 0.1, 1, None)
    assert st == binding.FA_ERR_INVALID_ARG
    msg = lib.fa_last_error_message().decode()
    assert "scratch" in msg and str(cap) in msg
    st = lib.fa_bwd_noalloc(*args, 1, 16, 8192 * 8 + 1, 128, 0.1, 1, None)
    assert st == binding.FA_ERR_INVALID_ARG
    # an empty problem needs nothing and is accepted without touching a device
    assert lib.fa_bwd_noalloc(*args, 0, 1, 64, 128, 0.1, 1, None) == binding.FA_OK

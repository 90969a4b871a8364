"""Keys that no query sees have exactly zero gradients.

dK_j = scale * sum_i dS_ij q_i and dV_j = sum_i P_ij dO_i run over the queries that see
key j; with none, both are empty sums.  The backward calls write those zeros: for a
sequence of a batch with keys but no queries, and for a whole call with keys and no
query rows (where the backward kernels have no query tile to run over).  Rows past a
sequence's key length stay untouched.  Every output starts as a sentinel.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_64_b200 import binding, inputs

pytestmark = pytest.mark.gpu

SENTINEL = 7.0
DTYPES = [torch.bfloat16, torch.float32]


def _keys(B, H, Nk, d, dtype, seed):
    b = inputs.make_inputs(B, H, Nk, d, seed=seed, dtype=dtype)
    return b["K"].cuda(), b["V"].cuda()


def _no_queries(B, H, d, dtype):
    q = torch.empty(B, H, 0, d, device="cuda", dtype=dtype)
    return q, torch.empty_like(q), torch.empty_like(q), torch.empty(B, H, 0, device="cuda")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", DTYPES)
def test_dense_call_without_queries(dtype, causal):
    B, H, Nk, d = 2, 3, 300, 64
    k, v = _keys(B, H, Nk, d, dtype, seed=5)
    q, O, do, LSE = _no_queries(B, H, d, dtype)
    dK, dV = torch.full_like(k, SENTINEL), torch.full_like(v, SENTINEL)
    dQ, _, _ = binding.bwd(q, k, v, O, do, LSE, causal=causal, dK=dK, dV=dV)
    binding.check_device_error()
    assert dQ.numel() == 0
    assert bool((dK == 0).all()) and bool((dV == 0).all())


@pytest.mark.parametrize("dtype", DTYPES)
def test_padded_call_without_queries(dtype):
    B, H, Nk, d = 3, 2, 260, 128
    lk = [260, 0, 17]
    k, v = _keys(B, H, Nk, d, dtype, seed=6)
    q, O, do, LSE = _no_queries(B, H, d, dtype)
    sq = torch.zeros(B, dtype=torch.int32, device="cuda")
    sk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    dK, dV = torch.full_like(k, SENTINEL), torch.full_like(v, SENTINEL)
    binding.bwd_varlen(q, k, v, O, do, LSE, sq, sk, dK=dK, dV=dV)
    binding.check_device_error()
    for b, n in enumerate(lk):
        for g in (dK, dV):
            assert bool((g[b, :, :n] == 0).all()), f"sequence {b}: key rows not zeroed"
            assert bool((g[b, :, n:] == SENTINEL).all()), f"sequence {b}: padding written"


@pytest.mark.parametrize("dtype", DTYPES)
def test_packed_call_without_query_tokens(dtype):
    H, d = 2, 64
    lk = [100, 0, 29]
    tk = sum(lk)
    x = inputs.make_inputs(1, H, tk, d, seed=7, dtype=dtype)
    k, v = (x[n][0].transpose(0, 1).contiguous().cuda() for n in ("K", "V"))
    q = torch.empty(0, H, d, device="cuda", dtype=dtype)
    O, do = torch.empty_like(q), torch.empty_like(q)
    LSE = torch.empty(H, 0, device="cuda")
    cq = torch.zeros(len(lk) + 1, dtype=torch.int32, device="cuda")
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32, device="cuda")
    dK, dV = torch.full_like(k, SENTINEL), torch.full_like(v, SENTINEL)
    binding.bwd_packed(q, k, v, O, do, LSE, cq, ck, 0, max(lk), dK=dK, dV=dV)
    binding.check_device_error()
    assert bool((dK == 0).all()) and bool((dV == 0).all())


def test_keys_without_queries_stop_at_the_key_length():
    """A padded call whose queries exist for some sequences only: the sequence without
    queries gets zeros in its key rows and nothing past them (bf16 path, several key
    tiles, so every key-tile unit of that sequence writes its zeros)."""
    B, H, Nq, Nk, d = 2, 2, 200, 700, 128
    a = inputs.make_inputs(B, H, Nq, d, seed=8, with_dO=True)
    k, v = _keys(B, H, Nk, d, torch.bfloat16, seed=9)
    q, do = a["Q"].cuda(), a["dO"].cuda()
    sq = torch.tensor([200, 0], dtype=torch.int32, device="cuda")
    sk = torch.tensor([500, 650], dtype=torch.int32, device="cuda")
    O, LSE = binding.fwd_varlen(q, k, v, sq, sk)
    dK, dV = torch.full_like(k, SENTINEL), torch.full_like(v, SENTINEL)
    binding.bwd_varlen(q, k, v, O, do, LSE, sq, sk, dK=dK, dV=dV)
    binding.check_device_error()
    for g in (dK, dV):
        assert bool((g[1, :, :650] == 0).all()) and bool((g[1, :, 650:] == SENTINEL).all())
        assert bool((g[0, :, 500:] == SENTINEL).all())
        assert bool(torch.isfinite(g[0, :, :500].float()).all())

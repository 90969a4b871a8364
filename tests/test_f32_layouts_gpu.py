"""Parity of the float32 path outside square problems: fewer (or more) queries than keys
(fa_fwd_f32_qk, fa_bwd_f32_qk), padded batches (fa_fwd_f32_varlen, fa_bwd_f32_varlen) and
packed batches (fa_fwd_f32_packed, fa_bwd_f32_packed), against the exact fp64 gradient
within the float32 tolerance.  The queries of a sequence are the last of its tokens
(causal masking aligned at the bottom right); rows past a sequence's lengths, and query
rows of a sequence without keys, must keep the values they had before the call."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, inputs
from parity import assert_f32_close, assert_lse_close, to64

pytestmark = pytest.mark.gpu

SENTINEL = 7.0


def _f32(B, H, N, d, seed, with_dO=False):
    return inputs.make_inputs(B, H, N, d, seed=seed, dtype=torch.float32, with_dO=with_dO)


def _check_head(Q, K, V, dO, O, LSE, grads, scale, causal, what):
    """One head of one sequence: O, LSE and (dQ, dK, dV) against the oracle."""
    nq, nk = Q.shape[0], K.shape[0]
    pos = oracle.chunk_positions(nq, nk) if causal else None
    rO, rL, _ = oracle.attention_head(Q, K, V, scale, causal, pos)
    assert_f32_close(O, rO, "O " + what)
    assert_lse_close(LSE, rL, "LSE " + what)
    ref = oracle.attention_bwd_head(Q, K, V, dO, scale, causal, q_index=pos)
    for k_, name in enumerate(("dQ", "dK", "dV")):
        assert_f32_close(grads[k_], ref[k_], f"{name} {what}")


# (Nq, Nk): ragged 32-row blocks on both sides, offsets Nk - Nq that are and are not
# multiples of 32, one query, and (non-causal only) more queries than keys
SHAPES = [(1, 5), (100, 300), (129, 200), (77, 77), (256, 1000), (200, 130)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nq,Nk", SHAPES)
def test_f32_qk(Nq, Nk, d, causal):
    if causal and Nq > Nk:
        pytest.skip("causal needs Nq <= Nk")
    a = _f32(1, 2, Nq, d, seed=4000 + Nq, with_dO=True)
    b = _f32(1, 2, Nk, d, seed=4100 + Nk)
    scale = d ** -0.5
    q, do = a["Q"].cuda(), a["dO"].cuda()
    k, v = b["K"].cuda(), b["V"].cuda()
    O, LSE = binding.fwd(q, k, v, scale=scale, causal=causal)
    grads = binding.bwd(q, k, v, O, do, LSE, scale=scale, causal=causal)
    binding.check_device_error()
    assert O.dtype == torch.float32 and all(g.dtype == torch.float32 for g in grads)
    for h in range(2):
        _check_head(to64(a["Q"][0, h]), to64(b["K"][0, h]), to64(b["V"][0, h]),
                    to64(a["dO"][0, h]), to64(O[0, h]), to64(LSE[0, h]),
                    [to64(g[0, h]) for g in grads], scale, causal,
                    f"f32 Nq={Nq} Nk={Nk} d={d} causal={causal}")


def test_f32_qk_equal_lengths_match_square_entry_points():
    """fa_fwd_f32_qk / fa_bwd_f32_qk with Nq == Nk are the square calls: same bits."""
    a = _f32(1, 2, 150, 64, seed=11, with_dO=True)
    q, k, v, do = (a[n].cuda() for n in ("Q", "K", "V", "dO"))
    O1, L1 = binding.fwd(q, k, v, causal=True)
    O2, L2 = torch.empty_like(O1), torch.empty_like(L1)
    stream = torch.cuda.current_stream().cuda_stream
    st = binding.lib().fa_fwd_f32_qk(q.data_ptr(), k.data_ptr(), v.data_ptr(), O2.data_ptr(),
                                     L2.data_ptr(), 1, 2, 150, 150, 64, 64 ** -0.5, 1, stream)
    assert st == binding.FA_OK
    g1 = binding.bwd(q, k, v, O1, do, L1, causal=True)
    g2 = [torch.empty_like(q) for _ in range(3)]
    ws = torch.empty(binding.workspace_bytes(1, 2, 150, 64), dtype=torch.uint8, device="cuda")
    st = binding.lib().fa_bwd_f32_qk(q.data_ptr(), k.data_ptr(), v.data_ptr(), O1.data_ptr(),
                                     do.data_ptr(), L1.data_ptr(), g2[0].data_ptr(),
                                     g2[1].data_ptr(), g2[2].data_ptr(), 1, 2, 150, 150, 64,
                                     64 ** -0.5, 1, ws.data_ptr(), ws.numel(), stream)
    assert st == binding.FA_OK
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    assert all(torch.equal(x, y) for x, y in zip(g1, g2))


VARLEN = [([100, 0, 33, 256], [300, 17, 33, 256], 256, 300),
          ([1, 64, 200], [5, 64, 0], 200, 64)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", range(len(VARLEN)))
def test_f32_varlen(case, d, causal):
    lq, lk, Nq, Nk = VARLEN[case]
    lq = list(lq)
    if causal:
        lq = [min(a, b) for a, b in zip(lq, lk)]
    if causal and Nq > Nk:
        Nk = Nq  # the padded shapes follow the causal rule too
    B, H, scale = len(lq), 2, d ** -0.5
    a = _f32(B, H, Nq, d, seed=4200 + case, with_dO=True)
    b = _f32(B, H, Nk, d, seed=4300 + case)
    q, do = a["Q"].cuda(), a["dO"].cuda()
    k, v = b["K"].cuda(), b["V"].cuda()
    sq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    sk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    O = torch.full_like(q, SENTINEL)
    LSE = torch.full((B, H, Nq), SENTINEL, device="cuda")
    binding.fwd_varlen(q, k, v, sq, sk, scale=scale, causal=causal, O=O, LSE=LSE)
    grads = [torch.full_like(t, SENTINEL) for t in (q, k, v)]
    binding.bwd_varlen(q, k, v, O, do, LSE, sq, sk, scale=scale, causal=causal, dQ=grads[0],
                       dK=grads[1], dV=grads[2])
    binding.check_device_error()
    for bi in range(B):
        nq, nk = lq[bi], lk[bi]
        for h in range(H):
            what = f"f32 varlen b={bi} h={h} lq={nq} lk={nk} d={d} causal={causal}"
            skipped = nq == 0 or nk == 0
            q_end = 0 if skipped else nq  # a skipped sequence writes no query row
            # keys without queries get zero gradients; a sequence without keys, none
            k_end = 0 if nk == 0 else nk
            assert bool((O[bi, h, q_end:] == SENTINEL).all()), "O past the rows " + what
            assert bool((LSE[bi, h, q_end:] == SENTINEL).all()), "LSE past the rows " + what
            assert bool((grads[0][bi, h, q_end:] == SENTINEL).all()), "dQ past " + what
            assert bool((grads[1][bi, h, k_end:] == SENTINEL).all()), "dK past " + what
            assert bool((grads[2][bi, h, k_end:] == SENTINEL).all()), "dV past " + what
            if nq == 0:
                assert bool((grads[1][bi, h, :nk] == 0).all()), "dK of unseen keys " + what
                assert bool((grads[2][bi, h, :nk] == 0).all()), "dV of unseen keys " + what
            if skipped:
                continue
            _check_head(to64(a["Q"][bi, h, :nq]), to64(b["K"][bi, h, :nk]),
                        to64(b["V"][bi, h, :nk]), to64(a["dO"][bi, h, :nq]),
                        to64(O[bi, h, :nq]), to64(LSE[bi, h, :nq]),
                        [to64(g[bi, h, :n]) for g, n in zip(grads, (nq, nk, nk))], scale,
                        causal, what)


def _packed(total, H, d, seed, with_dO=False):
    """[total, H, d] float32 tensors drawn like make_inputs (head-major, then packed)."""
    x = _f32(1, H, total, d, seed=seed, with_dO=with_dO)
    return {n: t[0].transpose(0, 1).contiguous() for n, t in x.items()}


def _cu(lengths):
    return torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32,
                        device="cuda")


PACKED = [([300, 1, 129, 0, 77, 256], [300, 1, 129, 5, 200, 256]),
          ([256, 100, 1, 200, 0], [640, 100, 33, 513, 0])]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", range(len(PACKED)))
def test_f32_packed(case, d, causal):
    lq, lk = PACKED[case]
    if causal:
        lq = [min(a, b) for a, b in zip(lq, lk)]
    H, scale = 2, d ** -0.5
    tq, tk = sum(lq), sum(lk)
    a = _packed(tq, H, d, seed=4400 + case, with_dO=True)
    b = _packed(tk, H, d, seed=4500 + case)
    q, do = a["Q"].cuda(), a["dO"].cuda()
    k, v = b["K"].cuda(), b["V"].cuda()
    cq, ck = _cu(lq), _cu(lk)
    O = torch.full_like(q, SENTINEL)
    LSE = torch.full((H, tq), SENTINEL, device="cuda")
    binding.fwd_packed(q, k, v, cq, ck, max(lq), max(lk), scale=scale, causal=causal, O=O,
                       LSE=LSE)
    dQ, dK, dV = (torch.full_like(t, SENTINEL) for t in (q, k, v))
    binding.bwd_packed(q, k, v, O, do, LSE, cq, ck, max(lq), max(lk), scale=scale,
                       causal=causal, dQ=dQ, dK=dK, dV=dV)
    binding.check_device_error()
    q0s, k0s = np.cumsum([0] + lq), np.cumsum([0] + lk)
    for s, (nq, nk) in enumerate(zip(lq, lk)):
        qs, ks = slice(q0s[s], q0s[s] + nq), slice(k0s[s], k0s[s] + nk)
        if nk == 0 or nq == 0:
            assert bool((O[qs] == SENTINEL).all()) and bool((dQ[qs] == SENTINEL).all())
            # keys no query sees: exactly zero gradients
            assert bool((dK[ks] == 0).all()) and bool((dV[ks] == 0).all())
            continue
        for h in range(H):
            _check_head(to64(a["Q"][qs, h]), to64(b["K"][ks, h]), to64(b["V"][ks, h]),
                        to64(a["dO"][qs, h]), to64(O[qs, h]), to64(LSE[h, qs]),
                        [to64(g[sl, h]) for g, sl in ((dQ, qs), (dK, ks), (dV, ks))], scale,
                        causal, f"f32 packed seq {s} h={h} lq={nq} lk={nk} d={d} "
                                f"causal={causal}")


def test_f32_varlen_bad_length_is_reported():
    """A length above the padded size skips that sequence and is reported as
    FA_ERR_INVALID_ARG by fa_check_device_error; the other sequences are computed."""
    a = _f32(2, 1, 64, 64, seed=5, with_dO=True)
    q, k, v = (a[n].cuda() for n in ("Q", "K", "V"))
    sq = torch.tensor([64, 65], dtype=torch.int32, device="cuda")
    sk = torch.tensor([64, 64], dtype=torch.int32, device="cuda")
    O = torch.full_like(q, SENTINEL)
    binding.fwd_varlen(q, k, v, sq, sk, causal=True, O=O)
    with pytest.raises(binding.FAError) as err:
        binding.check_device_error()
    assert err.value.status == binding.FA_ERR_INVALID_ARG
    assert bool((O[1] == SENTINEL).all())
    rO, _, _ = oracle.attention_head(to64(a["Q"][0, 0]), to64(a["K"][0, 0]),
                                     to64(a["V"][0, 0]), 64 ** -0.5, True)
    assert_f32_close(to64(O[0, 0]), rO, "f32 varlen sequence 0 beside a bad one")
    binding.check_device_error()  # the report cleared the error word

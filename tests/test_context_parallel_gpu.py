"""fa_merge and the context-parallel forward's blocks on one GPU, against the oracle.

fa_merge is checked on partial results the oracle computes over disjoint key sets: the
merged result must be attention over all of them.  ``blockwise_forward`` runs the ring's
blocks and merges with the library's kernels for every rank of an emulated ring (the
exchange itself needs several GPUs and is tested on CPU)."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, context_parallel as cp, inputs
from parity import assert_bf16_close, assert_lse_close, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
def test_merge_of_key_blocks_is_attention_over_all_keys(d):
    B, H, N, Nk = 2, 3, 200, 700
    a = inputs.make_inputs(B, H, N, d, seed=61)
    b = inputs.make_inputs(B, H, Nk, d, seed=62)
    Q, K, V = a["Q"], b["K"], b["V"]
    cuts = [0, 130, 131, 450, Nk]  # blocks of 130, 1, 319 and 250 keys
    scale = d ** -0.5
    O_acc = torch.full((B, H, N, d), float("nan"), device="cuda")  # ignored while empty
    L_acc = torch.full((B, H, N), float("-inf"), device="cuda")
    O_out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    parts = []
    for s0, s1 in zip(cuts, cuts[1:]):
        Op = np.empty((B, H, N, d))
        Lp = np.empty((B, H, N))
        for bb in range(B):
            for h in range(H):
                Op[bb, h], Lp[bb, h], _ = oracle.attention_head(
                    to64(Q[bb, h]), to64(K[bb, h, s0:s1]), to64(V[bb, h, s0:s1]), scale, False)
        parts.append((torch.from_numpy(Op).to(torch.bfloat16).cuda(),
                      torch.from_numpy(Lp).float().cuda()))
    # an empty block in the middle: LSE -inf and NaN values that must not leak
    parts.insert(2, (torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda"),
                     torch.full((B, H, N), float("-inf"), device="cuda")))
    for i, (Op, Lp) in enumerate(parts):
        binding.merge(O_acc, L_acc, Op, Lp, O_out=O_out if i == len(parts) - 1 else None)
    binding.check_device_error()
    for bb in range(B):
        for h in range(H):
            rO, rL, _ = oracle.attention_head(to64(Q[bb, h]), to64(K[bb, h]), to64(V[bb, h]),
                                              scale, False)
            assert_bf16_close(to64(O_out[bb, h]), rO, f"merged O b={bb} h={h}")
            assert_bf16_close(to64(O_acc[bb, h]), rO, f"float32 accumulator b={bb} h={h}")
            assert_lse_close(to64(L_acc[bb, h]), rL, f"merged LSE b={bb} h={h}")


def test_merge_of_two_empty_sides_stays_empty():
    O_acc = torch.full((1, 1, 4, 64), float("nan"), device="cuda")
    L_acc = torch.full((1, 1, 4), float("-inf"), device="cuda")
    Op = torch.full((1, 1, 4, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
    Lp = torch.full((1, 1, 4), float("-inf"), device="cuda")
    binding.merge(O_acc, L_acc, Op, Lp)
    torch.cuda.synchronize()
    assert bool((O_acc == 0).all()) and bool(torch.isinf(L_acc).all())


@pytest.mark.parametrize("causal", [False, True])
def test_blockwise_forward_every_rank(causal):
    """An emulated ring of 4 ranks with 384-token chunks (N = 1536): each rank's output,
    formed from its key blocks with fa_fwd and fa_merge, equals those rows of attention
    over the whole sequence."""
    W, B, H, L, d = 4, 1, 2, 384, 128
    ins = inputs.make_inputs(B, H, W * L, d, seed=63)
    q, k, v = (ins[n].cuda() for n in ("Q", "K", "V"))
    chunks = lambda t: [t[:, :, s * L:(s + 1) * L].contiguous() for s in range(W)]  # noqa: E731
    qs, ks, vs = chunks(q), chunks(k), chunks(v)
    scale = d ** -0.5
    refs = [oracle.attention_head(to64(ins["Q"][0, h]), to64(ins["K"][0, h]),
                                  to64(ins["V"][0, h]), scale, causal)[:2] for h in range(H)]
    for r in range(W):
        O, LSE = cp.blockwise_forward(qs[r], ks, vs, r, causal, scale=scale)
        binding.check_device_error()
        for h in range(H):
            sl = slice(r * L, (r + 1) * L)
            assert_bf16_close(to64(O[0, h]), refs[h][0][sl], f"rank {r} O h={h}")
            assert_lse_close(to64(LSE[0, h]), refs[h][1][sl], f"rank {r} LSE h={h}")


@pytest.mark.parametrize("causal", [False, True])
def test_blockwise_backward_every_rank(causal):
    """The emulated 4-rank ring's backward: block backwards with the global O and LSE,
    accumulated in float32 in the ring's order, give the gradients of attention over the
    whole sequence (with D formed from the bf16 output, as fa_bwd does)."""
    from parity import assert_bf16_close_scaled, assert_bwd_exact
    W, B, H, L, d = 4, 1, 2, 384, 128
    ins = inputs.make_inputs(B, H, W * L, d, seed=64, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    chunks = lambda t: [t[:, :, s * L:(s + 1) * L].contiguous() for s in range(W)]  # noqa: E731
    qs, ks, vs, dos = chunks(q), chunks(k), chunks(v), chunks(do)
    scale = d ** -0.5
    fw = [cp.blockwise_forward(qs[r], ks, vs, r, causal, scale=scale) for r in range(W)]
    Os, LSEs = [f[0] for f in fw], [f[1] for f in fw]
    dQs, dKs, dVs = cp.blockwise_backward(qs, ks, vs, Os, dos, LSEs, causal, scale=scale)
    binding.check_device_error()
    O_full = torch.cat(Os, dim=2)
    for h in range(H):
        args = [to64(ins[n][0, h]) for n in ("Q", "K", "V", "dO")]
        ref = oracle.attention_bwd_head(*args, scale, causal, O_given=to64(O_full[0, h]))
        exact = oracle.attention_bwd_head(*args, scale, causal)
        for k_, name, got in ((0, "dQ", dQs), (1, "dK", dKs), (2, "dV", dVs)):
            for r in range(W):
                sl = slice(r * L, (r + 1) * L)
                assert_bf16_close_scaled(to64(got[r][0, h]), ref[k_][sl],
                                         f"rank {r} {name} h={h}")
            # the whole sequence (1536 rows) against the exact gradient
            whole = np.concatenate([to64(got[r][0, h]) for r in range(W)])
            assert_bwd_exact(whole, exact[k_], f"ring {name} h={h} causal={causal}")


def test_accumulate():
    acc = torch.randn(1000, 8, device="cuda")
    part = torch.randn(1000, 8, device="cuda").to(torch.bfloat16)
    out = torch.empty(1000, 8, dtype=torch.bfloat16, device="cuda")
    ref = acc.double() + part.double()
    binding.accumulate(acc, part, out=out)
    torch.cuda.synchronize()
    assert torch.equal(acc, (ref).float())
    assert torch.equal(out, acc.to(torch.bfloat16))

"""Context-parallel forward, host side: which key block each rank attends to and how,
and the ring exchange, run with gloo ranks on CPU.  The attention of a block and the
merge are stand-ins here (the fp64 oracle per block and the merge's definition written
out in torch); the CUDA versions are checked on the GPU in test_context_parallel_gpu.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from exact_io_aware_64_b200 import context_parallel as cp


def test_block_kinds_and_ring_order():
    assert cp.ring_order(2, 4) == [2, 1, 0, 3]
    assert cp.ring_order(0, 3) == [0, 2, 1]
    assert cp.block_kind(2, 1, True) == "full"
    assert cp.block_kind(2, 2, True) == "causal"
    assert cp.block_kind(2, 3, True) is None
    assert all(cp.block_kind(1, s, False) == "full" for s in range(4))
    steps, last = cp._plan(1, 4, True)
    assert [k for _, k in steps] == ["causal", "full", None, None] and last == 1
    steps, last = cp._plan(3, 4, False)
    assert last == 3


def oracle_fwd(q, k, v, scale=None, causal=False):
    import oracle
    B, H, L, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    O = np.empty((B, H, L, v.shape[3]))
    LSE = np.empty((B, H, L))
    for b in range(B):
        for h in range(H):
            O[b, h], LSE[b, h], _ = oracle.attention_head(q[b, h].numpy(), k[b, h].numpy(),
                                                          v[b, h].numpy(), scale, causal)
    return torch.from_numpy(O), torch.from_numpy(LSE)


def torch_merge(O_acc, LSE_acc, O_part, LSE_part, O_out=None):
    """The merge written from its definition: weights exp(LSE - max) of the two key
    sets, an empty set (LSE -inf) weighing nothing."""
    la, lb = LSE_acc.double(), LSE_part.double()
    m = torch.maximum(la, lb)
    safe = torch.where(torch.isinf(m), torch.zeros_like(m), m)
    wa = torch.where(torch.isinf(la), torch.zeros_like(la), torch.exp(la - safe))
    wb = torch.where(torch.isinf(lb), torch.zeros_like(lb), torch.exp(lb - safe))
    s = wa + wb
    inv = torch.where(s > 0, 1.0 / s, torch.zeros_like(s))
    o = (torch.where(wa[..., None] > 0, wa[..., None] * O_acc.double(), torch.zeros_like(O_acc.double()))
         + wb[..., None] * O_part.double()) * inv[..., None]
    O_acc.copy_(o)
    LSE_acc.copy_(torch.where(s > 0, safe + torch.log(s), torch.full_like(s, float("-inf"))))
    if O_out is not None:
        O_out.copy_(o)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, causal, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    g = torch.Generator().manual_seed(11)
    B, H, L, d = 1, 2, 5, 3
    q, k, v = (torch.randn(B, H, world * L, d, generator=g, dtype=torch.float64)
               for _ in range(3))
    sl = slice(rank * L, (rank + 1) * L)
    O, LSE = cp.ring_forward(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                             v[:, :, sl].contiguous(), causal, scale=0.7, fwd=oracle_fwd,
                             merge=torch_merge)
    dist.destroy_process_group()
    out.put((rank, O.numpy(), LSE.numpy(), q.numpy(), k.numpy(), v.numpy()))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_forward_matches_full_attention(world, causal):
    import oracle
    port = _free_port()
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, q_)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted((q_.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    _, _, _, Q, K, V = results[0]
    L = Q.shape[2] // world
    for h in range(Q.shape[1]):
        rO, rL, _ = oracle.attention_head(Q[0, h], K[0, h], V[0, h], 0.7, causal)
        for rank, O, LSE, *_ in results:
            sl = slice(rank * L, (rank + 1) * L)
            # the accumulator is float32
            np.testing.assert_allclose(O[0, h], rO[sl], rtol=0, atol=1e-5)
            np.testing.assert_allclose(LSE[0, h], rL[sl], rtol=0, atol=1e-5)


def block_bwd_standin(q, k, v, O, dO, LSE, scale=None, causal=False):
    """One key block's share of the gradients with the global normalisers, float64,
    from the formulas: P = exp(S - LSE) on the block (0 where masked), dV = P^T dO,
    dS = P (dO V^T - rowsum(dO O)), dQ = scale dS K, dK = scale dS^T Q."""
    B, H, L, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    outs = [torch.empty_like(t, dtype=torch.float64) for t in (q, k, v)]
    for b in range(B):
        for h in range(H):
            Q, K, V = q[b, h].double(), k[b, h].double(), v[b, h].double()
            G, Oh, Lh = dO[b, h].double(), O[b, h].double(), LSE[b, h].double()
            P = torch.exp(scale * Q @ K.T - Lh[:, None])
            if causal:
                P = torch.tril(P)
            dS = P * (G @ V.T - (G * Oh).sum(1, keepdim=True))
            outs[0][b, h] = scale * dS @ K
            outs[1][b, h] = scale * dS.T @ Q
            outs[2][b, h] = P.T @ G
    return tuple(outs)


def add_standin(acc, part, out=None):
    acc += part.to(acc.dtype)
    if out is not None:
        out.copy_(acc)
    return acc


def _bwd_worker(rank, world, port, causal, out):
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    g = torch.Generator().manual_seed(12)
    B, H, L, d = 1, 2, 4, 3
    q, k, v, dO = (torch.randn(B, H, world * L, d, generator=g, dtype=torch.float64)
                   for _ in range(4))
    O, LSE = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), 0.6, causal)
    O, LSE = torch.from_numpy(O), torch.from_numpy(LSE)
    sl = slice(rank * L, (rank + 1) * L)
    c = lambda t: t[:, :, sl].contiguous()  # noqa: E731
    dQ, dK, dV = cp.ring_backward(c(q), c(k), c(v), c(O), c(dO), LSE[:, :, sl].contiguous(),
                                  causal, scale=0.6, bwd=block_bwd_standin,
                                  accumulate=add_standin)
    dist.destroy_process_group()
    out.put((rank, dQ.numpy(), dK.numpy(), dV.numpy(), q.numpy(), k.numpy(), v.numpy(),
             dO.numpy()))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_backward_matches_full_gradient(world, causal):
    import oracle
    port = _free_port()
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, causal, q_))
             for r in range(world)]
    for p in procs:
        p.start()
    results = sorted((q_.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    Q, K, V, G = results[0][4:]
    L = Q.shape[2] // world
    for h in range(Q.shape[1]):
        rQ, rK, rV, _ = oracle.attention_bwd_head(Q[0, h], K[0, h], V[0, h], G[0, h], 0.6,
                                                  causal)
        for rank, dQ, dK, dV, *_ in results:
            sl = slice(rank * L, (rank + 1) * L)
            # float32 accumulators
            np.testing.assert_allclose(dQ[0, h], rQ[sl], rtol=0, atol=1e-5)
            np.testing.assert_allclose(dK[0, h], rK[sl], rtol=0, atol=1e-5)
            np.testing.assert_allclose(dV[0, h], rV[sl], rtol=0, atol=1e-5)

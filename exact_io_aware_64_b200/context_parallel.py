"""Context-parallel attention: the sequence split across ranks, key/value blocks passed
around a ring, partial results merged (forward) and gradients accumulated (backward).

Rank r of W holds tokens [r*L, (r+1)*L) of every sequence: its queries Q_r and its keys
and values K_r, V_r ([B, H, L, d], bf16).  Over W steps each rank computes attention of
Q_r against one key block -- its own first, then the blocks of ranks r-1, r-2, ... as they
arrive -- and merges each partial result into a float32 accumulator (``fa_merge``: the
online-softmax rescale of "FlashAttention, simplified", "The trick", applied to whole
partial results).  Under causal masking a block from an earlier rank is visible in full,
the rank's own block needs the causal mask, and blocks from later ranks are skipped
(they are still forwarded).

The backward walks the same ring.  ``fa_bwd`` on one key block, given the global O and
LSE of the forward, yields exactly that block's share of the gradients (its
probabilities are the global ones restricted to the block), so each rank adds its dQ
share in float32 (``fa_accumulate``) and the block's dK and dV shares travel with the
block, in float32 accumulators, until every rank has added its part; one more hop takes
them home.

The exchange is torch.distributed point-to-point (NCCL between GPUs): at every step the
send of the current block to rank r+1 and the receive of the next one from rank r-1 are
posted before the step's attention, so the transfer overlaps it (in the backward the
gradient accumulators follow once the step has added to them).  ``blockwise_forward``
and ``blockwise_backward`` run the same blocks, merges and accumulations on one device
without the exchange; the exchange schedule is tested with gloo ranks on CPU.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch


def block_kind(q_rank: int, k_rank: int, causal: bool) -> Optional[str]:
    """How the queries of chunk ``q_rank`` see the keys of chunk ``k_rank``: "full",
    "causal" (the diagonal block: query i sees keys j <= i) or None (all hidden)."""
    if not causal or k_rank < q_rank:
        return "full"
    if k_rank == q_rank:
        return "causal"
    return None


def ring_order(rank: int, world: int) -> List[int]:
    """Key chunks in the order rank ``rank`` receives them: its own, then r-1, r-2, ..."""
    return [(rank - step) % world for step in range(world)]


def _default_fwd():
    from . import binding
    return binding.fwd


def _default_merge():
    from . import binding
    return binding.merge


def _default_bwd():
    from . import binding
    return binding.bwd


def _default_accumulate():
    from . import binding
    return binding.accumulate


def _accumulator(q: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    B, H, L, d = q.shape
    O = torch.zeros((B, H, L, d), dtype=torch.float32, device=q.device)
    LSE = torch.full((B, H, L), float("-inf"), dtype=torch.float32, device=q.device)
    return O, LSE


def _plan(q_rank: int, world: int, causal: bool):
    """(source chunk, kind) per step, and the last step that attends to its block (its
    merge writes the bf16 output)."""
    steps = [(src, block_kind(q_rank, src, causal)) for src in ring_order(q_rank, world)]
    last = max(i for i, (_, kind) in enumerate(steps) if kind is not None)
    return steps, last


def blockwise_forward(q: torch.Tensor, ks: List[torch.Tensor], vs: List[torch.Tensor],
                      q_rank: int, causal: bool, scale: Optional[float] = None,
                      fwd: Optional[Callable] = None, merge: Optional[Callable] = None):
    """Rank ``q_rank``'s result with every rank's key block at hand (ks[s], vs[s]): the
    ring's blocks and merges, in the ring's order, without the exchange.
    Returns (O [B, H, L, d] in q's dtype, LSE [B, H, L] float32)."""
    fwd = fwd or _default_fwd()
    merge = merge or _default_merge()
    O_acc, LSE_acc = _accumulator(q)
    O = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    steps, last = _plan(q_rank, len(ks), causal)
    for i, (src, kind) in enumerate(steps):
        if kind is None:
            continue
        O_p, LSE_p = fwd(q, ks[src], vs[src], scale=scale, causal=(kind == "causal"))
        merge(O_acc, LSE_acc, O_p, LSE_p, O_out=O if i == last else None)
    return O, LSE_acc


def ring_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool,
                 scale: Optional[float] = None, group=None, fwd: Optional[Callable] = None,
                 merge: Optional[Callable] = None):
    """This rank's attention output over the keys of all ranks in ``group`` (default:
    the whole job), exchanging key/value blocks around the ring.  Every rank calls it
    with its own chunk of the sequence (rank r: tokens [r*L, (r+1)*L)).
    Returns (O [B, H, L, d] in q's dtype, LSE [B, H, L] float32)."""
    import torch.distributed as dist
    fwd = fwd or _default_fwd()
    merge = merge or _default_merge()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    to_global = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    nxt, prv = to_global((rank + 1) % world), to_global((rank - 1) % world)
    O_acc, LSE_acc = _accumulator(q)
    O = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    steps, last = _plan(rank, world, causal)
    cur_k, cur_v = k.contiguous(), v.contiguous()
    for i, (src, kind) in enumerate(steps):
        reqs = []
        if i + 1 < world:
            nk, nv = torch.empty_like(cur_k), torch.empty_like(cur_v)
            reqs = [dist.isend(cur_k, nxt, group=group), dist.isend(cur_v, nxt, group=group),
                    dist.irecv(nk, prv, group=group), dist.irecv(nv, prv, group=group)]
        if kind is not None:
            O_p, LSE_p = fwd(q, cur_k, cur_v, scale=scale, causal=(kind == "causal"))
            merge(O_acc, LSE_acc, O_p, LSE_p, O_out=O if i == last else None)
        for rq in reqs:
            rq.wait()
        if i + 1 < world:
            cur_k, cur_v = nk, nv
    return O, LSE_acc


def _to_bf16(acc: torch.Tensor, like: torch.Tensor, accumulate: Callable) -> torch.Tensor:
    """acc rounded to like's dtype (a zero added through the accumulate call)."""
    out = torch.empty(acc.shape, dtype=like.dtype, device=acc.device)
    accumulate(acc, torch.zeros(acc.shape, dtype=like.dtype, device=acc.device), out=out)
    return out


def blockwise_backward(qs, ks, vs, Os, dOs, LSEs, causal: bool, scale: Optional[float] = None,
                       bwd: Optional[Callable] = None, accumulate: Optional[Callable] = None):
    """Every rank's gradients with all chunks at hand (lists indexed by rank): the ring's
    block backwards and accumulations in the ring's order (step by step, and within a
    step rank by rank, so each block's accumulators receive their shares in the order
    the ring delivers them), without the exchange.  Os and LSEs are the forward's global
    results.  Returns lists (dQ, dK, dV) indexed by rank, in the inputs' dtype."""
    bwd = bwd or _default_bwd()
    accumulate = accumulate or _default_accumulate()
    world = len(qs)
    dQ = [torch.zeros(q.shape, dtype=torch.float32, device=q.device) for q in qs]
    dK = [torch.zeros(k.shape, dtype=torch.float32, device=k.device) for k in ks]
    dV = [torch.zeros(v.shape, dtype=torch.float32, device=v.device) for v in vs]
    plans = [_plan(r, world, causal)[0] for r in range(world)]
    for i in range(world):
        for r in range(world):
            src, kind = plans[r][i]
            if kind is None:
                continue
            gq, gk, gv = bwd(qs[r], ks[src], vs[src], Os[r], dOs[r], LSEs[r], scale=scale,
                             causal=(kind == "causal"))
            accumulate(dQ[r], gq)
            accumulate(dK[src], gk)
            accumulate(dV[src], gv)
    return ([_to_bf16(a, qs[r], accumulate) for r, a in enumerate(dQ)],
            [_to_bf16(a, ks[r], accumulate) for r, a in enumerate(dK)],
            [_to_bf16(a, vs[r], accumulate) for r, a in enumerate(dV)])


def ring_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, O: torch.Tensor,
                  dO: torch.Tensor, LSE: torch.Tensor, causal: bool,
                  scale: Optional[float] = None, group=None, bwd: Optional[Callable] = None,
                  accumulate: Optional[Callable] = None):
    """This rank's (dQ, dK, dV) for ``ring_forward``'s output: O and LSE are what it
    returned, dO the gradient of O; every rank calls it with its own chunk."""
    import torch.distributed as dist
    bwd = bwd or _default_bwd()
    accumulate = accumulate or _default_accumulate()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    to_global = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    nxt, prv = to_global((rank + 1) % world), to_global((rank - 1) % world)
    steps, _ = _plan(rank, world, causal)
    dQ = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    cur_k, cur_v = k.contiguous(), v.contiguous()
    cur_dk = torch.zeros(k.shape, dtype=torch.float32, device=k.device)
    cur_dv = torch.zeros(v.shape, dtype=torch.float32, device=v.device)
    for i, (src, kind) in enumerate(steps):
        kv_reqs = []
        if i + 1 < world:
            nk, nv = torch.empty_like(cur_k), torch.empty_like(cur_v)
            kv_reqs = [dist.isend(cur_k, nxt, group=group), dist.isend(cur_v, nxt, group=group),
                       dist.irecv(nk, prv, group=group), dist.irecv(nv, prv, group=group)]
        if kind is not None:
            gq, gk, gv = bwd(q, cur_k, cur_v, O, dO, LSE, scale=scale,
                             causal=(kind == "causal"))
            accumulate(dQ, gq)
            accumulate(cur_dk, gk)
            accumulate(cur_dv, gv)
        # the block's gradient accumulators move on with it (after this step's share);
        # after the last step they go home: the block held now belongs to rank + 1
        ndk, ndv = torch.empty_like(cur_dk), torch.empty_like(cur_dv)
        g_reqs = [dist.isend(cur_dk, nxt, group=group), dist.isend(cur_dv, nxt, group=group),
                  dist.irecv(ndk, prv, group=group), dist.irecv(ndv, prv, group=group)]
        for rq in kv_reqs + g_reqs:
            rq.wait()
        cur_dk, cur_dv = ndk, ndv
        if i + 1 < world:
            cur_k, cur_v = nk, nv
    return _to_bf16(dQ, q, accumulate), _to_bf16(cur_dk, k, accumulate), \
        _to_bf16(cur_dv, v, accumulate)

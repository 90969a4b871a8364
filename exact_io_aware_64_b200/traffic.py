"""Work and memory-traffic arithmetic used for reporting (FLOPs, bytes, score sizes).

None of this runs on the data path; it turns shapes into the figures the benchmark
divides by.
"""
from __future__ import annotations


def score_entries(N: int) -> int:
    """Entries of one head's N x N score matrix ("FlashAttention" page, "A concrete
    example: 10,000 tokens")."""
    return N * N


def tile_entries(block: int) -> int:
    """Score entries held on chip for one block x block tile (same example)."""
    return block * block


def materialised_score_bytes(N: int, heads: int = 1, bytes_per_entry: int = 2,
                             passes: int = 1) -> int:
    """HBM bytes that standard attention moves for its score matrix.

    One pass is one write or one read of the N x N matrix for every head.  The
    "FlashAttention" page's example counts write S, read S, write P, read P: four passes.
    """
    return passes * bytes_per_entry * score_entries(N) * heads


def fwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """Credited forward FLOPs: two N x N x d matrix products, 4 B H N^2 d, halved when
    causal (only the lower triangle is needed)."""
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def bwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """Credited backward FLOPs: five N x N x d products (dV, dP, dQ, dK and the score
    recompute), 10 B H N^2 d, halved when causal."""
    f = 10.0 * B * H * N * N * d
    return f / 2 if causal else f


def bwd_executed_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """Tensor-core FLOPs the split backward actually executes: the dK/dV kernel's four
    products (S, dP, dV, dK) and the dQ kernel's three (S and dP again, then dQ),
    14 B H N^2 d, halved when causal.  The credited figure (bwd_flops) counts five."""
    f = 14.0 * B * H * N * N * d
    return f / 2 if causal else f


def visible_pairs(Nq: int, Nk: int, causal: bool) -> float:
    """(query, key) pairs the product covers per head: Nq * Nk, or, causal with the
    queries as the last Nq of the Nk tokens, Nq * Nk - Nq^2 / 2 (the same halving
    convention as the square case, where it gives N^2 / 2)."""
    return Nq * Nk - Nq * Nq / 2.0 if causal else float(Nq) * Nk


def fwd_flops_qk(B: int, H: int, Nq: int, Nk: int, d: int, causal: bool) -> float:
    """Credited forward FLOPs with Nq queries and Nk keys: 4 B H d per visible pair."""
    return 4.0 * B * H * d * visible_pairs(Nq, Nk, causal)


def bwd_flops_qk(B: int, H: int, Nq: int, Nk: int, d: int, causal: bool) -> float:
    """Credited backward FLOPs with Nq queries and Nk keys: 10 B H d per visible pair."""
    return 10.0 * B * H * d * visible_pairs(Nq, Nk, causal)


def fwd_compulsory_bytes(B: int, H: int, N: int, d: int, elem_bytes: int = 2,
                         lse: bool = True) -> int:
    """Bytes the forward must move at least once: read Q, K, V, write O (and the fp32
    LSE row statistics)."""
    b = 4 * B * H * N * d * elem_bytes
    if lse:
        b += 4 * B * H * N
    return b


def bwd_compulsory_bytes(B: int, H: int, N: int, d: int, elem_bytes: int = 2) -> int:
    """Bytes the backward must move at least once: read Q, K, V, O, dO, LSE; write dQ, dK,
    dV; write and read D once (fp32)."""
    return 8 * B * H * N * d * elem_bytes + 4 * B * H * N * 3


def bwd_prep_bytes(B: int, H: int, N: int, d: int, elem_bytes: int = 2) -> int:
    """Bytes of the backward's preparation pass: read O and dO and the LSE rows, write D
    and LSE*log2(e) for every row padded to whole 128-row tiles."""
    npad = (N + 127) // 128 * 128
    return 2 * B * H * N * d * elem_bytes + 4 * B * H * N + 8 * B * H * npad

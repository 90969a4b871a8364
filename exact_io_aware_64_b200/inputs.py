"""Seeded synthetic inputs and the named workloads.

This module draws random tensors and names shapes; it holds none of the attention
arithmetic, so both the CUDA path and the fp64 oracle can be fed from it.

Recipe: a ``torch.Generator`` seeded with ``seed`` draws float32 N(0, 1) tensors in the
fixed order Q, K, V, dO; Q and K are multiplied by ``sigma_qk``, V by ``sigma_v``; then
each is cast to the requested dtype.  The oracle reads the cast values upcast to float64,
so both sides see identical inputs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtype, masking and input distribution."""
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str          # "f32" or "bf16"
    causal: bool
    seed: int
    sigma_qk: float = 1.0
    sigma_v: float = 1.0
    backward: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The shapes of the pages' workloads: heads of 64 or 128 dims, contexts from a few
# hundred tokens to 32K, a length that is not a multiple of the 128-row tile
# ("FlashAttention" page, "A concrete example: 10,000 tokens"), and large logits that
# force frequent rescaling of the running max.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 1, 256, 64, "f32", False, seed=0),
    "n4096_d64": Workload("n4096_d64", 4, 16, 4096, 64, "bf16", False, seed=2),
    "n4096_d64_causal": Workload("n4096_d64_causal", 4, 16, 4096, 64, "bf16", True, seed=2),
    "n10000_d128_causal": Workload("n10000_d128_causal", 1, 32, 10000, 128, "bf16", True,
                                   seed=3),
    "n32768_d128_causal_sigma3": Workload("n32768_d128_causal_sigma3", 1, 8, 32768, 128,
                                          "bf16", True, seed=4, sigma_qk=3.0),
    "n8192_d128_causal_bwd": Workload("n8192_d128_causal_bwd", 2, 16, 8192, 128, "bf16",
                                      True, seed=5, backward=True),
}


def make_inputs(B: int, H: int, N: int, d: int, seed: int, dtype=torch.bfloat16,
                sigma_qk: float = 1.0, sigma_v: float = 1.0, with_dO: bool = False,
                device: str = "cpu") -> dict:
    """Draw Q, K, V (and dO) of shape [B, H, N, d] as described in the module docstring."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = (B, H, N, d)

    def draw(sigma: float) -> torch.Tensor:
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if sigma != 1.0:
            x.mul_(sigma)
        return x.to(dtype)

    out = {"Q": draw(sigma_qk), "K": draw(sigma_qk), "V": draw(sigma_v)}
    if with_dO:
        out["dO"] = draw(1.0)
    return out


def make_workload_inputs(w: Workload, device: str = "cpu") -> dict:
    return make_inputs(w.B, w.H, w.N, w.d, w.seed, w.torch_dtype, w.sigma_qk, w.sigma_v,
                       with_dO=w.backward, device=device)


def sample_rows(N: int, count: int, seed: int, tile: int = 128) -> list:
    """A seeded subset of query rows that always includes the rows around every tile
    boundary near the start and the whole last (possibly ragged) tile."""
    import numpy as np
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(count, N), replace=False).tolist())
    rows.update(r for r in (0, 1, tile - 1, tile, tile + 1, 2 * tile - 1, 2 * tile) if r < N)
    last_start = ((N - 1) // tile) * tile
    rows.update(range(last_start, N))
    return sorted(rows)

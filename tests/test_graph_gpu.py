"""The library's calls can be captured in a CUDA graph: they allocate nothing and never
synchronise, so a captured forward + backward replays to the same bits as direct calls."""
import pytest
import torch

from exact_io_aware_64_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def test_forward_backward_in_a_cuda_graph():
    B, H, N, d = 1, 4, 1000, 128
    ins = inputs.make_inputs(B, H, N, d, seed=21, with_dO=True)
    q, k, v, do = (ins[n].cuda() for n in ("Q", "K", "V", "dO"))
    O, LSE = torch.empty_like(q), torch.empty((B, H, N), device="cuda")
    dQ, dK, dV = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(binding.workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")

    def step():
        binding.fwd(q, k, v, causal=True, O=O, LSE=LSE)
        binding.bwd(q, k, v, O, do, LSE, causal=True, dQ=dQ, dK=dK, dV=dV, workspace=ws)

    step()  # the first call on a device looks up per-device facts; do it outside capture
    torch.cuda.synchronize()
    eager = [t.clone() for t in (O, LSE, dQ, dK, dV)]
    for t in (O, LSE, dQ, dK, dV):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    binding.check_device_error()
    for a, b in zip(eager, (O, LSE, dQ, dK, dV)):
        assert torch.equal(a, b)
    del g

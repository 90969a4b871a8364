"""Host-side logic: the traffic arithmetic against the pages' worked example, and the
seeded input generators."""
import json
import os

import torch

from exact_io_aware_64_b200 import inputs, traffic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_traffic_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "traffic_worked_examples.json")))
    assert traffic.score_entries(g["N"]) == g["score_entries"]
    assert traffic.materialised_score_bytes(g["N"], bytes_per_entry=g["bytes_per_entry"]) \
        == g["one_pass_bytes"]
    assert traffic.materialised_score_bytes(g["N"], bytes_per_entry=g["bytes_per_entry"],
                                            passes=g["passes"]) == g["four_pass_bytes"]
    assert traffic.tile_entries(g["tile"]) == g["tile_entries"]


def test_flop_convention():
    # 4 B H N^2 d forward, 10 B H N^2 d backward, halved when causal
    assert traffic.fwd_flops(1, 1, 2, 3, False) == 4 * 4 * 3
    assert traffic.fwd_flops(2, 16, 8192, 128, True) == 2 * 2 * 16 * 8192 ** 2 * 128
    assert traffic.bwd_flops(2, 16, 8192, 128, True) == 5 * 2 * 16 * 8192 ** 2 * 128
    # the split backward executes 7 products of 2*N^2*d per head (4 in dK/dV, 3 in dQ)
    assert traffic.bwd_executed_flops(2, 16, 8192, 128, True) == 7 * 2 * 16 * 8192 ** 2 * 128
    assert traffic.bwd_executed_flops(1, 1, 4, 2, False) == 7 * 2 * 4 ** 2 * 2


def test_flops_with_fewer_queries_than_keys():
    # equal lengths reduce to the square convention
    for causal in (False, True):
        assert traffic.fwd_flops_qk(2, 3, 256, 256, 64, causal) == \
            traffic.fwd_flops(2, 3, 256, 64, causal)
        assert traffic.bwd_flops_qk(2, 3, 256, 256, 64, causal) == \
            traffic.bwd_flops(2, 3, 256, 64, causal)
    # a chunk of 1024 queries at the end of 8192 keys: the rectangle before the chunk
    # plus half the square of the chunk
    assert traffic.visible_pairs(1024, 8192, True) == 1024 * 7168 + 1024 * 1024 / 2
    assert traffic.visible_pairs(1024, 8192, False) == 1024 * 8192


def test_inputs_are_seeded_and_ordered():
    a = inputs.make_inputs(1, 2, 9, 4, seed=7, with_dO=True)
    b = inputs.make_inputs(1, 2, 9, 4, seed=7, with_dO=True)
    for k in ("Q", "K", "V", "dO"):
        assert torch.equal(a[k], b[k])
        assert a[k].dtype == torch.bfloat16 and a[k].shape == (1, 2, 9, 4)
    # the draw order is Q, K, V, dO: dropping dO leaves the first three unchanged
    c = inputs.make_inputs(1, 2, 9, 4, seed=7, with_dO=False)
    for k in ("Q", "K", "V"):
        assert torch.equal(a[k], c[k])
    s = inputs.make_inputs(1, 2, 9, 4, seed=7, sigma_qk=3.0, dtype=torch.float32)
    f = inputs.make_inputs(1, 2, 9, 4, seed=7, dtype=torch.float32)
    assert torch.allclose(s["Q"], 3 * f["Q"]) and torch.equal(s["V"], f["V"])


def test_sample_rows_cover_tile_edges():
    rows = inputs.sample_rows(10000, 64, seed=1)
    assert rows == sorted(set(rows))
    for r in (0, 127, 128, 129, 9999, 9984):
        assert r in rows
    assert max(rows) < 10000


def test_workloads_have_expected_shapes():
    w = inputs.WORKLOADS
    assert (w["tiny_f32"].B, w["tiny_f32"].N, w["tiny_f32"].d) == (1, 256, 64)
    assert w["n10000_d128_causal"].N % 128 != 0
    assert w["n32768_d128_causal_sigma3"].sigma_qk == 3.0
    assert w["n8192_d128_causal_bwd"].backward

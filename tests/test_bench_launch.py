"""bench.py under torchrun, as the multi-GPU launch runs it, on CPU: the reference arm with
two ranks prints one JSON line from rank 0 and every rank exits 0."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_reference_arm_under_torchrun():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "3", "--ref-seconds", "0.5", "--workload", "n4096_d64"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"] == "n4096_d64"
    # the same config dict as the GPU arm of the same command line
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_cfg", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from exact_io_aware_64_b200 import inputs
    assert line["config"] == bench.config_dict(inputs.WORKLOADS["n4096_d64"], True, 2)


def test_per_kernel_rates():
    """The bench line's per-kernel figures: TFLOP/s for FLOP-credited kernels, GB/s for
    the bandwidth-bound preparation, executed TFLOP/s beside the credited figure."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    k = bench.add_rates({"fwd": {"ms": 0.5, "flops": 1e12},
                         "prep": {"ms": 0.04, "bytes": 1.4e8},
                         "dq": {"ms": 0.8, "flops": 2.75e11, "executed_flops": 8.25e11}})
    assert abs(k["fwd"]["tflops"] - 2000.0) < 1e-9 and "gbs" not in k["fwd"]
    assert abs(k["prep"]["gbs"] - 3500.0) < 1e-9 and "tflops" not in k["prep"]
    assert abs(k["dq"]["tflops"] - 343.75) < 1e-9
    assert abs(k["dq"]["executed_tflops"] - 1031.25) < 1e-9

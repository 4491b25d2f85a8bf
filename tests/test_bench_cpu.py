"""bench.py host logic without a GPU: the reference (CPU oracle) arm prints one
JSON line on rank 0, and under two ranks (gloo, as torchrun launches it) rank 1
exits cleanly without work."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARGS = ["--impl", "reference", "--workload", "fp32_n256_d64", "--steps", "2", "--warmup", "3"]


def _check_line(line):
    d = json.loads(line)
    assert d["impl"] == "reference"
    assert d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "fp32_n256_d64"
    return d


def test_reference_arm_single_process():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *ARGS], capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = _check_line(lines[0])
    assert d["n_gpus"] == 1


def test_reference_arm_two_ranks_gloo():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", "29517", os.path.join(ROOT, "bench.py"), *ARGS]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout
    d = _check_line(lines[0])
    assert d["n_gpus"] == 2


def test_gpu_arm_flags_are_validated():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "1"], capture_output=True,
                         text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "warmup" in out.stderr


def test_algorithmic_bytes_and_ridge_side():
    """The byte model behind the roofline entry, written out for the headline
    (bf16 B=2 H=16 N=8192 d=128): the forward moves Q, K, V in and O, LSE out;
    the backward kernel moves Q, K, V, dO, LSE, D in, dK, dV out and the fp32
    dQ accumulator in and out once.  The headline sits far above the ridge of
    the measured peaks, the narrow-band window workload below it."""
    sys.path.insert(0, ROOT)
    import bench
    from exact_io_aware_online_b200 import workloads as W
    w = W.WORKLOADS["bf16_causal_b2h16_n8192_d128"]
    t = 2 * 16 * 8192 * 128 * 2  # one bf16 [B, H, N, d] tensor
    rows = 2 * 16 * 8192
    assert bench.algorithmic_bytes(w, "fwd") == 4 * t + 4 * rows
    assert bench.algorithmic_bytes(w, "bwd") == 6 * t + 8 * rows + 8 * rows * 128
    pk, _ = bench.peaks()
    ridge = pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    f, b = W.flops(w)
    assert b / bench.algorithmic_bytes(w, "bwd") > 5 * ridge
    win = W.WORKLOADS["bf16_window128_h16_n32768_d64"]
    fw, bw = W.flops(win)
    assert bw / bench.algorithmic_bytes(win, "bwd") < ridge


def test_bench_rejects_bad_option_combinations():
    """Host-side option checks run before anything touches a GPU."""
    for extra in (["--warmup", "2"], ["--decode", "1", "--impl", "reference"], ["--packed", "10", "--impl", "reference"]):
        out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *extra], capture_output=True,
                             text=True, timeout=300, cwd=ROOT)
        assert out.returncode != 0
        assert any(w in out.stderr for w in ("warmup", "--decode", "--packed")), out.stderr[-500:]


def test_packed_workload_lengths_are_seeded_and_in_range():
    sys.path.insert(0, ROOT)
    import bench
    a, b = bench.packed_lengths(1000), bench.packed_lengths(1000)
    assert a == b and len(a) == 1000
    lo, hi = bench.PACKED_SHAPE["lo"], bench.PACKED_SHAPE["hi"]
    assert min(a) >= lo and max(a) <= hi and abs(sum(a) / len(a) - (lo + hi) / 2) < 10

"""The JSON line of bench.py's reference arm (the oracle on the host cores), on CPU.

The native arm needs a B200; the reference arm runs here, so its line is checked against the
keys and units the bench contract fixes, and against the native arm's workload description.
"""

import json
import os
import subprocess
import sys

ROOT = os.path.join(os.path.dirname(__file__), "..")


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=300, check=True)
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["scaling"] == "weak" and line["data"] == "synthetic" and line["vs_baseline"] is None
    cfg = line["config"]
    assert cfg["workload"] == "ttt_linear_B8_H12_T2048_b16" and (cfg["B"], cfg["H"], cfg["T"], cfg["chunk"]) == (8, 12,
                                                                                                              2048, 16)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_under_torchrun_prints_one_line(tmp_path):
    """Launched as the driver launches N > 1 (torch.distributed.run, two ranks on 127.0.0.1):
    rank 0 alone runs the oracle and prints the line; the other rank exits 0 without work."""
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    env = dict(os.environ, OMP_NUM_THREADS="1", TMPDIR=str(tmp_path))  # the launcher's scratch stays in tmp_path
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                          "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "0"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["config"]["parallelism"] == "replicas2"
    assert line["config"]["workload"] == "ttt_linear_B8_H12_T2048_b16"


def test_algorithmic_work_per_workload():
    """The flops and compulsory bytes the roofline divides by, per workload, from each
    workload's definition: In-Place 4·T·d·f flops (+ 2·T·d² for the fused target), Z, V̂ (or
    X0) read and O written once, W0 read and W written once in fp32; TTT-Linear 6·d²·T per
    (sequence, head) with queries (4·d²·T without), K, V (, Q) read and O written once in bf16,
    fp32 W0 and W, plus the losses and the cache with the gate."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from gen import workloads as wl
    MB = 1e6
    want = {
        "inplace_fp32_T2048_C512_d256_f512": (4 * 2048 * 256 * 512, 2048 * 512 * 4 + 2 * 2048 * 256 * 4 + 2 * 256 * 512 * 4),
        "ttt_linear_B8_H12_T2048_b16": (6 * 64 * 64 * 2048 * 96, 4 * 96 * 2048 * 64 * 2 + 2 * 96 * 64 * 64 * 4),
        "inplace_bf16_T32768_C1024_d2560_f9728": (4 * 32768 * 2560 * 9728,
                                                  32768 * 9728 * 2 + 2 * 32768 * 2560 * 2 + 2 * 2560 * 9728 * 4),
        "inplace_bf16_target_T131072_C1024_d2560_f9728": (
            4 * 131072 * 2560 * 9728 + 2 * 131072 * 2560 * 2560,
            131072 * 9728 * 2 + 2 * 131072 * 2560 * 2 + 2 * 2560 * 9728 * 4 + 2560 * 2560 * 2 + 2560 * 3 * 4),
        "srttt_gate_B4_H16_T8192_b16": (4 * 64 * 64 * 8192 * 64,
                                        2 * 64 * 8192 * 64 * 2 + 2 * 64 * 64 * 64 * 4 + 64 * 8192 * 4 + 64 * (256 * 3 + 2) * 4),
    }
    for name, (flops, byts) in want.items():
        w = bench.work(wl.WORKLOADS[name])
        assert w["flops"] == flops and w["bytes"] == byts, name
    # The figures quoted for the workloads: 4.83 GFLOP / 103.8 MB and 3.264 TFLOP / 1.17 GB.
    assert round(bench.work(wl.LINEAR_GD)["bytes"] / MB, 1) == 103.8
    assert round(bench.work(wl.INPLACE_4B)["flops"] / 1e12, 3) == 3.264

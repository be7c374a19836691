"""The N > 1 path of the benchmark on CPU: two ranks over gloo.

The attention path shards by heads with no data-path collective (each GPU
runs an independent replica), so what a multi-GPU run adds is host logic:
the ranks' environment, the max-over-ranks reduction of the timed region
and the whole-job aggregate, and that rank 0 alone prints the JSON line.
These tests run that logic as two real processes with the gloo backend.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


RANK_SCRIPT = r"""
import json, sys
from datetime import timedelta
import torch.distributed as dist
import bench
ws, rank, local = bench.dist_env()
dist.init_process_group("gloo", timeout=timedelta(seconds=60))
# rank r timed (r + 1) * 10 ms; the job's time is the slowest rank's
ms = bench.max_over_ranks(10.0 * (rank + 1), ws, "cpu")
v = bench.whole_job_tflops(ws, 2e12, ms)
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "ws": ws, "local": local, "ms": ms, "tflops": v}))
"""


def test_max_over_ranks_and_whole_job_value_with_two_gloo_ranks():
    port = free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", RANK_SCRIPT], cwd=ROOT, env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=240)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for r, o in enumerate(outs):
        assert (o["rank"], o["ws"], o["local"]) == (r, 2, r)
        assert o["ms"] == 20.0                       # the slower rank's time on both
        assert abs(o["tflops"] - 2 * 2e12 / 20e-3 / 1e12) < 1e-9   # both ranks' work


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_tflops(1, 1e12, 1000.0) == 1.0
    assert bench.dist_env() == (int(os.environ.get("WORLD_SIZE", "1")),
                                int(os.environ.get("RANK", "0")),
                                int(os.environ.get("LOCAL_RANK", "0")))


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", "fp32_small", "--steps", "1", "--warmup", "0", "--gpus",
           "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, OMP_NUM_THREADS="1"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0


def test_reference_arm_json_contract_on_one_rank():
    # one short step per workload kind (dense, FP8, decode); keys of the line
    for wl in ("fp32_small", "fp8_causal_d128", "decode_d128"):
        r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", wl,
                            "--steps", "1", "--warmup", "0"], cwd=ROOT, capture_output=True,
                           text=True, timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
        assert len(lines) == 1
        line = json.loads(lines[0])
        for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                    "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                    "impl", "cpu_baseline", "e2e"):
            assert key in line, (wl, key)
        assert line["impl"] == "reference" and line["n_gpus"] == 1
        assert line["config"]["workload"].startswith(wl)
        assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                               "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
        assert line["cpu_baseline"]["value"] == line["value"]
        assert line["cpu_baseline"]["cores"] >= 1

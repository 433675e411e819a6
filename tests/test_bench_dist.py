"""The benchmark's multi-rank plumbing on CPU: two `gloo` ranks, launched the way
torchrun would (RANK / WORLD_SIZE / MASTER_* in the environment). The timed
value must be the slowest rank's time and the sum of all ranks' units, and
non-zero ranks of the reference arm must leave without doing any work."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["ROOT"])
import bench
rank, world, local, dist = bench.dist_setup(2)
assert (rank, world) == (int(os.environ["RANK"]), 2) and dist is not None
# rank r reports elapsed 10 + 5r ms and 3 + r units
t, u = bench.aggregate(10.0 + 5.0 * rank, 3.0 + rank, dist)
print(json.dumps({"rank": rank, "t": t, "u": u}), flush=True)
dist.barrier()
dist.destroy_process_group()
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(code: str, extra_args=()):
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, ROOT=ROOT, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", code, *extra_args], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=240)
        except subprocess.TimeoutExpired:
            p.kill()
            out, err = p.communicate()
        outs.append((p.returncode, out, err))
    return outs


def test_aggregate_is_max_time_and_sum_of_units():
    outs = _launch(_WORKER)
    for rc, out, err in outs:
        assert rc == 0, err[-2000:]
    res = [json.loads(o.strip().splitlines()[-1]) for _, o, _ in outs]
    for r in res:
        assert r["t"] == 15.0   # the slower rank's time
        assert r["u"] == 7.0    # all ranks' units


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK") if k in os.environ}
    try:
        assert bench.dist_setup(1) == (0, 1, 0, None)
        assert bench.aggregate(12.5, 4.0, None) == (12.5, 4.0)
    finally:
        os.environ.update(env)


_REF_WORKER = r"""
import os, sys
sys.path.insert(0, os.environ["ROOT"])
import bench
if os.environ["RANK"] != "0":
    bench.run_reference(bench.parse_args(["--impl", "reference", "--gpus", "2"]))
    # a non-zero rank must return without loading the oracle or building weights
    assert "oracle" not in sys.modules
    print("rank1-done", flush=True)
else:
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    dist.destroy_process_group()
    print("rank0-done", flush=True)
"""


def test_reference_arm_other_ranks_exit_without_work():
    outs = _launch(_REF_WORKER)
    for rc, out, err in outs:
        assert rc == 0, err[-2000:]
    assert "rank1-done" in outs[1][1] and "rank0-done" in outs[0][1]


def test_reference_arm_prints_the_contract_line():
    """One process, no GPU: `bench.py --impl reference` times the CPU oracle on the
    benchmark's workload and prints one JSON line with the fields the benchmark
    contract names (the reference arm's value is the oracle's tokens/s)."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert "workload" in line["config"]
    assert line["dtype"] == "f32" and "fp32" in line["arithmetic"]  # the oracle computes in fp32

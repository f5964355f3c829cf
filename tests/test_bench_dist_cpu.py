"""bench.py's host logic on CPU.  Its multi-rank plumbing (gloo, world size 2), the path that
`bench.py --gpus N` takes under torch.distributed.run: every rank joins the
group, the timing is the maximum over ranks, the ranks meet at the barrier,
and the whole-job value counts every rank's work over the slowest rank's time.
The reference arm, launched the same way, prints one line from rank 0 only.
And the closed-form pair count behind the exact-mask figure."""

import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, sys
sys.path.insert(0, {root!r})
import torch.distributed as dist
import bench
world, rank, local = bench.dist_setup(None, backend="gloo")
t_ms = [3.0, 5.0][rank]  # this rank's own total time
m = bench.max_over_ranks(t_ms, world)
bench.barrier(world)
v = bench.whole_job_tflops(world, 10, 2e12, m)
json.dump({{"rank": rank, "world": world, "max": m, "value": v}}, open({out!r} % rank, "w"))
dist.destroy_process_group()
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(**kw):
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", CUDA_VISIBLE_DEVICES="")
    env.update({k: str(v) for k, v in kw.items()})
    return env


def test_two_gloo_ranks_take_the_max_and_count_both_ranks_work(tmp_path):
    out = str(tmp_path / "rank%d.json")
    port = _free_port()
    code = WORKER.format(root=ROOT, out=out)
    procs = [subprocess.Popen([sys.executable, "-c", code], cwd=ROOT,
                              env=_env(RANK=r, LOCAL_RANK=r, WORLD_SIZE=2, MASTER_PORT=port))
             for r in range(2)]
    try:
        for p in procs:
            assert p.wait(timeout=180) == 0
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    res = [json.load(open(out % r)) for r in range(2)]
    assert [x["world"] for x in res] == [2, 2]
    assert all(x["max"] == 5.0 for x in res)          # the slower rank's time, on both ranks
    expect = 2 * 10 * 2e12 / 5e-3 / 1e12              # both ranks' work over the max time
    assert all(abs(x["value"] - expect) < 1e-9 * expect for x in res)


def test_reference_arm_under_torchrun_prints_from_rank_zero_only():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1", "--small"]
    r = subprocess.run(cmd, cwd=ROOT, env=_env(), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_exact_mask_pair_count_matches_the_oracle_predicate():
    """bench.window_pairs (the closed form behind exact_mask_tflops) against a
    count of the oracle's allowed(i, j) on small windows, square and
    bottom-right rectangular, including the plain causal W = 0."""
    import types

    import numpy as np

    import bench
    import oracle
    for Sq, Skv, W in [(300, 300, 64), (200, 500, 128), (500, 200, 64), (257, 257, 0), (64, 640, 700)]:
        wl = types.SimpleNamespace(mask={"window": W}, Sq=Sq, Skv=Skv, B=2, H=3)
        allowed = oracle.allowed_rows(oracle.MaskDesc(window=W), 0, np.arange(Sq), Sq, Skv)
        assert bench.window_pairs(wl) == int(allowed.sum()) * 2 * 3, (Sq, Skv, W)
    assert bench.window_pairs(types.SimpleNamespace(mask={"window": 8, "dilation": 2})) is None

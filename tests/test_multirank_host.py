"""The bench's multi-rank path on CPU: two gloo ranks (world size 2) agree on
the slowest rank's time and on the whole-job throughput, and under torchrun
the oracle arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    env = dict(os.environ)
    env.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(port))
    return env


def test_two_gloo_ranks_take_the_slowest_time():
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, os.path.join(ROOT, "tests", "ranks_worker.py")],
                              env=_env(r, 2, port), stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
             for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["world"] == 2
        assert o["max_ms"] == 11.0  # rank 1's 11 ms, seen by both ranks
        assert abs(o["value"] - 2 * 100 / 0.011) < 1e-6


def test_reference_arm_runs_on_rank_zero_only():
    # a rank other than 0 leaves at once, without output and without work
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=_env(1, 2, _free_port()), capture_output=True, text=True,
                       timeout=120)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


def test_a_failing_extra_leg_is_reported_not_raised():
    import bench
    assert bench.leg(lambda: 1 / 0) == {"error": "ZeroDivisionError: division by zero"}
    assert bench.leg(lambda a, b: (a, b), 1, 2) == (1, 2)

"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks, one process
each, as torchrun launches them.  The hot path shards with no exchange
(every (batch row, head) is independent), so the process group carries only
the barrier and the max of the timings; these tests check that plumbing,
the weak-scaling aggregate, that replicas draw different data, and that a
rank which leaves early makes the other fail with an error instead of
waiting for ever."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    try:
        import torch
        import bench
        from channel_decay_softmax_b200 import inputs as I

        w, r, _ = bench.dist_setup("gloo", timeout_s=10)
        assert (w, r) == (world, rank)
        if mode == "ok":
            bench.barrier(w)
            # rank-dependent device times: everyone reports the slowest
            ms = bench.max_over_ranks(1.0 + rank, w)
            value = bench.weak_scaling_value(100.0, ms, w)
            s = I.spec(2, B=1, T=16, seed=bench.rank_seed(2, r))
            x = I.training_inputs(s)
            q.put((rank, ms, value, float(x["q"].float().sum())))
            bench.barrier(w)
        else:  # rank 1 leaves before the barrier; rank 0 must get an error
            if rank == 1:
                q.put((rank, "left"))
                return
            try:
                bench.barrier(w)
                q.put((rank, "no error"))
            except Exception as e:  # the process group's timeout
                q.put((rank, "error: " + type(e).__name__))
        torch.distributed.destroy_process_group()
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, "exception: %r" % (e,)))


def _run(mode, world=2, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=timeout) for _ in range(world)]
    for p in procs:
        p.join(timeout=timeout)
        if p.is_alive():
            p.kill()
    return sorted(out, key=lambda t: t[0])


def test_two_gloo_ranks_barrier_max_and_weak_scaling():
    out = _run("ok")
    assert [o[0] for o in out] == [0, 1], out
    for rank, ms, value, _ in out:
        assert ms == 2.0                      # max over ranks of 1.0 and 2.0
        assert value == 2 * 100.0 / 2e-3      # all ranks' units / the slowest time
    # the replicas draw different inputs
    assert out[0][3] != out[1][3]


def test_rank_leaving_early_fails_the_others():
    out = _run("leave")
    assert out[1][1] == "left"
    assert out[0][1].startswith("error"), out


def test_reference_arm_under_torchrun_prints_one_line():
    """`bench.py --impl reference` launched as torchrun launches it for N > 1:
    rank 0 alone runs the oracle and prints the line, the other rank exits
    0 without work."""
    import json
    import subprocess

    env = dict(os.environ, WALL_REF_T="128")  # a small oracle sample
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_gpus_flag_launches_the_ranks_itself():
    """`bench.py --gpus 2` run directly (no torchrun, no WORLD_SIZE) starts
    the two ranks itself; the reference arm runs on the host cores, so the
    launch path runs here: one line, from rank 0, with n_gpus = 2."""
    import json
    import subprocess

    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["WALL_REF_T"] = "128"
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2


def test_gpus_flag_refuses_missing_devices():
    """Our arm with more ranks than visible devices stops before any work,
    saying why, instead of measuring fewer replicas."""
    import subprocess

    import torch
    if torch.cuda.device_count() >= 2:
        pytest.skip("two devices are visible here")
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2"],
                         capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert res.returncode == 2
    assert "needs 2 visible CUDA devices" in res.stderr

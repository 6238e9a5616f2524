"""The benchmark's multi-process plumbing on CPU (gloo, world size 2): the
layer runs as independent replicas, so the only cross-rank steps are the
barriers around the timed region and the max over ranks of the time; rank 0
alone prints, and the reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(body: str, world: int = 2, timeout: float = 120.0):
    port = _free_port()
    script = textwrap.dedent(body)
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", script], cwd=ROOT, env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            p.kill()
            o, e = p.communicate()
        outs.append((p.returncode, o, e))
    return outs


def test_max_over_ranks_and_barrier_gloo():
    outs = _run_ranks("""
        import bench
        d = bench.Dist(backend="gloo", timeout_s=60)
        d.barrier()
        m = d.max(float(d.rank) * 3.0 + 1.0)     # rank 0: 1.0, rank 1: 4.0
        d.barrier()
        print("RESULT", d.rank, d.world, m)
        d.close()
    """)
    for rc, o, e in outs:
        assert rc == 0, e
    res = sorted(tuple(l.split()[1:]) for _, o, _ in outs for l in o.splitlines() if l.startswith("RESULT"))
    assert res == [("0", "2", "4.0"), ("1", "2", "4.0")]


def test_reference_arm_runs_on_rank_zero_only_gloo():
    # run_reference returns immediately on ranks other than 0 (no data, no work)
    outs = _run_ranks("""
        import argparse, bench
        d = bench.Dist(backend="gloo", timeout_s=60)
        called = []
        import mixture_experts_ffn_17_b200.workloads as wl
        orig = wl.make
        wl.make = lambda *a, **k: called.append(1) or (_ for _ in ()).throw(SystemExit(0))
        args = argparse.Namespace(workload="tiny", tokens=None, experts=None, ref_sample=1, warmup=0, steps=1,
                                  gpus=2)
        if d.rank != 0:
            bench.run_reference(args, d)
            print("RANK1_DONE", len(called))
        d.barrier()
        d.close()
    """)
    for rc, o, e in outs:
        assert rc == 0, e
    assert any("RANK1_DONE 0" in o for _, o, _ in outs)


def test_single_process_dist_is_a_no_op():
    import bench
    env_keep = {k: os.environ.pop(k, None) for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    try:
        d = bench.Dist()
        assert d.world == 1 and d.pg is None and d.max(2.5) == 2.5
        d.barrier()
        d.close()
    finally:
        for k, v in env_keep.items():
            if v is not None:
                os.environ[k] = v

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


def test_expert_parallel_split_and_all_reduce_gloo():
    # each rank slices the full weights with the package's shard_weights, runs
    # its share of the layer (here the oracle's per-rank forward stands in for
    # the GPU kernels), and all_reduce_partial sums the shares: every rank then
    # holds the whole layer's output
    outs = _run_ranks("""
        import datetime
        import numpy as np, torch, torch.distributed as dist
        import oracle
        from mixture_experts_ffn_17_b200 import expert_parallel as ep
        dist.init_process_group("gloo", init_method="env://", timeout=datetime.timedelta(seconds=60))
        r, W = dist.get_rank(), dist.get_world_size()
        rng = np.random.default_rng(7)            # same draws on every rank
        T, d, E, k, I, Is = 20, 16, 8, 3, 12, 8
        x = rng.standard_normal((T, d)); Wg = rng.standard_normal((E, d))
        W1, W3 = rng.standard_normal((E, d, I)) * .3, rng.standard_normal((E, d, I)) * .3
        W2 = rng.standard_normal((E, I, d)) * .3
        W1s, W3s, W2s = rng.standard_normal((d, Is)) * .3, rng.standard_normal((d, Is)) * .3, rng.standard_normal((Is, d)) * .3
        t = torch.from_numpy
        w = ep.shard_weights(t(W1), t(W3), t(W2), None, None, None, t(W1s), t(W3s), t(W2s), r, W)
        sl = ep.ep_slice(E, Is, r, W)
        y = t(oracle.moe_forward_ep_rank(x, Wg, w.W1.numpy(), w.W3.numpy(), w.W2.numpy(), w.W1s.numpy(),
                                         w.W3s.numpy(), w.W2s.numpy(), e_lo=sl.e_lo, k=k))
        ep.all_reduce_partial(y)
        y_full, *_ = oracle.moe_forward(x, Wg, W1, W3, W2, W1s, W3s, W2s, k=k)
        err = float(np.abs(y.numpy() - y_full).max() / np.sqrt(np.mean(y_full ** 2)))
        print("RESULT", r, sl.e_lo, sl.e_hi, sl.i_lo, sl.i_hi, err)
        dist.destroy_process_group()
    """)
    for rc, o, e in outs:
        assert rc == 0, e
    res = sorted(l.split()[1:] for _, o, _ in outs for l in o.splitlines() if l.startswith("RESULT"))
    assert [v[:5] for v in res] == [["0", "0", "4", "0", "4"], ["1", "4", "8", "4", "8"]]
    assert all(float(v[5]) <= 1e-12 for v in res)


def test_ep_slice_rejects_uneven_splits():
    from mixture_experts_ffn_17_b200 import expert_parallel as ep
    with pytest.raises(ValueError):
        ep.ep_slice(256, 2048, 0, 3)
    with pytest.raises(ValueError):
        ep.ep_slice(256, 2048, 2, 2)
    assert ep.ep_slice(256, 2048, 7, 8) == ep.EpSlice(224, 256, 1792, 2048)


def test_all_to_all_exchange_plumbing_gloo():
    # the all-to-all flavour's transport with host tensors, world size 2: the
    # per-expert counts, then variable-sized row blocks each way and back
    outs = _run_ranks("""
        import torch, torch.distributed as dist
        import bench
        from mixture_experts_ffn_17_b200 import expert_parallel as ep
        d = bench.Dist(backend="gloo", timeout_s=60)
        r, n, El = d.rank, d.world, 3
        g = torch.Generator().manual_seed(10 + r)
        counts = torch.randint(0, 4, (n, El), generator=g, dtype=torch.int32)   # rows this rank sends q, per expert
        rows = int(counts.sum())
        # row i of the send buffer encodes (source rank, i)
        send = torch.stack([torch.full((5,), 1000.0 * r + i) for i in range(rows)]) if rows else torch.zeros(0, 5)
        tr = ep.ProcessGroupTransport()
        recv_counts = tr.exchange_counts(counts)
        all_counts = [torch.zeros_like(counts) for _ in range(n)]
        dist.all_gather(all_counts, counts)
        assert torch.equal(recv_counts, torch.stack([all_counts[s][r] for s in range(n)]))
        ss, rs = ep._splits(counts), ep._splits(recv_counts)
        got, _ = tr.all_to_all(send, ss, rs)
        # block s of what arrives is source s's block for this rank, in its order
        at = 0
        for s in range(n):
            first = int(all_counts[s][:r].sum())
            for j in range(rs[s]):
                assert float(got[at + j, 0]) == 1000.0 * s + first + j
            at += rs[s]
        back, _ = tr.all_to_all(got, rs, ss)
        assert torch.equal(back, send)
        print("RESULT", r, rows, int(recv_counts.sum()))
        d.close()
    """)
    for rc, o, e in outs:
        assert rc == 0, e
    assert sum(1 for _, o, _ in outs for l in o.splitlines() if l.startswith("RESULT")) == 2

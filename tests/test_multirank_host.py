"""The multi-rank plumbing of bench.py on CPU: world size 2 over gloo (no GPU).
Ranks run independent replicas (different seeds, no data exchange), or split
one workload by KV-head group (no data exchange either); the only collectives
are the barrier and the max over ranks of the timed region; the reference arm
runs on rank 0 alone."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, ws: int, port: int, q):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from long_context_sparse_flash_b200 import workloads as wl
        w = wl.WORKLOADS["tiny"]
        # independent replicas: each rank draws its own inputs
        inp = wl.make_inputs(w, "cpu", seed=bench.replica_seed(w, rank), with_sparse=False)
        digest = float(inp["q"].float().sum())
        bench.barrier(ws)
        slowest = bench.max_over_ranks(10.0 + rank, ws)  # rank r "took" 10 + r ms
        value = bench.job_value(w.query_tokens, ws, 3, 3 * slowest)
        q.put((rank, digest, slowest, value))
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_over_gloo():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(ws))
    digests = [r[1] for r in res]
    assert digests[0] != digests[1]                     # different sequences per rank
    assert all(r[2] == 11.0 for r in res)               # every rank sees the slowest rank's time
    from long_context_sparse_flash_b200 import workloads as wl
    tokens = wl.WORKLOADS["tiny"].query_tokens
    assert all(abs(r[3] - tokens * ws / 11e-3) < 1e-6 * r[3] for r in res)  # all ranks' tokens / slowest time


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import argparse
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(workload="tiny", ref_rows=1, warmup=3, steps=2, gpus=2)
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""


def _failing_rank_main(rank: int, ws: int, port: int, q):
    """Rank 1 leaves between steps (an exception before the timing collective);
    rank 0 learns of it when its next collective ends with an error within the
    process group's short timeout, instead of waiting for good."""
    import datetime
    import time
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=5))
    import bench
    if rank == 1:
        q.put((rank, "left", 0.0))
        q.close()
        q.join_thread()  # the message is sent before the process vanishes
        os._exit(3)  # no destroy, no further collective: the rank is gone
    t0 = time.time()
    try:
        bench.max_over_ranks(10.0, ws)
        q.put((rank, "no error", time.time() - t0))
    except Exception as e:  # gloo reports the lost peer or the timeout
        q.put((rank, type(e).__name__, time.time() - t0))
    q.close()
    q.join_thread()
    os._exit(0)


def test_a_rank_that_leaves_ends_the_others_collective_with_an_error():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_failing_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert [p.exitcode for p in procs] == [0, 3]
    res = dict((r[0], r[1:]) for r in (q.get(timeout=5) for _ in range(ws)))
    assert res[1][0] == "left"
    assert res[0][0] != "no error", res
    assert res[0][1] < 60.0, res  # ended by the short timeout or the lost connection, not a hang


def _head_rank_main(rank: int, ws: int, port: int, q):
    """Rank r takes KV heads [r H_kv / ws, (r + 1) H_kv / ws) of ONE workload and
    their query heads.  The oracle run on that share alone reproduces exactly
    what the oracle computes for those heads on the whole workload: the split
    needs no exchange."""
    import datetime
    import numpy as np
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from long_context_sparse_flash_b200 import workloads as wl
        w = wl.custom("heads", n_q=160, q_pos0=200, h_q=8, h_kv=2, head_dim=64, window=32, topk=48, n_sparse=1,
                      seed=3)
        full = wl.make_inputs(w, "cpu", seed=w.seed)  # the same workload on every rank
        w_r, share = bench.head_shard(w, full, rank, ws)
        assert (w_r.h_q, w_r.h_kv) == (w.h_q // ws, w.h_kv // ws)
        assert all(t.is_contiguous() for t in (share["q"], share["k"], share["v"], *share["q_sparse"]))
        rows = np.array([0, 1, 31, 32, 100, 159])
        ts = w.q_pos0 + rows

        def run(qt, kt, vt, qs):
            qb = np.ascontiguousarray(wl.bf16_bits(qt[0][:, rows]).transpose(1, 0, 2))
            kb, vb = wl.bf16_bits(kt[0]), wl.bf16_bits(vt[0])
            r = oracle.full_select(qb, ts, kb, vb, window=w.window, topk=w.topk)
            qsb = np.ascontiguousarray(wl.bf16_bits(qs[0][:, rows]).transpose(1, 0, 2))
            return r, oracle.sparse(qsb, ts, kb, vb, r["idx"], window=w.window)

        part, part_sp = run(share["q"], share["k"], share["v"], share["q_sparse"][0])
        whole, whole_sp = run(full["q"], full["k"], full["v"], full["q_sparse"][0])
        h0, h1 = rank * w_r.h_q, (rank + 1) * w_r.h_q
        g0, g1 = rank * w_r.h_kv, (rank + 1) * w_r.h_kv
        same = (np.array_equal(part["out"], whole["out"][:, h0:h1]) and
                np.array_equal(part["lse"], whole["lse"][:, h0:h1]) and
                np.array_equal(part["idx"], whole["idx"][:, g0:g1]) and
                np.array_equal(part_sp, whole_sp[:, h0:h1]))
        # the shares cover every head once: gathered in rank order they are the whole
        got = [torch.empty_like(share["k"]) for _ in range(ws)]
        torch.distributed.all_gather(got, share["k"])
        covers = torch.equal(torch.cat(got, dim=1), full["k"])
        bench.barrier(ws)
        slowest = bench.max_over_ranks(10.0 + rank, ws)
        value = bench.job_value(w.query_tokens, 1, 3, 3 * slowest)  # one workload's tokens
        q.put((rank, same, covers, slowest, value))
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_split_one_workload_by_kv_head():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_head_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(ws))
    assert all(r[1] for r in res), "a share differs from the whole workload's heads"
    assert all(r[2] for r in res), "the shares do not cover the heads"
    assert all(r[3] == 11.0 for r in res)
    from long_context_sparse_flash_b200 import workloads as wl
    tokens = 160
    assert all(abs(r[4] - tokens / 11e-3) < 1e-6 * r[4] for r in res)  # one workload's tokens / slowest time


def test_head_split_rejects_an_uneven_split():
    import bench
    from long_context_sparse_flash_b200 import workloads as wl
    w = wl.custom("odd", n_q=8, h_q=6, h_kv=3, head_dim=64)
    inp = wl.make_inputs(w, "cpu", with_sparse=False)
    with pytest.raises(ValueError):
        bench.head_shard(w, inp, 0, 2)

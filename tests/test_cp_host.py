"""The multi-rank plumbing of context parallelism on CPU: world size 2 over gloo.
Each rank holds one slice; the step functions are replaced by stand-ins whose
outputs name the rank that made them, so the test sees that every exchange
stacks the slices' results in slice order, that the merges get the slices'
offsets and the combined LSE, and that every rank takes the same collective
steps (the kernels themselves are covered by the GPU tests)."""
import os
import socket
import sys
import types

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fake_ops(rank: int, ws: int, kv_offs, log):
    def attn_partial(q, k, v, *, kv_off, window, topk, q_pos0):
        assert kv_off == kv_offs[rank]
        return torch.full_like(q, float(rank + 1)), torch.full(q.shape[:3], float(rank))

    def combine(out_parts, lse_parts):
        assert out_parts.shape[0] == ws and lse_parts.shape[0] == ws
        for r in range(ws):  # slice order
            assert torch.all(out_parts[r] == out_parts[r].flatten()[0])
        log.append(("combine", [float(out_parts[r].flatten()[0]) for r in range(ws)]))
        return out_parts.sum(0), lse_parts.amax(0)

    def select_local(q, k, lse, *, kv_off, window, topk, q_pos0):
        assert torch.all(lse == ws - 1)  # the combined LSE, not this slice's
        B, Hq, nq, D = q.shape
        shape = (B, k.shape[1], nq, topk)
        return torch.full(shape, rank, dtype=torch.int32), torch.full(shape, rank / 10.0)

    def select_merge(idx_parts, score_parts, offs, *, shape):
        assert list(offs) == list(kv_offs)
        log.append(("merge", [int(idx_parts[r].flatten()[0]) for r in range(ws)],
                    [round(float(score_parts[r].flatten()[0]), 3) for r in range(ws)]))
        return idx_parts.sum(0)

    def sparse_partial(q, k, v, idx, *, kv_off, window, q_pos0):
        assert torch.all(idx == sum(range(ws)))  # the merged selection
        return torch.full_like(q, 10.0 * (rank + 1)), torch.full(q.shape[:3], float(rank))

    return types.SimpleNamespace(attn_partial=attn_partial, combine=combine, select_local=select_local,
                                 select_merge=select_merge, sparse_partial=sparse_partial)


def _rank_main(rank: int, ws: int, port: int, q):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        from long_context_sparse_flash_b200 import cp

        def gather(t):  # all_gather_into_tensor is NCCL-only; gloo stacks a list
            parts = [torch.empty_like(t) for _ in range(ws)]
            torch.distributed.all_gather(parts, t.contiguous())
            return torch.stack(parts)

        kv_len = 1000
        offs = cp.slice_offsets(kv_len, ws)
        ends = offs[1:] + [kv_len]
        B, Hq, Hkv, nq, D = 1, 4, 2, 8, 16
        k = torch.zeros(B, Hkv, ends[rank] - offs[rank], D, dtype=torch.bfloat16)
        log = []
        layer = cp.ContextParallel(k, k, rank=rank, kv_offs=offs, kv_len=kv_len, window=16, topk=32,
                                   gather=gather, ops=_fake_ops(rank, ws, offs, log))
        qq = torch.zeros(B, Hq, nq, D, dtype=torch.bfloat16)
        out, lse, idx = layer.full_attn_select(qq, q_pos0=kv_len - nq)
        sp = layer.sparse_attn(qq, idx, q_pos0=kv_len - nq)
        q.put((rank, float(out.flatten()[0]), float(lse.flatten()[0]), int(idx.flatten()[0]),
               float(sp.flatten()[0]), log))
    finally:
        torch.distributed.destroy_process_group()


def test_context_parallel_exchanges_over_two_ranks():
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
    for rank, out, lse, idx, sp, log in res:
        assert out == 1.0 + 2.0 and lse == 1.0 and idx == 0 + 1 and sp == 10.0 + 20.0
        # the same exchanges on every rank, each stacked in slice order
        assert log == [("combine", [1.0, 2.0]), ("merge", [0, 1], [0.0, 0.1]), ("combine", [10.0, 20.0])]

"""GPU parity of context parallelism: the KV cache cut into P contiguous
slices, each step run per slice through the C ABI and merged (all slices in
one process on one GPU: the steps and merges are the same ones each rank of a
multi-GPU run executes).  Checked against the fp64 oracle on the whole cache
and against the single-cache path."""
import numpy as np
import pytest
import torch

from long_context_sparse_flash_b200 import cp
from long_context_sparse_flash_b200 import native as nv
from long_context_sparse_flash_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from long_context_sparse_flash_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load()


def _run_cp(w, inp, n_slices):
    offs, ks, vs = cp.split_cache(inp["k"], inp["v"], n_slices)
    before = nv.hs2_launch_count()
    out, lse, idx, sp = cp.run_in_process(inp["q"], ks, vs, offs, kv_len=w.kv_len, window=w.window, topk=w.topk,
                                          q_pos0=w.q_pos0, q_sparse=inp["q_sparse"])
    torch.cuda.synchronize()
    assert nv.hs2_launch_count() > before
    return dict(out=out, lse=lse, idx=idx, sparse=sp)


CASES = [
    # name, n_slices, workload kwargs (None: the tiny workload)
    ("tiny_2", 2, None),
    ("tiny_3_uneven", 3, None),
    ("tiny_4", 4, None),
    ("chunk_after_slices", 3, dict(n_q=256, q_pos0=3000, kv_len=3256, h_q=16, h_kv=2, head_dim=128, window=128,
                                   topk=256)),
    ("g1_d64_slices_inside_chunk", 4, dict(n_q=700, q_pos0=100, h_q=2, h_kv=2, head_dim=64, window=32, topk=64)),
    ("one_slice", 1, dict(n_q=300, q_pos0=500, h_q=8, h_kv=2, head_dim=64, window=64, topk=128)),
]


@pytest.mark.parametrize("name,n_slices,kw", CASES, ids=[c[0] for c in CASES])
def test_context_parallel_every_row(name, n_slices, kw):
    """Every row of out, lse, idx and the sparse layers against the oracle over
    the whole cache (queries before a slice, after it and inside it)."""
    w = wl.WORKLOADS["tiny"] if kw is None else wl.custom(name, n_sparse=1, seed=17, **kw)
    inp = wl.make_inputs(w, "cuda")
    gpu = _run_cp(w, inp, n_slices)
    res = P.compare_rows(w, inp, gpu, 0, np.arange(w.n_q))
    print(name, res["idx"], res["out_err"], res["sparse_err"])


def test_context_parallel_matches_the_single_cache_path():
    """Against the one-cache kernels: outputs and LSE within rounding, and the
    selections equal except at near-ties of the k-th score."""
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda")
    gpu = _run_cp(w, inp, 4)
    ref = P.run_gpu(w, inp)
    P.assert_close(P.to_f64(gpu["out"]), P.to_f64(ref["out"]), "cp vs single out")
    P.assert_close(P.to_f64(gpu["lse"]), P.to_f64(ref["lse"]), "cp vs single lse", atol=1e-4, rtol=0.0)
    same = (gpu["idx"] == ref["idx"]).all(dim=-1).float().mean().item()
    assert same > 0.99, f"only {same:.4f} of the rows select identically"
    for a, b in zip(gpu["sparse"], ref["sparse"]):
        P.assert_close(P.to_f64(a), P.to_f64(b), "cp vs single sparse")


def test_prefill_32k_context_parallel_sampled():
    w = wl.WORKLOADS["prefill_32k"]
    inp = wl.make_inputs(w, "cuda")
    gpu = _run_cp(w, inp, 4)
    rows = wl.stratified_rows(w, 8)
    res = P.compare_rows(w, inp, gpu, 0, rows)
    print("32k cp4", res["idx"], res["out_err"], res["sparse_err"])


def test_chunk_256k_context_parallel_sampled():
    """8192 new queries on a 270336-token cache in 8 slices: every query sits
    after seven slices and inside the last."""
    w = wl.WORKLOADS["chunk_256k"]
    inp = wl.make_inputs(w, "cuda")
    gpu = _run_cp(w, inp, 8)
    rows = np.array([0, 1, 4095, 8191])
    res = P.compare_rows(w, inp, gpu, 0, rows)
    print("256k cp8", res["idx"], res["out_err"], res["sparse_err"])


def test_merge_handles_rows_with_fewer_candidates_than_the_budget():
    """Queries whose whole-context candidates number fewer than K, spread over
    slices: the merge keeps every candidate, ascending."""
    w = wl.custom("few_cands", n_q=256, q_pos0=100, kv_len=356, h_q=8, h_kv=2, head_dim=64, window=32, topk=512,
                  n_sparse=0, seed=19)
    inp = wl.make_inputs(w, "cuda", with_sparse=False)
    gpu = _run_cp(w, inp, 3)
    idx = gpu["idx"].cpu().numpy()
    for i in range(w.n_q):
        t = w.q_pos0 + i
        n = max(0, t - w.window + 1)
        want = np.concatenate([np.arange(n), -np.ones(w.topk - n)]).astype(np.int32)
        assert np.array_equal(idx[0, :, i], np.broadcast_to(want, idx[0, :, i].shape)), f"row t={t}"


def test_slice_steps_report_timeouts_and_checks_through_their_workspace():
    """A slice call's workspace carries the error word: a valid run leaves it clear."""
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda")
    offs, ks, vs = cp.split_cache(inp["k"], inp["v"], 2)
    shape = nv.shape_of(inp["q"], ks[1], window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    ws = torch.empty(nv.hs2_cp_workspace_size(shape, offs[1], nv.HS2_ENTRY_CP_ATTN), dtype=torch.uint8,
                     device="cuda")
    nv.hs2_workspace_init(ws)
    out = torch.empty_like(inp["q"])
    lse = torch.empty(inp["q"].shape[:3], dtype=torch.float32, device="cuda")
    nv.hs2_cp_attn_partial(shape, offs[1], inp["q"], ks[1], vs[1], out, lse, ws)
    rc, info = nv.hs2_get_device_status(ws)
    assert rc == nv.HS2_OK, (rc, info)
    # queries before the slice have no key there: output 0, LSE -inf
    first = offs[1] - w.q_pos0
    assert torch.all(torch.isneginf(lse[:, :, :first])) and torch.all(out[:, :, :first] == 0)
    assert torch.all(torch.isfinite(lse[:, :, first:]))


def test_context_parallel_class_over_nccl_one_rank():
    """The ContextParallel class as each rank of a multi-GPU run drives it: the
    library's kernels for the slice steps and merges, and the NCCL all-gather
    (dist_gather) to stack the per-slice results, here as rank 0 of a one-rank
    process group on this GPU (the collective runs on the device but exchanges
    nothing).  Its results equal those of the one-process path over the same
    single slice bit for bit, and match the oracle on every row."""
    import datetime
    import socket
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        w = wl.custom("cp_nccl", n_q=300, q_pos0=500, h_q=8, h_kv=2, head_dim=64, window=64, topk=128, n_sparse=1,
                      seed=23)
        inp = wl.make_inputs(w, "cuda")
        rank = cp.ContextParallel(inp["k"], inp["v"], rank=0, kv_offs=[0], kv_len=w.kv_len, window=w.window,
                                  topk=w.topk)
        before = nv.hs2_launch_count()
        out, lse, idx = rank.full_attn_select(inp["q"], w.q_pos0)
        sp = [rank.sparse_attn(qs, idx, w.q_pos0) for qs in inp["q_sparse"]]
        torch.cuda.synchronize()
        assert nv.hs2_launch_count() > before
        ref = _run_cp(w, inp, 1)
        assert torch.equal(out, ref["out"]) and torch.equal(lse, ref["lse"]) and torch.equal(idx, ref["idx"])
        assert all(torch.equal(a, b) for a, b in zip(sp, ref["sparse"]))
        P.compare_rows(w, inp, dict(out=out, lse=lse, idx=idx, sparse=sp), 0, np.arange(w.n_q))
    finally:
        dist.destroy_process_group()

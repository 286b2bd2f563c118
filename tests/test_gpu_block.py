"""GPU parity of block-level selection (the design token-level selection
replaces: whole blocks of contiguous keys ranked by their summed group score,
at the same key budget) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
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


def run_block(w: wl.Workload, inp: dict, blk: int):
    out, lse, idx = nv.full_attn_block_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk,
                                              block=blk, q_pos0=w.q_pos0)
    sp = [nv.sparse_attn(qs, inp["k"], inp["v"], idx, window=w.window, q_pos0=w.q_pos0)
          for qs in inp["q_sparse"]]
    torch.cuda.synchronize()
    return dict(out=out, lse=lse, idx=idx, sparse=sp)


def compare_block_rows(w: wl.Workload, inp: dict, gpu: dict, b: int, rows: np.ndarray, blk: int,
                       n_threads: int = 0) -> dict:
    rows = np.asarray(rows, dtype=np.int64)
    ts = w.q_pos0 + rows
    kb, vb = P.bits(inp["k"][b]), P.bits(inp["v"][b])
    qb = np.ascontiguousarray(P.bits(inp["q"][b][:, rows, :]).transpose(1, 0, 2))
    ores = oracle.block_select(qb, ts, kb, vb, window=w.window, topk=w.topk, block=blk, n_threads=n_threads)
    rows_t = torch.as_tensor(rows, device=gpu["out"].device)
    g_out = P.to_f64(gpu["out"][b][:, rows_t, :]).transpose(1, 0, 2)
    g_lse = P.to_f64(gpu["lse"][b][:, rows_t]).T
    g_idx = np.ascontiguousarray(gpu["idx"][b][:, rows_t, :].cpu().numpy().transpose(1, 0, 2))
    res = dict(out_err=P.assert_close(g_out, ores["full"]["out"], f"{w.name} full out"))
    res["lse_err"] = P.assert_close(g_lse, ores["full"]["lse"], f"{w.name} lse", atol=P.LSE_ATOL, rtol=0.0)
    res["idx"] = P.check_block_idx(g_idx, ores, ts, w.window, w.topk, blk, f"{w.name} block idx")
    res["sparse_err"] = []
    for layer, (qs, so) in enumerate(zip(inp["q_sparse"], gpu["sparse"])):
        qsb = np.ascontiguousarray(P.bits(qs[b][:, rows, :]).transpose(1, 0, 2))
        got = P.to_f64(so[b][:, rows_t, :]).transpose(1, 0, 2)
        ref = oracle.sparse(qsb, ts, kb, vb, g_idx, window=w.window, n_threads=n_threads)
        res["sparse_err"].append(P.assert_close(got, ref, f"{w.name} sparse layer {layer} on block idx"))
        if layer == 0:
            ref_e2e = oracle.sparse(qsb, ts, kb, vb, ores["idx"], window=w.window, n_threads=n_threads)
            res["sparse_e2e_err"] = P.assert_close(got, ref_e2e, f"{w.name} sparse layer 0 end to end")
    return res


def test_tiny_every_row_block64():
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda")
    before = nv.hs2_launch_count()
    gpu = run_block(w, inp, 64)
    assert nv.hs2_launch_count() > before
    res = compare_block_rows(w, inp, gpu, 0, np.arange(w.n_q), 64)
    print("tiny block 64", res["idx"], res["out_err"], res["sparse_err"])


BLOCK_SHAPES = [
    # name, block, kwargs for workloads.custom
    ("b32_g4_d64_chunk", 32, dict(n_q=333, q_pos0=700, h_q=8, h_kv=2, head_dim=64, window=32, topk=100)),
    ("b64_g8_d128_tail", 64, dict(n_q=200, q_pos0=900, h_q=16, h_kv=2, head_dim=128, window=128, topk=256)),
    ("b128_g2_d64", 128, dict(n_q=161, q_pos0=1200, h_q=4, h_kv=2, head_dim=64, window=16, topk=384)),
    ("b64_g1_d128_window1", 64, dict(n_q=257, q_pos0=300, h_q=2, h_kv=2, head_dim=128, window=1, topk=130)),
    ("b64_batch2_extra_cache", 64, dict(batch=2, n_q=150, q_pos0=500, kv_len=800, h_q=8, h_kv=1, head_dim=64,
                                        window=64, topk=192)),
    ("b32_topk_below_block", 32, dict(n_q=64, q_pos0=200, h_q=8, h_kv=2, head_dim=64, window=8, topk=20)),
    ("b128_topk_2048", 128, dict(n_q=64, q_pos0=3000, h_q=16, h_kv=2, head_dim=64, window=128, topk=2048)),
    # more than 2^18 candidates per row: the sweep's 28-query geometry (COUNTER)
    ("b64_counter_270k", 64, dict(n_q=64, q_pos0=270000, h_q=16, h_kv=2, head_dim=128, window=128, topk=1024)),
    ("b32_counter_g4_d64", 32, dict(n_q=40, q_pos0=270000, h_q=8, h_kv=2, head_dim=64, window=64, topk=512)),
    ("b64_counter_g8_d64", 64, dict(n_q=36, q_pos0=262300, h_q=16, h_kv=2, head_dim=64, window=128, topk=1024)),
    # G = 2 above 2^18 candidates keeps the 32-query geometry
    ("b128_long_g2", 128, dict(n_q=40, q_pos0=270000, h_q=4, h_kv=2, head_dim=64, window=64, topk=1024)),
]


@pytest.mark.parametrize("name,blk,kw", BLOCK_SHAPES, ids=[r[0] for r in BLOCK_SHAPES])
def test_block_shapes_every_row(name, blk, kw):
    w = wl.custom(name, n_sparse=1, seed=11, **kw)
    inp = wl.make_inputs(w, "cuda")
    gpu = run_block(w, inp, blk)
    for b in range(w.batch):
        compare_block_rows(w, inp, gpu, b, np.arange(w.n_q), blk)


def test_block_ties_take_the_lowest_blocks():
    """q = 0: every key of a row has the same probability, so every candidate
    block the same score; the kept blocks are the lowest ones, bit-exactly."""
    w = wl.custom("block_ties", n_q=96, q_pos0=1000, h_q=8, h_kv=2, head_dim=64, window=64, topk=256, n_sparse=0,
                  seed=5)
    inp = wl.make_inputs(w, "cuda", with_sparse=False)
    q = torch.zeros_like(inp["q"])
    out, lse, idx = nv.full_attn_block_select(q, inp["k"], inp["v"], window=w.window, topk=w.topk, block=64,
                                              q_pos0=w.q_pos0)
    torch.cuda.synchronize()
    want = torch.arange(w.topk, dtype=torch.int32, device="cuda")
    assert torch.equal(idx, want.expand_as(idx))


def test_block_entry_rejects_other_block_sizes():
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda", with_sparse=False)
    for blk in (0, 16, 48, 256):
        with pytest.raises(nv.HS2Error) as e:
            nv.full_attn_block_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk, block=blk)
        assert e.value.status == 2


def test_prefill_32k_block64_sampled():
    w = wl.WORKLOADS["prefill_32k"]
    inp = wl.make_inputs(w, "cuda")
    gpu = run_block(w, inp, 64)
    rows = wl.stratified_rows(w, 10)
    res = compare_block_rows(w, inp, gpu, 0, rows, 64)
    print("32k block 64", res["idx"], res["out_err"], res["sparse_err"])
    _block_row_properties(gpu["idx"], w, 64)


def test_chunk_1m_block64_sampled():
    """1M-token cache, 4096 new queries: the chunk sums (one float per 32 keys per
    row, 1 GiB budget) take query chunks of whole waves of CTAs, 1036 queries
    each (148 CTAs of 28 queries) and 988 last; rows on both sides of every
    chunk boundary, and seeded random ones."""
    w = wl.WORKLOADS["chunk_1m"]
    inp = wl.make_inputs(w, "cuda")
    gpu = run_block(w, inp, 64)
    edges = np.array([0, 1035, 1036, 2071, 2072, 3107, 3108, 4095])
    rows = np.union1d(edges, np.random.default_rng(7).integers(0, w.n_q, size=8))
    res = compare_block_rows(w, inp, gpu, 0, rows, 64)
    print("1m block 64", res["idx"], res["out_err"])
    _block_row_properties(gpu["idx"], w, 64)


def _block_row_properties(idx: torch.Tensor, w: wl.Workload, blk: int):
    """Every row of a full-size call, on the device: keep whole blocks, aligned,
    contiguous, ascending, below the window; -1 after."""
    B, Hkv, nq, K = idx.shape
    t = w.q_pos0 + torch.arange(nq, device=idx.device, dtype=torch.int64)
    n_blk = torch.clamp(t - w.window + 1, min=0) // blk
    keep = torch.clamp(n_blk, max=K // blk)  # [nq]
    pos = torch.arange(K, device=idx.device)
    valid = pos[None, :] < (keep * blk)[:, None]  # [nq, K]
    x = idx.to(torch.int64)
    assert torch.all(torch.where(valid, x >= 0, x == -1))
    starts = x[..., ::blk]  # [B, Hkv, nq, K / blk]
    body = starts.repeat_interleave(blk, dim=-1)[..., :K] + (pos % blk)
    assert torch.all(torch.where(valid, x == body, True))
    assert torch.all(torch.where(valid, x % blk == pos % blk, True))
    sv = valid[:, ::blk]
    nxt = torch.where(sv[:, 1:], starts[..., 1:] - starts[..., :-1], torch.full_like(starts[..., 1:], blk))
    assert torch.all(nxt >= blk)
    assert torch.all(torch.where(valid, x <= (t - w.window)[:, None], True))

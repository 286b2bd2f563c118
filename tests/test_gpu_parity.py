"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded bf16 inputs.  Small cases are checked on every row; the full-size
workloads on stratified samples (window / top-k boundary rows plus seeded
random rows) and on properties that hold for every row."""
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
    nv.load(True)


def test_tiny_every_row():
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda")
    before = nv.hs2_launch_count()
    gpu = P.run_gpu(w, inp)
    assert nv.hs2_launch_count() > before  # the CUDA kernels ran
    res = P.compare_rows(w, inp, gpu, 0, np.arange(w.n_q))
    print("tiny", {k: v for k, v in res.items() if k != "oracle"})


def test_prefill_entry_matches_full_select():
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda", with_sparse=False)
    a = nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk, entry="full")
    b = nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk, entry="prefill")
    torch.cuda.synchronize()
    assert torch.equal(a[2], b[2])
    P.assert_close(P.to_f64(a[0]), P.to_f64(b[0]), "prefill vs full out")


RAGGED = [
    # name, kwargs for workloads.custom
    ("g8_d128_tail", dict(n_q=200, h_q=16, h_kv=2, head_dim=128, window=128, topk=64)),
    ("g4_d64_chunk", dict(n_q=333, q_pos0=700, h_q=8, h_kv=2, head_dim=64, window=32, topk=100)),
    ("g2_d64_extra_cache", dict(n_q=130, q_pos0=50, kv_len=400, h_q=4, h_kv=2, head_dim=64, window=16, topk=20)),
    ("g1_d128", dict(n_q=257, h_q=2, h_kv=2, head_dim=128, window=8, topk=33)),
    ("window1_topk_large", dict(n_q=190, h_q=8, h_kv=1, head_dim=64, window=1, topk=300)),
    ("topk0", dict(n_q=160, h_q=8, h_kv=1, head_dim=128, window=40, topk=0)),
    ("batch3", dict(batch=3, n_q=150, q_pos0=100, h_q=8, h_kv=1, head_dim=64, window=64, topk=48)),
    ("topk_2048", dict(n_q=64, q_pos0=3000, h_q=16, h_kv=2, head_dim=64, window=128, topk=2048)),
    ("window1024", dict(n_q=96, q_pos0=1500, h_q=8, h_kv=1, head_dim=128, window=1024, topk=256)),
]


@pytest.mark.parametrize("name,kw", RAGGED, ids=[r[0] for r in RAGGED])
def test_ragged_shapes_every_row(name, kw):
    w = wl.custom(name, n_sparse=2, seed=7, **kw)
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    for b in range(w.batch):
        P.compare_rows(w, inp, gpu, b, np.arange(w.n_q))


def test_sparse_kernel_with_oracle_selection():
    """K3 alone, fed the oracle's idx row by row (one-query calls)."""
    w = wl.custom("k3_oracle_idx", n_q=700, h_q=16, h_kv=2, head_dim=128, window=128, topk=128, seed=3)
    inp = wl.make_inputs(w, "cuda")
    rows = np.array([0, 127, 128, 129, 255, 256, 257, 400, 699])
    kb, vb = P.bits(inp["k"][0]), P.bits(inp["v"][0])
    qb = np.ascontiguousarray(P.bits(inp["q"][0][:, rows]).transpose(1, 0, 2))
    ores = oracle.full_select(qb, rows, kb, vb, window=w.window, topk=w.topk)
    qs = inp["q_sparse"][0]
    qsb = np.ascontiguousarray(P.bits(qs[0][:, rows]).transpose(1, 0, 2))
    ref = oracle.sparse(qsb, rows, kb, vb, ores["idx"], window=w.window)
    for r, i in enumerate(rows):
        q1 = qs[:, :, i:i + 1].contiguous()
        idx1 = torch.as_tensor(ores["idx"][r][None, :, None, :], device="cuda").contiguous()
        o = nv.sparse_attn(q1, inp["k"], inp["v"], idx1, window=w.window, q_pos0=int(i))
        P.assert_close(P.to_f64(o[0, :, 0]), ref[r], f"K3 row {i}")


def test_prefill_32k_sampled():
    w = wl.WORKLOADS["prefill_32k"]
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    rows = wl.stratified_rows(w, 32)
    res = P.compare_rows(w, inp, gpu, 0, rows)
    print("32k", res["idx"], res["out_err"], res["sparse_err"])
    _row_properties(gpu["idx"], w)


def _row_properties(idx: torch.Tensor, w: wl.Workload, seq_len=None):
    """Every row of a full-size call: size min(K, t-W+1), strictly ascending,
    inside [0, t-W], -1 padded (checked on the device)."""
    B, Hkv, nq, K = idx.shape
    if seq_len is None:
        t = torch.arange(w.q_pos0, w.q_pos0 + nq, device=idx.device).view(1, 1, nq, 1).expand(B, 1, nq, 1)
    else:
        t = (seq_len - 1).view(B, 1, 1, 1)
    n_sel = torch.clamp(t - w.window + 1, min=0).clamp(max=K)
    pos = torch.arange(K, device=idx.device).view(1, 1, 1, K)
    valid = pos < n_sel
    assert torch.all(torch.where(valid, idx >= 0, idx == -1))
    assert torch.all(torch.where(valid, idx <= t - w.window, True))
    if K > 1:
        d = idx[..., 1:] - idx[..., :-1]
        assert torch.all(torch.where(valid[..., 1:], d > 0, True))


def test_chunk_256k_sampled():
    w = wl.WORKLOADS["chunk_256k"]
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    rows = wl.stratified_rows(w, 32)
    res = P.compare_rows(w, inp, gpu, 0, rows)
    print("256k", res["idx"], res["out_err"], res["sparse_err"])
    _row_properties(gpu["idx"], w)


def test_decode_128k_every_sequence():
    w = wl.WORKLOADS["decode_128k"]
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    t = np.array([w.kv_len - 1])
    for b in range(w.batch):
        P.compare_rows(w, inp, gpu, b, np.array([0]), ts=t)
    _row_properties(gpu["idx"], w)


def test_decode_ragged_lengths():
    w = wl.custom("decode_ragged", batch=5, n_q=1, q_pos0=4999, kv_len=5000, h_q=32, h_kv=4, head_dim=128,
                  window=128, topk=1024, n_sparse=2, decode=True, seed=9)
    inp = wl.make_inputs(w, "cuda")
    lens = torch.tensor([5000, 1, 128, 1153, 3001], dtype=torch.int64, device="cuda")
    gpu = P.run_gpu(w, inp, seq_len=lens)
    for b, ln in enumerate(lens.tolist()):
        P.compare_rows(w, inp, gpu, b, np.array([0]), ts=np.array([ln - 1]))
    _row_properties(gpu["idx"], w, seq_len=lens)


def test_chunk_1m_sampled():
    w = wl.WORKLOADS["chunk_1m"]
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    rows = wl.stratified_rows(w, 32)
    res = P.compare_rows(w, inp, gpu, 0, rows)
    print("1m chunk", res["idx"], res["out_err"], res["sparse_err"])
    _row_properties(gpu["idx"], w)


def test_decode_1m_every_sequence():
    w = wl.WORKLOADS["decode_1m"]
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    t = np.array([w.kv_len - 1])
    for b in range(w.batch):
        P.compare_rows(w, inp, gpu, b, np.array([0]), ts=t)
    _row_properties(gpu["idx"], w)


def test_checked_build_reports_invalid_selection():
    """A selection row that breaks the contract (an index inside the window) is
    reported through the error word; the kernel skips nothing out of bounds."""
    w = wl.custom("bad_idx", n_q=64, q_pos0=500, h_q=8, h_kv=1, head_dim=64, window=32, topk=16, seed=2)
    inp = wl.make_inputs(w, "cuda")
    _, _, idx = nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk,
                                    q_pos0=w.q_pos0, checked=True)
    shape = nv.shape_of(inp["q"], inp["k"], window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    ws = nv.alloc_workspace(shape, nv.HS2_ENTRY_SPARSE, checked=True)
    out = torch.empty_like(inp["q"])
    nv.hs2_sparse_attn(shape, inp["q"], inp["k"], inp["v"], idx, out, ws, checked=True)
    rc, info = nv.hs2_get_device_status(ws, checked=True)
    assert rc == nv.HS2_OK, (rc, info)
    bad = idx.clone()
    bad[0, 0, 5, 3] = w.q_pos0 + 5  # the query itself: inside the window
    nv.hs2_sparse_attn(shape, inp["q"], inp["k"], inp["v"], bad, out, ws, checked=True)
    rc, info = nv.hs2_get_device_status(ws, checked=True)
    assert rc == 5 and info[1] == 4, (rc, info)  # HS2_ERR_DEVICE_CHECK from the sparse kernel
    rc, info = nv.hs2_get_device_status(ws, checked=True)
    assert rc == nv.HS2_OK  # reading clears the word


def test_empty_call_launches_nothing():
    q = torch.zeros(1, 8, 0, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16, device="cuda")
    before = nv.hs2_launch_count()
    out, lse, idx = nv.full_attn_select(q, k, k, window=4, topk=4, q_pos0=0)
    assert nv.hs2_launch_count() == before


def test_exact_ties_force_list_compaction():
    """q = 0 makes every candidate's score exactly G/(t+1): the tie rule fixes the
    selection to indices 0..K-1, and with more than 4096 candidates per row every
    survivor list overflows and is compacted (the rare path of the selection)."""
    w = wl.custom("all_ties", n_q=96, q_pos0=9000, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024,
                  n_sparse=1, seed=4)
    inp = wl.make_inputs(w, "cuda")
    inp["q"].zero_()
    gpu = P.run_gpu(w, inp)
    want = torch.arange(w.topk, dtype=torch.int32, device="cuda")
    assert torch.equal(gpu["idx"], want.expand_as(gpu["idx"]))
    rows = np.array([0, 1, 47, 95])
    P.compare_rows(w, inp, gpu, 0, rows)


def test_decode_exact_ties_take_the_full_radix_path():
    """q = 0 gives every candidate the same score G/(t+1): the sampled threshold
    then admits all 19873 candidates, more than the survivor buffer holds, so
    the decode top-k falls back to the exact passes over the whole row; the tie
    rule fixes the selection to indices 0..K-1."""
    w = wl.custom("decode_ties", batch=2, n_q=1, q_pos0=19999, kv_len=20000, h_q=32, h_kv=4, head_dim=128,
                  window=128, topk=1024, n_sparse=1, decode=True, seed=6)
    inp = wl.make_inputs(w, "cuda")
    inp["q"].zero_()
    gpu = P.run_gpu(w, inp)
    want = torch.arange(w.topk, dtype=torch.int32, device="cuda")
    assert torch.equal(gpu["idx"], want.expand_as(gpu["idx"]))
    P.compare_rows(w, inp, gpu, 1, np.array([0]), ts=np.array([w.kv_len - 1]))


@pytest.mark.parametrize("head_dim,h_q,h_kv", [(128, 8, 2), (64, 8, 1)])
def test_split_key_range_full_attention(head_dim, h_q, h_kv):
    """Few query tiles over a long cache: the full layer splits each CTA's key
    range in parts and merges them exactly (out, lse and the selection built on
    the merged lse)."""
    w = wl.custom("split_kv", n_q=256, q_pos0=70000, kv_len=70256, h_q=h_q, h_kv=h_kv, head_dim=head_dim,
                  window=128, topk=256, n_sparse=1, seed=8)
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    P.compare_rows(w, inp, gpu, 0, np.array([0, 1, 127, 128, 200, 255]))
    _row_properties(gpu["idx"], w)


DECODE_SHAPES = [
    # name, kwargs: other head dims, group sizes, budgets and windows than the decode workloads
    ("d64_g4_k2048_w1024", dict(batch=2, q_pos0=49999, kv_len=50000, h_q=16, h_kv=4, head_dim=64, window=1024,
                                topk=2048)),
    ("d128_g2_k512_w16", dict(batch=3, q_pos0=2999, kv_len=3000, h_q=8, h_kv=4, head_dim=128, window=16, topk=512)),
    ("d128_g1_k64", dict(batch=2, q_pos0=20479, kv_len=20480, h_q=4, h_kv=4, head_dim=128, window=128, topk=64)),
]


@pytest.mark.parametrize("name,kw", DECODE_SHAPES, ids=[d[0] for d in DECODE_SHAPES])
def test_decode_shapes_every_sequence(name, kw):
    w = wl.custom(name, n_q=1, n_sparse=2, decode=True, seed=11, **kw)
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    for b in range(w.batch):
        P.compare_rows(w, inp, gpu, b, np.array([0]), ts=np.array([w.kv_len - 1]))
    _row_properties(gpu["idx"], w)


@pytest.mark.parametrize("head_dim,h_q,h_kv", [(128, 8, 1), (64, 8, 2)])
def test_full_attention_rescale_of_single_rows(head_dim, h_q, h_kv):
    """Keys far above every earlier logit of a few rows, several key tiles after
    the first: those rows rescale their running output at that tile, and each
    other row of their warps does or does not, at random (the spike key is a
    large random direction for them).  The rescale of the output in tensor
    memory is a warp-collective pass; every row must still match the oracle."""
    w = wl.custom(f"spike_d{head_dim}", n_q=256, q_pos0=512, kv_len=768, h_q=h_q, h_kv=h_kv, head_dim=head_dim,
                  window=128, topk=64, n_sparse=0, seed=5)
    inp = wl.make_inputs(w, "cuda", with_sparse=False)
    q, k = inp["q"], inp["k"]
    G = h_q // h_kv
    for r in (3, 45, 130, 250):
        j = w.q_pos0 + r - 2  # a later key tile than the rows' first one, still causal for row r
        for g in range(h_kv):
            u = q[0, g * G:(g + 1) * G, r].float().sum(0)
            k[0, g, j] = (160.0 * u / u.norm()).to(torch.bfloat16)
    gpu = P.run_gpu(w, inp)
    P.compare_rows(w, inp, gpu, 0, np.arange(w.n_q))


def _check_selection_and_scores(g_idx, g_score, ores, ts, w, what):
    """g_idx, g_score [n_rows, H_kv, K] from the selection pass; the selected
    sets against the oracle's (near-tie rule) and the score the pass returns for
    each selected row against the oracle's score of that row."""
    P.check_idx(g_idx, ores, ts, w.window, w.topk, what)
    for r, t in enumerate(ts):
        n_sel = min(w.topk, max(0, int(t) - w.window + 1))
        for g in range(g_idx.shape[1]):
            sel = g_idx[r, g, :n_sel]
            want = ores["scores"][r, g, sel]
            got = g_score[r, g, :n_sel].astype(np.float64)
            assert np.all(np.abs(got - want) <= 1e-9 + 1e-4 * np.abs(want)), f"{what} row t={t} g={g}: scores"


@pytest.mark.parametrize("n_q,q_pos0,topk", [(600, 1400, 256), (64, 270000, 1024)], ids=["ordered", "counter"])
def test_selection_pass_fed_the_oracle_lse(n_q, q_pos0, topk):
    """The selection pass alone (the slice step of context parallelism over the
    whole cache), fed the oracle's LSE instead of the full-attention kernel's:
    isolates the selection kernel from the LSE the first kernel computes.  It
    also returns each selected key's score, checked against the oracle's.  The
    second case has more than 2^18 candidates per row (the COUNTER layout, as
    each slice of a 1M context split four ways has)."""
    from long_context_sparse_flash_b200 import cp
    w = wl.custom("k2_oracle_lse", n_q=n_q, q_pos0=q_pos0, h_q=16, h_kv=2, head_dim=128, window=128, topk=topk,
                  n_sparse=0, seed=9)
    inp = wl.make_inputs(w, "cuda", with_sparse=False)
    ts = w.q_pos0 + np.arange(w.n_q)
    qb = np.ascontiguousarray(P.bits(inp["q"][0]).transpose(1, 0, 2))
    ores = oracle.full_select(qb, ts, P.bits(inp["k"][0]), P.bits(inp["v"][0]), window=w.window, topk=w.topk,
                              want_scores=True)
    lse = torch.as_tensor(np.ascontiguousarray(ores["lse"].T[None]).astype(np.float32), device="cuda")
    idx, score = cp.select_local(inp["q"], inp["k"], lse, kv_off=0, window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    torch.cuda.synchronize()
    g_idx = np.ascontiguousarray(idx[0].cpu().numpy().transpose(1, 0, 2))
    g_score = np.ascontiguousarray(score[0].cpu().numpy().transpose(1, 0, 2))
    _check_selection_and_scores(g_idx, g_score, ores, ts, w, "selection on the oracle LSE")


def test_overshooting_threshold_forces_the_retry_pass():
    """The selection's retry pass, forced.  Every query carries a shared
    per-group direction u_g, and the keys at the sampling stride (j = m S,
    S = kv_len // 1024, the keys the threshold estimate is drawn from) are
    strong plants along u_g.  The estimate is then the r-th best plant, far
    above the K-th best candidate of every row: fewer than K candidates pass
    the filtered sweep, every row is marked, and the retry pass re-sweeps it
    with bound 0.  Every row must still match the oracle."""
    w = wl.custom("retry", n_q=96, q_pos0=20000, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024,
                  n_sparse=1, seed=12)
    inp = wl.make_inputs(w, "cuda")
    q, k = inp["q"], inp["k"]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(77)
    u = torch.randn(w.h_kv, w.head_dim, generator=gen, device="cuda")
    u = u / u.norm(dim=-1, keepdim=True)
    G = w.group
    q_f = q.float().view(1, w.h_kv, G, w.n_q, w.head_dim) + 2.0 * u.view(1, w.h_kv, 1, 1, w.head_dim)
    q.copy_(q_f.view_as(q).to(torch.bfloat16))
    S = w.kv_len // 1024
    pos = torch.arange(0, w.kv_len, S, device="cuda")
    noise = torch.randn(w.h_kv, pos.numel(), w.head_dim, generator=gen, device="cuda")
    k[0][:, pos, :] = (8.0 * u[:, None, :] + 0.1 * noise).to(torch.bfloat16)
    shape = nv.shape_of(q, k, window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    ws = nv.alloc_workspace(shape, nv.HS2_ENTRY_FULL_SELECT)
    out, lse, idx = nv.full_attn_select(q, k, inp["v"], window=w.window, topk=w.topk, q_pos0=w.q_pos0, ws=ws)
    retried = nv.hs2_select_retry_rows(shape, ws)
    assert retried == w.batch * w.h_kv * w.n_q, retried  # every row took the retry pass
    sp = [nv.sparse_attn(qs, k, inp["v"], idx, window=w.window, q_pos0=w.q_pos0) for qs in inp["q_sparse"]]
    torch.cuda.synchronize()
    gpu = dict(out=out, lse=lse, idx=idx, sparse=sp)
    P.compare_rows(w, inp, gpu, 0, np.arange(w.n_q))
    _row_properties(idx, w)


def test_ordinary_inputs_take_no_retry():
    """The counterpart: on the needle workload's inputs the estimate holds and
    no row is retried (the retry pass exists for inputs like the test above)."""
    w = wl.custom("no_retry", n_q=96, q_pos0=20000, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024,
                  n_sparse=0, needles=16, seed=12)
    inp = wl.make_inputs(w, "cuda", with_sparse=False)
    shape = nv.shape_of(inp["q"], inp["k"], window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    ws = nv.alloc_workspace(shape, nv.HS2_ENTRY_FULL_SELECT)
    nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk, q_pos0=w.q_pos0, ws=ws)
    assert nv.hs2_select_retry_rows(shape, ws) == 0


def test_kv_head_halves_match_the_whole_call():
    """One workload's KV-head groups split in two, each half run as its own set
    of calls (what each GPU of a head-split run computes): every output of a
    half is bit-identical to the whole call's output for those heads, and the
    halves match the oracle."""
    import bench
    w = wl.custom("head_split", n_q=512, q_pos0=6000, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024,
                  n_sparse=1, seed=14)
    inp = wl.make_inputs(w, "cuda")
    whole = P.run_gpu(w, inp)
    for r in range(2):
        w_r, share = bench.head_shard(w, inp, r, 2)
        half = P.run_gpu(w_r, share)
        h0, h1 = r * w_r.h_q, (r + 1) * w_r.h_q
        g0, g1 = r * w_r.h_kv, (r + 1) * w_r.h_kv
        assert torch.equal(half["idx"], whole["idx"][:, g0:g1])
        assert torch.equal(half["out"], whole["out"][:, h0:h1])
        assert torch.equal(half["lse"], whole["lse"][:, h0:h1])
        assert torch.equal(half["sparse"][0], whole["sparse"][0][:, h0:h1])
        P.compare_rows(w_r, share, half, 0, np.array([0, 1, 255, 511]))


# The selection sweep has two epilogue layouts (ORDERED for calls whose longest
# row has fewer than 2^18 candidates, COUNTER from 2^18 on).  The small shapes
# above exercise ORDERED; these put every row of a COUNTER call next to the
# oracle: ragged tails of 28-query CTAs, exact ties (list compaction, the j
# tie-break and the run-ranked output), the retry pass, and a budget above the
# shared-memory staging of the final select.
COUNTER_MIN_CAND = 1 << 18


@pytest.mark.parametrize("name,kw", [
    ("counter_segments", dict(n_q=60, q_pos0=280000, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024,
                              keys="segments", needles=16)),
    ("counter_d64_g4", dict(n_q=33, q_pos0=270000, h_q=16, h_kv=4, head_dim=64, window=64, topk=512)),
    ("counter_topk2048", dict(n_q=30, q_pos0=265000, h_q=16, h_kv=2, head_dim=128, window=128, topk=2048)),
    ("counter_batch2", dict(batch=2, n_q=31, q_pos0=263000, h_q=8, h_kv=2, head_dim=128, window=128, topk=1024)),
    ("counter_d64_g8", dict(n_q=30, q_pos0=262300, h_q=16, h_kv=2, head_dim=64, window=128, topk=1024)),
], ids=["segments", "d64_g4", "topk2048", "batch2", "d64_g8"])
def test_counter_layout_every_row(name, kw):
    w = wl.custom(name, n_sparse=1, seed=15, **kw)
    assert w.q_pos0 + w.n_q - w.window >= COUNTER_MIN_CAND
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    for b in range(w.batch):
        P.compare_rows(w, inp, gpu, b, np.arange(w.n_q))
    _row_properties(gpu["idx"], w)


@pytest.mark.parametrize("name,kw", [
    ("long_g1", dict(n_q=40, q_pos0=270000, h_q=2, h_kv=2, head_dim=128, window=128, topk=1024)),
    ("long_g2", dict(n_q=40, q_pos0=270000, h_q=4, h_kv=2, head_dim=64, window=64, topk=512)),
], ids=["g1", "g2"])
def test_long_rows_with_one_or_two_heads_per_group(name, kw):
    """More than 2^18 candidates per row with G = 1 or 2 query heads per KV head:
    the COUNTER layout's MMA (N = 28 G columns) is not a valid tcgen05 shape for
    these G, so the sweep keeps ORDERED (N = 32 G); every row against the oracle."""
    w = wl.custom(name, n_sparse=1, seed=16, **kw)
    assert w.q_pos0 + w.n_q - w.window >= COUNTER_MIN_CAND
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    P.compare_rows(w, inp, gpu, 0, np.arange(w.n_q))
    _row_properties(gpu["idx"], w)


def test_counter_layout_exact_ties():
    """q = 0 over 270K candidates: every score is G/(t+1), every candidate passes
    the bound, the lists overflow and are compacted with the lower-j tie-break,
    and the selection must be exactly 0..K-1 (eight full key tiles, ranked
    inside their runs)."""
    w = wl.custom("counter_ties", n_q=56, q_pos0=270000, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024,
                  n_sparse=1, seed=16)
    inp = wl.make_inputs(w, "cuda")
    inp["q"].zero_()
    gpu = P.run_gpu(w, inp)
    want = torch.arange(w.topk, dtype=torch.int32, device="cuda")
    assert torch.equal(gpu["idx"], want.expand_as(gpu["idx"]))
    P.compare_rows(w, inp, gpu, 0, np.array([0, 27, 28, 55]))


def test_counter_layout_forced_retry():
    """The retry pass of the COUNTER layout: strong plants at the sampling stride
    make the estimated bound overshoot on every row."""
    w = wl.custom("counter_retry", n_q=40, q_pos0=270000, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024,
                  n_sparse=1, seed=17)
    inp = wl.make_inputs(w, "cuda")
    q, k = inp["q"], inp["k"]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(78)
    u = torch.randn(w.h_kv, w.head_dim, generator=gen, device="cuda")
    u = u / u.norm(dim=-1, keepdim=True)
    q_f = q.float().view(1, w.h_kv, w.group, w.n_q, w.head_dim) + 2.0 * u.view(1, w.h_kv, 1, 1, w.head_dim)
    q.copy_(q_f.view_as(q).to(torch.bfloat16))
    S = w.kv_len // 1024
    pos = torch.arange(0, w.kv_len, S, device="cuda")
    noise = torch.randn(w.h_kv, pos.numel(), w.head_dim, generator=gen, device="cuda")
    k[0][:, pos, :] = (8.0 * u[:, None, :] + 0.1 * noise).to(torch.bfloat16)
    shape = nv.shape_of(q, k, window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    ws = nv.alloc_workspace(shape, nv.HS2_ENTRY_FULL_SELECT)
    out, lse, idx = nv.full_attn_select(q, k, inp["v"], window=w.window, topk=w.topk, q_pos0=w.q_pos0, ws=ws)
    assert nv.hs2_select_retry_rows(shape, ws) == w.h_kv * w.n_q
    sp = [nv.sparse_attn(qs, k, inp["v"], idx, window=w.window, q_pos0=w.q_pos0) for qs in inp["q_sparse"]]
    torch.cuda.synchronize()
    P.compare_rows(w, inp, dict(out=out, lse=lse, idx=idx, sparse=sp), 0, np.arange(w.n_q))

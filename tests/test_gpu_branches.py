"""GPU parity of the predecessor design's two-branch sparse layer (a sliding-
window branch over its own cache and a selected-tokens branch over the shared
cache; the HySparse2 layer replaces both by one softmax over idx U window),
through the C ABI, against the fp64 oracle on the same seeded bf16 inputs."""
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


def _check_rows(w, inp, swa, idx, res, b, rows):
    """Both branches of sequence b on query indices `rows`, oracle on the same idx."""
    rows = np.asarray(rows, dtype=np.int64)
    ts = w.q_pos0 + rows
    rows_t = torch.as_tensor(rows, device="cuda")
    q = inp["q_sparse"][0] if inp["q_sparse"] else inp["q"]
    qb = np.ascontiguousarray(P.bits(q[b][:, rows, :]).transpose(1, 0, 2))
    g_idx = np.ascontiguousarray(idx[b][:, rows_t, :].cpu().numpy().transpose(1, 0, 2))
    ref = oracle.branches(qb, ts, P.bits(swa["k_swa"][b]), P.bits(swa["v_swa"][b]), P.bits(inp["k"][b]),
                          P.bits(inp["v"][b]), g_idx, window=w.window)
    out_swa, lse_swa, out_sel, lse_sel = res
    errs = {}
    for name, o, l in (("swa", out_swa, lse_swa), ("sel", out_sel, lse_sel)):
        go = P.to_f64(o[b][:, rows_t, :]).transpose(1, 0, 2)
        gl = P.to_f64(l[b][:, rows_t]).T
        rl = ref["lse_" + name]
        empty = np.isneginf(rl)
        assert np.array_equal(np.isneginf(gl), empty), f"{w.name} {name}: empty rows differ"
        assert np.all(go[empty] == 0.0), f"{w.name} {name}: empty rows must be zero"
        errs[name] = P.assert_close(go, ref["out_" + name], f"{w.name} {name} out")
        if (~empty).any():
            P.assert_close(gl[~empty], rl[~empty], f"{w.name} {name} lse", atol=P.LSE_ATOL, rtol=0.0)
    return errs


def _run(w, inp, swa, idx):
    q = inp["q_sparse"][0] if inp["q_sparse"] else inp["q"]
    res = nv.swa_branches(q, swa["k_swa"], swa["v_swa"], inp["k"], inp["v"], idx, window=w.window, q_pos0=w.q_pos0)
    torch.cuda.synchronize()
    return res


SHAPES = [
    ("tiny", None),
    ("g8_d128_chunk", dict(n_q=200, q_pos0=900, h_q=16, h_kv=2, head_dim=128, window=128, topk=256)),
    ("g4_d64_window1", dict(n_q=161, q_pos0=40, h_q=8, h_kv=2, head_dim=64, window=1, topk=64)),
    ("g2_d64_batch2", dict(batch=2, n_q=130, q_pos0=50, kv_len=400, h_q=4, h_kv=2, head_dim=64, window=16,
                           topk=20)),
    ("g1_d128_short", dict(n_q=190, h_q=2, h_kv=2, head_dim=128, window=128, topk=33)),
]


@pytest.mark.parametrize("name,kw", SHAPES, ids=[s[0] for s in SHAPES])
def test_branches_every_row(name, kw):
    """idx from the GPU's own token selection; every row, both branches (rows
    with t < W have an empty selected branch)."""
    w = wl.WORKLOADS["tiny"] if kw is None else wl.custom(name, n_sparse=1, seed=13, **kw)
    inp = wl.make_inputs(w, "cuda")
    swa = wl.make_swa_cache(w, "cuda")
    _, _, idx = nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    before = nv.hs2_launch_count()
    res = _run(w, inp, swa, idx)
    assert nv.hs2_launch_count() - before == 2
    for b in range(w.batch):
        _check_rows(w, inp, swa, idx, res, b, np.arange(w.n_q))


def test_branches_on_block_selection():
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda")
    swa = wl.make_swa_cache(w, "cuda")
    _, _, idx = nv.full_attn_block_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk, block=64)
    res = _run(w, inp, swa, idx)
    _check_rows(w, inp, swa, idx, res, 0, np.arange(0, w.n_q, 3))


def test_merged_branches_on_the_shared_cache_are_the_union_layer():
    """With the window branch reading the shared cache, the LSE merge of the two
    GPU branches reproduces the GPU's HySparse2 sparse layer (idx U window)."""
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda")
    _, _, idx = nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk)
    q = inp["q_sparse"][0]
    o_w, l_w, o_s, l_s = nv.swa_branches(q, inp["k"], inp["v"], inp["k"], inp["v"], idx, window=w.window)
    union = nv.sparse_attn(q, inp["k"], inp["v"], idx, window=w.window)
    torch.cuda.synchronize()
    lse = torch.logaddexp(l_w, l_s)
    a = torch.exp(l_w - lse)[..., None]
    b = torch.exp(l_s - lse)[..., None]
    merged = a * o_w.double() + b * o_s.double()
    P.assert_close(P.to_f64(merged), P.to_f64(union), "merged branches vs union layer")


def test_prefill_32k_branches_sampled():
    w = wl.WORKLOADS["prefill_32k"]
    inp = wl.make_inputs(w, "cuda")
    swa = wl.make_swa_cache(w, "cuda")
    _, _, idx = nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk)
    res = _run(w, inp, swa, idx)
    errs = _check_rows(w, inp, swa, idx, res, 0, wl.stratified_rows(w, 8))
    print("32k branches", errs)


def test_checked_build_reports_invalid_selection_in_the_selected_branch():
    """The checked build validates the selected branch's idx rows like the union
    layer's: an index inside the window is reported through the error word."""
    w = wl.custom("bad_branch_idx", n_q=64, q_pos0=500, h_q=8, h_kv=1, head_dim=64, window=32, topk=16, seed=2)
    inp = wl.make_inputs(w, "cuda")
    swa = wl.make_swa_cache(w, "cuda")
    nv.load(True)
    _, _, idx = nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk, q_pos0=w.q_pos0,
                                    checked=True)
    shape = nv.shape_of(inp["q"], inp["k"], window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    ws = nv.alloc_workspace(shape, nv.HS2_ENTRY_SPARSE, checked=True)
    q = inp["q_sparse"][0]
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    l1 = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    l2 = torch.empty_like(l1)
    nv.hs2_swa_branches(shape, q, swa["k_swa"], swa["v_swa"], inp["k"], inp["v"], idx, o1, l1, o2, l2, ws,
                        checked=True)
    rc, info = nv.hs2_get_device_status(ws, checked=True)
    assert rc == nv.HS2_OK, (rc, info)
    bad = idx.clone()
    bad[0, 0, 7, 2] = w.q_pos0 + 7  # the query itself: inside the window
    nv.hs2_swa_branches(shape, q, swa["k_swa"], swa["v_swa"], inp["k"], inp["v"], bad, o1, l1, o2, l2, ws,
                        checked=True)
    rc, info = nv.hs2_get_device_status(ws, checked=True)
    assert rc == 5 and info[1] == 4, (rc, info)

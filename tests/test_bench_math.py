"""The measurement arithmetic of bench.py on CPU: the algorithmic work per
kernel (the numerators of every roofline fraction) against the figures worked
out by hand for the workloads (causal pairs, FLOPs, gathered bytes), and the
roofline assembly on a made-up per-kernel profile."""
import math

import pytest

import bench
from long_context_sparse_flash_b200 import workloads as wl


@pytest.mark.parametrize("name,pairs,full_tf,qk_tf,kv_mb,attended", [
    # P = sum over queries of (t + 1); K1 FLOPs = 4 D H_q P; QK^T over every pair = 2 D H_q P;
    # K+V bytes = 2 B H_kv kv_len D 2; A = sum of min(K, n_cand) + min(t + 1, W)
    ("tiny", 2.10e6, 4.30e-3, 2.15e-3, 1.05, 7.13e5),
    ("prefill_32k", 5.37e8, 8.80, 4.40, 67.1, 3.71e7),
    ("chunk_256k", 2.18e9, 35.7, 17.9, 554, 9.44e6),
    ("chunk_1m", 4.30e9, 70.5, 35.3, 2156, 4.72e6),
])
def test_algorithmic_work_matches_the_hand_figures(name, pairs, full_tf, qk_tf, kv_mb, attended):
    w = wl.WORKLOADS[name]
    f = wl.flops_and_bytes(w)
    assert f["pairs"] == pytest.approx(pairs, rel=6e-3)
    assert f["full_flops"] / 1e12 == pytest.approx(full_tf, rel=6e-3)
    # the hand figure counts QK^T over every causal pair; the selection sweep only
    # recomputes it for the candidates, i.e. without each query's min(t + 1, W) window pairs
    D, Hq = w.head_dim, w.h_q
    assert 2 * D * Hq * f["pairs"] / 1e12 == pytest.approx(qk_tf, rel=6e-3)
    t = range(w.q_pos0, w.q_pos0 + w.n_q)
    window_pairs = sum(min(x + 1, w.window) for x in t) * w.batch
    assert f["select_qk_flops"] == pytest.approx(2 * D * Hq * (f["pairs"] - window_pairs), rel=1e-12)
    assert f["kv_bytes"] / 1e6 == pytest.approx(kv_mb, rel=6e-3)
    assert f["attended"] == pytest.approx(attended, rel=6e-3)


def test_closed_forms_for_a_small_case():
    """n_q = 300 from position 0, W = 16, K = 40: sums written out."""
    w = wl.custom("cf", n_q=300, h_q=8, h_kv=2, head_dim=64, window=16, topk=40)
    f = wl.flops_and_bytes(w)
    assert f["pairs"] == 300 * 301 / 2
    n_cand = [max(0, t - 15) for t in range(300)]
    assert f["cand"] == sum(n_cand) * 2
    A = sum(min(c, 40) + min(t + 1, 16) for t, c in zip(range(300), n_cand))
    assert f["attended"] == A
    assert f["sparse_bytes_per_layer"] == A * 2 * 64 * 2 * 2
    assert f["full_flops"] == 4 * 64 * 8 * f["pairs"]


def test_roofline_assembly():
    """Each kernel's achieved figure is its work per call x calls / event time,
    against the peak of its bound; the reported kernel is the slowest."""
    w = wl.WORKLOADS["prefill_32k"]
    work = bench.kernel_work(w)
    K = 2
    prof = {"full_attn": (14.0, 2), "sparse_attn": (36.0, 8), "select_filter": (18.0, 2), "select_thresh": (0.4, 2)}
    pk = dict(hbm=6552.0, tc=1590.0, tc_sustained=1403.2, src="measured", l2_gather=19000.0, ex2=4.6e12)
    rf, per = bench.roofline(w, prof, K, pk)
    tf = work["full_attn"]["flops"] * K / (14.0 / 1e3) / 1e12
    assert per["full_attn"]["achieved"] == pytest.approx(tf, rel=1e-4)
    assert per["full_attn"]["frac"] == pytest.approx(tf / 1403.2, rel=1e-3)
    gbs = work["sparse_attn"]["bytes"] * K * w.n_sparse / (36.0 / 1e3) / 1e9
    assert per["sparse_attn"]["bound"] == "l2" and per["sparse_attn"]["achieved"] == pytest.approx(gbs, rel=1e-4)
    gex = work["select_filter"]["ex2"] * K / (18.0 / 1e3) / 1e9
    assert per["select_filter"]["bound"] == "alu" and per["select_filter"]["achieved"] == pytest.approx(gex, rel=1e-4)
    assert "bound" not in per["select_thresh"]  # no roofline for the small helper kernels
    assert rf["kernel"] == "sparse_attn" and rf["frac"] == per["sparse_attn"]["frac"]


def test_job_value_is_whole_job_tokens_over_the_slowest_rank():
    assert bench.job_value(1000, 4, 10, 2000.0) == pytest.approx(1000 * 4 * 10 / 2.0)
    assert math.isclose(bench.job_value(32768, 1, 10, 350.0), 32768 * 10 / 0.35)


def test_sparse_layer_two_roofs():
    """With the distinct rows known, the sparse layer carries two roofs: every
    attended row against the L2 gather peak, each distinct row once against HBM;
    the one nearer its roof is the reported bound."""
    w = wl.WORKLOADS["chunk_1m"]
    unique = 4 * 900_000.0
    work = bench.kernel_work(w, unique)
    f = wl.flops_and_bytes(w)
    io = 2 * f["q_bytes"] + f["idx_bytes"]
    assert work["sparse_attn"]["hbm_bytes"] == unique * 128 * 2 * 2 + io
    assert work["sparse_attn"]["bytes"] == f["sparse_bytes_per_layer"] + io
    K = 2
    pk = dict(hbm=6552.0, tc=1590.0, tc_sustained=1403.2, src="measured", l2_gather=19000.0, ex2=4.6e12)
    ms = 6.0  # 8 launches
    rf, per = bench.roofline(w, {"sparse_attn": (ms, 8)}, K, pk, unique)
    e = per["sparse_attn"]
    l2 = work["sparse_attn"]["bytes"] * 8 / (ms / 1e3) / 1e9
    hbm = work["sparse_attn"]["hbm_bytes"] * 8 / (ms / 1e3) / 1e9
    assert e["l2"]["achieved"] == pytest.approx(l2, rel=1e-4)
    assert e["hbm"]["achieved"] == pytest.approx(hbm, rel=1e-4)
    want = "l2" if l2 / 19000.0 >= hbm / 6552.0 else "hbm"
    assert e["bound"] == want and rf["bound"] == want
    assert rf["frac"] == e[want]["frac"]


def test_unique_rows_counts_the_union_of_selections_and_windows():
    import torch
    w = wl.custom("u", n_q=3, q_pos0=20, kv_len=23, h_q=2, h_kv=2, head_dim=64, window=4, topk=3)
    idx = torch.full((1, 2, 3, 3), -1, dtype=torch.int32)
    idx[0, 0, 0] = torch.tensor([0, 5, 9])
    idx[0, 0, 1] = torch.tensor([5, 9, 16])   # 16 lies just below the windows' union [17, 22]
    idx[0, 1, 2] = torch.tensor([1, -1, -1])
    # windows: t in [20, 22] -> rows [17, 22] (6 rows) per head
    assert bench.unique_kv_rows(w, idx) == (6 + 4) + (6 + 1)

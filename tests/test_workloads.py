"""The workload table follows the pages' constants and the generator is seeded."""
import json
import os

import numpy as np
import torch

from long_context_sparse_flash_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_constants.json")


def test_paper_scale_workloads_use_page_constants():
    c = json.load(open(GOLDEN))
    for name in ("prefill_32k", "chunk_256k", "decode_128k", "chunk_1m", "decode_1m"):
        w = wl.WORKLOADS[name]
        assert w.window == c["window"]["value"]
        assert w.topk == c["topk"]["value"]
        assert w.n_sparse >= 1


def test_generator_is_deterministic_and_shaped():
    w = wl.custom(n_q=300, h_q=8, h_kv=2, head_dim=32, topk=16, needles=4, n_sparse=2)
    a = wl.make_inputs(w, "cpu")
    b = wl.make_inputs(w, "cpu")
    for key in ("q", "k", "v"):
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key])
    assert a["q"].shape == (1, 8, 300, 32)
    assert a["k"].shape == (1, 2, 300, 32)
    assert len(a["q_sparse"]) == 2 and not torch.equal(a["q_sparse"][0], a["q_sparse"][1])
    c = wl.make_inputs(w, "cpu", seed=5)
    assert not torch.equal(a["k"], c["k"])


def test_needles_are_planted_older_than_window():
    w = wl.custom(n_q=2048, h_q=8, h_kv=2, head_dim=64, topk=64, needles=8)
    x = wl.make_inputs(w, "cpu")
    probes = x["probes"][0]
    assert len(probes) == 2048 // 64
    # a planted key is 2 * unit vector + 0.1 noise: its norm is close to 2,
    # far below a N(0, 0.25) key's norm (about 0.5 * sqrt(64) = 4)
    norms = x["k"][0].float().norm(dim=-1)
    planted = (norms < 2.6).sum().item()
    assert planted >= 8 * len([p for p in probes if p - w.window + 1 >= 8]) * 2 * 0.9


def test_segment_keys_cluster():
    w = wl.custom(n_q=64, q_pos0=40000, kv_len=40064, h_q=4, h_kv=1, head_dim=32, keys="segments")
    x = wl.make_inputs(w, "cpu", with_sparse=False)
    k = x["k"][0, 0].float()
    # document segments have per-token spread 0.3 around a centroid: adjacent
    # keys inside one are much closer than two independent N(0,1) keys
    d = (k[1:] - k[:-1]).norm(dim=-1)
    assert (d < 0.3 * np.sqrt(2 * 32) * 1.3).float().mean() > 0.2


def test_stratified_rows_cover_boundaries():
    w = wl.WORKLOADS["prefill_32k"]
    rows = wl.stratified_rows(w, 8)
    for t in (0, 127, 128, 129, 127 + 1024, 32767):
        assert t in rows

"""GPU parity of the KV-bridging projection (xiawanshe.com report, section
"两级KV共享", first level): the tcgen05 kernel through the C ABI against the
fp64 oracle on the same seeded bf16 inputs.  Every written cache row is compared;
rows the call must not touch are checked to be unchanged."""
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


def _sentinel_caches(batch, h_kv, kv_cap, d):
    k = torch.full((batch, h_kv, kv_cap, d), 7.0, dtype=torch.bfloat16, device="cuda")
    v = torch.full((batch, h_kv, kv_cap, d), -3.0, dtype=torch.bfloat16, device="cuda")
    return k, v


def _check(inp, k_cache, v_cache, rows_of_b, h_kv, d, sample=None):
    """rows_of_b[b] = cache rows written for sequence b (in token order)."""
    hidden, w = inp["hidden"], inp["w_kv"]
    B, n_new, d_model = hidden.shape
    toks = range(n_new) if sample is None else sample
    for b in range(B):
        rows = np.asarray(rows_of_b[b])
        sel = np.asarray(list(toks))
        ok_, ov_ = oracle.kv_bridge(P.bits(hidden[b, sel]), P.bits(w), h_kv=h_kv, head_dim=d)
        gk = P.to_f64(k_cache[b][:, rows[sel]].permute(1, 0, 2))
        gv = P.to_f64(v_cache[b][:, rows[sel]].permute(1, 0, 2))
        P.assert_close(gk, ok_, f"K of sequence {b}")
        P.assert_close(gv, ov_, f"V of sequence {b}")
        untouched = np.setdiff1d(np.arange(k_cache.shape[2]), rows)
        assert torch.all(k_cache[b][:, untouched] == 7.0) and torch.all(v_cache[b][:, untouched] == -3.0)


@pytest.mark.parametrize("batch,n_new,d_model,h_kv,d,pos0,kv_cap", [
    (2, 300, 1024, 4, 128, 600, 1000),   # ragged token tile, prefill-chunk placement
    (1, 128, 512, 4, 64, 0, 128),        # D = 64, exact tiles, cache filled from 0
    (3, 77, 192, 2, 128, 5, 90),         # three K-steps, 2 heads
])
def test_bridge_prefill_placement(batch, n_new, d_model, h_kv, d, pos0, kv_cap):
    inp = wl.make_bridge_inputs(batch, n_new, d_model, h_kv, d, "cuda", seed=3)
    k, v = _sentinel_caches(batch, h_kv, kv_cap, d)
    before = nv.hs2_launch_count()
    nv.kv_bridge(inp["hidden"], inp["w_kv"], k, v, pos0=pos0)
    torch.cuda.synchronize()
    assert nv.hs2_launch_count() == before + 1
    _check(inp, k, v, [np.arange(pos0, pos0 + n_new)] * batch, h_kv, d)


def test_bridge_decode_append_ragged_positions():
    """The decode-time cache append: one new token per sequence at its own row."""
    batch, d_model, h_kv, d, kv_cap = 5, wl.BRIDGE_D_MODEL, 4, 128, 2048
    inp = wl.make_bridge_inputs(batch, 1, d_model, h_kv, d, "cuda", seed=4)
    k, v = _sentinel_caches(batch, h_kv, kv_cap, d)
    pos = torch.tensor([0, 17, 1000, 2047, 5], dtype=torch.int64, device="cuda")
    nv.kv_bridge(inp["hidden"], inp["w_kv"], k, v, seq_pos=pos)
    torch.cuda.synchronize()
    _check(inp, k, v, [[p] for p in pos.tolist()], h_kv, d)


def test_bridge_full_size_chunk_sampled_rows():
    """32768 new tokens of a 4096-wide hidden state (the 32K prefill's bridging),
    compared on seeded rows across every token tile and the tail."""
    n_new, h_kv, d = 32768, 4, 128
    inp = wl.make_bridge_inputs(1, n_new, wl.BRIDGE_D_MODEL, h_kv, d, "cuda", seed=5)
    k, v = _sentinel_caches(1, h_kv, n_new, d)
    nv.kv_bridge(inp["hidden"], inp["w_kv"], k, v, pos0=0)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    sample = sorted(set(rng.choice(n_new, 48, replace=False).tolist()) | {0, 127, 128, n_new - 1})
    hidden, w = inp["hidden"], inp["w_kv"]
    ok_, ov_ = oracle.kv_bridge(P.bits(hidden[0, sample]), P.bits(w), h_kv=h_kv, head_dim=d)
    P.assert_close(P.to_f64(k[0][:, sample].permute(1, 0, 2)), ok_, "K")
    P.assert_close(P.to_f64(v[0][:, sample].permute(1, 0, 2)), ov_, "V")


def test_bridge_out_of_range_position_reported_and_skipped():
    batch, d_model, h_kv, d, kv_cap = 3, 256, 4, 64, 32
    inp = wl.make_bridge_inputs(batch, 2, d_model, h_kv, d, "cuda", seed=6)
    k, v = _sentinel_caches(batch, h_kv, kv_cap, d)
    pos = torch.tensor([3, 31, 10], dtype=torch.int64, device="cuda")  # sequence 1 would write row 32
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    nv.kv_bridge(inp["hidden"], inp["w_kv"], k, v, seq_pos=pos, ws=ws)
    rc, info = nv.hs2_get_device_status(ws)
    assert rc == 5 and info[1] == 11, (rc, info)  # HS2_ERR_DEVICE_CHECK from the bridging kernel
    assert torch.all(k[1] == 7.0) and torch.all(v[1] == -3.0)  # nothing of sequence 1 is written
    _check({"hidden": inp["hidden"][[0, 2]], "w_kv": inp["w_kv"]}, k[[0, 2]], v[[0, 2]],
           [[3, 4], [10, 11]], h_kv, d)


@pytest.mark.parametrize("batch,n_new,d_model,h_kv,d", [
    (64, 1, wl.BRIDGE_D_MODEL, 4, 128),   # the 128K decode step's append: 4 CTAs without the split
    (8, 1, 448, 2, 128),                  # 7 K-steps: a split into uneven parts
    (3, 40, 1024, 4, 64),                 # several tokens per sequence, D = 64
])
def test_bridge_split_path(batch, n_new, d_model, h_kv, d):
    """With hs2_kv_bridge_workspace_size bytes, few-token calls split d_model over
    more CTAs and sum fp32 partials in a second kernel; same rows, oracle parity."""
    from long_context_sparse_flash_b200 import native
    inp = wl.make_bridge_inputs(batch, n_new, d_model, h_kv, d, "cuda", seed=8)
    kv_cap = 300
    k, v = _sentinel_caches(batch, h_kv, kv_cap, d)
    ws = native.kv_bridge_workspace(inp["hidden"], k)
    assert ws.numel() > 256  # the split path is taken
    pos = torch.tensor([(37 * b) % (kv_cap - n_new + 1) for b in range(batch)], dtype=torch.int64, device="cuda")
    before = nv.hs2_launch_count()
    nv.kv_bridge(inp["hidden"], inp["w_kv"], k, v, seq_pos=pos, ws=ws)
    rc, info = nv.hs2_get_device_status(ws)
    assert rc == 0, info
    assert nv.hs2_launch_count() == before + 2  # partials + reduce
    _check(inp, k, v, [list(range(p, p + n_new)) for p in pos.tolist()], h_kv, d)
    # the split and the one-pass kernels agree to fp32 rounding (bf16 outputs within one ulp)
    k2, v2 = _sentinel_caches(batch, h_kv, kv_cap, d)
    nv.kv_bridge(inp["hidden"], inp["w_kv"], k2, v2, seq_pos=pos)
    torch.cuda.synchronize()
    P.assert_close(P.to_f64(k), P.to_f64(k2), "split vs one-pass K", atol=1e-2, rtol=1e-2)


def test_bridge_split_path_reports_out_of_range_sequences():
    batch, d_model, h_kv, d, kv_cap = 4, 512, 4, 64, 16
    inp = wl.make_bridge_inputs(batch, 1, d_model, h_kv, d, "cuda", seed=9)
    k, v = _sentinel_caches(batch, h_kv, kv_cap, d)
    ws = nv.kv_bridge_workspace(inp["hidden"], k)
    pos = torch.tensor([0, 16, 5, -1], dtype=torch.int64, device="cuda")  # sequences 1 and 3 out of range
    nv.kv_bridge(inp["hidden"], inp["w_kv"], k, v, seq_pos=pos, ws=ws)
    rc, info = nv.hs2_get_device_status(ws)
    assert rc == 5 and info[1] == 11, (rc, info)
    for b in (1, 3):
        assert torch.all(k[b] == 7.0) and torch.all(v[b] == -3.0)
    _check({"hidden": inp["hidden"][[0, 2]], "w_kv": inp["w_kv"]}, k[[0, 2]], v[[0, 2]], [[0], [5]], h_kv, d)

"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/hs2.h declares, sizes workspaces, and rejects invalid
arguments before touching the device."""
import ctypes
import os
import re

import pytest

from long_context_sparse_flash_b200 import native as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hs2.h")

# a fake, 256-byte-aligned device address: never dereferenced by host validation
FAKE = ctypes.c_void_p(1 << 40)


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hs2_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module", params=[False, True], ids=["release", "checked"])
def lib(request):
    return request.param, nv.load(request.param)


def test_every_declared_symbol_is_exported(lib):
    checked, L = lib
    syms = declared_symbols()
    assert len(syms) >= 10
    for s in syms:
        assert hasattr(L, s), s
    assert set(syms) == set(nv.EXPORTS)
    assert nv.hs2_is_checked_build(checked) == checked


def shape(**kw):
    base = dict(batch=1, n_q=256, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024, q_pos0=0,
                kv_len=256)
    base.update(kw)
    return nv.make_shape(**base)


def test_workspace_size_rules():
    assert nv.hs2_workspace_size(shape(), nv.HS2_ENTRY_SPARSE) == 256
    # no row has more than topk candidates: header only
    assert nv.hs2_workspace_size(shape(), nv.HS2_ENTRY_FULL_SELECT) == 256
    s = shape(n_q=4096, kv_len=4096)
    n = nv.hs2_workspace_size(s, nv.HS2_ENTRY_FULL_SELECT)
    cand = 4096 - 128
    # prefill: per-SM survivor lists (256 slots x 32 rows x capacity) + 4108 B of state per row
    cap = (cand + 31) // 32 * 32
    assert n == 256 + 256 * 32 * cap * 8 + 4 * 4096 * (1024 * 4 + 12)
    # decode: every candidate's score, the chunk states and the stored logits
    d = shape(n_q=1, batch=8, q_pos0=4095, kv_len=4096)
    scores = 8 * 4 * ((cand + 3) // 4 * 4) * 4
    want = -(-(4 * 148 + 31) // 32)                 # chunks wanted per (sequence, group)
    chunk = max(256, -(-(-(-4096 // want)) // 64) * 64)
    n_chunks = -(-4096 // chunk)
    part = 8 * 4 * n_chunks * (8 * 128 + 16) * 4
    logits = 8 * 4 * 4096 * 8 * 4
    rnd = lambda x: -(-x // 256) * 256
    assert nv.hs2_workspace_size(d, nv.HS2_ENTRY_DECODE) == 256 + rnd(scores) + rnd(part) + rnd(logits)
    # invalid shapes size to 0
    assert nv.hs2_workspace_size(shape(h_q=30), nv.HS2_ENTRY_FULL_SELECT) == 0
    assert nv.hs2_workspace_size(shape(q_pos0=1), nv.HS2_ENTRY_FULL_SELECT) == 0
    assert nv.hs2_workspace_size(shape(), 99) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(h_q=30), 1),                                      # h_q % h_kv != 0
    (dict(h_q=48, h_kv=4), 2),                              # G = 12 unsupported
    (dict(head_dim=96), 2),
    (dict(window=0), 1),
    (dict(window=2048), 2),
    (dict(topk=-1), 1),
    (dict(topk=4096), 2),
    (dict(q_pos0=10), 1),                                   # q_pos0 + n_q > kv_len
    (dict(n_q=-1), 1),
    (dict(batch=70000), 2),
])
def test_invalid_shapes_rejected_without_launch(kw, status):
    L = nv.load()
    before = nv.hs2_launch_count()
    s = shape(**kw)
    rc = L.hs2_full_attn_select(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert rc == status
    rc = L.hs2_sparse_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None)
    assert rc == status
    assert nv.hs2_launch_count() == before


def test_pointer_and_workspace_checks():
    L = nv.load()
    s = shape(n_q=4096, kv_len=4096)
    need = nv.hs2_workspace_size(s, nv.HS2_ENTRY_FULL_SELECT)
    args = [FAKE] * 7
    assert L.hs2_full_attn_select(None, *args, need, None) == 1
    assert L.hs2_full_attn_select(ctypes.byref(s), None, *args[1:], need, None) == 1
    assert L.hs2_full_attn_select(ctypes.byref(s), *args, need - 1, None) == 3
    mis = ctypes.c_void_p((1 << 40) + 8)
    assert L.hs2_full_attn_select(ctypes.byref(s), mis, *args[1:], need, None) == 1
    bad = shape()
    bad.reserved = 1
    assert L.hs2_full_attn_select(ctypes.byref(bad), *args, need, None) == 1
    # decode needs n_q == 1
    assert L.hs2_decode(ctypes.byref(s), None, *args, need, None) == 1
    # sparse: ws_bytes without ws
    assert L.hs2_sparse_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, 64, None) == 1
    # nan scale
    s2 = shape(n_q=4096, kv_len=4096, softmax_scale=float("nan"))
    assert L.hs2_full_attn_select(ctypes.byref(s2), *args, need, None) == 1


def test_selftest_wait_argument_checks():
    """The bounded-wait self-test validates its workspace and bound on the host,
    before any launch."""
    L = nv.load()
    before = nv.hs2_launch_count()
    ws = ctypes.c_void_p(1 << 40)  # 256-byte aligned fake device address
    assert L.hs2_selftest_wait(None, 256, 1 << 20, None) == 1
    assert L.hs2_selftest_wait(ws, 255, 1 << 20, None) == 1
    assert L.hs2_selftest_wait(ctypes.c_void_p((1 << 40) + 16), 256, 1 << 20, None) == 1
    assert L.hs2_selftest_wait(ws, 256, 0, None) == 1
    assert L.hs2_selftest_wait(ws, 256, (1 << 32) + 1, None) == 1
    assert nv.hs2_launch_count() == before


def test_empty_calls_are_noops():
    L = nv.load()
    before = nv.hs2_launch_count()
    for kw in (dict(batch=0), dict(n_q=0)):
        s = shape(**kw)
        assert L.hs2_full_attn_select(ctypes.byref(s), None, None, None, None, None, None, None, 0, None) == 0
        assert L.hs2_sparse_attn(ctypes.byref(s), None, None, None, None, None, None, 0, None) == 0
        d = shape(**kw, **({} if "n_q" in kw else {"n_q": 1}))
        assert L.hs2_decode(ctypes.byref(d), None, None, None, None, None, None, None, None, 0, None) == 0
    assert nv.hs2_launch_count() == before


def test_status_strings():
    for code in range(7):
        assert nv.hs2_status_string(code) != "unknown status"
    assert nv.hs2_status_string(42) == "unknown status"


def test_binding_refuses_host_tensors():
    import torch
    q = torch.zeros(1, 8, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        nv.sparse_attn(q, q[:, :2], q[:, :2], torch.zeros(1, 2, 4, 1, dtype=torch.int32), window=2)


def test_gather_probe_argument_checks():
    """The diagnostic gather probe rejects bad sizes and pointers on the host."""
    L = nv.load()
    before = nv.hs2_launch_count()
    assert L.hs2_gather_probe(None, 16, FAKE, 32, 1, FAKE, None) == 1
    assert L.hs2_gather_probe(FAKE, 16, FAKE, 16, 1, FAKE, None) == 1   # n_order not a multiple of 32
    assert L.hs2_gather_probe(FAKE, 16, FAKE, 32, 0, FAKE, None) == 1   # passes < 1
    assert L.hs2_gather_probe(FAKE, 0, FAKE, 32, 1, FAKE, None) == 1    # no rows
    assert L.hs2_gather_probe(ctypes.c_void_p((1 << 40) + 4), 16, FAKE, 32, 1, FAKE, None) == 1  # misaligned
    assert nv.hs2_launch_count() == before


def test_ex2_probe_argument_checks():
    L = nv.load()
    n = ctypes.c_int64(0)
    before = nv.hs2_launch_count()
    assert L.hs2_ex2_probe(0, FAKE, None, ctypes.byref(n)) == 1
    assert L.hs2_ex2_probe(4, None, None, ctypes.byref(n)) == 1
    assert L.hs2_ex2_probe(4, FAKE, None, None) == 1
    assert nv.hs2_launch_count() == before


def test_kv_bridge_validation_without_launch():
    L = nv.load()
    before = nv.hs2_launch_count()

    def bs(**kw):
        base = dict(batch=1, n_new=16, d_model=256, h_kv=4, head_dim=128, reserved=0, pos0=0, kv_cap=64)
        base.update(kw)
        return nv.hs2_bridge_shape(**base)

    def call(s, seq=None, ws=None, ws_bytes=0):
        return L.hs2_kv_bridge(ctypes.byref(s), seq, FAKE, FAKE, FAKE, FAKE, ws, ws_bytes, None)

    assert L.hs2_kv_bridge(None, None, FAKE, FAKE, FAKE, FAKE, None, 0, None) == 1
    assert call(bs(reserved=1)) == 1
    assert call(bs(d_model=100)) == 2            # d_model not a multiple of 64
    assert call(bs(head_dim=96)) == 2
    assert call(bs(h_kv=1)) == 2                 # h_kv * D = 128: a 256-feature tile would span K and V
    assert call(bs(pos0=60)) == 1                # pos0 + n_new > kv_cap
    assert call(bs(pos0=-1)) == 1
    assert call(bs(), ws=FAKE, ws_bytes=100) == 3  # workspace smaller than the header
    assert call(bs(), ws=None, ws_bytes=256) == 1
    assert call(bs(n_new=0)) == 0                # empty: no launch
    assert call(bs(batch=0)) == 0
    # workspace for the split path: fp32 partials of every split when few CTAs would stream W_kv
    ws_size = lambda sh: L.hs2_kv_bridge_workspace_size(ctypes.byref(sh))
    assert ws_size(bs(batch=64, n_new=1, d_model=4096, kv_cap=300)) == 256 + 32 * 64 * 1024 * 4
    assert ws_size(bs(batch=1, n_new=32768, d_model=4096, kv_cap=32768)) == 256  # enough token tiles
    assert ws_size(bs(d_model=100)) == 0
    assert nv.hs2_launch_count() == before


def test_block_select_validation_without_launch():
    """Block-level selection entry: block size, workspace, pointers, empty calls."""
    L = nv.load()
    before = nv.hs2_launch_count()
    s = shape(n_q=4096, kv_len=4096)
    need = nv.hs2_workspace_size(s, nv.HS2_ENTRY_BLOCK_SELECT)
    # one float per 32 candidate keys of every 128-key tile, for every (query, group) row
    cand = 4096 - 128
    assert need == 256 + 4 * 4096 * (-(-cand // 128) * 4) * 4
    args = [FAKE] * 7

    def call(sh, blk, *a, ws_bytes=need):
        return L.hs2_full_attn_block_select(ctypes.byref(sh) if sh is not None else None, blk, *a, ws_bytes, None)

    for blk in (0, 16, 48, 96, 256, -64):
        assert call(s, blk, *args) == 2
    assert call(None, 64, *args) == 1
    assert call(s, 64, None, *args[1:]) == 1
    assert call(s, 64, *args, ws_bytes=need - 1) == 3
    assert call(s, 64, ctypes.c_void_p((1 << 40) + 8), *args[1:]) == 1
    assert call(shape(h_q=30), 64, *args) == 1
    for kw in (dict(batch=0), dict(n_q=0)):
        assert call(shape(**kw), 64, None, None, None, None, None, None, None, ws_bytes=0) == 0
    # no candidate at all: the header only (plus the full layer's own split scratch, none here)
    assert nv.hs2_workspace_size(shape(n_q=100, kv_len=100), nv.HS2_ENTRY_BLOCK_SELECT) == 256
    assert nv.hs2_launch_count() == before


def test_block_select_chunks_in_whole_waves():
    """At the 1M chunk the chunk sums of all 4096 queries exceed the 1 GiB budget,
    so the sweep runs over chunks of queries; each chunk is a whole number of
    waves of one-CTA-per-SM sweeps (148 CTAs of 28 queries for G = 8 above 2^18
    candidates, 32 queries for G = 2), and the workspace holds one chunk."""
    def expected(s_kw, qt):
        s = shape(**s_kw)
        B, hkv, nq, D, hq = s_kw["batch"], s_kw["h_kv"], s_kw["n_q"], s_kw["head_dim"], s_kw["h_q"]
        cand = s_kw["q_pos0"] + nq - s_kw["window"]
        per_q = B * hkv * (-(-cand // 128) * 4) * 4
        fit = (1 << 30) // per_q
        wave_q = 148 // (hkv * B) * qt
        chunk = fit // wave_q * wave_q
        # the full layer's split parts (2 key ranges at this shape) share the body with the sums
        split = 2 * B * hq * nq * (D * 4 + 4) + 256
        return nv.hs2_workspace_size(s, nv.HS2_ENTRY_BLOCK_SELECT), 256 + max(split, chunk * per_q), chunk
    kw = dict(batch=1, n_q=4096, h_q=32, h_kv=4, head_dim=128, window=128, topk=1024, q_pos0=1048576,
              kv_len=1052672)
    got, want, chunk = expected(kw, 28)
    assert chunk == 1036 and got == want
    kw2 = dict(kw, h_q=8)  # G = 2: the 32-query geometry
    got, want, chunk = expected(kw2, 32)
    assert chunk == 1184 and got == want


def test_swa_branches_validation_without_launch():
    """The two-branch comparator entry: shape, pointers, alignment, workspace, empty calls."""
    L = nv.load()
    before = nv.hs2_launch_count()
    s = shape(n_q=512, kv_len=4096, q_pos0=3584)
    ptrs = [FAKE] * 10  # q, k_swa, v_swa, k, v, idx, out_swa, lse_swa, out_sel, lse_sel

    def call(sh, *a, ws=None, ws_bytes=0):
        return L.hs2_swa_branches(ctypes.byref(sh) if sh is not None else None, *a, ws, ws_bytes, None)

    assert call(None, *ptrs) == 1
    assert call(shape(h_q=30), *ptrs) == 1
    assert call(shape(head_dim=96), *ptrs) == 2
    for i in range(10):
        bad = list(ptrs)
        bad[i] = None
        assert call(s, *bad) == 1, i
    mis = list(ptrs)
    mis[1] = ctypes.c_void_p((1 << 40) + 8)  # k_swa not 16-byte aligned
    assert call(s, *mis) == 1
    assert call(s, *ptrs, ws=FAKE, ws_bytes=100) == 3
    assert call(s, *ptrs, ws=None, ws_bytes=256) == 1
    for kw in (dict(batch=0), dict(n_q=0)):
        assert call(shape(**kw), *([None] * 10)) == 0
    assert nv.hs2_launch_count() == before


def test_context_parallel_validation_without_launch():
    """Slice calls and merges: shapes, offsets, workspace, sizes -- checked on the host."""
    L = nv.load()
    before = nv.hs2_launch_count()
    s = shape(n_q=256, q_pos0=5000, kv_len=2000)  # a slice of 2000 keys; queries after it
    for e in (nv.HS2_ENTRY_CP_ATTN, nv.HS2_ENTRY_CP_SELECT, nv.HS2_ENTRY_CP_SPARSE):
        assert nv.hs2_cp_workspace_size(s, 1000, e) >= 256
        assert nv.hs2_cp_workspace_size(s, -1, e) == 0
    assert nv.hs2_cp_workspace_size(s, 0, nv.HS2_ENTRY_FULL_SELECT) == 0
    assert nv.hs2_workspace_size(s, nv.HS2_ENTRY_CP_ATTN) == 0  # slices are sized by the slice call
    # local rows of the sparse step: one int32 per selected entry
    assert nv.hs2_cp_workspace_size(s, 0, nv.HS2_ENTRY_CP_SPARSE) == 256 + 4 * 256 * 1024 * 4
    need = nv.hs2_cp_workspace_size(s, 1000, nv.HS2_ENTRY_CP_ATTN)
    assert L.hs2_cp_attn_partial(ctypes.byref(s), 1000, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None) == 1
    assert L.hs2_cp_attn_partial(ctypes.byref(s), 1000, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, None) == 3
    assert L.hs2_cp_attn_partial(ctypes.byref(s), -5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, None) == 1
    small = shape(n_q=32, q_pos0=5000, kv_len=2000)
    assert L.hs2_cp_attn_partial(ctypes.byref(small), 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, None) == 2
    need_sel = nv.hs2_cp_workspace_size(s, 1000, nv.HS2_ENTRY_CP_SELECT)
    assert L.hs2_cp_select_local(ctypes.byref(s), 1000, FAKE, FAKE, FAKE, None, FAKE, FAKE, need_sel, None) == 1
    # merges
    assert L.hs2_cp_combine(0, 10, 128, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert L.hs2_cp_combine(2, 10, 96, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert L.hs2_cp_combine(2, 0, 128, None, None, None, None, None) == 0
    whole = shape(n_q=256, q_pos0=4000, kv_len=4256)
    offs = (ctypes.c_int64 * 3)(0, 2000, 1000)  # not ascending
    assert L.hs2_cp_select_merge(ctypes.byref(whole), 3, offs, FAKE, FAKE, FAKE, None) == 1
    many = (ctypes.c_int64 * 17)(*range(0, 17 * 100, 100))
    assert L.hs2_cp_select_merge(ctypes.byref(whole), 17, many, FAKE, FAKE, FAKE, None) == 2
    assert nv.hs2_launch_count() == before


def test_slice_offsets():
    from long_context_sparse_flash_b200 import cp
    assert cp.slice_offsets(10, 3) == [0, 4, 7]
    assert cp.slice_offsets(8, 4) == [0, 2, 4, 6]
    assert cp.slice_offsets(5, 1) == [0]
    with pytest.raises(ValueError):
        cp.slice_offsets(2, 3)

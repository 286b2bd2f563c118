"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same bf16 bits, compare.

Comparison rules (the stated tolerance of the method's target, plus the
reading of its near-tie exception):
  * attention outputs: |gpu - ref| <= 1e-2 + 1e-2 * |ref| elementwise;
  * LSE: |gpu - ref| <= 1e-3;
  * selection: every GPU row has the right size min(K, t-W+1), no duplicate,
    ascending entries inside [0, t-W], -1 padding; the GPU set must equal the
    oracle set, except that an index in the symmetric difference is accepted
    when its oracle score lies within min(1e-6, 2e-4 * kth) of the oracle's
    k-th score (a near-tie the fp32 GPU arithmetic cannot order reliably).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from long_context_sparse_flash_b200 import native as nv
from long_context_sparse_flash_b200 import workloads as wl

OUT_ATOL, OUT_RTOL = 1e-2, 1e-2
LSE_ATOL = 1e-3
IDX_ABS_MARGIN, IDX_REL_MARGIN = 1e-6, 2e-4


def bits(t: torch.Tensor) -> np.ndarray:
    return wl.bf16_bits(t)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str, atol=OUT_ATOL, rtol=OUT_RTOL) -> float:
    err = np.abs(gpu - ref)
    tol = atol + rtol * np.abs(ref)
    bad = err > tol
    if bad.any():
        where = np.argwhere(bad)[:5].tolist()
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance, "
                             f"max err {err.max():.3g}, first at {where}")
    return float(err.max()) if err.size else 0.0


def check_idx(gpu_idx: np.ndarray, ores: dict, ts: np.ndarray, window: int, topk: int, what="idx") -> dict:
    """gpu_idx [n_rows, H_kv, topk]; ores from oracle.full_select(..., want_scores=True)."""
    n_rows, h_kv, _ = gpu_idx.shape
    stats = dict(rows=0, rows_differing=0, max_sym_diff=0)
    for r in range(n_rows):
        t = int(ts[r])
        n_sel = min(topk, max(0, t - window + 1))
        for g in range(h_kv):
            row = gpu_idx[r, g]
            sel = row[:n_sel]
            assert np.all(row[n_sel:] == -1), f"{what} row t={t} g={g}: bad padding"
            if n_sel:
                assert np.all(np.diff(sel) > 0), f"{what} row t={t} g={g}: not strictly ascending"
                assert sel[0] >= 0 and sel[-1] <= t - window, f"{what} row t={t} g={g}: out of range"
            got, want = set(sel.tolist()), set(ores["idx"][r, g, :n_sel].tolist())
            stats["rows"] += 1
            diff = got ^ want
            if diff:
                kth = float(ores["kth"][r, g])
                margin = min(IDX_ABS_MARGIN, IDX_REL_MARGIN * kth)
                sc = ores["scores"][r, g]
                for j in diff:
                    gap = abs(float(sc[j]) - kth)
                    assert gap <= margin, (f"{what} row t={t} g={g}: index {j} differs with score gap "
                                           f"{gap:.3g} > margin {margin:.3g} (kth {kth:.6g})")
                stats["rows_differing"] += 1
                stats["max_sym_diff"] = max(stats["max_sym_diff"], len(diff))
    return stats


def check_block_idx(gpu_idx: np.ndarray, ores: dict, ts: np.ndarray, window: int, topk: int, blk: int,
                    what="block idx") -> dict:
    """gpu_idx [n_rows, H_kv, topk]; ores from oracle.block_select.  Every row: the
    first keep * blk entries are keep whole candidate blocks, ascending, then -1;
    the GPU's block set equals the oracle's except for blocks whose oracle score
    lies within min(blk * 1e-6, 2e-4 * kth) of the oracle's last kept block (the
    token near-tie rule, scaled to a sum of blk token scores)."""
    n_rows, h_kv, _ = gpu_idx.shape
    stats = dict(rows=0, rows_differing=0, max_sym_diff=0)
    sc = ores["full"]["scores"]
    for r in range(n_rows):
        t = int(ts[r])
        n_blk = max(0, t - window + 1) // blk
        keep = min(topk // blk, n_blk)
        for g in range(h_kv):
            row = gpu_idx[r, g]
            assert np.all(row[keep * blk:] == -1), f"{what} row t={t} g={g}: bad padding"
            body = row[:keep * blk].reshape(keep, blk) if keep else np.zeros((0, blk), np.int32)
            starts = body[:, 0]
            assert np.all(starts % blk == 0), f"{what} row t={t} g={g}: block not aligned"
            assert np.array_equal(body, starts[:, None] + np.arange(blk)[None, :]), \
                f"{what} row t={t} g={g}: block not contiguous"
            if keep:
                assert np.all(np.diff(starts) > 0), f"{what} row t={t} g={g}: blocks not ascending"
                assert starts[-1] // blk < n_blk, f"{what} row t={t} g={g}: block beyond the candidates"
            got = set((starts // blk).tolist())
            want = set((ores["idx"][r, g, :keep * blk:blk] // blk).tolist())
            stats["rows"] += 1
            diff = got ^ want
            if diff:
                kth = float(ores["kth_block"][r, g])
                margin = min(blk * IDX_ABS_MARGIN, IDX_REL_MARGIN * kth)
                for bb in diff:
                    gap = abs(float(sc[r, g, bb * blk:(bb + 1) * blk].sum()) - kth)
                    assert gap <= margin, (f"{what} row t={t} g={g}: block {bb} differs with score gap "
                                           f"{gap:.3g} > margin {margin:.3g} (kth {kth:.6g})")
                stats["rows_differing"] += 1
                stats["max_sym_diff"] = max(stats["max_sym_diff"], len(diff))
    return stats


def run_gpu(w: wl.Workload, inp: dict, entry: str = "full", checked: bool = False, seq_len=None):
    """Full-attention + selection layer, then every sparse layer, through the C ABI."""
    q, k, v = inp["q"], inp["k"], inp["v"]
    if w.decode:
        out, lse, idx = nv.decode(q, k, v, window=w.window, topk=w.topk, kv_len_per_seq=seq_len,
                                  checked=checked)
        sp = [nv.decode_sparse(qs, k, v, idx, window=w.window, kv_len_per_seq=seq_len, checked=checked)
              for qs in inp["q_sparse"]]
    else:
        out, lse, idx = nv.full_attn_select(q, k, v, window=w.window, topk=w.topk, q_pos0=w.q_pos0,
                                            entry=entry, checked=checked)
        sp = [nv.sparse_attn(qs, k, v, idx, window=w.window, q_pos0=w.q_pos0, checked=checked)
              for qs in inp["q_sparse"]]
    torch.cuda.synchronize()
    return dict(out=out, lse=lse, idx=idx, sparse=sp)


def compare_rows(w: wl.Workload, inp: dict, gpu: dict, b: int, rows: np.ndarray, ts: np.ndarray = None,
                 n_threads: int = 0) -> dict:
    """Oracle on query indices `rows` of sequence b; every check of the module docstring."""
    rows = np.asarray(rows, dtype=np.int64)
    if ts is None:
        ts = w.q_pos0 + rows
    kb = bits(inp["k"][b])
    vb = bits(inp["v"][b])
    qb = np.ascontiguousarray(bits(inp["q"][b][:, rows, :]).transpose(1, 0, 2))
    ores = oracle.full_select(qb, ts, kb, vb, window=w.window, topk=w.topk, want_scores=True,
                              n_threads=n_threads)
    rows_t = torch.as_tensor(rows, device=gpu["out"].device)
    g_out = to_f64(gpu["out"][b][:, rows_t, :]).transpose(1, 0, 2)
    g_lse = to_f64(gpu["lse"][b][:, rows_t]).T
    g_idx = gpu["idx"][b][:, rows_t, :].cpu().numpy().transpose(1, 0, 2)
    res = {}
    res["out_err"] = assert_close(g_out, ores["out"], f"{w.name} full out")
    res["lse_err"] = assert_close(g_lse, ores["lse"], f"{w.name} lse", atol=LSE_ATOL, rtol=0.0)
    res["idx"] = check_idx(g_idx, ores, ts, w.window, w.topk, f"{w.name} idx")
    # each sparse layer, with the GPU's own selection (isolates the sparse kernel)
    g_idx_c = np.ascontiguousarray(g_idx)
    res["sparse_err"] = []
    for layer, (qs, so) in enumerate(zip(inp["q_sparse"], gpu["sparse"])):
        qsb = np.ascontiguousarray(bits(qs[b][:, rows, :]).transpose(1, 0, 2))
        ref = oracle.sparse(qsb, ts, kb, vb, g_idx_c, window=w.window, n_threads=n_threads)
        got = to_f64(so[b][:, rows_t, :]).transpose(1, 0, 2)
        res["sparse_err"].append(assert_close(got, ref, f"{w.name} sparse layer {layer}"))
        if layer == 0:
            # end to end: the oracle's own selection in the oracle's sparse layer
            ref_e2e = oracle.sparse(qsb, ts, kb, vb, ores["idx"], window=w.window, n_threads=n_threads)
            res["sparse_e2e_err"] = assert_close(got, ref_e2e, f"{w.name} sparse layer 0 end to end")
    res["oracle"] = ores
    return res

#!/usr/bin/env python
"""Throughput of the HySparse2 Cross-Decoder attention hot path on B200.

One step = the full-attention + selection layer (hs2_full_attn_select, or
hs2_decode for decode workloads) followed by every sparse KV-reuse layer
(hs2_sparse_attn / hs2_decode_sparse, one call per layer, each with its own
query), over one batch of seeded synthetic input already resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...    # the fp64 CPU oracle, same workload

Prints ONE JSON line on rank 0.  Metric: query tokens/s through the whole
step.  With N > 1 (torchrun), every rank runs an independent replica of the
workload (its own sequences: weak scaling, no data-path collective); value =
all ranks' query tokens / the slowest rank's time.  With --split heads the
ranks instead share one workload by KV-head group (strong scaling, still no
exchange); value = its query tokens / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
from typing import Optional

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_sparse_flash_b200 import native as nv  # noqa: E402
from long_context_sparse_flash_b200 import workloads as wl  # noqa: E402

METRIC = "query tokens/s (full-attn+select + sparse-reuse layers) and % of TC/HBM roofline"
UNIT = "query tokens/s"
FLUSH_BYTES = 256 << 20  # > 126 MB L2
# a call whose K/V (both tensors) is at most this large keeps it in the 126 MB
# L2 between the sparse layer's gathers: that kernel is then bound by L2 gather
# bandwidth, not by HBM
L2_RESIDENT_BYTES = 96 << 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), tc=float(d["bf16_tflops"]),
                    tc_sustained=float(d["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, tc=1590.0, tc_sustained=1400.0, src="fallback")


# ---------------------------------------------------------------------------
# algorithmic work per kernel (per call of the entry point, all sequences)


def kernel_work(w: wl.Workload, unique_rows: Optional[float] = None):
    """Algorithmic work of each kernel per call (all sequences of the call).

    unique_rows: distinct K/V rows the sparse layer touches per call (summed over
    sequences and KV heads: the union of every query's selected rows and window),
    counted from the step's selection; it gives the sparse layer's compulsory
    HBM bytes."""
    f = wl.flops_and_bytes(w)
    Hq = w.h_q
    n_rows = w.batch * w.n_q
    cand = f["cand"]  # sum over (sequence, query, KV head) of candidate counts
    io = 2 * f["q_bytes"] + f["idx_bytes"]
    sparse = dict(bound="l2" if f["kv_bytes"] <= L2_RESIDENT_BYTES else "hbm",
                  bytes=f["sparse_bytes_per_layer"] + io)
    if unique_rows is not None:
        # two roofs: the logical gather (every attended row of every query) against the
        # random-row L2 gather peak, and the compulsory bytes (each distinct row once)
        # against HBM bandwidth; the one nearer its roof binds
        sparse = dict(bound="gather", bytes=f["sparse_bytes_per_layer"] + io,
                      hbm_bytes=unique_rows * w.head_dim * 2 * 2 + io)
    work = {
        # dense causal contraction: QK^T and PV over the causal pairs
        "full_attn": dict(bound="tensor", flops=f["full_flops"]),
        "decode_attn": dict(bound="hbm", bytes=f["kv_bytes"] + 2 * f["q_bytes"] + 4 * n_rows * Hq),
        # gathered K/V rows + q + out + idx, per layer
        "sparse_attn": sparse,
    }
    if w.decode:
        # decode: the attention pass stores each candidate's G scaled logits (fp32); the score
        # kernel streams them (32 B per candidate for G = 8) and writes one fp32 score each;
        # the radix top-k reads every score (at least once) and writes idx
        work["decode_attn"] = dict(bound="hbm", bytes=f["kv_bytes"] + 2 * f["q_bytes"] + 4 * n_rows * Hq
                                   + 4.0 * 8 * cand)
        work["select_score"] = dict(bound="hbm", bytes=(4.0 * 8 + 4.0) * cand)
        work["select_topk"] = dict(bound="hbm", bytes=4.0 * cand + f["idx_bytes"])
    else:
        # prefill: the filtered sweep recomputes QK^T over every candidate of every query
        # and takes one 2^x per (candidate, head): the special-function unit's ex2 rate is
        # the binding limit ("alu"); the tensor-core fraction is reported beside it
        G = w.h_q // w.h_kv
        work["select_filter"] = dict(bound="alu", ex2=G * cand, flops=f["select_qk_flops"],
                                     stream_bytes=select_stream_bytes(w))
    return work


def unique_kv_rows(w: wl.Workload, idx: torch.Tensor) -> float:
    """Distinct K/V rows one sparse layer reads: per (sequence, KV head), the
    union over the call's queries of the selected rows and the window."""
    B, H, nq, K = idx.shape
    total = 0
    for b in range(B):
        # padding (-1) goes to an extra column that is dropped
        mask = torch.zeros(H, w.kv_len + 1, dtype=torch.bool, device=idx.device)
        sel = idx[b].reshape(H, -1).long()
        mask.scatter_(1, torch.where(sel >= 0, sel, w.kv_len), True)
        mask = mask[:, :w.kv_len]
        t_lo = (w.kv_len - 1) if w.decode else w.q_pos0
        t_hi = (w.kv_len - 1) if w.decode else w.q_pos0 + nq - 1
        mask[:, max(0, t_lo - w.window + 1):t_hi + 1] = True
        total += int(mask.sum().item())
    return float(total)


# the selection sweep's CTAs hold 32 queries below this many candidates in the
# call's longest row (the ORDERED layout) and 28 from it on (COUNTER)
SELECT_COUNTER_MIN_CAND = 1 << 18


def select_stream_bytes(w: wl.Workload) -> float:
    """Bytes the filtered sweep streams per call: every CTA (32 queries of one KV
    group, or 28 in the layout used for long rows) reads the K rows of its
    candidate tiles (128 keys each) once, plus the queries, the LSE and the
    written selection.  The fraction of HBM bandwidth this gives is the one
    usually quoted for a select pass; most of the K reads are L2 hits, and the
    binding unit is the ex2 rate."""
    D = w.head_dim
    longest = w.q_pos0 + w.n_q - w.window
    qt = 28 if longest >= SELECT_COUNTER_MIN_CAND else 32
    tiles = 0
    for q0 in range(0, w.n_q, qt):
        t_max = w.q_pos0 + min(q0 + qt, w.n_q) - 1
        cand_end = t_max - w.window + 1
        tiles += max(0, -(-cand_end // 128))
    k_bytes = tiles * 128 * D * 2 * w.h_kv * w.batch
    f = wl.flops_and_bytes(w)
    return float(k_bytes + f["q_bytes"] + 4.0 * w.batch * w.h_q * w.n_q + f["idx_bytes"])


def measure_l2_gather(dev, reps: int = 10) -> float:
    """GB/s of a random 256-byte-row gather from a 64 MiB L2-resident buffer
    (the sparse layer's access pattern), measured here with the library's probe:
    the fastest of `reps` individually timed calls, as a peak should be."""
    g = torch.Generator().manual_seed(7)
    rows = torch.randint(0, 255, (64 << 20,), dtype=torch.uint8, generator=g).to(dev)
    order = torch.randint(0, (64 << 20) // 256, (1 << 22,), dtype=torch.int32, generator=g).to(dev)
    sink = torch.zeros(4, dtype=torch.int32, device=dev)
    passes = 4
    for _ in range(5):
        nv.hs2_gather_probe(rows, order, passes, sink)
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        e0.record(st)
        nv.hs2_gather_probe(rows, order, passes, sink)
        e1.record(st)
    torch.cuda.synchronize()
    ms = min(e0.elapsed_time(e1) for e0, e1 in ev)
    return order.numel() * 256.0 * passes / (ms / 1e3) / 1e9


def measure_ex2(dev, reps: int = 10) -> float:
    """ex2 per second of the special-function units (the library's probe: 8
    independent 2^x chains per thread, 2048 threads per SM), fastest of `reps`."""
    sink = torch.zeros(4, dtype=torch.float32, device=dev)
    iters = 4096
    for _ in range(3):
        n = nv.hs2_ex2_probe(iters, sink)
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        e0.record(st)
        n = nv.hs2_ex2_probe(iters, sink)
        e1.record(st)
    torch.cuda.synchronize()
    ms = min(e0.elapsed_time(e1) for e0, e1 in ev)
    return n / (ms / 1e3)


def bench_bridge(w: wl.Workload, dev, K: int, warmup: int, pk: dict) -> dict:
    """The KV-bridging projection (a next row of the path) for the workload's new
    tokens: prefill-shaped workloads project all n_q tokens of every sequence and
    write them at q_pos0; decode workloads append one token per sequence.  Timed
    on its own (CUDA events per call, hidden states > L2), not part of `value`."""
    d_model = wl.BRIDGE_D_MODEL
    n_new = 1 if w.decode else w.n_q
    inp = wl.make_bridge_inputs(w.batch, n_new, d_model, w.h_kv, w.head_dim, dev, seed=w.seed)
    cap = w.kv_len
    k = torch.empty(w.batch, w.h_kv, cap, w.head_dim, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    pos = None if not w.decode else torch.full((w.batch,), cap - 1, dtype=torch.int64, device=dev)
    pos0 = 0 if w.decode else w.q_pos0
    ws = nv.kv_bridge_workspace(inp["hidden"], k)  # enables the split path for the decode append
    run = lambda: nv.kv_bridge(inp["hidden"], inp["w_kv"], k, v, pos0=pos0, seq_pos=pos, ws=ws)
    for _ in range(warmup):
        run()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    st = torch.cuda.current_stream()
    torch.cuda.synchronize()
    for e0, e1 in ev:
        e0.record(st)
        run()
        e1.record(st)
    torch.cuda.synchronize()
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    feats = 2 * w.h_kv * w.head_dim
    flops = 2.0 * w.batch * n_new * d_model * feats
    note = "hidden [tokens, d_model] x W_kv^T -> bf16 K/V cache rows (synthetic weights)"
    if w.decode:  # one token per sequence: streaming the weights is the cost
        nbytes = 2.0 * feats * d_model + 2.0 * w.batch * (d_model + feats)
        gbs = nbytes / (ms / 1e3) / 1e9
        return {"ms": round(ms, 4), "tokens": w.batch * n_new, "d_model": d_model, "bound": "hbm",
                "achieved": round(gbs, 2), "peak": pk["hbm"], "unit": "GB/s", "frac": round(gbs / pk["hbm"], 4),
                "note": note}
    tf = flops / (ms / 1e3) / 1e12
    return {"ms": round(ms, 4), "tokens": w.batch * n_new, "d_model": d_model, "bound": "tensor",
            "achieved": round(tf, 2), "peak": pk["tc_sustained"], "unit": "TFLOP/s",
            "frac": round(tf / pk["tc_sustained"], 4), "note": note}


def bench_block_select(w: wl.Workload, inp: dict, dev, K: int, warmup: int, pk: dict, flush: torch.Tensor,
                       token_select_ms: float, blk: int = 64):
    """Block-level selection at the same budget (a next row of the path: the
    design token-level selection replaces), through its own C-ABI entry on the
    same inputs, L2 flushed before every call; per-kernel times from the
    library's event pairs.  Prefill-shaped workloads only; not part of `value`."""
    if w.decode:
        return None
    shape = nv.shape_of(inp["q"], inp["k"], window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    ws = nv.alloc_workspace(shape, nv.HS2_ENTRY_BLOCK_SELECT, dev)
    B, Hq, nq, D = inp["q"].shape
    out = torch.empty_like(inp["q"])
    lse = torch.empty(B, Hq, nq, dtype=torch.float32, device=dev)
    idx = torch.empty(B, w.h_kv, nq, w.topk, dtype=torch.int32, device=dev)
    run = lambda: nv.hs2_full_attn_block_select(shape, blk, inp["q"], inp["k"], inp["v"], out, lse, idx, ws)
    for _ in range(warmup):
        flush.zero_()
        run()
    torch.cuda.synchronize()
    nv.hs2_profile_start()
    for _ in range(K):
        flush.zero_()
        run()
    prof = nv.hs2_profile_stop()
    st, info = nv.hs2_get_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device error word after block selection: {st} {info}")
    sweep_ms = prof.get("block_sweep", (0.0, 0))[0] / K
    topk_ms = prof.get("block_topk", (0.0, 0))[0] / K
    G = w.h_q // w.h_kv
    ex2 = G * wl.flops_and_bytes(w)["cand"]
    res = {"block": blk, "select_ms": round(sweep_ms + topk_ms, 4), "sweep_ms": round(sweep_ms, 4),
           "topk_ms": round(topk_ms, 4), "token_select_ms": round(token_select_ms, 4),
           "note": "chunk-sum sweep (every candidate's group probability, summed per 32 keys) + per-row block "
                   "top-k; token_select_ms = the token-level selection kernels of the timed step"}
    if sweep_ms > 0 and pk.get("ex2"):
        achieved = ex2 / (sweep_ms / 1e3) / 1e9
        res.update({"bound": "alu", "kernel": "block_sweep", "achieved": round(achieved, 2),
                    "peak": round(pk["ex2"] / 1e9, 1), "unit": "Gex2/s",
                    "frac": round(achieved / (pk["ex2"] / 1e9), 4)})
    return res


def bench_swa_comparator(w: wl.Workload, inp: dict, dev, K: int, warmup: int, flush: torch.Tensor,
                         idx: torch.Tensor) -> dict:
    """One sparse layer three ways on the workload's inputs (a next row of the
    path: the cost comparison the pages make against the predecessor designs),
    each call timed alone with CUDA events, L2 flushed before every call:
      hysparse2   one softmax over idx U window, all from the shared cache
                  (hs2_sparse_attn, the layer of the timed step);
      two_branch  the predecessor's sparse layer: a sliding-window branch over
                  its own cache plus the selected rows alone (hs2_swa_branches);
      swa_only    a plain sliding-window layer over its own cache (the SWA layers
                  of a hybrid full/SWA model: hs2_sparse_attn with top-k 0)."""
    swa = wl.make_swa_cache(w, dev, seed=w.seed)
    q = inp["q_sparse"][0] if inp["q_sparse"] else inp["q"]
    q_pos0 = (w.kv_len - 1) if w.decode else w.q_pos0
    shape = nv.shape_of(q, inp["k"], window=w.window, topk=w.topk, q_pos0=q_pos0)
    shape0 = nv.shape_of(q, inp["k"], window=w.window, topk=0, q_pos0=q_pos0)
    B, Hq, nq, D = q.shape
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    l1 = torch.empty(B, Hq, nq, dtype=torch.float32, device=dev)
    l2 = torch.empty_like(l1)
    calls = {
        "hysparse2": lambda: nv.hs2_sparse_attn(shape, q, inp["k"], inp["v"], idx, o1, None),
        "two_branch": lambda: nv.hs2_swa_branches(shape, q, swa["k_swa"], swa["v_swa"], inp["k"], inp["v"], idx,
                                                  o1, l1, o2, l2),
        "swa_only": lambda: nv.hs2_sparse_attn(shape0, q, swa["k_swa"], swa["v_swa"], None, o1, None),
    }
    st = torch.cuda.current_stream()
    ms = {}
    for name, fn in calls.items():
        for _ in range(warmup):
            flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record(st)
            fn()
            e1.record(st)
        torch.cuda.synchronize()
        ms[name] = round(statistics.median(e0.elapsed_time(e1) for e0, e1 in ev), 4)
    del swa
    return {"ms_per_layer": ms, "two_branch_over_hysparse2": round(ms["two_branch"] / ms["hysparse2"], 3),
            "kv_caches_per_layer": {"hysparse2": 1, "two_branch": 2, "swa_only": 1},
            "note": "same q, idx and shared cache; the window branch's own cache is a seeded N(0,1)*0.5 draw "
                    "of the same shape; L2 flushed before each call"}


def bench_context_parallel(w: wl.Workload, inp: dict, dev, K: int, warmup: int, flush: torch.Tensor,
                           n_slices: int = 4):
    """Context parallelism (a next row of the path) on one GPU: the cache cut into
    n_slices slices, every slice's steps and every merge timed alone with CUDA
    events (median of K, L2 flushed before each).  A rank of an n-GPU run would
    execute one slice's steps plus every merge, so the per-rank time is the
    slowest slice per step plus the merges; the exchanges (all-gathers) cannot
    run on one GPU and are given as bytes received per rank and the time they
    take at the measured 770 GB/s NVLink peer bandwidth."""
    if w.decode or w.n_q < 64:
        return None
    from long_context_sparse_flash_b200 import cp
    st = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(warmup):
            flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        res = None
        for e0, e1 in ev:
            flush.zero_()
            e0.record(st)
            res = fn()
            e1.record(st)
        torch.cuda.synchronize()
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in ev), res

    offs, ks, vs = cp.split_cache(inp["k"], inp["v"], n_slices)
    q, W, Kk, p0 = inp["q"], w.window, w.topk, w.q_pos0
    t1, parts = zip(*[timed(lambda s=s: cp.attn_partial(q, ks[s], vs[s], kv_off=offs[s], window=W, topk=Kk,
                                                        q_pos0=p0)) for s in range(n_slices)])
    O, L = torch.stack([x[0] for x in parts]), torch.stack([x[1] for x in parts])
    tc1, (out, lse) = timed(lambda: cp.combine(O, L))
    t2, sel = zip(*[timed(lambda s=s: cp.select_local(q, ks[s], lse, kv_off=offs[s], window=W, topk=Kk, q_pos0=p0))
                    for s in range(n_slices)])
    I, S = torch.stack([x[0] for x in sel]), torch.stack([x[1] for x in sel])
    shape = nv.make_shape(w.batch, w.n_q, w.h_q, w.h_kv, w.head_dim, W, Kk, p0, w.kv_len)
    tm, idx = timed(lambda: cp.select_merge(I, S, offs, shape=shape))
    t3, sp = zip(*[timed(lambda s=s: cp.sparse_partial(inp["q_sparse"][0], ks[s], vs[s], idx, kv_off=offs[s],
                                                       window=W, q_pos0=p0)) for s in range(n_slices)])
    O3, L3 = torch.stack([x[0] for x in sp]), torch.stack([x[1] for x in sp])
    tc3, _ = timed(lambda: cp.combine(O3, L3))
    layers = w.n_sparse
    per_rank = max(t1) + tc1 + max(t2) + tm + layers * (max(t3) + tc3)
    rows_q = w.batch * w.h_q * w.n_q
    rows_g = w.batch * w.h_kv * w.n_q
    recv = (n_slices - 1) * (rows_q * (w.head_dim * 2 + 4) * (1 + layers) + rows_g * w.topk * 8)
    nvlink_ms = recv / 770e9 * 1e3
    del ks, vs
    return {"slices": n_slices, "ms": {"attn_partial_max": round(max(t1), 4), "combine": round(tc1, 4),
                                       "select_local_max": round(max(t2), 4), "select_merge": round(tm, 4),
                                       "sparse_partial_max": round(max(t3), 4), "sparse_combine": round(tc3, 4)},
            "per_rank_compute_ms": round(per_rank, 4), "bytes_received_per_rank": int(recv),
            "exchange_ms_at_770GBs": round(nvlink_ms, 4),
            "note": "slices run one after another on one GPU; per rank = slowest slice per step + the merges "
                    "(every rank runs them); exchanges not run (one GPU), given as bytes and NVLink time"}


def source_sha(path: str) -> str:
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


KERNEL_SOURCE = {
    "full_attn": "k1_full_tc.cu", "select_score": "k1_decode.cu", "select_topk": "k2_select.cu",
    "decode_attn": "k1_decode.cu",
    "select_filter": "k2_select_tc.cu", "sparse_attn": "k3_sparse_attn.cu",
}


def dram_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the current source of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    src = KERNEL_SOURCE.get(kernel)
    if not src or not os.path.exists(path):
        return None
    cur = source_sha(os.path.join(ROOT, "long_context_sparse_flash_b200", "csrc", src))
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload:
            if parts[2] == cur:
                return float(parts[3])
    return None


# ---------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    """SM clocks and clock-event reasons of this process's GPU while the timed
    region runs: read through NVML every 5 ms on a background thread (so a short
    region still gets samples), or through `nvidia-smi -lms 200` if NVML is not
    available.  Read-only: no clock or other GPU setting is changed."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device: int):
        self.proc = None
        self.uuid = None
        self.nvml = None
        self.handle = None
        self.thread = None
        self.samples = []
        try:
            u = str(torch.cuda.get_device_properties(device).uuid)
            self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            # this process's GPU: by PCI address (CUDA and NVML number GPUs differently)
            pr = torch.cuda.get_device_properties(device)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.handle = None
                for i in range(pynvml.nvmlDeviceGetCount()):
                    h = pynvml.nvmlDeviceGetHandleByIndex(i)
                    uid = pynvml.nvmlDeviceGetUUID(h)
                    uid = uid.decode() if isinstance(uid, bytes) else uid
                    if self.uuid is not None and uid == self.uuid:
                        self.handle = h
                        break
            if self.handle is not None:
                self.nvml = pynvml
            else:
                self.error = f"no NVML device at {bus} or {self.uuid}"
        except Exception as e:
            self.nvml = None
            self.error = f"NVML: {type(e).__name__}: {e}"

    def _run_nvml(self):
        nv_ = self.nvml
        bits = [nv_.nvmlClocksEventReasonHwSlowdown, nv_.nvmlClocksEventReasonHwThermalSlowdown,
                nv_.nvmlClocksEventReasonSwThermalSlowdown, nv_.nvmlClocksEventReasonSwPowerCap]
        mx = nv_.nvmlDeviceGetMaxClockInfo(self.handle, nv_.NVML_CLOCK_SM)
        while not self._stop.is_set():
            try:
                sm = nv_.nvmlDeviceGetClockInfo(self.handle, nv_.NVML_CLOCK_SM)
                r = nv_.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((float(sm), float(mx), [n for n, b in zip(self.NAMES, bits) if r & b]))
            except Exception:
                pass
            self._stop.wait(0.005)

    def start(self):
        if self.nvml is not None:
            import threading
            self._stop = threading.Event()
            self.thread = threading.Thread(target=self._run_nvml, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
            rows = self.samples
        elif self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            rows = []
            for r in (x.split(", ") for x in out.strip().splitlines() if x.strip()):
                if self.uuid and r[0] != self.uuid:
                    continue
                try:
                    rows.append((float(r[1]), float(r[2]),
                                 [n for n, v in zip(self.NAMES, r[4:8]) if v.strip().lower() == "active"]))
                except (ValueError, IndexError):
                    continue
        else:
            return None
        if not rows:
            return {"samples": 0, "error": self.error or "no sample during the timed region"}
        reasons = sorted({n for _, _, rs in rows for n in rs})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


# ---------------------------------------------------------------------------
# our arm


class Step:
    """Buffers and the C-ABI calls of one step."""

    def __init__(self, w: wl.Workload, inp: dict, device):
        self.w = w
        self.q, self.k, self.v = inp["q"], inp["k"], inp["v"]
        self.qs = inp["q_sparse"]
        B, Hq, nq, D = self.q.shape
        self.shape = nv.shape_of(self.q, self.k, window=w.window, topk=w.topk,
                                 q_pos0=(w.kv_len - 1) if w.decode else w.q_pos0)
        entry = nv.HS2_ENTRY_DECODE if w.decode else nv.HS2_ENTRY_FULL_SELECT
        self.ws = nv.alloc_workspace(self.shape, entry, device)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(B, Hq, nq, dtype=torch.float32, device=device)
        self.idx = torch.empty(B, w.h_kv, nq, w.topk, dtype=torch.int32, device=device)
        self.sp_out = [torch.empty_like(self.q) for _ in self.qs]

    def __call__(self):
        if self.w.decode:
            nv.hs2_decode(self.shape, None, self.q, self.k, self.v, self.out, self.lse, self.idx, self.ws)
            for qs, o in zip(self.qs, self.sp_out):
                nv.hs2_decode_sparse(self.shape, None, qs, self.k, self.v, self.idx, o, None)
        else:
            nv.hs2_full_attn_select(self.shape, self.q, self.k, self.v, self.out, self.lse, self.idx, self.ws)
            for qs, o in zip(self.qs, self.sp_out):
                nv.hs2_sparse_attn(self.shape, qs, self.k, self.v, self.idx, o, None)

    def inputs(self):
        return [self.q, self.k, self.v, *self.qs]

    def outputs(self):
        return [self.out, self.lse, self.idx, *self.sp_out]


def dist_setup(n_gpus: int):
    """One process per GPU.  A process group (NCCL) is set up whenever the
    launcher is torchrun, a one-rank run included, so the barrier and the max
    over ranks take the same collective path at every N."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1 or os.environ.get("TORCHELASTIC_RUN_ID"):
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return ws, rank, local


def dist_on() -> bool:
    return torch.distributed.is_available() and torch.distributed.is_initialized()


def barrier(ws):
    if dist_on():
        torch.distributed.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """The slowest rank's time (every rank gets it)."""
    if not dist_on():
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_seed(w: wl.Workload, rank: int) -> int:
    """Each rank runs its own independent sequences (weak scaling, no exchange)."""
    return w.seed + 1000 * rank


def job_value(query_tokens: int, ws: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: the query tokens of all ranks over the slowest rank's time."""
    return query_tokens * ws * steps / (total_ms / 1e3)


def head_shard(w: wl.Workload, inp: dict, rank: int, ws: int):
    """Rank `rank`'s share of one workload split by KV-head group: KV heads
    [rank H_kv / ws, (rank + 1) H_kv / ws) with the G query heads of each
    (head h belongs to group h // G), copied into contiguous tensors, and the
    workload of that share.  Every (query, group) is computed from its own
    heads' q, K and V alone (full attention, selection and every sparse layer),
    so the shares need no exchange."""
    if w.h_kv % ws:
        raise ValueError(f"{w.h_kv} KV heads do not split over {ws} ranks")
    per, G = w.h_kv // ws, w.group
    g0, g1 = rank * per, (rank + 1) * per
    cut = lambda t, a, b: t[:, a:b].contiguous()
    share = dict(q=cut(inp["q"], g0 * G, g1 * G), k=cut(inp["k"], g0, g1), v=cut(inp["v"], g0, g1),
                 q_sparse=[cut(x, g0 * G, g1 * G) for x in inp["q_sparse"]],
                 probes=inp.get("probes"), needles=inp.get("needles"))
    return dataclasses.replace(w, h_q=per * G, h_kv=per), share


def input_digests(inp: dict) -> dict:
    """SHA-256 (first 16 hex digits) of the first 64 MiB of each input tensor, for reproducibility."""
    def dig(t):
        b = t.reshape(-1).view(torch.uint8)[: 64 << 20].cpu().numpy().tobytes()
        return hashlib.sha256(b).hexdigest()[:16]
    d = {"q": dig(inp["q"]), "k": dig(inp["k"]), "v": dig(inp["v"])}
    for i, qs in enumerate(inp["q_sparse"]):
        d[f"q_sparse_{i}"] = dig(qs)
    return d


def time_steps(step, K: int, flush_buf: Optional[torch.Tensor], ws: int):
    """K steps, L2 flushed (outside the timed events) before each unless flush_buf is None."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier(ws)
    torch.cuda.synchronize()
    for a, b in evs:
        if flush_buf is not None:
            flush_buf.zero_()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    barrier(ws)
    return [a.elapsed_time(b) for a, b in evs]


def time_e2e(step: Step, K: int, ws: int, inp: dict, device):
    """Same metric end to end through the C ABI: every step copies its inputs in
    from pinned host memory and its results (out, lse, idx, every sparse layer's
    out) back to pinned host memory.  Steps are pipelined the way a serving loop
    would run them: three streams and two device buffer sets, so the upload of
    step i+1 and the download of step i-1 overlap the compute of step i.  The
    time is from the first upload's start to the last download's end."""
    steps = [step, Step(step.w, {k: torch.empty_like(v) if torch.is_tensor(v) else [torch.empty_like(t) for t in v]
                                 for k, v in inp.items() if k in ("q", "k", "v", "q_sparse")}, device)]
    h_in = [t.cpu().pin_memory() for t in step.inputs()]
    h_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in s.outputs()] for s in steps]
    s_up, s_comp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    comp_done, down_done = [None, None], [None, None]

    def one(i):
        u = i % 2
        with torch.cuda.stream(s_up):
            if comp_done[u] is not None:
                s_up.wait_event(comp_done[u])      # step i-2 no longer reads these inputs
            for h, d in zip(h_in, steps[u].inputs()):
                d.copy_(h, non_blocking=True)
            up_done = ev()
            up_done.record(s_up)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(up_done)
            if down_done[u] is not None:
                s_comp.wait_event(down_done[u])    # step i-2's results are already downloaded
            steps[u]()
            comp_done[u] = ev()
            comp_done[u].record(s_comp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[u])
            for h, d in zip(h_out[u], steps[u].outputs()):
                h.copy_(d, non_blocking=True)
            down_done[u] = ev()
            down_done[u].record(s_down)

    for i in range(2):  # untimed: pins and warms both buffer sets
        one(i)
    torch.cuda.synchronize()
    barrier(ws)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_up)
    for i in range(K):
        one(i)
    t1.record(s_down)
    torch.cuda.synchronize()
    barrier(ws)
    bi = sum(t.numel() * t.element_size() for t in h_in)
    bo = sum(t.numel() * t.element_size() for t in h_out[0])
    return t0.elapsed_time(t1), bi, bo


def cpu_baseline(w: wl.Workload, inp: dict, n_rows: int, seed: int = 2024) -> dict:
    """The oracle, as it stands, on a bounded seeded sample of the workload's
    query rows (full attention + selection + every sparse layer per row)."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(seed)
    if w.decode:
        seqs = rng.choice(w.batch, size=min(n_rows, w.batch), replace=False)
        picks = [(int(b), np.array([0]), np.array([w.kv_len - 1])) for b in seqs]
    else:
        rows = np.sort(rng.choice(w.n_q, size=min(n_rows, w.n_q), replace=False))
        picks = [(0, rows, w.q_pos0 + rows)]
    prepared = []
    for b, rows, ts in picks:
        rt = torch.as_tensor(rows, device=inp["q"].device)
        kb, vb = wl.bf16_bits(inp["k"][b]), wl.bf16_bits(inp["v"][b])
        qb = np.ascontiguousarray(wl.bf16_bits(inp["q"][b][:, rt]).transpose(1, 0, 2))
        qsb = [np.ascontiguousarray(wl.bf16_bits(qs[b][:, rt]).transpose(1, 0, 2)) for qs in inp["q_sparse"]]
        prepared.append((ts, qb, qsb, kb, vb))
    t0 = time.perf_counter()
    n = 0
    for ts, qb, qsb, kb, vb in prepared:
        res = oracle.full_select(qb, ts, kb, vb, window=w.window, topk=w.topk, n_threads=cores)
        for q2 in qsb:
            oracle.sparse(q2, ts, kb, vb, res["idx"], window=w.window, n_threads=cores)
        n += len(ts)
    dt = time.perf_counter() - t0
    mean_t = float(np.mean(np.concatenate([p[0] for p in prepared]))) + 1
    return {"value": n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} seeded random query rows of {w.name} (mean context {mean_t:.0f} tokens), "
                      f"full-attn+select and {w.n_sparse} sparse layers each, {dt:.2f} s",
            "_rows": n, "_seconds": dt}


def roofline(w: wl.Workload, prof: dict, K: int, pk: dict, unique_rows: Optional[float] = None):
    work = kernel_work(w, unique_rows)
    per = {}
    for name, (ms, launches) in prof.items():
        if name not in work or ms <= 0:
            per[name] = dict(ms=ms / K, launches=launches // K if K else launches)
            continue
        wk = work[name]
        calls = K * (w.n_sparse if name == "sparse_attn" else 1)
        if wk["bound"] == "tensor":
            achieved = wk["flops"] * calls / (ms / 1e3) / 1e12
            peak, unit = pk["tc_sustained"], "TFLOP/s"
        elif wk["bound"] == "l2":
            achieved = wk["bytes"] * calls / (ms / 1e3) / 1e9
            peak, unit = round(pk["l2_gather"], 1), "GB/s"
        elif wk["bound"] == "alu":
            achieved = wk["ex2"] * calls / (ms / 1e3) / 1e9
            peak, unit = round(pk["ex2"] / 1e9, 1), "Gex2/s"
        elif wk["bound"] == "gather":
            l2 = wk["bytes"] * calls / (ms / 1e3) / 1e9
            hbm = wk["hbm_bytes"] * calls / (ms / 1e3) / 1e9
            l2_frac, hbm_frac = l2 / pk["l2_gather"], hbm / pk["hbm"]
            entry = dict(ms=ms / K, launches=launches // K if K else launches,
                         l2=dict(achieved=round(l2, 2), peak=round(pk["l2_gather"], 1), unit="GB/s",
                                 frac=round(l2_frac, 4), bytes="every attended row of every query"),
                         hbm=dict(achieved=round(hbm, 2), peak=pk["hbm"], unit="GB/s", frac=round(hbm_frac, 4),
                                  bytes="each distinct row once (compulsory)"))
            b = "l2" if l2_frac >= hbm_frac else "hbm"
            entry.update(bound=b, achieved=entry[b]["achieved"], peak=entry[b]["peak"], unit="GB/s",
                         frac=entry[b]["frac"])
            per[name] = entry
            continue
        else:
            achieved = wk["bytes"] * calls / (ms / 1e3) / 1e9
            peak, unit = pk["hbm"], "GB/s"
        per[name] = dict(ms=ms / K, launches=launches // K if K else launches, bound=wk["bound"],
                         achieved=round(achieved, 2), peak=peak, unit=unit, frac=round(achieved / peak, 4))
        if wk["bound"] == "alu" and "flops" in wk:  # the contraction's share of the tensor peak, for reference
            per[name]["tensor_frac"] = round(wk["flops"] * calls / (ms / 1e3) / 1e12 / pk["tc_sustained"], 4)
        if "stream_bytes" in wk:  # the bytes it streams against HBM bandwidth, for reference
            per[name]["hbm_frac"] = round(wk["stream_bytes"] * calls / (ms / 1e3) / 1e9 / pk["hbm"], 4)
    if not per:
        return None, per
    top = max((n for n in per if "bound" in per[n]), key=lambda n: per[n]["ms"])
    p = per[top]
    launches_total = prof[top][1]
    traffic = dram_traffic(top, w.name)
    for name, e in per.items():  # measured DRAM bytes of the kernel (ncu), where current
        tb = dram_traffic(name, w.name)
        if tb is not None and e.get("ms"):
            e["dram_bytes_per_launch"] = tb
            e["dram_frac"] = round(tb / (e["ms"] / max(1, e["launches"]) / 1e3) / 1e9 / pk["hbm"], 4)
    src = {"tensor": pk["src"] + " (sustained bf16)", "hbm": pk["src"] + " (copy GB/s)",
           "l2": "measured here (random 256-byte-row gather from a 64 MiB L2-resident buffer, hs2_gather_probe)",
           "alu": "measured here (special-function-unit ex2 rate, hs2_ex2_probe)"}
    rf = {"kernel": top, "bound": p["bound"], "achieved": p["achieved"],
          "peak": p["peak"], "unit": p["unit"], "frac": p["frac"],
          "peak_source": src[p["bound"]],
          "launches_per_step": launches_total / K, "traffic": traffic,
          "share_of_step": None}
    return rf, per


# the 1M-context configuration is one 4096-token prefill chunk and one batch-8
# decode step over independent 1M contexts: the chunk is the line's `value`,
# the decode step is measured in the same run and reported beside it
COMPANION = {"chunk_1m": "decode_1m"}


def default_cpu_rows(w: wl.Workload) -> int:
    """Oracle rows of the CPU baseline: about 12 s of host work on 16 cores
    (1536 rows at a 16K mean context), scaled by the workload's mean context."""
    return max(8, int(1536 * 16384 / wl.mean_context(w)))


def measure(w: wl.Workload, args, ws: int, rank: int, local: int, dev, pk: dict, flush: torch.Tensor,
            extras: bool) -> dict:
    """Time `args.steps` steps of workload w (after `args.warmup` untimed ones),
    L2 flushed before each; per-kernel times from the library's event pairs;
    with `extras`, also the warm-L2 figure, e2e, next rows and the CPU baseline."""
    if args.split == "heads":
        # one sequence (the same seed on every rank), its KV-head groups split over the ranks
        full = wl.make_inputs(w, dev, seed=w.seed)
        w_full, (w, inp) = w, head_shard(w, full, rank, ws)
        del full
        torch.cuda.empty_cache()
        tokens_per_rank = 0  # every rank serves the same query tokens
    else:
        inp = wl.make_inputs(w, dev, seed=replica_seed(w, rank))  # independent replica per rank
        w_full, tokens_per_rank = w, w.query_tokens
    step = Step(w, inp, dev)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    st, info = nv.hs2_get_device_status(step.ws)
    if st != 0:
        raise RuntimeError(f"device error word after warm-up: {st} {info}")

    clocks = ClockSampler(local)
    clocks.start()
    l0 = nv.hs2_launch_count()
    nv.hs2_profile_start()
    ms = time_steps(step, args.steps, flush, ws)
    prof = nv.hs2_profile_stop()
    launches = nv.hs2_launch_count() - l0
    clk = clocks.stop()
    total_ms = max_over_ranks(float(sum(ms)), ws)
    # replicas: all ranks' query tokens; head split: the one sequence's query tokens
    job_tokens, job_ranks = (w.query_tokens, ws) if tokens_per_rank else (w_full.query_tokens, 1)
    value = job_value(job_tokens, job_ranks, args.steps, total_ms)
    rf, per_kernel = roofline(w, prof, args.steps, pk, unique_kv_rows(w, step.idx) if w.topk else None)
    if rf is not None:
        rf["share_of_step"] = round(per_kernel[rf["kernel"]]["ms"] / (sum(ms) / args.steps), 4)
    res = {"workload": w_full.name, "value": round(value, 2), "ms_per_step": round(total_ms / args.steps, 4),
           "per_kernel": per_kernel, "roofline": rf, "gpu_launches": launches, "clocks": clk,
           "step_ms": {"median": round(statistics.median(ms), 4), "min": round(min(ms), 4),
                       "max": round(max(ms), 4)},
           "inputs_sha256_64MiB": input_digests(inp)}
    if not extras:
        del step, inp
        return res

    # the same steps with L2 left warm between them (a second figure, not `value`)
    warm_ms = max_over_ranks(float(sum(time_steps(step, args.steps, None, ws))), ws)
    res["warm_l2"] = {"ms_per_step": round(warm_ms / args.steps, 4),
                      "value": round(job_value(job_tokens, job_ranks, args.steps, warm_ms), 2)}
    res["e2e"] = None
    if not args.no_e2e:
        tokens = job_tokens * job_ranks * args.steps
        e_ms, bi, bo = time_e2e(step, args.steps, ws, inp, dev)
        e_total = max_over_ranks(float(e_ms), ws)
        res["e2e"] = {"value": round(tokens / (e_total / 1e3), 2), "unit": UNIT, "h2d_bytes_per_step": bi,
                      "d2h_bytes_per_step": bo, "ms_per_step": round(e_total / args.steps, 3)}
    res["next_rows"] = None
    if not args.no_next_rows:
        nr = {"kv_bridge": bench_bridge(w, dev, args.steps, args.warmup, pk)}
        sel_kernels = ("select_score", "select_thresh", "select_filter", "select_retry", "select_topk")
        token_sel_ms = sum(per_kernel[n]["ms"] for n in sel_kernels if n in per_kernel)
        blk = bench_block_select(w, inp, dev, args.steps, args.warmup, pk, flush, token_sel_ms)
        if blk is not None:
            nr["block_select"] = blk
        nr["swa_comparator"] = bench_swa_comparator(w, inp, dev, args.steps, args.warmup, flush, step.idx)
        cpr = bench_context_parallel(w, inp, dev, args.steps, args.warmup, flush)
        if cpr is not None:
            nr["context_parallel"] = cpr
        res["next_rows"] = nr
    res["cpu_baseline"] = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rows = args.cpu_rows if args.cpu_rows else default_cpu_rows(w)
        cpu = cpu_baseline(w, inp, rows)
        cpu.pop("_rows"), cpu.pop("_seconds")
        cpu["value"] = round(cpu["value"], 4)
        res["cpu_baseline"] = cpu
    del step, inp
    return res


def run_ours(args):
    ws, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    w = wl.WORKLOADS[args.workload]
    comp = None if args.no_companion else COMPANION.get(w.name)
    if args.split == "heads":
        for x in [w] + ([wl.WORKLOADS[comp]] if comp else []):
            if x.h_kv % ws:
                raise SystemExit(f"--split heads: {x.name} has {x.h_kv} KV heads, not divisible by {ws} ranks")
    nv.load()
    kinds = {wk["bound"] for x in [w] + ([wl.WORKLOADS[comp]] if comp else []) for wk in kernel_work(x, 0.0).values()}
    # the L2 gather and ex2 peaks are taken first, on an idle GPU (burst figures,
    # like the other measured peaks), before the workload's tensors exist
    pk = peaks()
    pk["l2_gather"] = measure_l2_gather(dev) if kinds & {"l2", "gather"} else None
    pk["ex2"] = measure_ex2(dev) if "alu" in kinds else None
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    main_res = measure(w, args, ws, rank, local, dev, pk, flush, extras=True)
    comp_res = None
    if comp:
        torch.cuda.empty_cache()
        comp_res = measure(wl.WORKLOADS[comp], args, ws, rank, local, dev, pk, flush, extras=False)
        comp_res["note"] = ("the other half of the 1M-context configuration, measured in the same run with the "
                            "same steps, warm-up and L2 flush; not part of `value`")

    if rank == 0:
        line = {
            "metric": METRIC, "value": main_res["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main_res["ms_per_step"], "higher_is_better": True,
            "scaling": "strong" if args.split == "heads" else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, shapes and value distributions of the workload; no dataset)",
            "config": {"workload": w.name, "batch": w.batch, "n_q": w.n_q, "q_pos0": w.q_pos0,
                       "kv_len": w.kv_len, "h_q": w.h_q, "h_kv": w.h_kv, "head_dim": w.head_dim,
                       "window": w.window, "topk": w.topk, "sparse_layers": w.n_sparse,
                       "parallelism": (f"heads x{ws} (the KV-head groups of one workload split over the GPUs, "
                                       f"no exchange)" if args.split == "heads"
                                       else f"replicas x{ws} (independent sequences per GPU)"),
                       "l2": f"flushed before every timed step ({FLUSH_BYTES >> 20} MiB write, outside the events)"},
            "per_kernel": main_res["per_kernel"],
            "roofline": main_res["roofline"],
            "warm_l2": main_res["warm_l2"],
            "inputs_sha256_64MiB": main_res["inputs_sha256_64MiB"],
            "next_rows": main_res["next_rows"],
            "cpu_baseline": main_res["cpu_baseline"],
            "e2e": main_res["e2e"],
            "gpu_launches": main_res["gpu_launches"],
            "clocks": main_res["clocks"],
            "step_ms": main_res["step_ms"],
        }
        if comp_res is not None:
            line[comp] = comp_res
        print(json.dumps(line), flush=True)
    else:
        line = None
    if dist_on():
        torch.distributed.destroy_process_group()
    return line


def run_reference(args):
    """The reference arm: the fp64 CPU oracle as it stands, on a bounded sample
    of the same workload per step (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    inp = wl.make_inputs(w, "cpu")
    rows_per_step = max(1, args.ref_rows)
    samples, cores = [], None
    total_rows, total_s = 0, 0.0
    for s in range(args.warmup + args.steps):
        c = cpu_baseline(w, inp, rows_per_step, seed=3000 + s)
        if s >= args.warmup:
            samples.append(c["sample"])
            cores = c["cores"]
            total_rows += c["_rows"]
            total_s += c["_seconds"]
    value = total_rows / total_s
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total_s / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, shapes and value distributions of the workload; no dataset)",
        "config": {"workload": w.name, "batch": w.batch, "n_q": w.n_q, "q_pos0": w.q_pos0, "kv_len": w.kv_len,
                   "h_q": w.h_q, "h_kv": w.h_kv, "head_dim": w.head_dim, "window": w.window, "topk": w.topk,
                   "sparse_layers": w.n_sparse, "parallelism": "host cores (OpenMP over rows)"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{rows_per_step} seeded random query rows per step; " + samples[-1]},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return line


def git_sha() -> str:
    """The commit the run measured (or "unknown" outside a git checkout)."""
    import subprocess
    try:
        r = subprocess.run(["git", "-C", ROOT, "rev-parse", "--short=12", "HEAD"], capture_output=True, text=True,
                           timeout=10)
        return r.stdout.strip() or "unknown"
    except Exception:
        return "unknown"


def run_key(args, sha: str) -> dict:
    """What identifies one bench entry in a JSONL log (a rerun with the same key is skipped)."""
    return {"impl": args.impl, "workload": args.workload, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "split": getattr(args, "split", "replicas"), "git_sha": sha}


def logged_line(path: str, key: dict):
    """The logged line with this key, or None (unreadable lines are ignored)."""
    if not path or not os.path.exists(path):
        return None
    with open(path) as f:
        for raw in f:
            try:
                d = json.loads(raw)
            except ValueError:
                continue
            if d.get("log_key") == key:
                return d
    return None


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="chunk_1m", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--split", choices=["replicas", "heads"], default="replicas",
                    help="with N > 1: independent replicas per GPU (weak scaling), or the KV-head groups of one "
                         "workload split over the GPUs (strong scaling; N must divide H_kv)")
    ap.add_argument("--no-companion", action="store_true",
                    help="chunk_1m only: skip the batch-8 1M decode step measured beside the chunk")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the next-row measurements (KV bridging, block selection, SWA comparator, "
                         "context parallelism) that run after the timed steps")
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="query rows in the oracle baseline sample (default: about 12 s of host work, "
                         "1536 rows at a 16K mean context, scaled by the workload's mean context)")
    ap.add_argument("--ref-rows", type=int, default=8, help="query rows per reference-arm step")
    ap.add_argument("--log", default="", help="append the JSON line, with the git commit and its key, to this "
                                                 "JSONL file (rank 0)")
    ap.add_argument("--skip-logged", action="store_true",
                    help="with --log: if the log already holds this entry (impl, workload, GPUs, steps, warm-up, "
                         "commit), print that line and run nothing, so a killed sweep resumes where it stopped")
    args = ap.parse_args()
    sha = git_sha() if args.log else None
    key = run_key(args, sha) if args.log else None
    if args.log and args.skip_logged:
        done = logged_line(args.log, key)
        if done is not None:
            if int(os.environ.get("RANK", "0")) == 0:
                print(json.dumps({k: v for k, v in done.items() if k not in ("log_key", "logged_at")}), flush=True)
            return
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    line = run_reference(args) if args.impl == "reference" else run_ours(args)
    if args.log and line is not None:
        with open(args.log, "a") as f:
            f.write(json.dumps({**line, "log_key": key, "logged_at": round(time.time(), 1)}) + "\n")


if __name__ == "__main__":
    main()

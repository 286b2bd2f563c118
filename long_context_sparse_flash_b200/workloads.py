"""Workload table and seeded synthetic inputs.

This module holds no attention arithmetic: it only draws seeded tensors with
the shapes, value distributions and structure of the HySparse2 setting
(xiawanshe.com report, sections "Token级选择" and "实测数据": a shared
Cross-Decoder KV cache, a 128-token forced window, a top-1024 token selection,
contexts up to 1M tokens).  The pages' retrieval suites (RULER-v2, MRCR-v2,
GraphWalks) are not available; planted "needle" keys stand in for retrieval
targets and clustered key segments stand in for multi-document context.  No
item of those suites is reproduced.

Both the CUDA path and the oracle read the tensors drawn here (the oracle
through their raw bf16 bits).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q: int          # query tokens per sequence in this call
    q_pos0: int       # absolute position of query 0 (decode: kv_len - 1)
    kv_len: int       # tokens in the shared cache per sequence (query tokens included)
    h_q: int
    h_kv: int
    head_dim: int
    window: int
    topk: int
    n_sparse: int     # sparse KV-reuse layers after the full-attention layer
    keys: str         # "gaussian" or "segments"
    needles: int      # planted keys per probe query (0: none)
    seed: int
    decode: bool = False

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def query_tokens(self) -> int:
        return self.batch * self.n_q


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        # 1 x 2048 prefill, 8/2 heads, D=64, top-256, 2 sparse layers, seed 0
        Workload("tiny", 1, 2048, 0, 2048, 8, 2, 64, 128, 256, 2, "gaussian", 8, 0),
        # 32K prefill, 32/4 heads, D=128, top-1024, 4 sparse layers, seed 1
        Workload("prefill_32k", 1, 32768, 0, 32768, 32, 4, 128, 128, 1024, 4, "gaussian", 16, 1),
        # 8192 new tokens appended to a 262144-token cache (clustered keys), seed 2
        Workload("chunk_256k", 1, 8192, 262144, 270336, 32, 4, 128, 128, 1024, 4, "segments", 0, 2),
        # decode: 64 sequences x 1 token, 131072-token context each, seed 3
        Workload("decode_128k", 64, 1, 131071, 131072, 32, 4, 128, 128, 1024, 4, "gaussian", 32, 3,
                 decode=True),
        # 1M context: a 4096-token chunk appended to a 1048576-token cache, seed 4
        Workload("chunk_1m", 1, 4096, 1048576, 1052672, 32, 4, 128, 128, 1024, 4, "segments", 64, 4),
        # 1M context: batch-8 decode over independent 1M contexts, seed 4
        Workload("decode_1m", 8, 1, 1048575, 1048576, 32, 4, 128, 128, 1024, 4, "segments", 64, 4,
                 decode=True),
        # profiling case: the last 4096 queries of the 32K prefill (same per-row work, 1/8 of the rows)
        Workload("prefill_32k_tail", 1, 4096, 28672, 32768, 32, 4, 128, 128, 1024, 4, "gaussian", 16, 1),
        # profiling case: 512 queries over the 1M cache (the sweep's per-CTA work of the 1M
        # chunk: about 8200 key tiles per CTA, on 64 CTAs; 2.15 GB of K+V)
        Workload("chunk_1m_prof", 1, 512, 1048576, 1049088, 32, 4, 128, 128, 1024, 4, "segments", 64, 4),
        # profiling case: 4 of the 128K decode sequences (1.07 GB of K+V, > L2)
        Workload("decode_128k_b4", 4, 1, 131071, 131072, 32, 4, 128, 128, 1024, 4, "gaussian", 32, 3,
                 decode=True),
    ]
}

# sub-seed offsets, one per drawn tensor: seed * 1000 + offset
SUB_Q, SUB_K, SUB_V, SUB_QS, SUB_NEEDLE, SUB_SEG = 1, 2, 3, 10, 50, 60
SUB_HIDDEN, SUB_WKV = 70, 71
SUB_KSWA, SUB_VSWA = 80, 81  # the sliding-window branch's own cache (comparator)
# hidden size of the Self-Decoder for the KV-bridging inputs (the pages give no
# model dimensions; a common size for a model of this class)
BRIDGE_D_MODEL = 4096


def custom(name="custom", *, batch=1, n_q=256, q_pos0=0, kv_len=None, h_q=8, h_kv=2, head_dim=64,
           window=128, topk=64, n_sparse=1, keys="gaussian", needles=0, seed=0,
           decode=False) -> Workload:
    """A small ad-hoc workload (tests: ragged tails, edge cases)."""
    if kv_len is None:
        kv_len = q_pos0 + n_q
    return Workload(name, batch, n_q, q_pos0, kv_len, h_q, h_kv, head_dim, window, topk, n_sparse,
                    keys, needles, seed, decode)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _segment_keys(w: Workload, device, gen: torch.Generator) -> torch.Tensor:
    """Keys of one sequence: seeded segments of length U[2048, 16384]; each is
    background N(0,1) with probability 1/2, else a 'document' whose keys are
    one of 64 per-KV-head Gaussian centroids plus 0.3 * N(0,1) noise."""
    H, N, D = w.h_kv, w.kv_len, w.head_dim
    cent = torch.randn(H, 64, D, generator=gen, device=device)
    k = torch.empty(H, N, D, dtype=torch.bfloat16, device=device)
    pos = 0
    while pos < N:
        ln = int(torch.randint(2048, 16385, (1,), generator=gen, device=device).item())
        ln = min(ln, N - pos)
        doc = bool(torch.rand(1, generator=gen, device=device).item() < 0.5)
        noise = torch.randn(H, ln, D, generator=gen, device=device)
        if doc:
            cid = int(torch.randint(0, 64, (1,), generator=gen, device=device).item())
            seg = cent[:, cid:cid + 1, :] + 0.3 * noise
        else:
            seg = noise
        k[:, pos:pos + ln] = seg.to(torch.bfloat16)
        pos += ln
    return k


def _plant(w: Workload, q_seq: torch.Tensor, k_seq: torch.Tensor, probes: List[int],
           gen: torch.Generator) -> Dict[int, List[int]]:
    """Plant w.needles keys per probe query i (absolute t = q_pos0 + i) at distinct
    older positions j <= t - window not used by an earlier plant:
    k_{g,j} = 2 * normalize(sum_{h in g} q_{h,t}) + 0.1 * N(0,1).
    Returns the planted positions of each probe query."""
    m = w.needles
    planted: Dict[int, List[int]] = {}
    dev = k_seq.device
    used = torch.zeros(w.kv_len, dtype=torch.bool, device=dev)
    G = w.group
    for i in probes:
        t = w.q_pos0 + i
        hi = t - w.window  # last candidate position
        if hi + 1 < m:
            continue
        # oversample, drop used / repeated positions, keep the first m
        cand = torch.randint(0, hi + 1, (4 * m + 64,), generator=gen, device=dev)
        cand = cand[~used[cand]]
        seen = []
        sset = set()
        for c in cand.tolist():
            if c not in sset:
                sset.add(c)
                seen.append(c)
            if len(seen) == m:
                break
        if len(seen) < m:
            continue
        pos = torch.tensor(seen, dtype=torch.long, device=dev)
        used[pos] = True
        qd = q_seq[:, i, :].float().view(w.h_kv, G, w.head_dim).sum(1)  # [H_kv, D]
        qd = qd / qd.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        noise = torch.randn(w.h_kv, m, w.head_dim, generator=gen, device=dev)
        k_seq[:, pos, :] = (2.0 * qd[:, None, :] + 0.1 * noise).to(torch.bfloat16)
        planted[i] = seen
    return planted


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None,
                with_sparse: bool = True) -> Dict[str, object]:
    """Seeded inputs for workload ``w``.

    Returns dict with
      q        bf16 [B, H_q, n_q, D]  full-attention layer queries
      k, v     bf16 [B, H_kv, kv_len, D] the shared Cross-Decoder cache
      q_sparse list of n_sparse bf16 [B, H_q, n_q, D] (fresh draw per layer)
      probes   list (per sequence) of query indices that got planted needles
      needles  list (per sequence) of {probe query index: planted key positions}
    """
    seed = w.seed if seed is None else int(seed)
    B, Hq, Hk, D, N, nq = w.batch, w.h_q, w.h_kv, w.head_dim, w.kv_len, w.n_q
    gq = _gen(device, seed * 1000 + SUB_Q)
    q = (torch.randn(B, Hq, nq, D, generator=gq, device=device) * 0.5).to(torch.bfloat16)
    gk = _gen(device, seed * 1000 + SUB_K)
    gs = _gen(device, seed * 1000 + SUB_SEG)
    gn = _gen(device, seed * 1000 + SUB_NEEDLE)
    k = torch.empty(B, Hk, N, D, dtype=torch.bfloat16, device=device)
    probes_all = []
    needles_all = []
    for b in range(B):
        if w.keys == "segments":
            k[b] = _segment_keys(w, device, gs)
        else:
            k[b] = (torch.randn(Hk, N, D, generator=gk, device=device) * 0.5).to(torch.bfloat16)
        probes = []
        planted = {}
        if w.needles > 0:
            n_probe = min(nq, max(1, N // (8 * w.needles)))
            # probe queries: seeded, distinct, increasing
            perm = torch.randperm(nq, generator=gn, device=device)[:n_probe]
            probes = sorted(int(x) for x in perm.tolist())
            planted = _plant(w, q[b], k[b], probes, gn)
        probes_all.append(probes)
        needles_all.append(planted)
    gv = _gen(device, seed * 1000 + SUB_V)
    v = torch.empty(B, Hk, N, D, dtype=torch.bfloat16, device=device)
    for b in range(B):
        v[b] = (torch.randn(Hk, N, D, generator=gv, device=device) * 0.5).to(torch.bfloat16)
    q_sparse = []
    if with_sparse:
        for layer in range(w.n_sparse):
            g = _gen(device, seed * 1000 + SUB_QS + layer)
            q_sparse.append((torch.randn(B, Hq, nq, D, generator=g, device=device) * 0.5)
                            .to(torch.bfloat16))
    return dict(q=q, k=k, v=v, q_sparse=q_sparse, probes=probes_all, needles=needles_all)


def make_bridge_inputs(batch: int, n_new: int, d_model: int, h_kv: int, head_dim: int, device="cpu",
                       seed: int = 0) -> Dict[str, torch.Tensor]:
    """Seeded inputs of the KV-bridging projection: hidden states
    hidden [batch, n_new, d_model] ~ N(0, 1) and weights w_kv [2 h_kv D, d_model]
    ~ N(0, 1/d_model) (so K and V come out near unit scale), both bf16."""
    gh = _gen(device, seed * 1000 + SUB_HIDDEN)
    gw = _gen(device, seed * 1000 + SUB_WKV)
    hidden = torch.randn(batch, n_new, d_model, generator=gh, device=device).to(torch.bfloat16)
    w = (torch.randn(2 * h_kv * head_dim, d_model, generator=gw, device=device) / math.sqrt(d_model)).to(torch.bfloat16)
    return dict(hidden=hidden, w_kv=w)


def make_swa_cache(w: Workload, device="cpu", seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """The own K/V cache of a separate sliding-window branch (the predecessor
    design's sparse layer), shaped like the shared cache: k_swa, v_swa bf16
    [B, H_kv, kv_len, D] ~ N(0,1) * 0.5."""
    seed = w.seed if seed is None else int(seed)
    shape = (w.batch, w.h_kv, w.kv_len, w.head_dim)
    gk = _gen(device, seed * 1000 + SUB_KSWA)
    gv = _gen(device, seed * 1000 + SUB_VSWA)
    k = (torch.randn(*shape, generator=gk, device=device) * 0.5).to(torch.bfloat16)
    v = (torch.randn(*shape, generator=gv, device=device) * 0.5).to(torch.bfloat16)
    return dict(k_swa=k, v_swa=v)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a host numpy uint16 array."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def positions(w: Workload) -> np.ndarray:
    """Absolute position of every query index of one sequence."""
    return np.arange(w.q_pos0, w.q_pos0 + w.n_q, dtype=np.int64)


def stratified_rows(w: Workload, n_random: int, seed: int = 12345) -> np.ndarray:
    """Query indices for sampled parity checks: the boundary positions of the
    window / top-K regime plus seeded random ones, restricted to this call."""
    W, K = w.window, w.topk
    t_special = [0, 1, W - 2, W - 1, W, W + 1, W + 2, W - 1 + K - 1, W - 1 + K, W + K,
                 w.q_pos0, w.q_pos0 + 1, w.q_pos0 + w.n_q - 1]
    rows = {t - w.q_pos0 for t in t_special if w.q_pos0 <= t < w.q_pos0 + w.n_q}
    rng = np.random.default_rng(seed)
    rows |= set(int(x) for x in rng.integers(0, w.n_q, size=n_random))
    return np.array(sorted(rows), dtype=np.int64)


def flops_and_bytes(w: Workload) -> Dict[str, float]:
    """Algorithmic work of one pass over the workload (per call, all sequences).

    P = causal (query, key) pairs; A = attended rows per (query, KV head) summed.
    """
    t = np.arange(w.q_pos0, w.q_pos0 + w.n_q, dtype=np.float64)
    P = float((t + 1).sum()) * w.batch
    n_cand = np.maximum(0.0, t - w.window + 1)
    A = float((np.minimum(n_cand, w.topk) + np.minimum(t + 1, w.window)).sum()) * w.batch
    D, Hq, Hk = w.head_dim, w.h_q, w.h_kv
    return dict(
        pairs=P,
        cand=float(n_cand.sum()) * w.batch * Hk,
        attended=A,
        full_flops=4.0 * D * Hq * P,
        select_qk_flops=2.0 * D * Hq * float(n_cand.sum()) * w.batch,
        sparse_flops_per_layer=4.0 * D * Hq * A,
        sparse_bytes_per_layer=A * Hk * D * 2 * 2,
        kv_bytes=2.0 * w.batch * Hk * w.kv_len * D * 2,
        q_bytes=2.0 * w.batch * Hq * w.n_q * D,
        idx_bytes=4.0 * w.batch * Hk * w.n_q * w.topk,
    )


def mean_context(w: Workload) -> float:
    return float(w.q_pos0 + (w.n_q - 1) / 2.0 + 1)


def _check():  # pragma: no cover - manual sanity
    for w in WORKLOADS.values():
        print(w.name, flops_and_bytes(w)["full_flops"] / 1e12, "TF")


if __name__ == "__main__":  # pragma: no cover
    _check()

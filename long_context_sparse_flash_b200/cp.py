"""Context parallelism: one context's KV cache cut into P contiguous slices,
one per GPU, with the full-attention + selection layer and the sparse layers
computed exactly as over the whole cache (HySparse2 pages: xiawanshe.com
report, sections "两级KV共享" and "Token级选择"; the steps and their merges are
those of the context-parallel section of include/hs2.h).

Every step runs in the library's kernels through the C ABI; this module only
allocates outputs and workspaces and moves the per-slice results between the
steps.  Two ways to move them:

* ``ContextParallel`` -- one rank per GPU, each holding its slice; the
  per-slice buffers are all-gathered in slice order with ``torch.distributed``
  (NCCL over NVLink on GPUs).  Every rank takes the same collective steps in the
  same order.
* ``run_in_process`` -- every slice held by one process on one device, the
  slices run one after another and their results are stacked.  It checks the
  steps and merges on a single GPU.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch

from . import native as nv


def slice_offsets(kv_len: int, n_slices: int) -> List[int]:
    """First key of each of n contiguous slices of [0, kv_len) (sizes differ by at most one)."""
    if n_slices < 1 or kv_len < n_slices:
        raise ValueError("need 1 <= n_slices <= kv_len")
    base, extra = divmod(kv_len, n_slices)
    offs, o = [], 0
    for s in range(n_slices):
        offs.append(o)
        o += base + (1 if s < extra else 0)
    return offs


# ---------------------------------------------------------------------------
# the steps on one slice (shape: the slice's kv_len, the absolute q_pos0)


def _ws(shape, kv_off: int, entry: int, device, stream=None) -> torch.Tensor:
    n = nv.hs2_cp_workspace_size(shape, kv_off, entry)
    if n == 0:
        # 0: the shape is invalid or not supported by the slice calls (n_q >= 64,
        # head_dim in {64, 128}, G in {1, 2, 4, 8}, ...)
        raise nv.HS2Error(1, "hs2_cp_workspace_size (shape not accepted by the slice calls)")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    nv.hs2_workspace_init(ws, stream=stream)
    return ws


def attn_partial(q, k_slice, v_slice, *, kv_off: int, window: int, topk: int, q_pos0: int, stream=None):
    """Step 1 on one slice: (out_p, lse_p) over the slice's causal keys."""
    shape = nv.shape_of(q, k_slice, window=window, topk=topk, q_pos0=q_pos0)
    ws = _ws(shape, kv_off, nv.HS2_ENTRY_CP_ATTN, q.device, stream)
    B, Hq, nq, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, nq, dtype=torch.float32, device=q.device)
    nv.hs2_cp_attn_partial(shape, kv_off, q, k_slice, v_slice, out, lse, ws, stream)
    return out, lse


def select_local(q, k_slice, lse, *, kv_off: int, window: int, topk: int, q_pos0: int, stream=None):
    """Step 2 on one slice, with the combined LSE: (local idx, scores) of its top-K."""
    shape = nv.shape_of(q, k_slice, window=window, topk=topk, q_pos0=q_pos0)
    ws = _ws(shape, kv_off, nv.HS2_ENTRY_CP_SELECT, q.device, stream)
    B, Hq, nq, D = q.shape
    idx = torch.empty(B, k_slice.shape[1], nq, topk, dtype=torch.int32, device=q.device)
    score = torch.empty(B, k_slice.shape[1], nq, topk, dtype=torch.float32, device=q.device)
    nv.hs2_cp_select_local(shape, kv_off, q, k_slice, lse, idx, score, ws, stream)
    return idx, score


def sparse_partial(q, k_slice, v_slice, idx, *, kv_off: int, window: int, q_pos0: int, stream=None):
    """Step 3 on one slice: (out_p, lse_p) of one sparse layer over the rows it holds."""
    shape = nv.shape_of(q, k_slice, window=window, topk=idx.shape[-1], q_pos0=q_pos0)
    ws = _ws(shape, kv_off, nv.HS2_ENTRY_CP_SPARSE, q.device, stream)
    B, Hq, nq, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, nq, dtype=torch.float32, device=q.device)
    nv.hs2_cp_sparse_partial(shape, kv_off, q, k_slice, v_slice, idx, out, lse, ws, stream)
    return out, lse


def combine(out_parts: torch.Tensor, lse_parts: torch.Tensor, stream=None):
    """Merge of steps 1 and 3: stacked [P, B, H_q, n_q, D] / [P, B, H_q, n_q] -> (out, lse)."""
    P = out_parts.shape[0]
    out = torch.empty(out_parts.shape[1:], dtype=out_parts.dtype, device=out_parts.device)
    lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=out_parts.device)
    nv.hs2_cp_combine(P, lse.numel(), out.shape[-1], out_parts, lse_parts, out, lse, stream)
    return out, lse


def select_merge(idx_parts: torch.Tensor, score_parts: torch.Tensor, kv_offs: Sequence[int], *, shape, stream=None):
    """Merge of step 2: stacked [P, B, H_kv, n_q, K] lists -> whole-context idx."""
    idx = torch.empty(idx_parts.shape[1:], dtype=torch.int32, device=idx_parts.device)
    nv.hs2_cp_select_merge(shape, kv_offs, idx_parts, score_parts, idx, stream)
    return idx


def _whole_shape(q, kv_len: int, h_kv: int, *, window: int, topk: int, q_pos0: int):
    B, Hq, nq, D = q.shape
    return nv.make_shape(B, nq, Hq, h_kv, D, window, topk, q_pos0, kv_len)


# ---------------------------------------------------------------------------
# one rank per GPU


def dist_gather(t: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of one per-slice tensor, stacked in rank (= slice) order."""
    import torch.distributed as dist
    ws = dist.get_world_size(group)
    out = torch.empty((ws,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    return out


class ContextParallel:
    """This rank's slice of the context and the steps over it.

    k_slice, v_slice: [B, H_kv, len, D] bf16, keys [kv_off, kv_off + len) of the
    whole context; kv_offs: every slice's first key (ascending, this rank's at
    index rank); kv_len: the whole context's length.  ``gather`` stacks one
    tensor from every rank in slice order (``dist_gather`` by default); ``ops``
    holds the step functions (this module's by default)."""

    def __init__(self, k_slice, v_slice, *, rank: int, kv_offs: Sequence[int], kv_len: int, window: int, topk: int,
                 gather: Optional[Callable[[torch.Tensor], torch.Tensor]] = None, ops=None):
        import sys
        self.k, self.v = k_slice, v_slice
        self.rank = rank
        self.kv_offs = list(kv_offs)
        self.kv_off = self.kv_offs[rank]
        self.kv_len = kv_len
        self.window, self.topk = window, topk
        self.gather = gather if gather is not None else dist_gather
        self.ops = ops if ops is not None else sys.modules[__name__]

    def full_attn_select(self, q, q_pos0: int):
        """The full-attention layer with selection: (out, lse, idx) of the whole context."""
        o = self.ops
        out_p, lse_p = o.attn_partial(q, self.k, self.v, kv_off=self.kv_off, window=self.window, topk=self.topk,
                                      q_pos0=q_pos0)
        out, lse = o.combine(self.gather(out_p), self.gather(lse_p))
        idx_p, score_p = o.select_local(q, self.k, lse, kv_off=self.kv_off, window=self.window, topk=self.topk,
                                        q_pos0=q_pos0)
        shape = _whole_shape(q, self.kv_len, self.k.shape[1], window=self.window, topk=self.topk, q_pos0=q_pos0)
        idx = o.select_merge(self.gather(idx_p), self.gather(score_p), self.kv_offs, shape=shape)
        return out, lse, idx

    def sparse_attn(self, q, idx, q_pos0: int):
        """One sparse layer of the whole context (q its own query, idx the selection)."""
        o = self.ops
        out_p, lse_p = o.sparse_partial(q, self.k, self.v, idx, kv_off=self.kv_off, window=self.window,
                                        q_pos0=q_pos0)
        out, _ = o.combine(self.gather(out_p), self.gather(lse_p))
        return out


# ---------------------------------------------------------------------------
# every slice in one process


def split_cache(k: torch.Tensor, v: torch.Tensor, n_slices: int):
    """Contiguous copies of n slices of a whole cache (for one-process runs)."""
    offs = slice_offsets(k.shape[2], n_slices)
    ends = offs[1:] + [k.shape[2]]
    ks = [k[:, :, a:b].contiguous() for a, b in zip(offs, ends)]
    vs = [v[:, :, a:b].contiguous() for a, b in zip(offs, ends)]
    return offs, ks, vs


def run_in_process(q, ks: List[torch.Tensor], vs: List[torch.Tensor], offs: Sequence[int], *, kv_len: int,
                   window: int, topk: int, q_pos0: int, q_sparse: Sequence[torch.Tensor] = ()):
    """Every step over every slice in this process: (out, lse, idx, [sparse outs])."""
    P = len(offs)
    parts = [attn_partial(q, ks[s], vs[s], kv_off=offs[s], window=window, topk=topk, q_pos0=q_pos0)
             for s in range(P)]
    out, lse = combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    sel = [select_local(q, ks[s], lse, kv_off=offs[s], window=window, topk=topk, q_pos0=q_pos0) for s in range(P)]
    shape = _whole_shape(q, kv_len, ks[0].shape[1], window=window, topk=topk, q_pos0=q_pos0)
    idx = select_merge(torch.stack([x[0] for x in sel]), torch.stack([x[1] for x in sel]), offs, shape=shape)
    sp_out = []
    for qs in q_sparse:
        parts = [sparse_partial(qs, ks[s], vs[s], idx, kv_off=offs[s], window=window, q_pos0=q_pos0)
                 for s in range(P)]
        sp_out.append(combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))[0])
    return out, lse, idx, sp_out

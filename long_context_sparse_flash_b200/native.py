"""Thin ctypes binding of libhs2 (include/hs2.h), same names as the C ABI.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are passed as device pointers (``tensor.data_ptr()``) and the
current torch CUDA stream is passed as the library's stream unless one is given.
There is no fallback: if ``libhs2.so`` is missing or a call fails, an exception
is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))

HS2_OK = 0
STATUS = {0: "HS2_OK", 1: "HS2_ERR_INVALID_ARG", 2: "HS2_ERR_UNSUPPORTED", 3: "HS2_ERR_WORKSPACE",
          4: "HS2_ERR_CUDA", 5: "HS2_ERR_DEVICE_CHECK", 6: "HS2_ERR_TIMEOUT"}
HS2_ENTRY_FULL_SELECT, HS2_ENTRY_SPARSE, HS2_ENTRY_PREFILL, HS2_ENTRY_DECODE = 0, 1, 2, 3
HS2_ENTRY_BLOCK_SELECT = 4
HS2_ENTRY_CP_ATTN, HS2_ENTRY_CP_SELECT, HS2_ENTRY_CP_SPARSE = 5, 6, 7

# every symbol include/hs2.h declares
EXPORTS = ("hs2_workspace_size", "hs2_workspace_init", "hs2_full_attn_select", "hs2_sparse_attn",
           "hs2_prefill_chunk", "hs2_decode", "hs2_decode_sparse", "hs2_get_device_status", "hs2_status_string",
           "hs2_launch_count", "hs2_is_checked_build", "hs2_profile_start", "hs2_profile_stop",
           "hs2_full_attn_select_static", "hs2_static_scratch_bytes", "hs2_selftest_exp2",
           "hs2_gather_probe", "hs2_ex2_probe", "hs2_kv_bridge", "hs2_full_attn_block_select",
           "hs2_swa_branches", "hs2_cp_workspace_size", "hs2_cp_attn_partial", "hs2_cp_select_local",
           "hs2_cp_sparse_partial", "hs2_cp_combine", "hs2_cp_select_merge",
           "hs2_kv_bridge_workspace_size", "hs2_selftest_wait", "hs2_static_scratch_status",
           "hs2_select_retry_rows")

KERNEL_NAMES = {1: "full_attn", 2: "select_score", 3: "select_topk", 4: "sparse_attn", 5: "decode_attn",
                6: "decode_combine", 7: "fused_attn_select", 8: "select_thresh", 9: "select_filter",
                10: "select_retry", 11: "kv_bridge", 12: "block_sweep", 13: "block_topk",
                14: "cp_combine", 15: "cp_select_merge", 16: "cp_idx_local", 17: "selftest_wait"}


class HS2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class hs2_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("h_q", ctypes.c_int32),
                ("h_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("window", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("reserved", ctypes.c_int32), ("q_pos0", ctypes.c_int64),
                ("kv_len", ctypes.c_int64), ("softmax_scale", ctypes.c_float)]


class hs2_bridge_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_new", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("h_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("pos0", ctypes.c_int64), ("kv_cap", ctypes.c_int64)]


_libs = {}


def lib_path(checked: bool = False) -> str:
    return os.path.join(_PKG, "libhs2_checked.so" if checked else "libhs2.so")


def load(checked: bool = False) -> ctypes.CDLL:
    """Load (once) libhs2.so or libhs2_checked.so from the package directory."""
    if checked in _libs:
        return _libs[checked]
    path = lib_path(checked)
    if not os.path.exists(path):
        raise RuntimeError(f"{os.path.basename(path)} is not built; run "
                           "`python -m long_context_sparse_flash_b200.build`")
    lib = ctypes.CDLL(path)
    P, S, U64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64
    sh = ctypes.POINTER(hs2_shape)
    lib.hs2_workspace_size.argtypes = [sh, ctypes.c_int]
    lib.hs2_workspace_size.restype = S
    lib.hs2_workspace_init.argtypes = [P, S, P]
    lib.hs2_full_attn_select.argtypes = [sh, P, P, P, P, P, P, P, S, P]
    lib.hs2_prefill_chunk.argtypes = [sh, P, P, P, P, P, P, P, S, P]
    lib.hs2_full_attn_block_select.argtypes = [sh, ctypes.c_int32, P, P, P, P, P, P, P, S, P]
    lib.hs2_swa_branches.argtypes = [sh, P, P, P, P, P, P, P, P, P, P, P, S, P]
    I64, I32 = ctypes.c_int64, ctypes.c_int32
    lib.hs2_cp_workspace_size.argtypes = [sh, I64, ctypes.c_int]
    lib.hs2_cp_workspace_size.restype = S
    lib.hs2_cp_attn_partial.argtypes = [sh, I64, P, P, P, P, P, P, S, P]
    lib.hs2_cp_select_local.argtypes = [sh, I64, P, P, P, P, P, P, S, P]
    lib.hs2_cp_sparse_partial.argtypes = [sh, I64, P, P, P, P, P, P, P, S, P]
    lib.hs2_cp_combine.argtypes = [I32, I64, I32, P, P, P, P, P]
    lib.hs2_cp_select_merge.argtypes = [sh, I32, ctypes.POINTER(ctypes.c_int64), P, P, P, P]
    lib.hs2_decode.argtypes = [sh, P, P, P, P, P, P, P, P, S, P]
    lib.hs2_sparse_attn.argtypes = [sh, P, P, P, P, P, P, S, P]
    lib.hs2_decode_sparse.argtypes = [sh, P, P, P, P, P, P, P, S, P]
    lib.hs2_get_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
    lib.hs2_status_string.argtypes = [ctypes.c_int]
    lib.hs2_status_string.restype = ctypes.c_char_p
    lib.hs2_launch_count.argtypes = []
    lib.hs2_launch_count.restype = U64
    lib.hs2_is_checked_build.argtypes = []
    lib.hs2_profile_start.argtypes = []
    lib.hs2_profile_stop.argtypes = [ctypes.c_uint32, P, P]
    lib.hs2_full_attn_select_static.argtypes = [sh, P, P, P, P, P, P, P]
    lib.hs2_static_scratch_bytes.argtypes = []
    lib.hs2_static_scratch_bytes.restype = S
    lib.hs2_static_scratch_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.hs2_static_scratch_status.restype = ctypes.c_int
    lib.hs2_select_retry_rows.argtypes = [sh, P, S, P, ctypes.POINTER(ctypes.c_int64)]
    lib.hs2_select_retry_rows.restype = ctypes.c_int
    lib.hs2_selftest_exp2.argtypes = [P, P, ctypes.c_int, P]
    lib.hs2_gather_probe.argtypes = [P, ctypes.c_int64, P, ctypes.c_int64, ctypes.c_int32, P, P]
    lib.hs2_ex2_probe.argtypes = [ctypes.c_int32, P, P, ctypes.POINTER(ctypes.c_int64)]
    lib.hs2_selftest_wait.argtypes = [P, S, ctypes.c_int64, P]
    lib.hs2_kv_bridge.argtypes = [ctypes.POINTER(hs2_bridge_shape), P, P, P, P, P, P, S, P]
    lib.hs2_kv_bridge_workspace_size.argtypes = [ctypes.POINTER(hs2_bridge_shape)]
    lib.hs2_kv_bridge_workspace_size.restype = S
    for name in ("hs2_workspace_init", "hs2_full_attn_select", "hs2_prefill_chunk", "hs2_decode",
                 "hs2_sparse_attn", "hs2_decode_sparse", "hs2_get_device_status", "hs2_is_checked_build",
                 "hs2_profile_start", "hs2_profile_stop", "hs2_full_attn_select_static", "hs2_selftest_exp2",
                 "hs2_gather_probe", "hs2_ex2_probe", "hs2_kv_bridge", "hs2_full_attn_block_select",
                 "hs2_swa_branches", "hs2_cp_attn_partial", "hs2_cp_select_local", "hs2_cp_sparse_partial",
                 "hs2_cp_combine", "hs2_cp_select_merge"):
        getattr(lib, name).restype = ctypes.c_int
    _libs[checked] = lib
    return lib


def make_shape(batch, n_q, h_q, h_kv, head_dim, window, topk, q_pos0, kv_len,
               softmax_scale: float = 0.0) -> hs2_shape:
    return hs2_shape(int(batch), int(n_q), int(h_q), int(h_kv), int(head_dim), int(window), int(topk), 0,
                     int(q_pos0), int(kv_len), float(softmax_scale))


def shape_of(q: torch.Tensor, k: torch.Tensor, *, window: int, topk: int, q_pos0: int,
             softmax_scale: float = 0.0) -> hs2_shape:
    B, Hq, nq, D = q.shape
    Bk, Hkv, N, Dk = k.shape
    if (B, D) != (Bk, Dk):
        raise ValueError("q and k disagree on batch or head_dim")
    return make_shape(B, nq, Hq, Hkv, D, window, topk, q_pos0, N, softmax_scale)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libhs2 takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libhs2 takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, where: str) -> None:
    if rc != HS2_OK:
        raise HS2Error(rc, where)


def hs2_workspace_size(shape: hs2_shape, entry: int, checked: bool = False) -> int:
    return int(load(checked).hs2_workspace_size(ctypes.byref(shape), int(entry)))


def alloc_workspace(shape: hs2_shape, entry: int, device="cuda", checked: bool = False,
                    stream=None) -> torch.Tensor:
    """Allocate (with torch) and initialise a workspace for `entry`."""
    n = hs2_workspace_size(shape, entry, checked)
    if n == 0:
        raise HS2Error(1, "hs2_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    hs2_workspace_init(ws, stream=stream, checked=checked)
    return ws


def hs2_workspace_init(ws: torch.Tensor, stream=None, checked: bool = False) -> None:
    _check(load(checked).hs2_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "hs2_workspace_init")


def _ws(ws):
    return (None, 0) if ws is None else (_ptr(ws), ws.numel() * ws.element_size())


def hs2_full_attn_select(shape, q, k, v, out, lse, idx, ws, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_full_attn_select(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                              _ptr(lse), _ptr(idx), wp, wn, _stream(stream)),
           "hs2_full_attn_select")


def hs2_full_attn_block_select(shape, block, q, k, v, out, lse, idx, ws, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_full_attn_block_select(ctypes.byref(shape), int(block), _ptr(q), _ptr(k), _ptr(v),
                                                    _ptr(out), _ptr(lse), _ptr(idx), wp, wn, _stream(stream)),
           "hs2_full_attn_block_select")


def hs2_swa_branches(shape, q, k_swa, v_swa, k, v, idx, out_swa, lse_swa, out_sel, lse_sel, ws=None, stream=None,
                     checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_swa_branches(ctypes.byref(shape), _ptr(q), _ptr(k_swa), _ptr(v_swa), _ptr(k), _ptr(v),
                                          _ptr(idx), _ptr(out_swa), _ptr(lse_swa), _ptr(out_sel), _ptr(lse_sel),
                                          wp, wn, _stream(stream)),
           "hs2_swa_branches")


def hs2_cp_workspace_size(shape, kv_off: int, entry: int, checked=False) -> int:
    return int(load(checked).hs2_cp_workspace_size(ctypes.byref(shape), int(kv_off), int(entry)))


def hs2_cp_attn_partial(shape, kv_off, q, k, v, out, lse, ws, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_cp_attn_partial(ctypes.byref(shape), int(kv_off), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                             _ptr(lse), wp, wn, _stream(stream)), "hs2_cp_attn_partial")


def hs2_cp_select_local(shape, kv_off, q, k, lse, idx, score, ws, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_cp_select_local(ctypes.byref(shape), int(kv_off), _ptr(q), _ptr(k), _ptr(lse),
                                             _ptr(idx), _ptr(score), wp, wn, _stream(stream)), "hs2_cp_select_local")


def hs2_cp_sparse_partial(shape, kv_off, q, k, v, idx, out, lse, ws, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_cp_sparse_partial(ctypes.byref(shape), int(kv_off), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
                                               _ptr(out), _ptr(lse), wp, wn, _stream(stream)),
           "hs2_cp_sparse_partial")


def hs2_cp_combine(n_parts, n_rows, head_dim, out_parts, lse_parts, out, lse, stream=None, checked=False) -> None:
    _check(load(checked).hs2_cp_combine(int(n_parts), int(n_rows), int(head_dim), _ptr(out_parts), _ptr(lse_parts),
                                        _ptr(out), _ptr(lse), _stream(stream)), "hs2_cp_combine")


def hs2_cp_select_merge(shape, kv_offs, idx_parts, score_parts, idx, stream=None, checked=False) -> None:
    offs = (ctypes.c_int64 * len(kv_offs))(*[int(o) for o in kv_offs])
    _check(load(checked).hs2_cp_select_merge(ctypes.byref(shape), len(kv_offs), offs, _ptr(idx_parts),
                                             _ptr(score_parts), _ptr(idx), _stream(stream)), "hs2_cp_select_merge")


def hs2_prefill_chunk(shape, q, k, v, out, lse, idx, ws, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_prefill_chunk(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                           _ptr(lse), _ptr(idx), wp, wn, _stream(stream)),
           "hs2_prefill_chunk")


def hs2_decode(shape, kv_len_per_seq, q, k, v, out, lse, idx, ws, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_decode(ctypes.byref(shape), _ptr(kv_len_per_seq), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(out), _ptr(lse), _ptr(idx), wp, wn, _stream(stream)),
           "hs2_decode")


def hs2_sparse_attn(shape, q, k, v, idx, out, ws=None, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_sparse_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
                                         _ptr(out), wp, wn, _stream(stream)),
           "hs2_sparse_attn")


def hs2_decode_sparse(shape, kv_len_per_seq, q, k, v, idx, out, ws=None, stream=None, checked=False) -> None:
    wp, wn = _ws(ws)
    _check(load(checked).hs2_decode_sparse(ctypes.byref(shape), _ptr(kv_len_per_seq), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(idx), _ptr(out), wp, wn, _stream(stream)),
           "hs2_decode_sparse")


def hs2_full_attn_select_static(shape, q, k, v, out, lse, idx, stream=None, checked=False) -> None:
    """hs2_full_attn_select without a workspace (library-internal static scratch)."""
    _check(load(checked).hs2_full_attn_select_static(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                                     _ptr(lse), _ptr(idx), _stream(stream)),
           "hs2_full_attn_select_static")


def hs2_static_scratch_status(stream=None, checked=False):
    """Returns (status, [code, kernel, a, b]) of the static array's error word; synchronises."""
    info = (ctypes.c_uint32 * 4)()
    rc = load(checked).hs2_static_scratch_status(_stream(stream), info)
    return int(rc), list(info)


def hs2_selftest_exp2(x: torch.Tensor, stream=None):
    """(hardware ex2, degree-3, degree-5, packed degree-5 at x, packed degree-5
    at x/2) evaluations of 2^x on the device."""
    n = x.numel()
    y = torch.empty(5 * n, dtype=torch.float32, device=x.device)
    _check(load().hs2_selftest_exp2(_ptr(x), _ptr(y), int(n), _stream(stream)), "hs2_selftest_exp2")
    return tuple(y[u * n:(u + 1) * n] for u in range(5))


def hs2_gather_probe(rows: torch.Tensor, order: torch.Tensor, passes: int, sink: torch.Tensor, stream=None):
    """Gather-bandwidth probe: reads rows[order[u]] (256-byte rows) `passes` times."""
    if rows.numel() * rows.element_size() % 256:
        raise ValueError("rows must hold whole 256-byte rows")
    n_rows = rows.numel() * rows.element_size() // 256
    _check(load().hs2_gather_probe(_ptr(rows), int(n_rows), _ptr(order), int(order.numel()), int(passes),
                                   _ptr(sink), _stream(stream)), "hs2_gather_probe")


def hs2_ex2_probe(iters: int, sink: torch.Tensor, stream=None) -> int:
    """Special-function-unit probe; returns the number of ex2 it executes."""
    n = ctypes.c_int64(0)
    _check(load().hs2_ex2_probe(int(iters), _ptr(sink), _stream(stream), ctypes.byref(n)), "hs2_ex2_probe")
    return int(n.value)


def hs2_selftest_wait(ws: torch.Tensor, limit_cycles: int, stream=None, checked=False) -> None:
    """The bounded-wait self-test: its timeout lands in the error word of ws."""
    _check(load(checked).hs2_selftest_wait(_ptr(ws), ws.numel() * ws.element_size(), int(limit_cycles),
                                           _stream(stream)), "hs2_selftest_wait")


def hs2_kv_bridge(shape: hs2_bridge_shape, seq_pos, hidden, w_kv, k_cache, v_cache, ws=None, stream=None,
                  checked=False):
    _check(load(checked).hs2_kv_bridge(ctypes.byref(shape), _ptr(seq_pos), _ptr(hidden), _ptr(w_kv),
                                       _ptr(k_cache), _ptr(v_cache), _ptr(ws),
                                       0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)),
           "hs2_kv_bridge")


def kv_bridge(hidden: torch.Tensor, w_kv: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, *,
              pos0: int = 0, seq_pos: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
              stream=None, checked: bool = False) -> None:
    """K/V of the new tokens, hidden [B, n_new, d_model] @ w_kv^T, written into the
    caches [B, H_kv, kv_cap, D] at rows pos_b + i (pos_b = seq_pos[b] or pos0)."""
    B, n_new, d_model = hidden.shape
    _, h_kv, kv_cap, D = k_cache.shape
    shape = hs2_bridge_shape(batch=B, n_new=n_new, d_model=d_model, h_kv=h_kv, head_dim=D, reserved=0,
                             pos0=pos0, kv_cap=kv_cap)
    hs2_kv_bridge(shape, seq_pos, hidden, w_kv, k_cache, v_cache, ws, stream, checked)


def kv_bridge_workspace(hidden: torch.Tensor, k_cache: torch.Tensor, stream=None, checked: bool = False):
    """A workspace of hs2_kv_bridge_workspace_size bytes (enables the split path), initialised."""
    B, n_new, d_model = hidden.shape
    _, h_kv, kv_cap, D = k_cache.shape
    shape = hs2_bridge_shape(batch=B, n_new=n_new, d_model=d_model, h_kv=h_kv, head_dim=D, reserved=0, pos0=0,
                             kv_cap=kv_cap)
    n = int(load(checked).hs2_kv_bridge_workspace_size(ctypes.byref(shape)))
    if n == 0:
        raise HS2Error(1, "hs2_kv_bridge_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=hidden.device)
    hs2_workspace_init(ws, stream=stream, checked=checked)
    return ws


def hs2_get_device_status(ws: torch.Tensor, stream=None, checked=False):
    """Returns (status, [code, kernel, a, b]); synchronises the stream."""
    info = (ctypes.c_uint32 * 4)()
    rc = load(checked).hs2_get_device_status(_ptr(ws), _stream(stream), info)
    return int(rc), list(info)


def hs2_select_retry_rows(shape, ws, stream=None, checked=False) -> int:
    """Rows of the last query chunk of the last selection on `ws` that ran the retry pass."""
    n = ctypes.c_int64(0)
    wp, wn = _ws(ws)
    _check(load(checked).hs2_select_retry_rows(ctypes.byref(shape), wp, wn, _stream(stream), ctypes.byref(n)),
           "hs2_select_retry_rows")
    return int(n.value)


def hs2_status_string(status: int, checked=False) -> str:
    return load(checked).hs2_status_string(int(status)).decode()


def hs2_launch_count(checked=False) -> int:
    return int(load(checked).hs2_launch_count())


def hs2_profile_start(checked=False) -> None:
    _check(load(checked).hs2_profile_start(), "hs2_profile_start")


def hs2_profile_stop(checked=False) -> dict:
    """{kernel name: (total ms, launches)} recorded since hs2_profile_start."""
    n = 24
    ms = (ctypes.c_float * n)()
    cnt = (ctypes.c_uint64 * n)()
    _check(load(checked).hs2_profile_stop(n, ms, cnt), "hs2_profile_stop")
    return {KERNEL_NAMES[u]: (float(ms[u]), int(cnt[u])) for u in range(1, n) if cnt[u]}


def hs2_is_checked_build(checked=False) -> bool:
    return bool(load(checked).hs2_is_checked_build())


# ---------------------------------------------------------------------------
# convenience: allocate outputs and run one layer (still one C-ABI call each)


def full_attn_select(q, k, v, *, window: int, topk: int, q_pos0: int = 0, ws=None, stream=None,
                     entry: str = "full", checked: bool = False):
    """Allocate out/lse/idx and run hs2_full_attn_select (or hs2_prefill_chunk)."""
    shape = shape_of(q, k, window=window, topk=topk, q_pos0=q_pos0)
    e = HS2_ENTRY_PREFILL if entry == "prefill" else HS2_ENTRY_FULL_SELECT
    if ws is None:
        ws = alloc_workspace(shape, e, q.device, checked, stream)
    out = torch.empty_like(q)
    B, Hq, nq, D = q.shape
    lse = torch.empty(B, Hq, nq, dtype=torch.float32, device=q.device)
    idx = torch.empty(B, k.shape[1], nq, topk, dtype=torch.int32, device=q.device)
    fn = hs2_prefill_chunk if entry == "prefill" else hs2_full_attn_select
    fn(shape, q, k, v, out, lse, idx, ws, stream, checked)
    return out, lse, idx


def full_attn_block_select(q, k, v, *, window: int, topk: int, block: int, q_pos0: int = 0, ws=None,
                           stream=None, checked: bool = False):
    """Allocate out/lse/idx and run hs2_full_attn_block_select."""
    shape = shape_of(q, k, window=window, topk=topk, q_pos0=q_pos0)
    if ws is None:
        ws = alloc_workspace(shape, HS2_ENTRY_BLOCK_SELECT, q.device, checked, stream)
    out = torch.empty_like(q)
    B, Hq, nq, D = q.shape
    lse = torch.empty(B, Hq, nq, dtype=torch.float32, device=q.device)
    idx = torch.empty(B, k.shape[1], nq, topk, dtype=torch.int32, device=q.device)
    hs2_full_attn_block_select(shape, block, q, k, v, out, lse, idx, ws, stream, checked)
    return out, lse, idx


def swa_branches(q, k_swa, v_swa, k, v, idx, *, window: int, q_pos0: int = 0, stream=None, ws=None,
                 checked: bool = False):
    """The predecessor design's two branches: returns (out_swa, lse_swa, out_sel, lse_sel)."""
    shape = shape_of(q, k, window=window, topk=idx.shape[-1], q_pos0=q_pos0)
    B, Hq, nq, D = q.shape
    out_swa, out_sel = torch.empty_like(q), torch.empty_like(q)
    lse_swa = torch.empty(B, Hq, nq, dtype=torch.float32, device=q.device)
    lse_sel = torch.empty_like(lse_swa)
    hs2_swa_branches(shape, q, k_swa, v_swa, k, v, idx, out_swa, lse_swa, out_sel, lse_sel, ws, stream, checked)
    return out_swa, lse_swa, out_sel, lse_sel


def decode(q, k, v, *, window: int, topk: int, kv_len_per_seq=None, ws=None, stream=None,
           checked: bool = False):
    shape = shape_of(q, k, window=window, topk=topk, q_pos0=k.shape[2] - 1)
    if ws is None:
        ws = alloc_workspace(shape, HS2_ENTRY_DECODE, q.device, checked, stream)
    out = torch.empty_like(q)
    B, Hq, nq, D = q.shape
    lse = torch.empty(B, Hq, nq, dtype=torch.float32, device=q.device)
    idx = torch.empty(B, k.shape[1], nq, topk, dtype=torch.int32, device=q.device)
    hs2_decode(shape, kv_len_per_seq, q, k, v, out, lse, idx, ws, stream, checked)
    return out, lse, idx


def sparse_attn(q, k, v, idx, *, window: int, q_pos0: int = 0, stream=None, ws=None,
                checked: bool = False):
    """Run one sparse KV-reuse layer (queries at q_pos0 + i)."""
    shape = shape_of(q, k, window=window, topk=idx.shape[-1], q_pos0=q_pos0)
    out = torch.empty_like(q)
    hs2_sparse_attn(shape, q, k, v, idx, out, ws, stream, checked)
    return out


def decode_sparse(q, k, v, idx, *, window: int, kv_len_per_seq=None, stream=None, ws=None,
                  checked: bool = False):
    """Run one sparse KV-reuse layer for a decode step (one query per sequence)."""
    shape = shape_of(q, k, window=window, topk=idx.shape[-1], q_pos0=k.shape[2] - 1)
    out = torch.empty_like(q)
    hs2_decode_sparse(shape, kv_len_per_seq, q, k, v, idx, out, ws, stream, checked)
    return out

"""fp64 CPU oracle for the HySparse2 full-attention + selection + sparse-reuse path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code with the CUDA library.

The arithmetic lives in ``hs2_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only compiles it with gcc and marshals numpy arrays through ctypes.
Inputs are raw bf16 bit patterns (``numpy.uint16``), so the oracle reads exactly
the bits the GPU reads.

Method (HySparse2 pages: xiawanshe.com report, sections "两级KV共享" /
"Token级选择"; davidyin.dev notes, section "HySparse2 的解法"):

* ``full_select`` -- one full-attention layer over the shared cache: causal
  softmax attention output and LSE per head, plus the per-(token, KV-head)
  selection of min(K, t-W+1) candidates j <= t-W ranked by the group-summed
  causal probability, ties to the lower index, emitted ascending, -1 padded.
* ``sparse`` -- one KV-reuse layer: softmax attention of the layer's own query
  over idx U window(t).
* ``block_select`` -- the predecessor block-level selection at the same
  budget: whole blocks of contiguous candidates, ranked by summed score.
* ``branches`` -- the predecessor design's sparse layer: a sliding-window
  branch over its own cache and a selected-tokens branch over the shared one,
  each with its own softmax (outputs and LSEs, uncombined).
* ``kv_bridge`` -- KV bridging (same report, section "两级KV共享", first
  level): a token's Cross-Decoder K and V from its Self-Decoder hidden state by
  one projection, output features [K heads | V heads], D per head.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hs2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhs2_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``hs2_oracle.c`` into ``libhs2_oracle.so`` (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    # -O2 without -ffast-math: the oracle keeps IEEE fp64 semantics.
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def open_library(path: str):
    """Open a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    i32 = ctypes.c_int
    lib.hs2o_full_select.argtypes = [i32, i32, i32, i32, i32, ctypes.c_double,
                                     i64, P, P, P, P, i64, i64,
                                     P, P, P, P, P, P, i64, i32]
    lib.hs2o_full_select.restype = i32
    lib.hs2o_sparse.argtypes = [i32, i32, i32, i32, i32, ctypes.c_double,
                                i64, P, P, P, P, i64, i64, P, P, i32]
    lib.hs2o_sparse.restype = i32
    lib.hs2o_kv_bridge.argtypes = [i64, i32, i32, i32, P, P, P, P, i32]
    lib.hs2o_block_select.argtypes = [i64, i32, i32, i32, i32, P, P, i64, P, P, P]
    lib.hs2o_block_select.restype = i32
    lib.hs2o_kv_bridge.restype = i32
    lib.hs2o_branches.argtypes = [i32, i32, i32, i32, i32, ctypes.c_double, i64, P, P, P, P, P, P, i64, P,
                                  P, P, P, P, i32]
    lib.hs2o_branches.restype = i32
    lib.hs2o_max_threads.argtypes = []
    lib.hs2o_max_threads.restype = i32
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = open_library(_LIB_PATH)
    return _lib


def max_threads() -> int:
    return int(_load().hs2o_max_threads())


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _as_bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (numpy.uint16)")
    return a


def full_select(q_rows, t, k, v, *, window: int, topk: int, scale: float | None = None,
                want_scores: bool = False, n_threads: int = 0):
    """Full causal attention + selection for query rows of ONE sequence.

    q_rows: uint16 [n_rows, H_q, D] (bf16 bits); t: int64 [n_rows] absolute positions;
    k, v: uint16 [H_kv, kv_len, D].
    Returns dict(out [n,H_q,D] f64, lse [n,H_q] f64, idx [n,H_kv,topk] i32,
    kth [n,H_kv] f64, next [n,H_kv] f64, scores [n,H_kv,max_cand] f64 or None).
    """
    q_rows = _as_bits(q_rows)
    k = _as_bits(k)
    v = _as_bits(v)
    t = np.ascontiguousarray(t, dtype=np.int64)
    n, h_q, d = q_rows.shape
    h_kv, kv_len, d2 = k.shape
    assert d2 == d and v.shape == k.shape and t.shape == (n,)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((n, h_q, d), np.float64)
    lse = np.zeros((n, h_q), np.float64)
    idx = np.full((n, h_kv, topk), -7, np.int32)
    kth = np.zeros((n, h_kv), np.float64)
    nxt = np.zeros((n, h_kv), np.float64)
    scores = None
    stride = 0
    if want_scores:
        stride = int(max(1, (t.max() - window + 1) if n else 1))
        scores = np.full((n, h_kv, stride), np.nan, np.float64)
    rc = _load().hs2o_full_select(h_q, h_kv, d, window, topk, float(scale), n, _ptr(t),
                                  _ptr(q_rows), _ptr(k), _ptr(v), kv_len, kv_len,
                                  _ptr(out), _ptr(lse), _ptr(idx), _ptr(kth), _ptr(nxt),
                                  _ptr(scores), stride, int(n_threads))
    if rc != 0:
        raise RuntimeError(f"hs2o_full_select failed with code {rc}")
    return dict(out=out, lse=lse, idx=idx, kth=kth, next=nxt, scores=scores)


def sparse(q_rows, t, k, v, idx, *, window: int, scale: float | None = None,
           n_threads: int = 0) -> np.ndarray:
    """One KV-reuse sparse layer for query rows of ONE sequence.

    idx: int32 [n_rows, H_kv, topk] (ascending or not; -1 = unused).
    Returns out [n_rows, H_q, D] f64.
    """
    q_rows = _as_bits(q_rows)
    k = _as_bits(k)
    v = _as_bits(v)
    t = np.ascontiguousarray(t, dtype=np.int64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    n, h_q, d = q_rows.shape
    h_kv, kv_len, _ = k.shape
    topk = idx.shape[2]
    assert idx.shape[:2] == (n, h_kv)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((n, h_q, d), np.float64)
    rc = _load().hs2o_sparse(h_q, h_kv, d, window, topk, float(scale), n, _ptr(t),
                             _ptr(q_rows), _ptr(k), _ptr(v), kv_len, kv_len,
                             _ptr(idx), _ptr(out), int(n_threads))
    if rc != 0:
        raise RuntimeError(f"hs2o_sparse failed with code {rc}")
    return out


def kv_bridge(hidden, w, *, h_kv: int, head_dim: int, n_threads: int = 0):
    """K and V of each token from its hidden state: ``hidden`` [n_rows, d_model]
    and ``w`` [2 * h_kv * head_dim, d_model] as bf16 bit patterns; returns
    (k, v), each [n_rows, h_kv, head_dim] float64."""
    x = _as_bits(hidden)
    wb = _as_bits(w)
    n_rows, d_model = x.shape
    assert wb.shape == (2 * h_kv * head_dim, d_model)
    k = np.empty((n_rows, h_kv, head_dim), dtype=np.float64)
    v = np.empty_like(k)
    rc = _load().hs2o_kv_bridge(n_rows, d_model, h_kv, head_dim, _ptr(x), _ptr(wb), _ptr(k), _ptr(v),
                                int(n_threads))
    if rc != 0:
        raise ValueError(f"hs2o_kv_bridge: error {rc}")
    return k, v


def block_select(q_rows, t, k, v, *, window: int, topk: int, block: int, scale: float | None = None,
                 n_threads: int = 0):
    """Block-level selection from the same per-candidate scores as ``full_select``:
    returns dict(idx [n_rows, h_kv, topk] token indices of the kept blocks,
    ascending, -1 padded; kth_block / next_block [n_rows, h_kv]: score of the last
    kept block and of the best block left out (-1 if none); and the full_select
    result under "full")."""
    full = full_select(q_rows, t, k, v, window=window, topk=0, scale=scale, want_scores=True,
                       n_threads=n_threads)
    t = np.ascontiguousarray(np.asarray(t, dtype=np.int64))
    sc = np.ascontiguousarray(full["scores"], dtype=np.float64)
    n_rows, h_kv = sc.shape[0], sc.shape[1]
    idx = np.empty((n_rows, h_kv, topk), dtype=np.int32)
    kth = np.empty((n_rows, h_kv), dtype=np.float64)
    nxt = np.empty((n_rows, h_kv), dtype=np.float64)
    rc = _load().hs2o_block_select(n_rows, h_kv, window, topk, block, _ptr(t), _ptr(sc), sc.shape[2],
                                   _ptr(idx), _ptr(kth), _ptr(nxt))
    if rc != 0:
        raise ValueError(f"hs2o_block_select: error {rc}")
    return dict(idx=idx, kth_block=kth, next_block=nxt, full=full)


def branches(q_rows, t, k_swa, v_swa, k, v, idx, *, window: int, scale: float | None = None,
             n_threads: int = 0):
    """The two branches of a predecessor-design sparse layer for query rows of ONE
    sequence: returns dict(out_swa, lse_swa, out_sel, lse_sel); out [n, H_q, D]
    f64, lse [n, H_q] f64 (natural log; -inf for a row with no selected key).
    k_swa, v_swa: the window branch's own cache; k, v: the shared cache, all
    uint16 [H_kv, kv_len, D]; idx int32 [n, H_kv, topk]."""
    q_rows = _as_bits(q_rows)
    k_swa, v_swa, k, v = _as_bits(k_swa), _as_bits(v_swa), _as_bits(k), _as_bits(v)
    t = np.ascontiguousarray(t, dtype=np.int64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    n, h_q, d = q_rows.shape
    h_kv, kv_len, _ = k.shape
    assert k_swa.shape == k.shape and v_swa.shape == k.shape and v.shape == k.shape
    assert idx.shape[:2] == (n, h_kv)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    res = dict(out_swa=np.zeros((n, h_q, d)), lse_swa=np.zeros((n, h_q)),
               out_sel=np.zeros((n, h_q, d)), lse_sel=np.zeros((n, h_q)))
    rc = _load().hs2o_branches(h_q, h_kv, d, window, idx.shape[2], float(scale), n, _ptr(t), _ptr(q_rows),
                               _ptr(k_swa), _ptr(v_swa), _ptr(k), _ptr(v), kv_len, _ptr(idx),
                               _ptr(res["out_swa"]), _ptr(res["lse_swa"]), _ptr(res["out_sel"]),
                               _ptr(res["lse_sel"]), int(n_threads))
    if rc != 0:
        raise RuntimeError(f"hs2o_branches failed with code {rc}")
    return res

"""The entry point that allocates nothing: hs2_full_attn_select_static.

It exists for callers that cannot allocate device memory where they run the
layer (a pre-sized memory pool they may not grow, a host runtime that hands
them only input and output buffers, a step that must not synchronise the
device).  Its scratch is a fixed static array inside the library; these tests
check that, called through the C ABI, it gives the same outputs as
hs2_full_attn_select with a caller-allocated workspace on two calls in a row
with different inputs, that those outputs also match the fp64 oracle, that
its error word reads clean afterwards, that a warm call leaves the device's
free memory unchanged, and that it refuses shapes whose scratch would not fit.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sparse_flash_b200 import native as nv
from long_context_sparse_flash_b200 import workloads as wl
from tests import parity as P


def _static_call(shape, q, k, v, out, lse, idx):
    lib = nv.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.hs2_full_attn_select_static(ctypes.byref(shape), nv._ptr(q), nv._ptr(k), nv._ptr(v), nv._ptr(out),
                                           nv._ptr(lse), nv._ptr(idx), stream)


@pytest.mark.gpu
def test_static_scratch_entry_matches_allocating_entry():
    from long_context_sparse_flash_b200 import build
    build.build()
    assert torch.cuda.is_available()
    # more candidates than topk, so the selection pass uses its score scratch
    w = wl.custom("static_scratch", n_q=700, q_pos0=300, h_q=16, h_kv=2, head_dim=128, window=128, topk=256,
                  n_sparse=0)
    for call, seed in enumerate((21, 22)):
        inp = wl.make_inputs(w, "cuda", seed=seed, with_sparse=False)
        q, k, v = inp["q"], inp["k"], inp["v"]
        ref_out, ref_lse, ref_idx = nv.full_attn_select(q, k, v, window=w.window, topk=w.topk, q_pos0=w.q_pos0)
        shape = nv.shape_of(q, k, window=w.window, topk=w.topk, q_pos0=w.q_pos0)
        assert nv.hs2_workspace_size(shape, nv.HS2_ENTRY_FULL_SELECT) > 256
        out = torch.full_like(q, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        idx = torch.full_like(ref_idx, -7)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        assert _static_call(shape, q, k, v, out, lse, idx) == nv.HS2_OK
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        if call == 1:
            # the first call may load the library's kernels (and its static
            # array) onto the device; a warm call takes no device memory
            assert free_after == free_before, (free_before, free_after)
        rc, info = nv.hs2_static_scratch_status()
        assert rc == nv.HS2_OK, (rc, info)
        P.assert_close(P.to_f64(out), P.to_f64(ref_out), f"call {call} out")
        P.assert_close(P.to_f64(lse), P.to_f64(ref_lse), f"call {call} lse", atol=P.LSE_ATOL, rtol=0.0)
        assert torch.equal(idx, ref_idx), f"call {call}: selection differs"
        # and against the oracle itself, on rows around the window and top-k boundaries
        gpu = dict(out=out, lse=lse, idx=idx, sparse=[])
        P.compare_rows(w, inp, gpu, 0, np.array([0, 1, 127, 128, 300, 383, 384, 385, 600, 699]))


def test_static_scratch_entry_rejects_oversized_shapes():
    lib = nv.load()
    limit = lib.hs2_static_scratch_bytes()
    # 32K prefill needs about 1 GiB of score scratch: beyond the static array
    shape = nv.make_shape(1, 32768, 32, 4, 128, 128, 1024, 0, 32768)
    assert nv.hs2_workspace_size(shape, nv.HS2_ENTRY_FULL_SELECT) > limit
    before = nv.hs2_launch_count()
    fake = ctypes.c_void_p(1 << 40)
    rc = lib.hs2_full_attn_select_static(ctypes.byref(shape), fake, fake, fake, fake, fake, fake, None)
    assert rc == 3  # HS2_ERR_WORKSPACE
    assert nv.hs2_launch_count() == before

"""Needle recall on the GPU path (a sanity check beside parity): the keys planted
for a probe query, k = 2 normalize(sum of the group's queries) + 0.1 noise at
positions older than the window, must be in that query's selection for every KV
group.  The oracle selects all of them on sampled rows of these workloads.

Only the workloads with N(0,1)*0.5 keys: against the 1M workloads' segment keys
(unit-variance centroids plus noise) a needle's logit sits well inside the
spread of ordinary keys, so neither the oracle nor the kernels select it (the
sampled-row parity tests show the two agree there)."""
import numpy as np
import pytest
import torch

from long_context_sparse_flash_b200 import native as nv
from long_context_sparse_flash_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from long_context_sparse_flash_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load()


def _recall(w, inp, idx):
    idx = idx.cpu().numpy()  # [B, H_kv, n_q, K]
    rec = []
    for b, planted in enumerate(inp["needles"]):
        for i, pos in planted.items():
            for g in range(w.h_kv):
                sel = set(idx[b, g, i].tolist())
                rec.append(len(sel & set(pos)) / len(pos))
    return np.array(rec)


@pytest.mark.parametrize("name", ["tiny", "prefill_32k", "decode_128k"])
def test_planted_needles_are_selected(name):
    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w, "cuda", with_sparse=False)
    if w.decode:
        _, _, idx = nv.decode(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk)
    else:
        _, _, idx = nv.full_attn_select(inp["q"], inp["k"], inp["v"], window=w.window, topk=w.topk, q_pos0=w.q_pos0)
    torch.cuda.synchronize()
    rec = _recall(w, inp, idx)
    assert rec.size > 0
    print(name, "probes x groups", rec.size, "mean recall", rec.mean(), "min", rec.min())
    assert rec.mean() >= 0.99 and rec.min() >= 0.9

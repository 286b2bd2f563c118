"""Why the selection sweep does not prune candidates with the max-head bound.

Each candidate's score is a sum over the G heads of its group, so it is at
most G * max_h p_h.  A sweep could skip a candidate's G exponentials when that
bound falls below the row's threshold.  On these workloads' inputs the bound
is loose: the logits of one key differ across the heads of a group by about
half a nat, so G * max_h p_h is above the threshold for most candidates.  On
the GPU a warp holds 32 consecutive keys and takes the exponentials for all of
them if any one needs them, so nearly every warp would still compute them.
This test measures both fractions in fp64 (numpy, CPU) on the 1M-context key
structure (clustered segments plus needles) and on Gaussian keys, at a 32K
context, with the threshold the sweep uses (the r-th largest of a fixed-stride
sample of 1024 keys)."""
import numpy as np
import pytest

from long_context_sparse_flash_b200 import workloads as wl


@pytest.mark.parametrize("keys,needles", [("segments", 64), ("gaussian", 16)])
def test_max_head_bound_rejects_almost_no_warp(keys, needles):
    N, G, D = 32768, 8, 128
    w = wl.custom("bound", n_q=64, q_pos0=N - 64, kv_len=N, h_q=32, h_kv=4, head_dim=D, window=128, topk=1024,
                  keys=keys, needles=needles, seed=4, n_sparse=0)
    inp = wl.make_inputs(w, "cpu", with_sparse=False)
    q = inp["q"][0].float().numpy().astype(np.float64)
    k = inp["k"][0].float().numpy().astype(np.float64)
    tot = passes = warps = warps_pass = 0
    for i in range(0, 64, 16):
        t = w.q_pos0 + i
        n = t - w.window + 1
        for g in range(w.h_kv):
            s = q[g * G:(g + 1) * G, i] @ k[g, :t + 1].T / np.sqrt(D)
            m = s.max(1, keepdims=True)
            p = np.exp(s - (m + np.log(np.exp(s - m).sum(1, keepdims=True))))[:, :n]
            score = p.sum(0)
            samp = score[::N // 1024][:1024]
            lam = w.topk * len(samp) / n
            r = int(np.ceil(lam + 4.5 * np.sqrt(lam) + 2))
            tau = np.sort(samp)[::-1][r - 1]
            admitted = G * p.max(0) >= tau
            assert np.all(admitted[score >= tau])  # the bound never drops a survivor
            tot += n
            passes += admitted.sum()
            nw = n // 32
            warps += nw
            warps_pass += admitted[:nw * 32].reshape(nw, 32).any(1).sum()
    assert passes / tot > 0.5, passes / tot
    assert warps_pass / warps > 0.9, warps_pass / warps

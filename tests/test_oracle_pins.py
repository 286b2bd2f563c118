"""Pins for the fp64 CPU oracle: each test checks it against something other
than its own formula -- closed forms, library routines on special cases,
invariants the method fixes, and brute force on tiny inputs -- chosen so that a
plausible mistake (wrong scale, causal or window off-by-one, wrong head->group
map, reversed tie rule, score normalised over the wrong set, wrong LSE base)
fails at least one of them.

Method: HySparse2 pages, xiawanshe.com report sections "两级KV共享" (KV reuse:
one full-attention layer's KV cache and token selection are reused by the
following sparse layers) and "Token级选择" (token-level selection, forced last
128 tokens + 1024 selected older tokens, one shared KV cache).
"""
import decimal
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle


def bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (RNE) and return their bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def unbits(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_qkv(rng, n_rows, h_q, h_kv, n, d, scale=0.5):
    q = bits(rng.standard_normal((n_rows, h_q, d)) * scale)
    k = bits(rng.standard_normal((h_kv, n, d)) * scale)
    v = bits(rng.standard_normal((h_kv, n, d)) * scale)
    return q, k, v


# ---------------------------------------------------------------------------
# closed forms


@pytest.mark.parametrize("G", [1, 2, 4])
def test_zero_query_closed_form(G):
    """q = 0: every s_j = 0, so p_j = 1/(t+1), lse = ln(t+1), out = mean(v[0..t]),
    every score = G/(t+1); the tie rule then selects exactly the lowest indices
    [0, min(K, t-W+1)), and a sparse layer with q' = 0 returns the plain mean of v
    over selected U window."""
    rng = np.random.default_rng(1)
    h_kv, d, n, W, K = 2, 8, 60, 16, 8
    h_q = G * h_kv
    ts = np.array([0, 1, W - 2, W - 1, W, W + 1, W + K - 2, W + K - 1, W + K, W + K + 1, n - 1])
    q = np.zeros((len(ts), h_q, d), np.uint16)  # bf16 +0.0
    _, k, v = rand_qkv(rng, 1, h_q, h_kv, n, d)
    res = oracle.full_select(q, ts, k, v, window=W, topk=K, want_scores=True)
    vf = unbits(v)
    for r, t in enumerate(ts):
        n_cand = max(0, t - W + 1)
        n_sel = min(K, n_cand)
        for h in range(h_q):
            g = h // G
            assert res["lse"][r, h] == pytest.approx(math.log(t + 1), abs=1e-12)
            np.testing.assert_allclose(res["out"][r, h], vf[g, :t + 1].mean(0), rtol=0, atol=1e-12)
        for g in range(h_kv):
            want = list(range(n_sel)) + [-1] * (K - n_sel)
            assert res["idx"][r, g].tolist() == want, (t, g)
            if n_cand:
                np.testing.assert_allclose(res["scores"][r, g, :n_cand], G / (t + 1), rtol=1e-13)
                assert res["kth"][r, g] == pytest.approx(G / (t + 1), rel=1e-13)
            else:
                assert math.isnan(res["kth"][r, g])
    out_sp = oracle.sparse(q, ts, k, v, res["idx"], window=W)
    for r, t in enumerate(ts):
        for h in range(h_q):
            g = h // G
            sel = [j for j in res["idx"][r, g] if j >= 0] + list(range(max(0, t - W + 1), t + 1))
            np.testing.assert_allclose(out_sp[r, h], vf[g, sel].mean(0), rtol=0, atol=1e-12)


def test_two_key_scale_and_lse():
    """t = 1 with k_0 = 0 and k_1 = b e_0, q = a e_0: s_1 = a b / sqrt(D), so
    lse = ln(1 + e^{s_1}) and out = sigmoid(s_1) v_1 + (1 - sigmoid(s_1)) v_0.
    Catches a wrong softmax scale (1/D, none) and a wrong LSE base."""
    d, a, b = 16, 2.0, 1.5
    q = np.zeros((1, 1, d)); q[0, 0, 0] = a
    k = np.zeros((1, 2, d)); k[0, 1, 0] = b
    rng = np.random.default_rng(2)
    v = rng.standard_normal((1, 2, d))
    res = oracle.full_select(bits(q), np.array([1]), bits(k), bits(v), window=1, topk=1)
    s1 = a * b / math.sqrt(d)
    assert res["lse"][0, 0] == pytest.approx(math.log1p(math.exp(s1)), abs=1e-14)
    p1 = scipy.special.expit(s1)
    vv = unbits(bits(v))
    np.testing.assert_allclose(res["out"][0, 0], p1 * vv[0, 1] + (1 - p1) * vv[0, 0], atol=1e-14)
    # window = 1 leaves j = 0 as the only candidate: selected, with score 1 - p1
    assert res["idx"][0, 0].tolist() == [0]
    assert res["kth"][0, 0] == pytest.approx(1 - p1, abs=1e-14)


def test_identity_values_link_score_to_probabilities():
    """V = identity rows (v_j = e_j, N <= D): out_h[j] = p_{h,j}.  The selection
    score must equal sum over the group's heads of out_h[j] for j <= t-W --
    i.e. the causal probability normalised over the WHOLE row, window included --
    and every probability row must sum to 1."""
    rng = np.random.default_rng(3)
    h_q, h_kv, d, W, K = 8, 2, 64, 8, 10
    n = d
    G = h_q // h_kv
    ts = np.array([5, 8, 20, 40, 63])
    q = bits(rng.standard_normal((len(ts), h_q, d)))
    k = bits(rng.standard_normal((h_kv, n, d)))
    v = bits(np.tile(np.eye(n, d)[None], (h_kv, 1, 1)))
    res = oracle.full_select(q, ts, k, v, window=W, topk=K, want_scores=True)
    for r, t in enumerate(ts):
        np.testing.assert_allclose(res["out"][r].sum(-1), 1.0, atol=1e-12)
        assert np.all(res["out"][r][:, t + 1:] == 0.0)  # causal: no future key
        n_cand = max(0, t - W + 1)
        for g in range(h_kv):
            want = res["out"][r, g * G:(g + 1) * G, :n_cand].sum(0)
            np.testing.assert_allclose(res["scores"][r, g, :n_cand], want, rtol=1e-12, atol=1e-15)


def test_library_softmax_special_case():
    """Outputs against scipy's softmax/logsumexp on the materialised score row."""
    rng = np.random.default_rng(4)
    h_q, h_kv, d, n = 4, 2, 32, 50
    ts = np.array([0, 7, 31, 49])
    q, k, v = rand_qkv(rng, len(ts), h_q, h_kv, n, d, scale=1.0)
    res = oracle.full_select(q, ts, k, v, window=4, topk=3)
    qf, kf, vf = unbits(q), unbits(k), unbits(v)
    for r, t in enumerate(ts):
        for h in range(h_q):
            g = h // (h_q // h_kv)
            s = kf[g, :t + 1] @ qf[r, h] / math.sqrt(d)
            assert res["lse"][r, h] == pytest.approx(scipy.special.logsumexp(s), abs=1e-12)
            np.testing.assert_allclose(res["out"][r, h], scipy.special.softmax(s) @ vf[g, :t + 1],
                                       atol=1e-12)


# ---------------------------------------------------------------------------
# structure of the method


def test_head_to_group_map_is_contiguous():
    """g = h // G: with group 1's keys all zero, heads G..2G-1 see a uniform row
    (lse = ln(t+1)) while heads 0..G-1 do not.  A modulo map (g = h % H_kv)
    would make heads 1, 3, ... uniform instead."""
    rng = np.random.default_rng(5)
    h_q, h_kv, d, n = 4, 2, 16, 40
    q = bits(rng.standard_normal((1, h_q, d)) * 2)
    k = rng.standard_normal((h_kv, n, d)) * 2
    k[1] = 0.0
    v = rng.standard_normal((h_kv, n, d))
    t = 39
    res = oracle.full_select(q, np.array([t]), bits(k), bits(v), window=8, topk=4)
    for h in (2, 3):
        assert res["lse"][0, h] == pytest.approx(math.log(t + 1), abs=1e-12)
    for h in (0, 1):
        assert abs(res["lse"][0, h] - math.log(t + 1)) > 1e-3


def test_group_of_identical_heads_scales_score():
    """G copies of one head with identical queries: score = G * p, so the
    selection equals the single-head (G = 1) selection and kth scales by G."""
    rng = np.random.default_rng(6)
    d, n, W, K = 16, 300, 32, 20
    ts = np.array([40, 100, 299])
    q1 = bits(rng.standard_normal((len(ts), 1, d)))
    k = bits(rng.standard_normal((1, n, d)))
    v = bits(rng.standard_normal((1, n, d)))
    one = oracle.full_select(q1, ts, k, v, window=W, topk=K, want_scores=True)
    for G in (2, 4, 8):
        qg = np.repeat(q1, G, axis=1)
        many = oracle.full_select(qg, ts, k, v, window=W, topk=K, want_scores=True)
        np.testing.assert_array_equal(many["idx"], one["idx"])
        np.testing.assert_allclose(many["kth"], G * one["kth"], rtol=1e-13)


def test_dominant_planted_key_is_selected():
    """A key planted as c * q_hat with large c dominates its row: it is selected
    whenever it is a candidate (t >= j + W) and the output approaches its value."""
    rng = np.random.default_rng(7)
    h_q, h_kv, d, n, W, K = 4, 1, 32, 400, 64, 16
    q = rng.standard_normal((1, h_q, d))
    qhat = q[0].sum(0) / np.linalg.norm(q[0].sum(0))
    k = rng.standard_normal((h_kv, n, d)) * 0.3
    v = rng.standard_normal((h_kv, n, d))
    j = 57
    k[0, j] = 200.0 * qhat
    qb, kb, vb = bits(q), bits(k), bits(v)
    for t in (j + W - 1, j + W, j + W + 1, n - 1):
        res = oracle.full_select(qb, np.array([t]), kb, vb, window=W, topk=K)
        sel = res["idx"][0, 0]
        if t >= j + W:
            assert j in sel.tolist()
        else:
            assert j not in sel.tolist()  # still inside the forced window
        # the planted key carries almost all probability mass of every head
        np.testing.assert_allclose(res["out"][0], np.tile(unbits(vb)[0, j], (h_q, 1)), atol=0.05)


def test_selection_invariants_random():
    """Size min(K, t-W+1); unique; ascending; inside [0, t-W]; -1 padded;
    every selected score >= kth >= every unselected score; among candidates
    tied with kth the selected ones have the lowest indices."""
    rng = np.random.default_rng(8)
    h_q, h_kv, d, n, W, K = 8, 2, 16, 500, 32, 40
    ts = np.array([0, 10, 31, 32, 33, 71, 72, 73, 250, 499])
    q, k, v = rand_qkv(rng, len(ts), h_q, h_kv, n, d)
    res = oracle.full_select(q, ts, k, v, window=W, topk=K, want_scores=True)
    for r, t in enumerate(ts):
        n_cand = max(0, t - W + 1)
        n_sel = min(K, n_cand)
        for g in range(h_kv):
            row = res["idx"][r, g]
            sel = row[:n_sel]
            assert np.all(row[n_sel:] == -1)
            assert np.all(np.diff(sel) > 0)
            assert (sel.min() >= 0 and sel.max() <= t - W) if n_sel else True
            if n_sel == 0:
                continue
            sc = res["scores"][r, g, :n_cand]
            kth = res["kth"][r, g]
            mask = np.zeros(n_cand, bool); mask[sel] = True
            assert sc[mask].min() == kth
            if (~mask).any():
                assert sc[~mask].max() <= kth
                assert res["next"][r, g] == sc[~mask].max()
                tied_out = np.nonzero((~mask) & (sc == kth))[0]
                tied_in = np.nonzero(mask & (sc == kth))[0]
                if len(tied_out):
                    assert tied_in.max() < tied_out.min()


def test_exact_ties_go_to_lower_index():
    """Duplicate key rows give bitwise-equal scores; with K cutting through the
    tied group the lower indices must win (reversed tie rule fails)."""
    rng = np.random.default_rng(9)
    h_q, h_kv, d, n, W = 2, 1, 8, 64, 4
    q = rng.standard_normal((1, h_q, d))
    k = rng.standard_normal((h_kv, n, d)) * 0.1
    best = q[0].sum(0) / np.linalg.norm(q[0].sum(0))
    dup = [3, 11, 20, 41]  # four identical, clearly highest-scoring keys
    for j in dup:
        k[0, j] = 3.0 * best
    v = rng.standard_normal((h_kv, n, d))
    res = oracle.full_select(bits(q), np.array([n - 1]), bits(k), bits(v), window=W, topk=2,
                             want_scores=True)
    assert res["idx"][0, 0].tolist() == [3, 11]
    assert res["scores"][0, 0, 3] == res["scores"][0, 0, 41]


# ---------------------------------------------------------------------------
# sparse (KV reuse) layer


def test_sparse_with_full_budget_equals_full_attention():
    """topk >= t-W+1 selects every candidate: the sparse layer with the SAME query
    is exactly full causal attention."""
    rng = np.random.default_rng(10)
    h_q, h_kv, d, n, W = 8, 2, 32, 300, 16
    ts = np.array([0, 5, 15, 16, 17, 120, 299])
    q, k, v = rand_qkv(rng, len(ts), h_q, h_kv, n, d)
    res = oracle.full_select(q, ts, k, v, window=W, topk=n)
    out = oracle.sparse(q, ts, k, v, res["idx"], window=W)
    np.testing.assert_allclose(out, res["out"], rtol=0, atol=1e-12)


def test_sparse_with_zero_budget_is_sliding_window():
    """topk = 0: the sparse layer is textbook sliding-window attention of width W,
    checked against scipy's softmax over the window."""
    rng = np.random.default_rng(11)
    h_q, h_kv, d, n, W = 4, 2, 32, 200, 24
    ts = np.array([0, 3, 23, 24, 25, 150, 199])
    q, k, v = rand_qkv(rng, len(ts), h_q, h_kv, n, d, scale=1.0)
    idx = np.zeros((len(ts), h_kv, 0), np.int32)
    out = oracle.sparse(q, ts, k, v, idx, window=W)
    qf, kf, vf = unbits(q), unbits(k), unbits(v)
    for r, t in enumerate(ts):
        lo = max(0, t - W + 1)
        for h in range(h_q):
            g = h // (h_q // h_kv)
            s = kf[g, lo:t + 1] @ qf[r, h] / math.sqrt(d)
            np.testing.assert_allclose(out[r, h], scipy.special.softmax(s) @ vf[g, lo:t + 1],
                                       atol=1e-12)


def test_short_context_selects_nothing():
    """t < W: no candidate exists, idx is all -1, and sparse = full attention."""
    rng = np.random.default_rng(12)
    h_q, h_kv, d, n, W, K = 4, 1, 16, 128, 128, 32
    ts = np.array([0, 1, 64, 126, 127, 128])
    q, k, v = rand_qkv(rng, len(ts), h_q, h_kv, n + 1, d)
    res = oracle.full_select(q, ts, k, v, window=W, topk=K)
    assert np.all(res["idx"][:5] == -1)
    assert res["idx"][5, 0, 0] == 0 and np.all(res["idx"][5, 0, 1:] == -1)  # t = 128: j = 0
    out = oracle.sparse(q, ts, k, v, res["idx"], window=W)
    np.testing.assert_allclose(out, res["out"], atol=1e-12)


def test_sparse_rejects_invalid_indices():
    rng = np.random.default_rng(13)
    q, k, v = rand_qkv(rng, 1, 2, 1, 64, 8)
    t = np.array([63])
    for bad in ([60, -1], [5, 5], [-3, -1]):  # inside the window; duplicate; negative
        with pytest.raises(RuntimeError):
            oracle.sparse(q, t, k, v, np.array([[bad]], np.int32), window=8)


# ---------------------------------------------------------------------------
# brute force / high precision on tiny inputs


def _decimal_row(qr, kf, vf, t, W, K, G, prec=50):
    """Everything for one row in 50-digit decimal arithmetic, with the selection
    done by a full sort of (score desc, j asc)."""
    decimal.getcontext().prec = prec
    D = decimal.Decimal
    h_q, d = qr.shape
    scale = D(1) / D(d).sqrt()
    lse, outs, probs = [], [], []
    for h in range(h_q):
        g = h // G
        s = [sum(D(float(qr[h, e])) * D(float(kf[g, j, e])) for e in range(d)) * scale
             for j in range(t + 1)]
        z = sum(x.exp() for x in s)
        l = z.ln()
        p = [(x - l).exp() for x in s]
        lse.append(l)
        probs.append(p)
        outs.append([sum(p[j] * D(float(vf[g, j, e])) for j in range(t + 1)) for e in range(d)])
    h_kv = h_q // G
    n_cand = max(0, t - W + 1)
    sel, scores = [], []
    for g in range(h_kv):
        sc = [sum(probs[h][j] for h in range(g * G, (g + 1) * G)) for j in range(n_cand)]
        order = sorted(range(n_cand), key=lambda j: (-sc[j], j))[:min(K, n_cand)]
        sel.append(sorted(order))
        scores.append(sc)
    return lse, outs, sel, scores


def test_high_precision_brute_force():
    """Tiny random rows recomputed in 50-digit decimal arithmetic."""
    rng = np.random.default_rng(14)
    h_q, h_kv, d, n, W, K = 4, 2, 4, 30, 6, 5
    G = h_q // h_kv
    ts = np.array([0, 5, 6, 12, 29])
    q, k, v = rand_qkv(rng, len(ts), h_q, h_kv, n, d, scale=1.0)
    res = oracle.full_select(q, ts, k, v, window=W, topk=K, want_scores=True)
    qf, kf, vf = unbits(q), unbits(k), unbits(v)
    for r, t in enumerate(ts):
        lse, outs, sel, scores = _decimal_row(qf[r], kf, vf, int(t), W, K, G)
        for h in range(h_q):
            assert res["lse"][r, h] == pytest.approx(float(lse[h]), abs=1e-13)
            np.testing.assert_allclose(res["out"][r, h], [float(x) for x in outs[h]], atol=1e-13)
        for g in range(h_kv):
            n_sel = len(sel[g])
            assert res["idx"][r, g, :n_sel].tolist() == sel[g]
            if n_sel:
                np.testing.assert_allclose(res["scores"][r, g, :len(scores[g])],
                                           [float(x) for x in scores[g]], rtol=1e-13)


def test_numpy_brute_force_matrix():
    """Whole score matrix materialised with numpy; selection by np.lexsort."""
    rng = np.random.default_rng(15)
    h_q, h_kv, d, n, W, K = 8, 2, 16, 256, 32, 48
    G = h_q // h_kv
    ts = np.arange(n)
    q, k, v = rand_qkv(rng, n, h_q, h_kv, n, d)
    res = oracle.full_select(q, ts, k, v, window=W, topk=K, want_scores=True)
    qf, kf, vf = unbits(q), unbits(k), unbits(v)
    causal = np.tril(np.ones((n, n), bool))
    for g in range(h_kv):
        P = np.zeros((n, n))
        for h in range(g * G, (g + 1) * G):
            S = qf[:, h] @ kf[g].T / math.sqrt(d)
            S = np.where(causal, S, -np.inf)
            L = scipy.special.logsumexp(S, axis=1)
            np.testing.assert_allclose(res["lse"][:, h], L, atol=1e-12)
            Ph = np.exp(S - L[:, None])
            np.testing.assert_allclose(res["out"][:, h], Ph @ vf[g], atol=1e-12)
            P += Ph
        for t in range(n):
            n_cand = max(0, t - W + 1)
            sc = P[t, :n_cand]
            order = np.lexsort((np.arange(n_cand), -sc))[:min(K, n_cand)]
            assert res["idx"][t, g, :len(order)].tolist() == sorted(order.tolist())


def test_oracle_is_deterministic_across_thread_counts():
    rng = np.random.default_rng(16)
    q, k, v = rand_qkv(rng, 12, 8, 2, 300, 16)
    ts = np.arange(288, 300)
    a = oracle.full_select(q, ts, k, v, window=16, topk=30, n_threads=1)
    b = oracle.full_select(q, ts, k, v, window=16, topk=30, n_threads=4)
    for key in ("out", "lse", "idx", "kth"):
        np.testing.assert_array_equal(a[key], b[key])


# ---------------------------------------------------------------------------
# KV bridging (xiawanshe.com report, section "两级KV共享", first level): a
# token's K and V come from its Self-Decoder hidden state by one projection.


def test_bridge_identity_weights_copy_the_hidden_state():
    """With W = I (d_model = 2 H_kv D), K is the first half of the hidden state and
    V the second, head-major, exactly."""
    rng = np.random.default_rng(21)
    h_kv, d = 2, 4
    x = rng.standard_normal((5, 2 * h_kv * d)).astype(np.float32)
    k, v = oracle.kv_bridge(bits(x), bits(np.eye(2 * h_kv * d, dtype=np.float32)), h_kv=h_kv, head_dim=d)
    xb = unbits(bits(x)).astype(np.float64)
    assert np.array_equal(k, xb[:, :h_kv * d].reshape(5, h_kv, d))
    assert np.array_equal(v, xb[:, h_kv * d:].reshape(5, h_kv, d))


def test_bridge_feature_layout_by_permuted_one_hot_rows():
    """Row f of W picks hidden column perm[f]: K[h][d] must equal hidden[perm[h D + d]]
    and V[h][d] hidden[perm[H D + h D + d]] -- fixes which output feature is
    which (K or V, head, dim)."""
    rng = np.random.default_rng(22)
    h_kv, d, d_model = 3, 2, 16
    f_total = 2 * h_kv * d
    perm = rng.permutation(d_model)[:f_total]
    w = np.zeros((f_total, d_model), dtype=np.float32)
    w[np.arange(f_total), perm] = 1.0
    x = rng.standard_normal((4, d_model)).astype(np.float32)
    xb = unbits(bits(x)).astype(np.float64)
    k, v = oracle.kv_bridge(bits(x), bits(w), h_kv=h_kv, head_dim=d)
    for h in range(h_kv):
        for dd in range(d):
            assert np.array_equal(k[:, h, dd], xb[:, perm[h * d + dd]])
            assert np.array_equal(v[:, h, dd], xb[:, perm[h_kv * d + h * d + dd]])


def test_bridge_one_hot_hidden_returns_a_weight_column():
    rng = np.random.default_rng(23)
    h_kv, d, d_model = 2, 8, 32
    w = rng.standard_normal((2 * h_kv * d, d_model)).astype(np.float32)
    wb = unbits(bits(w)).astype(np.float64)
    x = np.zeros((3, d_model), dtype=np.float32)
    cols = [0, 7, 31]
    x[np.arange(3), cols] = 1.0
    k, v = oracle.kv_bridge(bits(x), bits(w), h_kv=h_kv, head_dim=d)
    for r, c in enumerate(cols):
        assert np.array_equal(k[r].reshape(-1), wb[:h_kv * d, c])
        assert np.array_equal(v[r].reshape(-1), wb[h_kv * d:, c])


def test_bridge_decimal_brute_force():
    """Every output feature as a 50-digit decimal dot product of the bf16 values."""
    rng = np.random.default_rng(24)
    h_kv, d, d_model = 2, 3, 10
    x = rng.standard_normal((2, d_model)).astype(np.float32)
    w = rng.standard_normal((2 * h_kv * d, d_model)).astype(np.float32)
    xb, wb = unbits(bits(x)), unbits(bits(w))
    k, v = oracle.kv_bridge(bits(x), bits(w), h_kv=h_kv, head_dim=d)
    got = np.concatenate([k.reshape(2, -1), v.reshape(2, -1)], axis=1)
    with decimal.localcontext() as ctx:
        ctx.prec = 50
        for r in range(2):
            for f in range(2 * h_kv * d):
                ref = sum(decimal.Decimal(float(xb[r, c])) * decimal.Decimal(float(wb[f, c])) for c in range(d_model))
                assert abs(float(ref) - got[r, f]) <= 1e-12 * max(1.0, abs(float(ref)))


# ---------------------------------------------------------------------------
# Block-level selection (the predecessor design the "Token级选择" section of the
# xiawanshe.com report contrasts with), at the same budget.


def test_block_of_one_token_is_the_token_selection():
    """Blocks of one token rank exactly like tokens: the same idx as full_select."""
    rng = np.random.default_rng(31)
    q, k, v = rand_qkv(rng, 6, 4, 2, 300, 16)
    t = np.array([0, 130, 131, 200, 250, 299])
    ref = oracle.full_select(q, t, k, v, window=16, topk=40)
    got = oracle.block_select(q, t, k, v, window=16, topk=40, block=1)
    assert np.array_equal(got["idx"], ref["idx"])


def test_block_ties_take_the_lowest_blocks():
    """q = 0: every candidate has the same score, so every block too; the tie rule
    keeps the lowest-index blocks, i.e. tokens 0 .. K-1."""
    rng = np.random.default_rng(32)
    _, k, v = rand_qkv(rng, 1, 4, 2, 700, 8)
    q = np.zeros((2, 4, 8), np.float32)
    t = np.array([699, 600])
    got = oracle.block_select(bits(q), t, k, v, window=128, topk=256, block=64)
    assert np.array_equal(got["idx"], np.broadcast_to(np.arange(256, dtype=np.int32), (2, 2, 256)))


def test_blocks_lie_entirely_before_the_window():
    """With t - W + 1 = 3 * 64 + 10 candidates only blocks 0..2 are candidates; with
    a budget of 8 blocks every candidate block is kept and the rest is -1."""
    rng = np.random.default_rng(33)
    W, blk = 32, 64
    t_val = W - 1 + 3 * blk + 10
    q, k, v = rand_qkv(rng, 1, 2, 1, t_val + 1, 8)
    got = oracle.block_select(q, np.array([t_val]), k, v, window=W, topk=8 * blk, block=blk)
    row = got["idx"][0, 0]
    assert np.array_equal(row[:3 * blk], np.arange(3 * blk))
    assert np.all(row[3 * blk:] == -1)


def test_block_with_planted_key_is_kept():
    """A key that dominates the probabilities selects its block (budget: 2 blocks of 64)."""
    rng = np.random.default_rng(34)
    q = rng.standard_normal((1, 2, 16))
    qhat = q[0].sum(0) / np.linalg.norm(q[0].sum(0))
    k = rng.standard_normal((1, 1000, 16)) * 0.3
    v = rng.standard_normal((1, 1000, 16))
    k[0, 517] = 200.0 * qhat
    got = oracle.block_select(bits(q), np.array([999]), bits(k), bits(v), window=128, topk=128, block=64)
    blocks = sorted(set((got["idx"][0, 0] // 64).tolist()))
    assert 517 // 64 in blocks


def test_block_scores_sum_the_token_scores():
    """Every block's score equals the sum of its tokens' scores; the kept blocks are
    the top ones and the best left-out block is below the last kept one."""
    rng = np.random.default_rng(35)
    q, k, v = rand_qkv(rng, 3, 4, 2, 900, 16)
    t = np.array([899, 700, 560])
    W, K, blk = 64, 256, 64
    got = oracle.block_select(q, t, k, v, window=W, topk=K, block=blk)
    sc = got["full"]["scores"]
    for r in range(3):
        n_blk = (t[r] - W + 1) // blk
        for g in range(2):
            bs = np.array([sc[r, g, b * blk:(b + 1) * blk].sum() for b in range(n_blk)])
            kept = sorted(set((got["idx"][r, g][got["idx"][r, g] >= 0] // blk).tolist()))
            order = np.lexsort((np.arange(n_blk), -bs))[:K // blk]
            assert kept == sorted(order.tolist())
            assert got["kth_block"][r, g] == pytest.approx(bs[order[-1]], rel=1e-12)
            rest = np.setdiff1d(np.arange(n_blk), order)
            if rest.size:
                assert got["next_block"][r, g] == pytest.approx(bs[rest].max(), rel=1e-12)


# ---------------------------------------------------------------------------
# The predecessor design's two-branch sparse layer (the "Token级选择" section of
# the xiawanshe.com report: HySparse2 drops the separate sliding-window branch):
# a window branch over its own cache and a selected-tokens branch over the
# shared one, each with its own softmax.


def _branch_inputs(seed, n_rows=6, h_q=4, h_kv=2, n=300, d=16, W=24, K=40):
    rng = np.random.default_rng(seed)
    ts = np.array([0, 5, W - 1, W, W + 7, n - 1])[:n_rows]
    q, k, v = rand_qkv(rng, len(ts), h_q, h_kv, n, d, scale=1.0)
    _, k2, v2 = rand_qkv(rng, 1, h_q, h_kv, n, d, scale=1.0)
    idx = oracle.full_select(q, ts, k, v, window=W, topk=K)["idx"]
    return ts, q, k, v, k2, v2, idx, W


def test_branches_merged_by_lse_are_the_union_layer():
    """Softmaxes over two disjoint sets, merged by their log-sum-exp, are the
    softmax over the union: with the window branch on the shared cache the merge
    is the HySparse2 sparse layer (idx U window) exactly."""
    ts, q, k, v, _, _, idx, W = _branch_inputs(41)
    br = oracle.branches(q, ts, k, v, k, v, idx, window=W)
    union = oracle.sparse(q, ts, k, v, idx, window=W)
    lse = np.logaddexp(br["lse_swa"], br["lse_sel"])
    a = np.exp(br["lse_swa"] - lse)[..., None]
    b = np.exp(br["lse_sel"] - lse)[..., None]
    np.testing.assert_allclose(a * br["out_swa"] + b * br["out_sel"], union, atol=1e-12)


def test_window_branch_is_sliding_window_attention_of_its_own_cache():
    """The window branch against scipy's softmax over the window rows of k_swa."""
    ts, q, k, v, k2, v2, idx, W = _branch_inputs(42)
    br = oracle.branches(q, ts, k2, v2, k, v, idx, window=W)
    qf, kf, vf = unbits(q), unbits(k2), unbits(v2)
    d = q.shape[2]
    for r, t in enumerate(ts):
        lo = max(0, t - W + 1)
        for h in range(q.shape[1]):
            g = h // (q.shape[1] // k.shape[0])
            s = kf[g, lo:t + 1] @ qf[r, h] / math.sqrt(d)
            np.testing.assert_allclose(br["out_swa"][r, h], scipy.special.softmax(s) @ vf[g, lo:t + 1], atol=1e-12)
            assert br["lse_swa"][r, h] == pytest.approx(scipy.special.logsumexp(s), abs=1e-12)


def test_selected_branch_single_key_closed_form():
    """One selected key j: the branch output is v_j and its LSE is the logit s_j."""
    rng = np.random.default_rng(43)
    h_q, h_kv, d, n, W = 4, 2, 16, 100, 8
    q, k, v = rand_qkv(rng, 1, h_q, h_kv, n, d, scale=1.0)
    t = np.array([60])
    idx = np.full((1, h_kv, 3), -1, np.int32)
    idx[0, 0, 0], idx[0, 1, 0] = 17, 40
    br = oracle.branches(q, t, k, v, k, v, idx, window=W)
    qf, kf, vf = unbits(q), unbits(k), unbits(v)
    for h in range(h_q):
        g = h // (h_q // h_kv)
        j = idx[0, g, 0]
        np.testing.assert_array_equal(br["out_sel"][0, h], vf[g, j])
        assert br["lse_sel"][0, h] == pytest.approx(kf[g, j] @ qf[0, h] / math.sqrt(d), abs=1e-12)


def test_selected_branch_without_keys_is_empty():
    """Rows with no selected key (t < W, or an all -1 row): zero output, LSE -inf;
    the window branch is unaffected."""
    ts, q, k, v, k2, v2, idx, W = _branch_inputs(44)
    idx[:] = -1
    br = oracle.branches(q, ts, k2, v2, k, v, idx, window=W)
    assert np.all(br["out_sel"] == 0.0) and np.all(np.isneginf(br["lse_sel"]))
    assert np.all(np.isfinite(br["lse_swa"]))


def test_each_branch_reads_only_its_own_cache():
    """Changing the shared cache leaves the window branch unchanged, and changing
    the window branch's cache leaves the selected branch unchanged."""
    ts, q, k, v, k2, v2, idx, W = _branch_inputs(45)
    a = oracle.branches(q, ts, k2, v2, k, v, idx, window=W)
    b = oracle.branches(q, ts, k2, v2, v, k, idx, window=W)  # another shared cache
    c = oracle.branches(q, ts, v2, k2, k, v, idx, window=W)  # another window cache
    np.testing.assert_array_equal(a["out_swa"], b["out_swa"])
    np.testing.assert_array_equal(a["out_sel"], c["out_sel"])
    assert not np.allclose(a["out_sel"], b["out_sel"]) and not np.allclose(a["out_swa"], c["out_swa"])

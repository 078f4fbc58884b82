"""Pins of the fp64 oracle to facts fixed by the HiLS pages and by mathematics.

Each test checks the oracle against something other than itself: a
hand-worked example, a closed form, a library routine that is the textbook
definition (scipy logsumexp, torch's dense causal attention in float64), an
invariant, or a brute-force loop written independently below.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import hils_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


# --- hand-worked example (notes section 5.1) --------------------------------
def test_golden_two_key_summary():
    g = json.load(open(os.path.join(GOLD, "summary_two_keys.json")))
    keys = np.array(g["keys"])
    kbar, h = O.summarize_chunk(keys, np.array(g["landmark"]), g["scale"])
    assert np.allclose(kbar, g["kbar"], atol=1e-15, rtol=0)
    assert abs(h - g["hbias"]) < 1e-15
    for q, s, z in zip(g["queries"], g["score"], g["exact_log_mass"]):
        shat = q * kbar[0] * g["scale"] + h
        assert abs(shat - s) < 1e-14
        assert shat <= z + 1e-15
    # equality at the expansion point q = landmark (Proposition 3.1)
    assert abs(g["score"][0] - g["exact_log_mass"][0]) < 1e-14


# --- entropy limits (notes section 5.1: uniform -> log S, one-hot -> 0) ------
@pytest.mark.parametrize("B,d", [(64, 64), (64, 128), (16, 8)])
def test_uniform_p_gives_log_B(B, d):
    r = _rng(1)
    keys = r.standard_normal((B, d))
    kbar, h = O.summarize_chunk(keys, np.zeros(d), 1 / math.sqrt(d))
    assert abs(h - math.log(B)) < 1e-13
    assert np.allclose(kbar, keys.mean(axis=0), atol=1e-14)
    same = np.tile(r.standard_normal(d), (B, 1))
    kbar2, h2 = O.summarize_chunk(same, r.standard_normal(d), 1 / math.sqrt(d))
    assert abs(h2 - math.log(B)) < 1e-13
    assert np.allclose(kbar2, same[0], atol=1e-14)


def test_one_hot_p_gives_zero_entropy():
    r = _rng(2)
    B, d = 64, 64
    keys = r.standard_normal((B, d)) * 1e-3
    lm = np.zeros(d)
    lm[0] = 1.0
    keys[17, 0] = 900.0  # logit gap >= 800 -> other weights underflow to 0
    kbar, h = O.summarize_chunk(keys, lm, 1.0)
    assert h == 0.0
    assert np.array_equal(kbar, keys[17])


def test_entropy_bounds():
    r = _rng(3)
    k = r.standard_normal((2, 2, 64 * 8, 32)) * 3
    lm = r.standard_normal((2, 4, 8, 32)) * 3
    kbar, hb = O.summarize(k, lm, 64)
    assert np.all(hb >= -1e-15) and np.all(hb <= math.log(64) + 1e-12)


# --- identical keys: the score is the exact log-mass for every q ------------
def test_identical_keys_score_equals_exact_log_mass():
    r = _rng(4)
    b, h, g, B, d = 1, 2, 1, 64, 64
    n = 4 * B
    k = r.standard_normal((b, g, n, d))
    k[0, 0, B:2 * B] = k[0, 0, B]  # chunk 1: all keys identical
    lm = r.standard_normal((b, h, n // B, d))
    q = r.standard_normal((b, h, n, d))
    kbar, hb = O.summarize(k, lm, B)
    rows = np.arange(2 * B, n)
    s = O.chunk_scores(q, kbar, hb, B, rows=rows)[..., 1]
    sc = 1 / math.sqrt(d)
    for hi in range(h):
        exact = logsumexp(np.einsum("rd,jd->rj", q[0, hi, rows], k[0, 0, B:2 * B]) * sc, axis=1)
        assert np.allclose(s[0, hi], exact, atol=1e-12, rtol=0)


# --- Proposition 3.1: tangent plane of the chunk log-mass at l_c ------------
def test_tangent_plane_at_landmark_and_convexity():
    r = _rng(5)
    B, d = 64, 64
    sc = 1 / math.sqrt(d)
    for t in range(20):
        keys = r.standard_normal((B, d))
        lm = r.standard_normal(d) * (t % 4)
        kbar, h = O.summarize_chunk(keys, lm, sc)
        exact_at_l = logsumexp(keys @ lm * sc)
        assert abs(lm @ kbar * sc + h - exact_at_l) < 1e-12
        for _ in range(10):
            q = r.standard_normal(d) * 2
            assert q @ kbar * sc + h <= logsumexp(keys @ q * sc) + 1e-12


def test_kbar_is_gradient_of_log_mass():
    """d/dq log sum exp(q.k_j * s) at q = l equals s * kbar (first-order term)."""
    r = _rng(6)
    B, d = 64, 16
    sc = 0.3
    keys = r.standard_normal((B, d))
    lm = r.standard_normal(d)
    kbar, _ = O.summarize_chunk(keys, lm, sc)
    eps = 1e-5
    grad = np.zeros(d)
    for e in range(d):
        dq = np.zeros(d)
        dq[e] = eps
        grad[e] = (logsumexp(keys @ (lm + dq) * sc) - logsumexp(keys @ (lm - dq) * sc)) / (2 * eps)
    assert np.allclose(grad, sc * kbar, atol=1e-8)


# --- selection rules ---------------------------------------------------------
def test_topk_ties_go_to_lower_index():
    s = np.array([1.0, 3.0, 2.0, 3.0, 2.0, -np.inf]).reshape(1, 1, 1, 6)
    idx, _ = O.select_topk(s, 1, 3)
    assert idx[0, 0, 0].tolist() == [1, 3, 2]
    idx, _ = O.select_topk(s, 1, 8)
    assert idx[0, 0, 0].tolist() == [1, 3, 2, 4, 0, -1, -1, -1]


def test_topk_many_ties_keep_lowest_indices():
    r = _rng(13)
    s = np.zeros((1, 1, 3, 300))
    s[0, 0, 1] = r.integers(0, 3, 300).astype(float)   # heavy ties
    s[0, 0, 2, 150:] = -np.inf
    idx, _ = O.select_topk(s, 1, 64)
    assert idx[0, 0, 0].tolist() == list(range(64))
    expect = sorted(range(300), key=lambda c: (-s[0, 0, 1, c], c))[:64]
    assert idx[0, 0, 1].tolist() == expect
    assert idx[0, 0, 2].tolist() == list(range(64))


def test_summaries_survive_large_logits():
    """Logits near 1000 must not overflow (the exact value is still finite)."""
    r = _rng(14)
    B, d = 64, 8
    k = r.standard_normal((1, 1, 2 * B, d))
    lm = r.standard_normal((1, 1, 2, d)) * 2000.0
    kbar, hb = O.summarize(k, lm, B)
    for c in range(2):
        keys = k[0, 0, c * B:(c + 1) * B]
        sc = 1 / math.sqrt(d)
        exact = logsumexp(keys @ lm[0, 0, c] * sc)
        assert np.isfinite(exact)
        assert abs(lm[0, 0, c] @ kbar[0, 0, c] * sc + hb[0, 0, c] - exact) < 1e-9 * abs(exact)


def test_gqa_selection_takes_group_max():
    s = np.full((1, 4, 1, 5), 0.0)
    s[0, 0, 0] = [5, 4, 3, 2, 1]
    s[0, 1, 0] = [0, 0, 0, 0, 9]   # head 1 wants chunk 4
    s[0, 2, 0] = [0, 0, 0, 0, 0]
    s[0, 3, 0] = [0, 0, 0, 7, 0]   # head 3 (second group) wants chunk 3
    idx, key = O.select_topk(s, 2, 2)
    assert idx[0, 0, 0].tolist() == [4, 0]
    assert idx[0, 1, 0].tolist() == [3, 0]
    assert key[0, 0, 0].tolist() == [5, 4, 3, 2, 9]


# --- dense equivalence: exact scores + K = all is causal attention ----------
def _dense_causal(q, k, v, scale):
    """Textbook causal softmax attention (torch SDPA in float64), GQA expanded."""
    b, h, n, d = q.shape
    grp = h // k.shape[1]
    kt = torch.from_numpy(np.repeat(k, grp, axis=1))
    vt = torch.from_numpy(np.repeat(v, grp, axis=1))
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), kt, vt, is_causal=True, scale=scale)
    return out.numpy()


@pytest.mark.parametrize("n,h,g", [(256, 2, 2), (200, 4, 2), (64, 1, 1), (5, 1, 1)])
def test_exact_mode_all_chunks_is_dense_causal_attention(n, h, g):
    r = _rng(7)
    B, d = 64, 32
    q = r.standard_normal((1, h, n, d))
    k = r.standard_normal((1, g, n, d))
    v = r.standard_normal((1, g, n, d))
    lm = r.standard_normal((1, h, n // B, d))
    res = O.forward(q, k, v, lm, B, top_k=max(1, n // B), mode="exact")
    ref = _dense_causal(q, k, v, 1 / math.sqrt(d))
    assert np.allclose(res["out"], ref, atol=1e-12, rtol=0)


# --- V = 1 and convex hull --------------------------------------------------
def test_constant_values_and_convex_hull():
    r = _rng(8)
    B, d, n = 64, 16, 512
    q = r.standard_normal((1, 2, n, d))
    k = r.standard_normal((1, 1, n, d))
    lm = r.standard_normal((1, 2, n // B, d))
    res = O.forward(q, k, np.ones((1, 1, n, d)), lm, B, top_k=3)
    assert np.allclose(res["out"], 1.0, atol=1e-13)
    v = r.standard_normal((1, 1, n, d))
    res = O.forward(q, k, v, lm, B, top_k=3)
    for hi in range(2):
        for i in range(0, n, 37):
            sel = [c for c in res["idx"][0, 0, i] if c >= 0]
            own = i // B
            keys = list(range(own * B, i + 1)) + [j for c in sel for j in range(c * B, (c + 1) * B)]
            lo = v[0, 0, keys].min(axis=0)
            hi_ = v[0, 0, keys].max(axis=0)
            o = res["out"][0, hi, i]
            assert np.all(o >= lo - 1e-12) and np.all(o <= hi_ + 1e-12)


# --- K = 0 or queries in chunk 0: causal attention inside the own chunk -----
def test_no_remote_chunks_reduces_to_local_causal_attention():
    r = _rng(9)
    B, d, n = 64, 32, 256
    q = r.standard_normal((1, 2, n, d))
    k = r.standard_normal((1, 2, n, d))
    v = r.standard_normal((1, 2, n, d))
    lm = r.standard_normal((1, 2, n // B, d))
    res0 = O.forward(q, k, v, lm, B, top_k=0)
    resk = O.forward(q, k, v, lm, B, top_k=2)
    for c in range(n // B):
        sl = slice(c * B, (c + 1) * B)
        ref = _dense_causal(q[:, :, sl], k[:, :, sl], v[:, :, sl], 1 / math.sqrt(d))
        assert np.allclose(res0["out"][:, :, sl], ref, atol=1e-12, rtol=0)
    assert np.allclose(resk["out"][:, :, :B], res0["out"][:, :, :B], atol=1e-14, rtol=0)


# --- permutation inside a non-own chunk changes nothing ----------------------
def test_permutation_inside_remote_chunk():
    r = _rng(10)
    B, d, n = 64, 16, 384
    q = r.standard_normal((1, 2, n, d))
    k = r.standard_normal((1, 1, n, d))
    v = r.standard_normal((1, 1, n, d))
    lm = r.standard_normal((1, 2, n // B, d))
    base = O.forward(q, k, v, lm, B, top_k=2)
    perm = r.permutation(B) + 2 * B
    k2, v2 = k.copy(), v.copy()
    k2[0, 0, 2 * B:3 * B] = k[0, 0, perm]
    v2[0, 0, 2 * B:3 * B] = v[0, 0, perm]
    moved = O.forward(q, k2, v2, lm, B, top_k=2)
    assert np.array_equal(base["idx"][..., 3 * B:, :], moved["idx"][..., 3 * B:, :])
    assert np.allclose(base["out"][:, :, 3 * B:], moved["out"][:, :, 3 * B:], atol=1e-12, rtol=0)


# --- brute force: per-query, per-key loops (written independently) ----------
def _brute(q, k, v, lm, B, K, scale):
    b, h, n, d = q.shape
    g = k.shape[1]
    grp = h // g
    nc = n // B
    out = np.zeros((b, h, n, d))
    idx = np.full((b, g, n, K), -1)

    def dot(a, c):
        return sum(float(x) * float(y) for x, y in zip(a, c))

    summ = {}
    for bi in range(b):
        for hi in range(h):
            for c in range(nc):
                keys = [k[bi, hi // grp, c * B + j] for j in range(B)]
                logits = [dot(lm[bi, hi, c], kj) * scale for kj in keys]
                mx = max(logits)
                ex = [math.exp(x - mx) for x in logits]
                z = sum(ex)
                p = [e / z for e in ex]
                kb = [sum(p[j] * keys[j][e] for j in range(B)) for e in range(d)]
                ent = -sum(pj * math.log(pj) for pj in p if pj > 0)
                summ[bi, hi, c] = (kb, ent)
    for bi in range(b):
        for gi in range(g):
            for i in range(n):
                own = i // B
                scores = {}
                for hh in range(gi * grp, (gi + 1) * grp):
                    for c in range(own):
                        kb, ent = summ[bi, hh, c]
                        scores[hh, c] = dot(q[bi, hh, i], kb) * scale + ent
                keyed = sorted(range(own), key=lambda c: (-max(scores[hh, c] for hh in range(gi * grp, (gi + 1) * grp)), c))
                chosen = keyed[:K]
                for s_, c in enumerate(chosen):
                    idx[bi, gi, i, s_] = c
                for hh in range(gi * grp, (gi + 1) * grp):
                    # token-level weights of notes section 5.3:
                    # w_ij = exp(s_ij)/Z_c(j) * Zhat_c(j)/Zhat, local branch exact
                    own_l = [dot(q[bi, hh, i], k[bi, gi, j]) * scale for j in range(own * B, i + 1)]
                    zs = {c: sum(math.exp(dot(q[bi, hh, i], k[bi, gi, j]) * scale) for j in range(c * B, (c + 1) * B)) for c in chosen}
                    zown = sum(math.exp(x) for x in own_l)
                    zhat = sum(math.exp(scores[hh, c]) for c in chosen) + zown
                    o = [0.0] * d
                    for c in chosen:
                        for j in range(c * B, (c + 1) * B):
                            w = math.exp(dot(q[bi, hh, i], k[bi, gi, j]) * scale) / zs[c] * math.exp(scores[hh, c]) / zhat
                            for e in range(d):
                                o[e] += w * v[bi, gi, j, e]
                    for j in range(own * B, i + 1):
                        w = math.exp(dot(q[bi, hh, i], k[bi, gi, j]) * scale) / zhat
                        for e in range(d):
                            o[e] += w * v[bi, gi, j, e]
                    out[bi, hh, i] = o
    return out, idx


def test_brute_force_small_gqa():
    r = _rng(11)
    b, h, g, n, d, B, K = 1, 4, 2, 70, 4, 16, 2
    q = r.standard_normal((b, h, n, d))
    k = r.standard_normal((b, g, n, d))
    v = r.standard_normal((b, g, n, d))
    lm = r.standard_normal((b, h, n // B, d))
    sc = 1 / math.sqrt(d)
    ref_out, ref_idx = _brute(q, k, v, lm, B, K, sc)
    res = O.forward(q, k, v, lm, B, K)
    assert np.array_equal(res["idx"], ref_idx)
    assert np.allclose(res["out"], ref_out, atol=1e-12, rtol=0)


# --- decode equals the matching prefill row, paged or contiguous ------------
def test_decode_matches_prefill_rows():
    r = _rng(12)
    b, h, g, n, d, B, K = 2, 4, 2, 320, 16, 64, 2
    q = r.standard_normal((b, h, n, d))
    k = r.standard_normal((b, g, n, d))
    v = r.standard_normal((b, g, n, d))
    lm = r.standard_normal((b, h, n // B, d))
    pre = O.forward(q, k, v, lm, B, K)
    c_max = -(-n // B)
    n_pages = b * c_max
    perm = r.permutation(n_pages)
    bt = perm.reshape(b, c_max)
    kp = np.zeros((n_pages, g, B, d))
    vp = np.zeros((n_pages, g, B, d))
    lp = np.zeros((n_pages, h, d))
    for bi in range(b):
        for c in range(c_max):
            p = bt[bi, c]
            w = min(B, n - c * B)
            kp[p, :, :w] = k[bi, :, c * B:c * B + w].transpose(0, 1, 2)
            vp[p, :, :w] = v[bi, :, c * B:c * B + w]
            kp[p, :, w:] = 1e3  # garbage past the end must stay masked
            if c < n // B:
                lp[p] = lm[bi, :, c]
    for t in [0, 63, 64, 100, 200, 319]:
        dec = O.decode(q[:, :, t], kp, vp, lp, bt, [t + 1] * b, K)
        assert np.allclose(dec["out"], pre["out"][:, :, t], atol=1e-12, rtol=0)
        assert np.array_equal(dec["idx"], pre["idx"][:, :, t])


# --- separate scoring query (notes section 5.4, the Q-Cal interface) -------
def test_scoring_query_equal_to_q_changes_nothing():
    r = _rng(21)
    b, h, g, n, d, B, K = 1, 4, 2, 300, 16, 64, 2
    q, k, v = (r.standard_normal((b, x, n, d)) for x in (h, g, g))
    lm = r.standard_normal((b, h, n // B, d))
    a = O.forward(q, k, v, lm, B, K)
    c = O.forward(q, k, v, lm, B, K, q_score=q.copy())
    assert np.array_equal(a["idx"], c["idx"])
    assert np.allclose(a["out"], c["out"], atol=0, rtol=0)


def test_zero_scoring_query_selects_by_entropy_alone():
    # shat = 0 . kbar + H_c = H_c: the selection is the top K of H (group max, lower index on ties)
    r = _rng(22)
    b, h, g, n, d, B, K = 1, 4, 2, 640, 8, 64, 3
    q, k, v = (r.standard_normal((b, x, n, d)) for x in (h, g, g))
    lm = 3.0 * r.standard_normal((b, h, n // B, d))
    res = O.forward(q, k, v, lm, B, K, q_score=np.zeros_like(q))
    _, hb = O.summarize(k, lm, B)
    grp = h // g
    for gi in range(g):
        hmax = hb[0, gi * grp:(gi + 1) * grp].max(axis=0)
        for i in range(0, n, 37):
            cand = i // B
            want = sorted(range(cand), key=lambda c: (-hmax[c], c))[:K]
            got = [int(c) for c in res["idx"][0, gi, i] if c >= 0]
            assert got == want


def test_scoring_query_of_rows_without_candidates_is_unused():
    r = _rng(23)
    b, h, g, n, d, B, K = 1, 2, 2, 256, 16, 64, 2
    q, k, v = (r.standard_normal((b, x, n, d)) for x in (h, g, g))
    lm = r.standard_normal((b, h, n // B, d))
    qs = r.standard_normal((b, h, n, d))
    a = O.forward(q, k, v, lm, B, K, q_score=qs)
    qs2 = qs.copy()
    qs2[:, :, :B] = 1e3 * r.standard_normal((b, h, B, d))  # chunk 0 has no candidate chunk
    c = O.forward(q, k, v, lm, B, K, q_score=qs2)
    assert np.array_equal(a["out"], c["out"]) and np.array_equal(a["idx"], c["idx"])

"""Pins of the oracle's row normaliser, scoring-query weights, sliding-window
local branch and backward pass.

As in test_oracle_pins.py, each test checks the oracle against something other
than itself: a closed form built by hand from scipy/torch primitives, torch's
float64 dense attention (and its autograd gradient), finite differences of the
oracle's own forward pass (itself pinned in test_oracle_pins.py), or an
invariant that a dropped term or a wrong sign would break.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

from oracle import hils_oracle as O


def _rng(seed=0):
    return np.random.default_rng(seed)


def _dense_causal_t(q, k, v, scale, mask=None):
    """float64 torch SDPA (GQA by repeating KV heads); mask [N, N] bool or causal."""
    h, g = q.shape[1], k.shape[1]
    grp = h // g
    kt = torch.from_numpy(np.repeat(k, grp, axis=1)) if isinstance(k, np.ndarray) else k.repeat_interleave(grp, 1)
    vt = torch.from_numpy(np.repeat(v, grp, axis=1)) if isinstance(v, np.ndarray) else v.repeat_interleave(grp, 1)
    qt = torch.from_numpy(q) if isinstance(q, np.ndarray) else q
    if mask is None:
        return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask),
                                                            scale=scale)


def _dense_lse(q, k, scale, mask=None):
    b, h, n, d = q.shape
    grp = h // k.shape[1]
    out = np.zeros((b, h, n))
    for bi in range(b):
        for hi in range(h):
            lg = q[bi, hi] @ k[bi, hi // grp].T * scale
            m = np.tril(np.ones((n, n), bool)) if mask is None else mask
            lg = np.where(m, lg, -np.inf)
            out[bi, hi] = logsumexp(lg, axis=1)
    return out


def _window_mask(n, B, W):
    """Allowed keys of the chunk-aligned window: [max(0, (i//B + 1 - W/B) * B), i]."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    lo = np.maximum(0, (i // B + 1 - W // B) * B)
    return (j <= i) & (j >= lo)


# --- row normaliser log Zhat (notes section 5.3) ----------------------------
@pytest.mark.parametrize("n,h,g,window", [(256, 2, 2, None), (300, 4, 2, None), (320, 2, 1, 128)])
def test_row_lse_is_dense_lse_in_exact_mode_with_all_chunks(n, h, g, window):
    r = _rng(31)
    B, d = 64, 16
    q = r.standard_normal((1, h, n, d))
    k = r.standard_normal((1, g, n, d))
    v = r.standard_normal((1, g, n, d))
    lm = r.standard_normal((1, h, n // B, d))
    res = O.forward(q, k, v, lm, B, top_k=n // B, mode="exact", window=window)
    assert np.allclose(res["lse"], _dense_lse(q, k, 1 / math.sqrt(d)), atol=1e-12, rtol=0)


def test_row_lse_with_identical_chunk_keys_is_dense_lse():
    # identical keys inside every complete chunk make shat the exact chunk log-mass
    # (notes section 5.1), so log Zhat with K = all is the dense causal LSE
    r = _rng(32)
    B, d, n, h = 64, 8, 256 + 20, 2
    base = r.standard_normal((1, 1, n // B + 1, d))
    k = np.repeat(base, B, axis=2)[:, :, :n]
    q = r.standard_normal((1, h, n, d))
    v = r.standard_normal((1, 1, n, d))
    lm = r.standard_normal((1, h, n // B, d))
    res = O.forward(q, k, v, lm, B, top_k=n // B)
    assert np.allclose(res["lse"], _dense_lse(q, k, 1 / math.sqrt(d)), atol=1e-12, rtol=0)
    assert np.allclose(res["out"], _dense_causal_t(q, k, v, 1 / math.sqrt(d)).numpy(), atol=1e-12, rtol=0)


# --- scoring query: it alone sets the inter-chunk weights (notes 5.3, 5.4) ---
def test_scoring_query_sets_the_inter_chunk_weights():
    """One-hot values: V = e_c on every key of chunk c, so output component c is
    the fusion weight of chunk c.  The weights must be the softmax of
    q_score . kbar_c * scale + H_c over the selected chunks and LSE_own(q) for
    the own chunk; kbar, H and the logits are recomputed here with scipy."""
    r = _rng(33)
    B, d, n, h = 64, 16, 64 * 7 + 30, 2
    C = n // B
    sc = 1 / math.sqrt(d)
    q = r.standard_normal((1, h, n, d))
    qs = 2.0 * r.standard_normal((1, h, n, d))
    k = r.standard_normal((1, h, n, d))
    lm = r.standard_normal((1, h, C, d))
    v = np.zeros((1, h, n, d))
    for c in range(C + 1):
        v[0, :, c * B:(c + 1) * B, c] = 1.0
    K = 3
    res = O.forward(q, k, v, lm, B, K, q_score=qs)
    for hi in range(h):
        kb = np.zeros((C, d))
        hh = np.zeros(C)
        for c in range(C):
            p = softmax(k[0, hi, c * B:(c + 1) * B] @ lm[0, hi, c] * sc)
            kb[c] = p @ k[0, hi, c * B:(c + 1) * B]
            hh[c] = -np.sum(p * np.log(p))
        for i in range(B, n, 11):
            own = i // B
            sel = [int(c) for c in res["idx"][0, hi, i] if c >= 0]
            want_sel = sorted(range(own), key=lambda c: (-(qs[0, hi, i] @ kb[c] * sc + hh[c]), c))[:K]
            assert sel == want_sel
            logits = [qs[0, hi, i] @ kb[c] * sc + hh[c] for c in sel]
            logits.append(logsumexp(k[0, hi, own * B:i + 1] @ q[0, hi, i] * sc))
            w = softmax(np.array(logits))
            got = res["out"][0, hi, i]
            for c, wc in zip(sel + [own], w):
                assert abs(got[c] - wc) < 1e-12
            assert abs(got.sum() - 1.0) < 1e-12
            # the same row with q as the scoring query gives different weights
            alt = [q[0, hi, i] @ kb[c] * sc + hh[c] for c in sel] + [logits[-1]]
            if np.abs(softmax(np.array(alt)) - w).max() > 1e-3:
                assert np.abs(np.array([got[c] for c in sel + [own]]) - softmax(np.array(alt))).max() > 1e-6


# --- sliding-window local branch (notes sections 5.2, 5.3) ------------------
def test_window_of_one_chunk_is_the_own_chunk_branch():
    r = _rng(34)
    B, d, n = 64, 16, 64 * 6 + 9
    q, k, v = (r.standard_normal((1, x, n, d)) for x in (4, 2, 2))
    lm = r.standard_normal((1, 4, n // B, d))
    a = O.forward(q, k, v, lm, B, 2)
    c = O.forward(q, k, v, lm, B, 2, window=B)
    assert np.array_equal(a["idx"], c["idx"])
    assert np.array_equal(a["out"], c["out"]) and np.array_equal(a["lse"], c["lse"])


@pytest.mark.parametrize("W", [128, 256])
def test_window_with_no_remote_chunks_is_banded_causal_attention(W):
    r = _rng(35)
    B, d, n = 64, 16, 64 * 7 + 5
    q, k, v = (r.standard_normal((1, x, n, d)) for x in (2, 1, 1))
    lm = r.standard_normal((1, 2, n // B, d))
    res = O.forward(q, k, v, lm, B, 0, window=W)
    mask = _window_mask(n, B, W)
    ref = _dense_causal_t(q, k, v, 1 / math.sqrt(d), mask=mask).numpy()
    assert np.allclose(res["out"], ref, atol=1e-12, rtol=0)
    assert np.allclose(res["lse"], _dense_lse(q, k, 1 / math.sqrt(d), mask), atol=1e-12, rtol=0)


@pytest.mark.parametrize("W", [128, 192])
def test_window_exact_mode_all_chunks_is_dense_causal_attention(W):
    r = _rng(36)
    B, d, n = 64, 16, 64 * 6 + 33
    q, k, v = (r.standard_normal((1, x, n, d)) for x in (4, 2, 2))
    lm = r.standard_normal((1, 4, n // B, d))
    res = O.forward(q, k, v, lm, B, n // B, mode="exact", window=W)
    ref = _dense_causal_t(q, k, v, 1 / math.sqrt(d)).numpy()
    assert np.allclose(res["out"], ref, atol=1e-12, rtol=0)


def test_window_candidates_lie_before_the_window():
    r = _rng(37)
    B, d, n, W = 64, 8, 64 * 10, 256
    q, k, v = (r.standard_normal((1, x, n, d)) for x in (2, 2, 2))
    lm = r.standard_normal((1, 2, n // B, d))
    res = O.forward(q, k, v, lm, B, 4, window=W)
    for i in range(n):
        first_local = max(0, i // B + 1 - W // B)
        sel = [c for c in res["idx"][0, 0, i] if c >= 0]
        assert all(c < first_local for c in sel)
        assert len(sel) == min(4, first_local)


def test_window_decode_matches_prefill_rows():
    r = _rng(38)
    b, h, g, n, d, B, K, W = 2, 4, 2, 64 * 9 + 7, 8, 64, 2, 192
    q, k, v = (r.standard_normal((b, x, n, d)) for x in (h, g, g))
    lm = r.standard_normal((b, h, n // B, d))
    pre = O.forward(q, k, v, lm, B, K, window=W)
    c_max = -(-n // B)
    perm = r.permutation(b * c_max)
    bt = perm.reshape(b, c_max)
    kp = np.full((b * c_max, g, B, d), 1e3)
    vp = np.zeros((b * c_max, g, B, d))
    lp = np.zeros((b * c_max, h, d))
    for bi in range(b):
        for c in range(c_max):
            w = min(B, n - c * B)
            kp[bt[bi, c], :, :w] = k[bi, :, c * B:c * B + w]
            vp[bt[bi, c], :, :w] = v[bi, :, c * B:c * B + w]
            if c < n // B:
                lp[bt[bi, c]] = lm[bi, :, c]
    for t in [0, 63, 191, 192, 255, 256, 300, n - 1]:
        dec = O.decode(q[:, :, t], kp, vp, lp, bt, [t + 1] * b, K, window=W)
        assert np.allclose(dec["out"], pre["out"][:, :, t], atol=1e-12, rtol=0)
        assert np.allclose(dec["lse"], pre["lse"][:, :, t], atol=1e-12, rtol=0)
        assert np.array_equal(dec["idx"], pre["idx"][:, :, t])


# --- backward pass (notes section 5.3; Tide Figure 3 caption) ---------------
def _loss(res, dout):
    return float(np.sum(res["out"] * dout))


def _fd_check(fwd, x, grad, r, n_dirs=3, eps=1e-5, tol=2e-7):
    """Central difference along random directions against <grad, u>."""
    for _ in range(n_dirs):
        u = r.standard_normal(x.shape)
        x0 = x.copy()
        x[...] = x0 + eps * u
        lp, ip = fwd()
        x[...] = x0 - eps * u
        lm_, im = fwd()
        x[...] = x0
        assert np.array_equal(ip, im), "selection changed under the perturbation"
        fd = (lp - lm_) / (2 * eps)
        an = float(np.sum(grad * u))
        assert abs(fd - an) <= tol * max(1.0, abs(an)), (fd, an)


@pytest.mark.parametrize("window,q_sep", [(None, False), (128, False), (None, True)])
def test_backward_matches_finite_differences_on_a_256_token_slice(window, q_sep):
    r = _rng(40)
    b, h, g, n, d, B, K = 1, 4, 2, 256, 8, 64, 2
    q, k, v = (r.standard_normal((b, x, n, d)) for x in (h, g, g))
    lm = r.standard_normal((b, h, n // B, d))
    qs = r.standard_normal((b, h, n, d)) if q_sep else None
    dout = r.standard_normal((b, h, n, d))
    kw = dict(window=window, q_score=qs)
    gr = O.backward(q, k, v, lm, dout, B, K, **kw)

    def fwd():
        res = O.forward(q, k, v, lm, B, K, **kw)
        return _loss(res, dout), res["idx"]

    _fd_check(fwd, q, gr["dq"], r)
    _fd_check(fwd, k, gr["dk"], r)
    _fd_check(fwd, v, gr["dv"], r)
    _fd_check(fwd, lm, gr["dlandmark"], r)
    if q_sep:
        _fd_check(fwd, qs, gr["dq_score"], r)


def test_summary_backward_matches_finite_differences():
    r = _rng(41)
    B, d, sc = 64, 16, 0.3
    keys = r.standard_normal((B, d))
    lm = r.standard_normal(d)
    dkb = r.standard_normal(d)
    dh = 0.7
    dkeys, dl = O.summarize_backward(keys, lm, sc, dkb, dh)

    def f():
        kb, hh = O.summarize_chunk(keys, lm, sc)
        return float(dkb @ kb + dh * hh), np.zeros(1)

    _fd_check(f, keys, dkeys, r, n_dirs=4, tol=1e-8)
    _fd_check(f, lm, dl, r, n_dirs=4, tol=1e-8)


@pytest.mark.parametrize("n,h,g", [(256, 2, 2), (200, 4, 2)])
def test_backward_exact_mode_all_chunks_is_dense_attention_gradient(n, h, g):
    """Exact masses with K = all make the method dense causal attention, so its
    gradients are torch autograd's float64 SDPA gradients."""
    r = _rng(42)
    B, d = 64, 16
    sc = 1 / math.sqrt(d)
    q, k, v = (r.standard_normal((1, x, n, d)) for x in (h, g, g))
    lm = r.standard_normal((1, h, n // B, d))
    dout = r.standard_normal((1, h, n, d))
    gr = O.backward(q, k, v, lm, dout, B, n // B, mode="exact")
    qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = _dense_causal_t(qt, kt, vt, sc)
    out.backward(torch.from_numpy(dout))
    assert np.allclose(gr["dq"], qt.grad.numpy(), atol=1e-11, rtol=0)
    assert np.allclose(gr["dk"], kt.grad.numpy(), atol=1e-11, rtol=0)
    assert np.allclose(gr["dv"], vt.grad.numpy(), atol=1e-11, rtol=0)
    assert not gr["dlandmark"].any()


def test_backward_constant_values_leave_only_dv():
    """V = 1: every branch output is 1, so the weights carry no gradient:
    dq = dk = dlandmark = 0 and dv_j = sum_i (final weight of key j in row i) dout_i."""
    r = _rng(43)
    B, d, n, h, g, K = 64, 8, 64 * 5 + 10, 2, 1, 2
    q, k = r.standard_normal((1, h, n, d)), r.standard_normal((1, g, n, d))
    lm = r.standard_normal((1, h, n // B, d))
    dout = r.standard_normal((1, h, n, d))
    v = np.ones((1, g, n, d))
    gr = O.backward(q, k, v, lm, dout, B, K)
    assert np.abs(gr["dq"]).max() < 1e-12
    assert np.abs(gr["dk"]).max() < 1e-12
    assert np.abs(gr["dlandmark"]).max() < 1e-12
    # column sums: sum over rows and heads of the weights of each key times dout
    res = O.forward(q, k, v, lm, B, K, keep_terms=True)
    want = np.zeros((n, d))
    sc = 1 / math.sqrt(d)
    for (bi, hi, t), (lo, w, terms) in res["terms"].items():
        for wx, (_, _, c) in zip(w, terms):
            j0, j1 = (lo, t + 1) if c < 0 else (c * B, (c + 1) * B)
            p = softmax(k[0, 0, j0:j1] @ q[0, hi, t] * sc)
            want[j0:j1] += (wx * p)[:, None] * dout[0, hi, t][None, :]
    assert np.allclose(gr["dv"][0, 0], want, atol=1e-12, rtol=0)


def test_backward_unselected_chunks_get_no_gradient():
    r = _rng(44)
    B, d, n, h, K = 64, 8, 64 * 12, 2, 1
    q, k, v = (r.standard_normal((1, x, n, d)) for x in (h, 1, 1))
    q *= 0.05  # scores ~ H_c: every row picks the best-entropy candidate, few chunks are used
    lm = 3.0 * r.standard_normal((1, h, n // B, d))
    dout = r.standard_normal((1, h, n, d))
    res = O.forward(q, k, v, lm, B, K)
    used = set(int(c) for c in res["idx"].ravel() if c >= 0)
    unused = [c for c in range(n // B - 1) if c not in used]  # the last chunk is every row's own
    assert unused, "the seed should leave some chunk unselected"
    gr = O.backward(q, k, v, lm, dout, B, K)
    for c in unused:
        sl = slice(c * B, (c + 1) * B)
        # only the own-chunk rows of chunk c read its keys
        own_rows = O.backward(q, k, v, lm, dout[:, :, sl], B, K, rows=np.arange(c * B, (c + 1) * B))
        assert np.allclose(gr["dk"][0, 0, sl], own_rows["dk"][0, 0, sl], atol=1e-13, rtol=0)
        assert np.allclose(gr["dv"][0, 0, sl], own_rows["dv"][0, 0, sl], atol=1e-13, rtol=0)
        assert not gr["dlandmark"][0, :, c].any()
        assert not gr["dkbar"][0, :, c].any() and not gr["dhbias"][0, :, c].any()

"""Plain fp64 CPU oracle for the HiLS-Attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
C-ABI library and its Python binding) never calls it and shares no code with it.

What it computes, in the notation of the HiLS pages
("Hierarchical Sparse Attention Done Right: Toward Infinite Context Modeling",
reading notes, section 5; and the "Tide" digest of the same paper, Figure 3):

1. Landmark summary, notes section 5.1 (equations for s_j, p_j, k'_c, b'_c):
   s_j = l_c . k_j / sqrt(d) over the B keys of chunk c, p = softmax(s),
   kbar_c = sum_j p_j k_j, H_c = -sum_j p_j log p_j.
2. Chunk score and Top-K, notes section 5.2:
   shat_{i,c} = q_i . kbar_c / sqrt(d) + H_c over candidate chunks c, and
   I_i = the K candidates of highest score.  Under GQA the selection key is
   the maximum of the group's per-head scores (notes section 5.4, GQA
   paragraph); each head keeps its own score for the weights.
3. Intra-chunk softmax attention o_{i,c} over the B keys of each selected
   chunk (notes section 5.3, the "intra-chunk" factor exp(s_ij) / Z_{i,c}).
4. Inter-chunk fusion, notes section 5.3 and Tide Figure 3: the weight of
   chunk c is exp(shat_{i,c}) / Zhat_i where Zhat_i adds the surrogate masses
   of the selected chunks and the exact mass of the local branch.

Readings where the pages leave a step open (each one is listed with its
reason in the design notes of this repository):

* Local branch: the query's own (partial) chunk, keys [c_i*B, i], causally
  masked, entering the fusion with its exact log-mass LSE_own.
* Candidates: complete chunks strictly before the query's chunk, c < floor(i/B).
* K_eff = min(K, #candidates); unused index slots are -1; ties in the
  selection key go to the lower chunk index.
* One landmark query per (chunk, query head); the landmark is not a key.
* Scale 1/sqrt(d) everywhere unless a scale is given.
* 0 * log 0 = 0 in the entropy.

* Sliding-window local branch (notes section 5.2: the main configuration
  keeps a 512-token sliding window next to the remote chunks; section 5.3:
  the window's exact mass enters the normaliser Zhat_i beside the selected
  chunks' surrogate masses).  With window W (a multiple of B) the local branch
  is chunk-aligned: the own partial chunk and the W/B - 1 complete chunks
  before it, keys [max(0, (c_i + 1 - W/B) * B), i], at their exact mass; the
  remote candidates are the complete chunks before that, c < c_i + 1 - W/B.
  W = B (the default) is the own-chunk branch above.
* The row normaliser log Zhat_i (returned as "lse") is the log-sum-exp of the
  fusion logits: the selected chunks' shat and the local branch's LSE.
* Gradients (notes section 5.3: the hierarchical softmax lets the LM loss
  train the selector; Tide Figure 3 caption: gradients reach the compressed
  key): the Top-K indices are a constant of the backward pass; every other
  step (intra-chunk softmax, inter-chunk softmax, shat = q.kbar*scale + H,
  the landmark softmax that makes kbar and H) is differentiated exactly.

Modes: "landmark" (the method), "exact" (shat replaced by the exact chunk
log-mass log Z_{i,c}, notes section 3: naive block-sparse attention), and
forced selection (the caller supplies I_i).

Every routine works on float64 copies of its inputs.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "summarize",
    "chunk_scores",
    "exact_chunk_lse",
    "select_topk",
    "forward",
    "decode",
    "summarize_pages",
    "backward",
    "summarize_backward",
]


def _f64(x):
    if hasattr(x, "detach"):  # torch tensor -> numpy without importing torch here
        x = x.detach().cpu().float().numpy() if str(x.dtype) == "torch.bfloat16" else x.detach().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def _scale(d, scale):
    return 1.0 / math.sqrt(d) if (scale is None or scale == 0) else float(scale)


def _local_chunks(chunk, window):
    """Chunks in the local branch: 1 (own chunk only) or W / B for a window W."""
    if window is None or window == 0:
        return 1
    if window % chunk != 0 or window < chunk:
        raise ValueError("window must be a positive multiple of the chunk size")
    return window // chunk


def _n_cand(rows, chunk, window):
    """Number of remote candidate chunks of each query position: c < c_i + 1 - W/B."""
    return np.maximum(np.asarray(rows) // chunk + 1 - _local_chunks(chunk, window), 0)


def _local_start(i, chunk, window):
    """First key of query i's local branch."""
    return max(0, (i // chunk + 1 - _local_chunks(chunk, window)) * chunk)


# ---------------------------------------------------------------------------
# 1. Landmark summary (notes section 5.1; Proposition 3.1)
# ---------------------------------------------------------------------------
def summarize_chunk(keys, landmark, scale):
    """k̄ and H of one chunk: keys [B, d], landmark [d].

    s_j = l . k_j * scale; p = softmax(s); kbar = sum p_j k_j;
    H = -sum p_j log p_j with 0 log 0 = 0.
    """
    s = keys @ landmark * scale
    m = s.max()
    e = np.exp(s - m)
    p = e / e.sum()
    kbar = p @ keys
    nz = p > 0
    h = -np.sum(p[nz] * np.log(p[nz]))
    return kbar, h


def summarize(k, landmark, chunk, scale=None):
    """Summaries of every complete chunk of a contiguous sequence.

    k: [b, g, N, d]; landmark: [b, h, C, d] with C = N // chunk.
    Returns kbar [b, h, C, d] and hbias [b, h, C] (float64).
    Query head h reads the keys of KV head h // (h/g).
    """
    k = _f64(k)
    lm = _f64(landmark)
    b, g, n, d = k.shape
    h = lm.shape[1]
    c_all = n // chunk
    sc = _scale(d, scale)
    grp = h // g
    kc = k[:, :, : c_all * chunk].reshape(b, g, c_all, chunk, d)
    kbar = np.zeros((b, h, c_all, d))
    hb = np.zeros((b, h, c_all))
    for bi in range(b):
        for hi in range(h):
            for c in range(c_all):
                kbar[bi, hi, c], hb[bi, hi, c] = summarize_chunk(kc[bi, hi // grp, c], lm[bi, hi, c], sc)
    return kbar, hb


# ---------------------------------------------------------------------------
# 2. Chunk scores (notes section 5.2) and the exact chunk log-mass (section 3)
# ---------------------------------------------------------------------------
def chunk_scores(q, kbar, hbias, chunk, scale=None, rows=None, window=None):
    """shat [b, h, R, C]: q_i . kbar_c * scale + H_c, -inf where c is not a
    remote candidate (c >= floor(i/B), or inside the local window).

    rows: query positions to score (default: all).
    """
    q = _f64(q)
    kbar = _f64(kbar)
    hbias = _f64(hbias)
    b, h, n, d = q.shape
    sc = _scale(d, scale)
    rows = np.arange(n) if rows is None else np.asarray(rows)
    c_all = kbar.shape[2]
    s = np.einsum("bhrd,bhcd->bhrc", q[:, :, rows], kbar) * sc + hbias[:, :, None, :]
    cand = np.arange(c_all)[None, :] < _n_cand(rows, chunk, window)[:, None]
    return np.where(cand[None, None], s, -np.inf)


def exact_chunk_lse(q, k, chunk, scale=None, rows=None, window=None):
    """log Z_{i,c} = log sum_{j in chunk c} exp(q_i . k_j * scale) (notes section 3).

    Returned for the remote candidates c < floor(i/B) + 1 - W/B; -inf
    elsewhere.  [b, h, R, C]
    """
    q = _f64(q)
    k = _f64(k)
    b, h, n, d = q.shape
    g = k.shape[1]
    grp = h // g
    sc = _scale(d, scale)
    rows = np.arange(n) if rows is None else np.asarray(rows)
    c_all = n // chunk
    out = np.full((b, h, len(rows), c_all), -np.inf)
    kc = k[:, :, : c_all * chunk].reshape(b, g, c_all, chunk, d)
    for bi in range(b):
        for hi in range(h):
            lg = np.einsum("rd,cjd->rcj", q[bi, hi, rows], kc[bi, hi // grp]) * sc
            m = lg.max(axis=2, keepdims=True)
            lse = np.log(np.exp(lg - m).sum(axis=2)) + m[..., 0]
            cand = np.arange(c_all)[None, :] < _n_cand(rows, chunk, window)[:, None]
            out[bi, hi] = np.where(cand, lse, -np.inf)
    return out


# ---------------------------------------------------------------------------
# 3. Top-K selection (notes section 5.2; GQA max of section 5.4)
# ---------------------------------------------------------------------------
def select_topk(scores, heads_kv, top_k):
    """idx [b, g, R, K] (int64, -1 padded) and the selection key [b, g, R, C].

    The key is the max over the group's query heads; candidates are the
    finite entries; K_eff = min(K, #candidates); order: key descending,
    chunk index ascending on ties.
    """
    b, h, r, c_all = scores.shape
    grp = h // heads_kv
    key = scores.reshape(b, heads_kv, grp, r, c_all).max(axis=2)
    idx = np.full((b, heads_kv, r, top_k), -1, dtype=np.int64)
    if c_all == 0 or top_k == 0:
        return idx, key
    # stable sort of -key keeps the lower index first among equal keys
    order = np.argsort(-key, axis=-1, kind="stable")
    n_cand = np.isfinite(key).sum(axis=-1)
    k_eff = np.minimum(n_cand, top_k)
    take = order[..., :top_k]
    slot = np.arange(min(top_k, c_all))
    valid = slot[None, None, None, :] < k_eff[..., None]
    idx[..., : take.shape[-1]] = np.where(valid, take, -1)
    return idx, key


# ---------------------------------------------------------------------------
# 4. Forward pass: intra-chunk attention + hierarchical fusion (section 5.3)
# ---------------------------------------------------------------------------
def _softmax_attend(qv, keys, vals, sc):
    """o = softmax(q . k_j * sc) V and log-sum-exp, for one query, one key set."""
    lg = keys @ qv * sc
    m = lg.max()
    e = np.exp(lg - m)
    z = e.sum()
    return (e @ vals) / z, m + math.log(z)


def forward(q, k, v, landmark, chunk, top_k, scale=None, mode="landmark",
            forced_idx=None, rows=None, heads=None, q_score=None, window=None,
            keep_terms=False):
    """HiLS forward for a contiguous causal sequence.

    q [b,h,N,d], k/v [b,g,N,d], landmark [b,h,C,d] (C = N // chunk).
    mode: "landmark" or "exact".  forced_idx [b,g,R,K]: selection supplied by
    the caller (-1 = unused slot).  rows: query positions (default all);
    heads: (b, h) pairs to produce (default all; selection still uses the
    whole GQA group).  q_score [b,h,N,d]: a separate scoring query (notes
    section 5.4, the Q-Cal interface): it replaces q in the chunk scores, so it
    decides the selection and the inter-chunk weights, while q keeps the
    intra-chunk attention and the local branch.  window: None (own chunk) or
    a multiple W of the chunk size (sliding-window local branch).

    Returns a dict with out [b,h,R,d] (nan for heads not produced),
    idx [b,g,R,K], shat_sel [b,h,R,K] (-inf in unused slots), lse_own
    [b,h,R] (log-mass of the local branch), lse [b,h,R] (log Zhat_i, the
    log-sum-exp of all fusion logits), key [b,g,R,C] and shat [b,h,R,C].
    With keep_terms, "terms" maps (b, h, t) to the per-branch pieces the
    backward pass reuses.
    """
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    b, h, n, d = q64.shape
    g = k64.shape[1]
    grp = h // g
    sc = _scale(d, scale)
    rows = np.arange(n) if rows is None else np.asarray(rows)
    qs64 = q64 if q_score is None else _f64(q_score)
    if mode == "landmark":
        kbar, hb = summarize(k64, landmark, chunk, scale)
        shat = chunk_scores(qs64, kbar, hb, chunk, scale, rows, window)
    elif mode == "exact":
        shat = exact_chunk_lse(qs64, k64, chunk, scale, rows, window)
    else:
        raise ValueError(mode)
    if forced_idx is None:
        idx, key = select_topk(shat, g, top_k)
    else:
        idx = np.asarray(forced_idx, dtype=np.int64)
        key = None
    r = len(rows)
    kk = idx.shape[-1]
    out = np.full((b, h, r, d), np.nan)
    shat_sel = np.full((b, h, r, kk), -np.inf)
    lse_own = np.full((b, h, r), np.nan)
    lse = np.full((b, h, r), np.nan)
    terms_kept = {}
    want = set(heads) if heads is not None else None
    for bi in range(b):
        for hi in range(h):
            if want is not None and (bi, hi) not in want:
                continue
            gi = hi // grp
            for t, i in enumerate(rows):
                i = int(i)
                qv = q64[bi, hi, i]
                lo = _local_start(i, chunk, window)
                o_own, l_own = _softmax_attend(qv, k64[bi, gi, lo: i + 1], v64[bi, gi, lo: i + 1], sc)
                lse_own[bi, hi, t] = l_own
                terms = [(l_own, o_own, -1)]
                for s_, c in enumerate(idx[bi, gi, t]):
                    if c < 0:
                        continue
                    c = int(c)
                    o_c, _ = _softmax_attend(qv, k64[bi, gi, c * chunk:(c + 1) * chunk],
                                             v64[bi, gi, c * chunk:(c + 1) * chunk], sc)
                    sh = shat[bi, hi, t, c]
                    shat_sel[bi, hi, t, s_] = sh
                    terms.append((sh, o_c, c))
                mx = max(x for x, _, _ in terms)
                w = np.array([math.exp(x - mx) for x, _, _ in terms])
                z = w.sum()
                w /= z
                lse[bi, hi, t] = mx + math.log(z)
                out[bi, hi, t] = sum(wi * o for wi, (_, o, _) in zip(w, terms))
                if keep_terms:
                    terms_kept[bi, hi, t] = (lo, w, terms)
    res = dict(out=out, idx=idx, shat_sel=shat_sel, lse_own=lse_own, lse=lse, key=key, shat=shat)
    if keep_terms:
        res["terms"] = terms_kept
    return res


# ---------------------------------------------------------------------------
# 4b. Backward pass (notes section 5.3; Tide Figure 3 caption)
# ---------------------------------------------------------------------------
def summarize_backward(keys, landmark, scale, dkbar, dh):
    """Chain rule through one chunk summary (notes section 5.1).

    sigma_j = l . k_j * scale, pi = softmax(sigma), kbar = sum_j pi_j k_j,
    H = -sum_j pi_j log pi_j.  Given dL/dkbar [d] and dL/dH, returns
    dL/dkeys [B, d] and dL/dl [d]:
      dpi_j    = dkbar . k_j - dH (log pi_j + 1)
      dsigma_j = pi_j (dpi_j - sum_m pi_m dpi_m)
      dk_j     = pi_j dkbar + scale dsigma_j l,   dl = scale sum_j dsigma_j k_j.
    log pi_j is taken as sigma_j - LSE(sigma), finite even where pi_j
    underflows to 0 (there pi_j multiplies it, so 0 log 0 = 0 still holds).
    """
    sig = keys @ landmark * scale
    m = sig.max()
    e = np.exp(sig - m)
    z = e.sum()
    pi = e / z
    logpi = sig - (m + math.log(z))
    dpi = keys @ dkbar - dh * (logpi + 1.0)
    dsig = pi * (dpi - pi @ dpi)
    dkeys = pi[:, None] * dkbar[None, :] + scale * dsig[:, None] * landmark[None, :]
    dl = scale * (dsig @ keys)
    return dkeys, dl


def backward(q, k, v, landmark, dout, chunk, top_k, scale=None, mode="landmark",
             forced_idx=None, rows=None, heads=None, q_score=None, window=None):
    """Gradients of L = sum(dout * out) for the HiLS forward pass.

    Arguments as for forward(); dout has out's shape [b,h,R,d] for the rows
    given (default all).  The selection I_i is held fixed (Top-K is not
    differentiable); everything else is differentiated exactly.  Only the
    listed rows and (b, h) pairs contribute, so a caller can assemble the
    gradient of a key from the rows that attend to it.

    Per row i with fusion weights w (local branch l, selected chunks c),
    output o and D = dout . o:
      selected chunk c:  dshat_c = w_c (dout . o_c - D)
                         ds_ij   = w_c p_ij (dout . v_j - dout . o_c)
      local branch:      ds_ij   = w_l p_ij (dout . v_j - D)
                         (its logit is LSE_l, whose gradient is p_ij)
      every key j used:  dv_j += w p_ij dout,  dk_j += scale ds_ij q_i,
                         dq_i += scale ds_ij k_j
      scores:            dq_i (or dq_score_i) += scale dshat_c kbar_c,
                         dkbar_c += scale dshat_c q_i (q_score_i), dH_c += dshat_c
    then summarize_backward() carries dkbar, dH to the chunk keys and the
    landmark query.  In "exact" mode the chunk logit is LSE_c, so its
    keys get ds_ij = w_c p_ij (dout . v_j - D) and no summary gradient.

    Returns dict dq [b,h,N,d], dk, dv [b,g,N,d], dlandmark [b,h,C,d],
    dq_score [b,h,N,d] (None without q_score), dkbar [b,h,C,d], dhbias [b,h,C].
    """
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    lm64 = _f64(landmark)
    b, h, n, d = q64.shape
    g = k64.shape[1]
    grp = h // g
    sc = _scale(d, scale)
    rows = np.arange(n) if rows is None else np.asarray(rows)
    do = _f64(dout)
    qs64 = q64 if q_score is None else _f64(q_score)
    fw = forward(q64, k64, v64, lm64, chunk, top_k, scale, mode, forced_idx, rows, heads,
                 q_score=q_score, window=window, keep_terms=True)
    c_all = n // chunk
    dq = np.zeros_like(q64)
    dqs = np.zeros_like(q64)
    dk = np.zeros_like(k64)
    dv = np.zeros_like(v64)
    dkbar = np.zeros((b, h, c_all, d))
    dhb = np.zeros((b, h, c_all))
    kbar = None
    if mode == "landmark":
        kbar, _ = summarize(k64, lm64, chunk, scale)
    for (bi, hi, t), (lo, w, terms) in fw["terms"].items():
        gi = hi // grp
        i = int(rows[t])
        qv = q64[bi, hi, i]
        g_o = do[bi, hi, t]
        o = fw["out"][bi, hi, t]
        D = g_o @ o
        for wx, (_, o_x, c) in zip(w, terms):
            if c < 0:
                j0, j1 = lo, i + 1
            else:
                j0, j1 = c * chunk, (c + 1) * chunk
            keys, vals = k64[bi, gi, j0:j1], v64[bi, gi, j0:j1]
            lg = keys @ qv * sc
            p = np.exp(lg - lg.max())
            p /= p.sum()
            dov = vals @ g_o
            if c < 0 or mode == "exact":
                ds = wx * p * (dov - D)
            else:
                ds = wx * p * (dov - g_o @ o_x)
                dsh = wx * (g_o @ o_x - D)
                dqs[bi, hi, i] += sc * dsh * kbar[bi, hi, c]
                dkbar[bi, hi, c] += sc * dsh * qs64[bi, hi, i]
                dhb[bi, hi, c] += dsh
            dv[bi, gi, j0:j1] += (wx * p)[:, None] * g_o[None, :]
            dk[bi, gi, j0:j1] += sc * ds[:, None] * qv[None, :]
            dq[bi, hi, i] += sc * (ds @ keys)
    dlm = np.zeros_like(lm64)
    if mode == "landmark":
        for bi in range(b):
            for hi in range(h):
                gi = hi // grp
                for c in range(c_all):
                    if dhb[bi, hi, c] == 0.0 and not dkbar[bi, hi, c].any():
                        continue
                    sl = slice(c * chunk, (c + 1) * chunk)
                    dkeys, dl = summarize_backward(k64[bi, gi, sl], lm64[bi, hi, c], sc,
                                                   dkbar[bi, hi, c], dhb[bi, hi, c])
                    dk[bi, gi, sl] += dkeys
                    dlm[bi, hi, c] = dl
    if q_score is None:
        dq += dqs
        dqs = None
    return dict(dq=dq, dk=dk, dv=dv, dlandmark=dlm, dq_score=dqs, dkbar=dkbar, dhbias=dhb)


# ---------------------------------------------------------------------------
# 5. Decode over a paged chunk cache (one new query per sequence)
# ---------------------------------------------------------------------------
def summarize_pages(k_pages, landmark_pages, page_ids, heads_q, scale=None):
    """Summaries of the listed pages: returns {page: (kbar [h,d], hbias [h])}."""
    kp = _f64(k_pages)
    lp = _f64(landmark_pages)
    g = kp.shape[1]
    d = kp.shape[3]
    grp = heads_q // g
    sc = _scale(d, scale)
    res = {}
    for p in page_ids:
        p = int(p)
        kb = np.zeros((heads_q, d))
        hb = np.zeros(heads_q)
        for hi in range(heads_q):
            kb[hi], hb[hi] = summarize_chunk(kp[p, hi // grp], lp[p, hi], sc)
        res[p] = (kb, hb)
    return res


def decode(q, k_pages, v_pages, landmark_pages, block_table, seq_lens, top_k,
           scale=None, batches=None, window=None):
    """One decode step per sequence.

    q [b,h,d] is the query at position seq_lens[b]-1, whose key/value are
    already in the cache.  Chunk c of sequence b lives in page
    block_table[b, c] of the pools k_pages/v_pages [P,g,B,d].  The own chunk is
    floor((seq_len-1)/B); candidates are the complete chunks before the local
    branch (the own chunk, or with a window W the last W/B chunks), scored
    with summaries computed here from landmark_pages [P,h,d].
    Returns out [b,h,d] (zeros for seq_len <= 0), idx [b,g,K], lse [b,h]
    (log Zhat) and, per sequence, the selection key [g, n_cand] of its
    candidate chunks.
    """
    q64, kp, vp = _f64(q), _f64(k_pages), _f64(v_pages)
    bt = np.asarray(block_table).astype(np.int64)
    sl = np.asarray(seq_lens).astype(np.int64)
    b, h, d = q64.shape
    g = kp.shape[1]
    chunk = kp.shape[2]
    grp = h // g
    sc = _scale(d, scale)
    out = np.zeros((b, h, d))
    idx = np.full((b, g, top_k), -1, dtype=np.int64)
    shat_sel = np.full((b, h, top_k), -np.inf)
    lse = np.full((b, h), -np.inf)
    keys = {}
    for bi in range(b) if batches is None else batches:
        L = int(sl[bi])
        if L <= 0:
            continue
        own = (L - 1) // chunk
        n_cand = int(_n_cand(L - 1, chunk, window))
        pages = bt[bi, :n_cand]
        summ = summarize_pages(kp, landmark_pages, pages, h, scale)
        shat = np.full((h, n_cand), -np.inf)
        for c in range(n_cand):
            kb, hb = summ[int(pages[c])]
            shat[:, c] = np.einsum("hd,hd->h", kb, q64[bi]) * sc + hb
        sel, key = select_topk(shat[None, :, None, :], g, top_k)
        idx[bi] = sel[0, :, 0]
        keys[bi] = key[0, :, 0]
        lo_c = _local_start(L - 1, chunk, window) // chunk
        for hi in range(h):
            gi = hi // grp
            qv = q64[bi, hi]
            # local branch: chunks lo_c .. own, the last one up to the new token
            lk = np.concatenate([kp[int(bt[bi, c]), gi, :min(chunk, L - c * chunk)] for c in range(lo_c, own + 1)])
            lv = np.concatenate([vp[int(bt[bi, c]), gi, :min(chunk, L - c * chunk)] for c in range(lo_c, own + 1)])
            o_own, l_own = _softmax_attend(qv, lk, lv, sc)
            terms = [(l_own, o_own)]
            for s_, c in enumerate(idx[bi, gi]):
                if c < 0:
                    continue
                pg = int(bt[bi, int(c)])
                o_c, _ = _softmax_attend(qv, kp[pg, gi], vp[pg, gi], sc)
                terms.append((shat[hi, int(c)], o_c))
                shat_sel[bi, hi, s_] = shat[hi, int(c)]
            mx = max(x for x, _ in terms)
            w = np.array([math.exp(x - mx) for x, _ in terms])
            z = w.sum()
            w /= z
            lse[bi, hi] = mx + math.log(z)
            out[bi, hi] = sum(wi * o for wi, (_, o) in zip(w, terms))
    return dict(out=out, idx=idx, shat_sel=shat_sel, key=keys, lse=lse)

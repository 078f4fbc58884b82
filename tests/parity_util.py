"""Comparison helpers shared by the GPU parity tests (test infrastructure)."""
import numpy as np

TOL_BF16_MAX = 2e-2
TOL_BF16_MEAN = 2e-3
TOL_F32 = 1e-4
TIE_GAP = 1e-3


def check_indices(gpu_idx, key, top_k, gap=TIE_GAP):
    """Compares Top-K index sets row by row against the oracle's selection key.

    gpu_idx [..., K] (int, -1 padded); key [..., C] (oracle fp64 selection
    key, -inf for non-candidates).  Rows whose K-th vs (K+1)-th key gap is at
    least `gap` must match exactly (as sets); in near-tie rows the two sets
    may differ only in chunks whose key lies within `gap` of the K-th key.
    Returns the number of near-tie rows.
    """
    if top_k == 0:
        assert np.asarray(gpu_idx).size == 0
        return 0
    if np.asarray(key).shape[-1] == 0:  # no complete chunk before any query
        assert np.all(np.asarray(gpu_idx) == -1)
        return 0
    gpu_idx = np.asarray(gpu_idx).reshape(-1, gpu_idx.shape[-1])
    key = np.asarray(key).reshape(-1, key.shape[-1])
    ties = 0
    for r in range(key.shape[0]):
        kr = key[r]
        finite = np.isfinite(kr)
        n_cand = int(finite.sum())
        k_eff = min(top_k, n_cand)
        g = gpu_idx[r]
        got = [int(c) for c in g if c >= 0]
        assert len(got) == k_eff, f"row {r}: {len(got)} indices, expected {k_eff}"
        assert all(c >= 0 for c in g[:k_eff]) and all(c < 0 for c in g[k_eff:]), f"row {r}: padding"
        assert len(set(got)) == len(got), f"row {r}: duplicate index"
        if k_eff == 0:
            continue
        order = np.argsort(-kr, kind="stable")
        want = set(int(c) for c in order[:k_eff])
        kth = kr[order[k_eff - 1]]
        nxt = kr[order[k_eff]] if k_eff < n_cand else -np.inf
        if set(got) == want:
            continue
        assert kth - nxt < gap, f"row {r}: sets differ with gap {kth - nxt}"
        ties += 1
        for c in set(got) ^ want:
            assert abs(kr[c] - kth) < gap, f"row {r}: chunk {c} key {kr[c]} far from K-th {kth}"
    return ties


def check_close(gpu, ref, bf16):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape
    assert np.all(np.isfinite(gpu)), "non-finite GPU output"
    err = np.abs(gpu - ref)
    if bf16:
        assert err.max() <= TOL_BF16_MAX, f"max abs err {err.max():.3g}"
        assert err.mean() <= TOL_BF16_MEAN, f"mean abs err {err.mean():.3g}"
    else:
        assert err.max() <= TOL_F32, f"max abs err {err.max():.3g}"
    return float(err.max()), float(err.mean())

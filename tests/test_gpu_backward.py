"""GPU parity of hils_backward against the oracle's fp64 analytic gradients.

The GPU path runs the forward (hils_summarize, hils_select, hils_attend_selected
with lse_out) and then hils_backward; the oracle differentiates the same
forward with the GPU's selection held fixed (the Top-K is not differentiable).

Tolerance, derived from the arithmetic: inputs are bf16 (exact in the oracle),
every product and sum runs in fp32, and the two tensor-core operands formed on
the fly, P and dS, are rounded to bf16 (relative error 2^-9); D = dO . o reads
the forward's bf16 output (another 2^-9).  A gradient element is a sum of such
terms, so its error is bounded by about 2^-8 of the sum of the terms' absolute
values.  Per gradient tensor: mean |err| <= 2^-8 mean |ref| and
max |err| <= 1e-2 max |ref|.
"""
import numpy as np
import pytest
import torch

import chunk_wise_hierarchical_b200 as hils
from hils_inputs import CONFIGS, prefill_inputs
from oracle import hils_oracle as O

pytestmark = pytest.mark.gpu

REL_MEAN = 2.0 ** -8
REL_MAX = 1e-2


def _forward(inp, K, window=0):
    q, k, v, lm = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.landmark))
    kbar, hb = hils.summarize(k, lm)
    idx, sc = hils.select(q, kbar, hb, K, k.shape[1], window=window)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    out = hils.attend_selected(q, k, v, idx, sc, window=window, lse=lse)
    return q, k, v, lm, idx, sc, lse, out


def _check(name, got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{name}: non-finite gradient"
    err = np.abs(got - want)
    assert err.max() <= REL_MAX * np.abs(want).max() + 1e-6, f"{name}: max err {err.max():.3g} vs {np.abs(want).max():.3g}"
    assert err.mean() <= REL_MEAN * np.abs(want).mean() + 1e-7, f"{name}: mean err {err.mean():.3g} vs {np.abs(want).mean():.3g}"


@pytest.mark.parametrize("kw", [
    dict(batch=1, heads_q=2, heads_kv=2, seq_len=64 * 6 + 17, head_dim=64, K=3),
    dict(batch=1, heads_q=8, heads_kv=2, seq_len=64 * 8, head_dim=128, K=4, qkv_std=0.5),
    dict(batch=1, heads_q=2, heads_kv=2, seq_len=64 * 10, head_dim=64, K=2, window=192),
    dict(batch=2, heads_q=4, heads_kv=4, seq_len=64 * 12 + 5, head_dim=128, K=5),
    dict(batch=1, heads_q=4, heads_kv=1, seq_len=64 * 5 + 63, head_dim=64, K=0),
    dict(batch=1, heads_q=2, heads_kv=2, seq_len=37, head_dim=64, K=2),
])
def test_backward_matches_oracle_gradients(kw):
    kw = dict(kw)
    K = kw.pop("K")
    window = kw.pop("window", 0)
    inp = prefill_inputs(dtype="bf16", seed=5, **kw)
    q, k, v, lm, idx, sc, lse, out = _forward(inp, K, window)
    g = torch.Generator().manual_seed(12)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv, dl = hils.backward(q, k, v, lm, out, lse, idx, sc, dout.cuda(), window=window)
    torch.cuda.synchronize()
    ref = O.backward(inp.q, inp.k, inp.v, inp.landmark, dout, 64, K, forced_idx=idx.cpu().numpy(),
                     window=window or None)
    _check("dq", dq.cpu(), ref["dq"])
    _check("dk", dk.cpu(), ref["dk"])
    _check("dv", dv.cpu(), ref["dv"])
    if inp.landmark.shape[2] > 0:
        _check("dlandmark", dl.cpu(), ref["dlandmark"])


def test_backward_training_config_sampled():
    """The training workload (b2 h16 N16384 d128 K16): dq on sampled rows, and dk,
    dv, dlandmark on two late chunks of one head, from the oracle run over exactly
    the rows that read them (their selecting rows and their own-chunk rows)."""
    b, h, N, d, K = 2, 16, 16384, 128, 16
    inp = prefill_inputs(b, h, h, N, d, top_k=K, dtype="bf16", seed=0, device="cpu")
    q, k, v, lm, idx, sc, lse, out = _forward(inp, K)
    g = torch.Generator().manual_seed(3)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv, dl = hils.backward(q, k, v, lm, out, lse, idx, sc, dout.cuda())
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy()
    rng = np.random.default_rng(4)
    bi, hi = 1, 9
    rows = np.unique(np.concatenate([[0, 63, 64, N - 1], rng.integers(0, N, 24)]))
    ref = O.backward(inp.q, inp.k, inp.v, inp.landmark, dout[:, :, rows], 64, K, rows=rows, heads=[(bi, hi)],
                     forced_idx=gidx[:, :, rows])
    _check("dq rows", dq[bi, hi, rows].cpu(), ref["dq"][bi, hi, rows])
    for c in (240, 200):
        sel_rows = np.nonzero((gidx[bi, hi] == c).any(-1))[0]
        rr = np.unique(np.concatenate([sel_rows, np.arange(c * 64, c * 64 + 64)]))
        ref = O.backward(inp.q, inp.k, inp.v, inp.landmark, dout[:, :, rr], 64, K, rows=rr, heads=[(bi, hi)],
                         forced_idx=gidx[:, :, rr])
        sl = slice(c * 64, (c + 1) * 64)
        _check(f"dk chunk {c}", dk[bi, hi, sl].cpu(), ref["dk"][bi, hi, sl])
        _check(f"dv chunk {c}", dv[bi, hi, sl].cpu(), ref["dv"][bi, hi, sl])
        _check(f"dlandmark chunk {c}", dl[bi, hi, c].cpu(), ref["dlandmark"][bi, hi, c])

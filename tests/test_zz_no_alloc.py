"""hils_decode_static: decode through the C ABI with the library's own scratch
array instead of a caller workspace.  Its results must match hils_decode's on
the same inputs, call after call, across shapes that lay the scratch out
differently.  (File named to be collected last, so it also runs after every
other GPU test has used the library.)"""
import ctypes

import pytest
import torch

import chunk_wise_hierarchical_b200 as hils
from hils_inputs import decode_inputs

HILS_ERR_WORKSPACE = 3


def _prepare(batch, heads_q, heads_kv, head_dim, top_k, dtype, seq_lens, seed):
    di = decode_inputs(batch, heads_q, heads_kv, 0, head_dim, top_k=top_k, dtype=dtype, seed=seed,
                       seq_lens=seq_lens, spare_pages=3)
    dev = torch.device("cuda")
    kp, vp, lp = di.k_pages.to(dev), di.v_pages.to(dev), di.landmark_pages.to(dev)
    P = kp.shape[0]
    kbar = torch.empty((P, heads_q, head_dim), dtype=torch.float32, device=dev)
    hb = torch.empty((P, heads_q), dtype=torch.float32, device=dev)
    hils.summarize_paged(kp, lp, torch.arange(P, dtype=torch.int32, device=dev), kbar, hb)
    return dict(q=di.q.to(dev), k_pages=kp, v_pages=vp, kbar_pages=kbar, hbias_pages=hb,
                block_table=di.block_table.to(dev), seq_lens=di.seq_lens.to(dev)), top_k


def _with_workspace(t, K):
    return hils.decode(t["q"], t["k_pages"], t["v_pages"], t["kbar_pages"], t["hbias_pages"],
                       t["block_table"], t["seq_lens"], K, return_idx=True)


def _static(t, K, status_word):
    b, _, _ = t["q"].shape
    g = t["k_pages"].shape[1]
    idx = torch.full((b, g, K), -7, dtype=torch.int32, device="cuda")
    out = hils.decode_static(t["q"], t["k_pages"], t["v_pages"], t["kbar_pages"], t["hbias_pages"],
                             t["block_table"], t["seq_lens"], K, topk_idx=idx, status_word=status_word)
    return out, idx


def _same(got, want):
    out, idx = got
    ref_out, ref_idx = want
    assert torch.equal(idx, ref_idx)
    atol = 1e-2 if out.dtype == torch.bfloat16 else 1e-5
    torch.testing.assert_close(out.float(), ref_out.float(), atol=atol, rtol=0)


CASES = [
    dict(batch=5, heads_q=4, heads_kv=2, head_dim=64, top_k=4, dtype="bf16",
         seq_lens=[1, 64, 65, 300, 1000], seed=4),
    dict(batch=3, heads_q=8, heads_kv=1, head_dim=128, top_k=16, dtype="f32",
         seq_lens=[4000, 129, 2049], seed=5),
]


@pytest.mark.gpu
def test_static_scratch_matches_workspace_decode_call_after_call():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    prepared = [_prepare(**c) for c in CASES]
    wanted = [_with_workspace(t, K) for t, K in prepared]
    # two calls in a row per shape, then the shapes interleaved (the scratch is
    # laid out differently per shape; the ticket counters must stay at zero)
    for t_k, want in zip(prepared, wanted):
        for _ in range(2):
            _same(_static(*t_k, status), want)
    for _ in range(2):
        for t_k, want in zip(prepared, wanted):
            _same(_static(*t_k, None), want)
    torch.cuda.synchronize()
    assert hils.lib().hils_device_status(ctypes.c_void_p(status.data_ptr()), None) == 0


def test_static_scratch_rejects_shapes_beyond_its_size():
    lib = hils.lib()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: both calls fail the size check first
    # batch * heads_kv above the 4096 ticket slots
    s = hils.make_shape(4097, 1, 1, 64, 64, 4, 1)
    assert lib.hils_decode_static(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 1, fake, 4, fake,
                                  None, None, None) == HILS_ERR_WORKSPACE
    # partial Top-K lists alone: 64 * 64 * 64 splits * 64 keys * 8 B, far above 4 MiB
    s = hils.make_shape(64, 64, 64, 64, 64 * 8192, 64, 1)
    assert lib.hils_decode_static(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 8192, fake, 4, fake,
                                  None, None, None) == HILS_ERR_WORKSPACE

"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

import chunk_wise_hierarchical_b200 as hils
from chunk_wise_hierarchical_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "hils.h")).read()
    return sorted(set(re.findall(r"HILS_API[^;(]*?\b(hils_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    lib = hils.lib()
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(hils.EXPORTED) == names


def test_status_strings_and_version():
    lib = hils.lib()
    assert lib.hils_abi_version() == 3
    for code in range(7):
        assert lib.hils_status_string(code)
    assert lib.hils_status_string(99) == b"unknown status"


def _shape(**kw):
    base = dict(batch=2, heads_q=8, heads_kv=2, head_dim=64, seq_len=1000, top_k=16, dtype=1)
    base.update(kw)
    return _abi.make_shape(base["batch"], base["heads_q"], base["heads_kv"], base["head_dim"],
                           base["seq_len"], base["top_k"], base["dtype"],
                           chunk=base.get("chunk", 64), scale=base.get("scale", 0.0),
                           window=base.get("window", 0))


def test_workspace_sizes():
    # fp32 inputs: summaries, selection and scores only
    s = _shape(dtype=0)
    n = _abi.workspace_size(s, _abi.OP_ATTEND)
    C = 1000 // 64
    need = 2 * 8 * C * 64 * 4 + 2 * 8 * C * 4 + 2 * 2 * 1000 * 16 * 4 + 2 * 8 * 1000 * 16 * 4
    assert need <= n <= need + 6 * 256
    assert _abi.workspace_size(s, _abi.OP_ATTEND_SELECTED) == 256
    # bf16 inputs: also the chunk-major scratch, at least one d-wide bf16 partial per
    # (query, head, slot) and per local-branch row, plus their positions
    s = _shape()
    partials = (2 * 8 * 1000 * 16 + 2 * 8 * 1000) * 64 * 2 + 2 * 2 * 1000 * 16 * 4
    n = _abi.workspace_size(s, _abi.OP_ATTEND)
    assert need + partials <= n <= 2 * (need + partials)
    m = _abi.workspace_size(s, _abi.OP_ATTEND_SELECTED)
    assert 256 + partials <= m <= n - need + 256
    assert _abi.workspace_size(s, _abi.OP_SELECT) == 256
    assert _abi.workspace_size(s, _abi.OP_DECODE) >= 2 * 2 * 16 * 8


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), 2), (dict(chunk=32), 2), (dict(top_k=65), 2), (dict(heads_q=6, heads_kv=2), 2),
    (dict(heads_q=7, heads_kv=2), 1), (dict(batch=-1), 1), (dict(dtype=5), 1), (dict(top_k=-1), 1),
    (dict(scale=float("nan")), 1), (dict(heads_q=32, heads_kv=2), 2),
    (dict(window=-64), 1), (dict(window=100), 1), (dict(window=64 * 129), 2), (dict(window=512), 0),
    (dict(window=64), 0),
])
def test_shape_validation(kw, code):
    s = _shape(**kw)
    out = ctypes.c_size_t(0)
    assert hils.lib().hils_workspace_size(ctypes.byref(s), 1, ctypes.byref(out)) == code


def test_entry_points_reject_before_launch():
    lib = hils.lib()
    s = _shape()
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: every call below fails validation first
    assert lib.hils_workspace_size(None, 1, ctypes.byref(ctypes.c_size_t())) == 1
    assert lib.hils_attend(ctypes.byref(s), None, fake, fake, fake, fake, None, None, fake, 1 << 30, None) == 1
    assert lib.hils_attend(ctypes.byref(s), fake, fake, fake, fake, fake, None, None, None, 0, None) == 3
    assert lib.hils_attend(ctypes.byref(s), fake, fake, fake, fake, fake, None, None, fake, 16, None) == 3
    assert lib.hils_attend(ctypes.byref(s), P((1 << 20) + 4), fake, fake, fake, fake, None, None, fake,
                           1 << 30, None) == 1  # misaligned
    assert lib.hils_attend_selected(ctypes.byref(s), fake, fake, fake, None, fake, fake, None, fake,
                                    1 << 30, None) == 1  # top_k > 0 without indices
    assert lib.hils_select(ctypes.byref(s), fake, None, fake, fake, None, None, 0, None) == 1
    assert lib.hils_select(ctypes.byref(s), fake, fake, fake, fake, None, None, 0, None) == 3  # no error word
    assert lib.hils_summarize(ctypes.byref(s), fake, None, fake, fake, None) == 1
    assert lib.hils_summarize_paged(ctypes.byref(s), fake, fake, fake, -1, 4, fake, fake, None) == 1
    assert lib.hils_decode(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 0, fake, 4, fake, None,
                           fake, 1 << 30, None) == 1
    assert lib.hils_decode(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 100, fake, 4, fake, None,
                           fake, 1 << 30, None) == 1  # more chunks than seq_len allows
    assert lib.hils_device_status(None, None) == 1


def test_empty_problems_are_no_ops():
    lib = hils.lib()
    P = ctypes.c_void_p
    s0 = _shape(batch=0)
    assert lib.hils_attend(ctypes.byref(s0), None, None, None, None, None, None, None, None, 0, None) == 0
    assert lib.hils_decode(ctypes.byref(s0), None, None, None, None, None, None, 0, None, 0, None, None,
                           None, 0, None) == 0
    s1 = _shape(seq_len=0)
    assert lib.hils_attend(ctypes.byref(s1), None, None, None, None, None, None, None, None, 0, None) == 0
    assert lib.hils_summarize(ctypes.byref(s1), None, None, None, None, None) == 0
    s2 = _shape(top_k=0)
    assert lib.hils_select(ctypes.byref(s2), None, None, None, None, None, None, 0, None) == 0
    assert lib.hils_summarize_paged(ctypes.byref(s2), P(16), P(16), P(16), 0, 4, P(16), P(16), None) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 64, 64)
    with pytest.raises((ValueError, RuntimeError)):
        hils.attend(q, q, q, torch.zeros(1, 1, 1, 64), top_k=1)


def test_summary_dtype_validation():
    lib = hils.lib()
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: every call below fails validation first
    s_bf16 = _shape(dtype=1)
    s_f32 = _shape(dtype=0)
    # unknown summary dtype
    assert lib.hils_summarize_paged_ex(ctypes.byref(s_bf16), fake, fake, fake, 4, 4, fake, 7, fake, None) == 1
    assert lib.hils_decode_ex(ctypes.byref(s_bf16), fake, fake, fake, fake, 7, fake, fake, 1, fake, 4, fake,
                              None, fake, 1 << 30, None) == 1
    # a bf16 summary cache needs a bf16 model
    assert lib.hils_summarize_paged_ex(ctypes.byref(s_f32), fake, fake, fake, 4, 4, fake, 1, fake, None) == 2
    assert lib.hils_decode_ex(ctypes.byref(s_f32), fake, fake, fake, fake, 1, fake, fake, 1, fake, 4, fake,
                              None, fake, 1 << 30, None) == 2


def test_decode_window_beyond_the_decode_limit_is_unsupported():
    lib = hils.lib()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the call fails validation first
    s = _shape(window=64 * 17, seq_len=4096)
    assert lib.hils_decode(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 8, fake, 4, fake, None,
                           fake, 1 << 30, None) == 2


def test_decode_beyond_the_merge_limit_is_unsupported():
    """The attention kernel merges the scan's per-range Top-K lists in shared memory:
    more than 128 ranges are merged in groups of 128 whose results (groups x top_k keys)
    must fit 512 keys.  With one sequence and top_k = 64 that allows 8 groups, i.e.
    1024 ranges of 256 chunks: max_chunks = 2^18 passes this check, 2^18 + 256 does not.
    Both hils_decode and hils_decode_static refuse it before any launch."""
    lib = hils.lib()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the call fails validation first
    mc = (1 << 18) + 256
    s = _shape(batch=1, heads_q=8, heads_kv=8, top_k=64, seq_len=mc * 64)
    assert lib.hils_decode(ctypes.byref(s), fake, fake, fake, fake, fake, fake, mc, fake, 4, fake, None,
                           fake, 1 << 40, None) == 2
    assert lib.hils_decode_static(ctypes.byref(s), fake, fake, fake, fake, fake, fake, mc, fake, 4, fake,
                                  None, None, None) == 2
    # top_k = 16 allows 32 groups: the same cache is within the limit (the call then fails
    # later, for lack of a workspace, not as unsupported)
    s16 = _shape(batch=1, heads_q=8, heads_kv=8, top_k=16, seq_len=mc * 64)
    assert lib.hils_decode(ctypes.byref(s16), fake, fake, fake, fake, fake, fake, mc, fake, 4, fake, None,
                           fake, 0, None) == 3


def test_decode_static_binding_rejects_a_bf16_summary_cache():
    """hils_decode_static reads fp32 summaries only: the binding refuses a bf16
    cache before any pointer reaches the library."""
    import torch
    q = torch.zeros(2, 4, 64, dtype=torch.bfloat16)
    kp = torch.zeros(3, 2, 64, 64, dtype=torch.bfloat16)
    bt = torch.zeros(2, 1, dtype=torch.int32)
    sl = torch.ones(2, dtype=torch.int32)
    with pytest.raises(TypeError):
        hils.decode_static(q, kp, kp, torch.zeros(3, 4, 64, dtype=torch.bfloat16), torch.zeros(3, 4), bt, sl, 2)
    with pytest.raises(TypeError):
        hils.decode_static(q, kp, kp, torch.zeros(3, 4, 64), torch.zeros(3, 4), bt, sl, 2,
                           topk_idx=torch.zeros(2, 2, 2, dtype=torch.int64))


def test_backward_rejects_before_launch():
    lib = hils.lib()
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: every call below fails validation first
    s16 = _shape(dtype=1)
    s32 = _shape(dtype=0)
    args = [fake] * 13  # q k v landmark out lse idx score dout dq dk dv dl
    assert lib.hils_backward(ctypes.byref(s32), *args, fake, 1 << 30, None) == 2  # bf16 only
    no_lse = list(args)
    no_lse[5] = None
    assert lib.hils_backward(ctypes.byref(s16), *no_lse, fake, 1 << 30, None) == 1
    assert lib.hils_backward(ctypes.byref(s16), *args, None, 0, None) == 3
    n = ctypes.c_size_t(0)
    assert lib.hils_workspace_size(ctypes.byref(s16), 4, ctypes.byref(n)) == 0 and n.value > 256


def test_wait_limit_setter_returns_the_previous_limit():
    """hils_set_wait_limit is host state only: the default is HILS_DEFAULT_WAIT_LIMIT
    (parsed from the header) and each call returns the limit it replaces."""
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "hils.h")).read()
    m = re.search(r"#define HILS_DEFAULT_WAIT_LIMIT \(1u << (\d+)\)", hdr)
    assert m and hils.DEFAULT_WAIT_LIMIT == 1 << int(m.group(1))
    prev = hils.set_wait_limit(12345)
    try:
        assert prev == hils.DEFAULT_WAIT_LIMIT
        assert hils.set_wait_limit(0) == 12345
    finally:
        hils.set_wait_limit(prev)
    assert hils.set_wait_limit(prev) == prev

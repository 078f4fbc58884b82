"""The binding refuses tensors whose shape, dtype or device does not match the call
before any pointer reaches the library: the kernels read each tensor at the extent the
shape implies, so a short tensor would be read past its end.  Host-only (CPU tensors)."""
import pytest
import torch

import chunk_wise_hierarchical_b200 as hils
from chunk_wise_hierarchical_b200._abi import HILS_BF16, HILS_F32, check_decode_args, check_prefill_args, make_shape

B, H, G, N, D, K = 2, 8, 2, 200, 64, 4


def _prefill(dtype=torch.bfloat16):
    z = lambda *s: torch.zeros(*s, dtype=dtype)
    return dict(q=z(B, H, N, D), k=z(B, G, N, D), v=z(B, G, N, D), landmark=z(B, H, N // 64, D))


def test_prefill_arguments_of_the_right_shape_pass():
    sh = make_shape(B, H, G, D, N, K, HILS_BF16)
    a = _prefill()
    check_prefill_args(sh, a["q"], a["k"], a["v"], a["landmark"], torch.zeros_like(a["q"]))
    sh32 = make_shape(B, H, G, D, N, K, HILS_F32)
    a = _prefill(torch.float32)
    check_prefill_args(sh32, a["q"], a["k"], a["v"], None)


@pytest.mark.parametrize("name,bad", [
    ("k", torch.zeros(B, G, N - 1, D, dtype=torch.bfloat16)),
    ("v", torch.zeros(B, H, N, D, dtype=torch.bfloat16)),
    ("landmark", torch.zeros(B, H, N // 64 - 1, D, dtype=torch.bfloat16)),
    ("k", torch.zeros(B, G, N, D, dtype=torch.float32)),
    ("q", torch.zeros(B, H, N, D, dtype=torch.float32)),
])
def test_prefill_arguments_that_do_not_match_are_refused(name, bad):
    sh = make_shape(B, H, G, D, N, K, HILS_BF16)
    a = _prefill()
    a[name] = bad
    with pytest.raises((ValueError, TypeError)):
        check_prefill_args(sh, a["q"], a["k"], a["v"], a["landmark"])


def test_prefill_output_of_another_shape_is_refused():
    sh = make_shape(B, H, G, D, N, K, HILS_BF16)
    a = _prefill()
    with pytest.raises(ValueError):
        check_prefill_args(sh, a["q"], a["k"], a["v"], a["landmark"], torch.zeros(B, H, N, D + 64, dtype=torch.bfloat16))


def _decode(P=7, kbar_dtype=torch.float32):
    return dict(q=torch.zeros(B, H, D, dtype=torch.bfloat16),
                k_pages=torch.zeros(P, G, 64, D, dtype=torch.bfloat16),
                v_pages=torch.zeros(P, G, 64, D, dtype=torch.bfloat16),
                kbar_pages=torch.zeros(P, H, D, dtype=kbar_dtype),
                hbias_pages=torch.zeros(P, H),
                seq_lens=torch.zeros(B, dtype=torch.int32))


def test_decode_arguments_of_the_right_shape_pass():
    sh = make_shape(B, H, G, D, 5 * 64, K, HILS_BF16)
    for kd in (torch.float32, torch.bfloat16):
        a = _decode(kbar_dtype=kd)
        check_decode_args(sh, **a, out=torch.zeros_like(a["q"]), topk_idx=torch.zeros(B, G, K, dtype=torch.int32))


@pytest.mark.parametrize("name,bad", [
    ("v_pages", torch.zeros(6, G, 64, D, dtype=torch.bfloat16)),
    ("kbar_pages", torch.zeros(7, G, D)),
    ("kbar_pages", torch.zeros(7, H, D, dtype=torch.float16)),
    ("hbias_pages", torch.zeros(7, H, dtype=torch.bfloat16)),
    ("seq_lens", torch.zeros(B, dtype=torch.int64)),
    ("seq_lens", torch.zeros(B + 1, dtype=torch.int32)),
    ("k_pages", torch.zeros(7, G, 32, D, dtype=torch.bfloat16)),
])
def test_decode_arguments_that_do_not_match_are_refused(name, bad):
    sh = make_shape(B, H, G, D, 5 * 64, K, HILS_BF16)
    a = _decode()
    a[name] = bad
    with pytest.raises((ValueError, TypeError)):
        check_decode_args(sh, **a)


def test_decode_index_output_too_small_is_refused():
    sh = make_shape(B, H, G, D, 5 * 64, K, HILS_BF16)
    with pytest.raises(TypeError):
        check_decode_args(sh, **_decode(), topk_idx=torch.zeros(B * G * K - 1, dtype=torch.int32))


def test_select_refuses_summaries_of_another_shape():
    q = torch.zeros(B, H, N, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hils.select(q, torch.zeros(B, H, N // 64 + 1, D), torch.zeros(B, H, N // 64), K, G)
    with pytest.raises(TypeError):
        hils.select(q, torch.zeros(B, H, N // 64, D, dtype=torch.bfloat16), torch.zeros(B, H, N // 64), K, G)

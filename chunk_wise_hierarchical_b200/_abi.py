"""ctypes binding of libhils.so (argument marshalling only).

Every function takes torch tensors that already live on the GPU, checks their
dtype, shape and contiguity, and passes raw pointers to the C ABI declared in
include/hils.h.  All arithmetic happens in the CUDA kernels; there is no
fallback: if the library is missing or the tensors are on the CPU, the call
raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhils.so")

HILS_F32, HILS_BF16 = 0, 1
OP_SELECT, OP_ATTEND, OP_DECODE, OP_ATTEND_SELECTED, OP_BACKWARD = 0, 1, 2, 3, 4
STATUS = {
    0: "HILS_OK", 1: "HILS_ERR_INVALID_ARG", 2: "HILS_ERR_UNSUPPORTED", 3: "HILS_ERR_WORKSPACE",
    4: "HILS_ERR_CUDA", 5: "HILS_ERR_DEVICE_CHECK", 6: "HILS_ERR_DEVICE_TIMEOUT",
}


class HilsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class Shape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads_q", ctypes.c_int32), ("heads_kv", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("seq_len", ctypes.c_int32), ("chunk", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("scale", ctypes.c_float), ("dtype", ctypes.c_int32),
        ("window", ctypes.c_int32),
    ]


_lib = None
_P = ctypes.c_void_p


def lib():
    """Loads libhils.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libhils.so not built ({LIB_PATH}); run "
                           "`python -m chunk_wise_hierarchical_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    S = ctypes.POINTER(Shape)
    i32, sz = ctypes.c_int32, ctypes.c_size_t
    sig = {
        "hils_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "hils_abi_version": (i32, []),
        "hils_workspace_size": (i32, [S, i32, ctypes.POINTER(sz)]),
        "hils_summarize": (i32, [S, _P, _P, _P, _P, _P]),
        "hils_summarize_paged": (i32, [S, _P, _P, _P, i32, i32, _P, _P, _P]),
        "hils_select": (i32, [S, _P, _P, _P, _P, _P, _P, sz, _P]),
        "hils_attend": (i32, [S, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "hils_attend_selected": (i32, [S, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "hils_decode": (i32, [S, _P, _P, _P, _P, _P, _P, i32, _P, i32, _P, _P, _P, sz, _P]),
        "hils_summarize_paged_ex": (i32, [S, _P, _P, _P, i32, i32, _P, i32, _P, _P]),
        "hils_decode_ex": (i32, [S, _P, _P, _P, _P, i32, _P, _P, i32, _P, i32, _P, _P, _P, sz, _P]),
        "hils_decode_static": (i32, [S, _P, _P, _P, _P, _P, _P, i32, _P, i32, _P, _P, _P, _P]),
        "hils_device_status": (i32, [_P, _P]),
        "hils_set_wait_limit": (ctypes.c_uint32, [ctypes.c_uint32]),
        "hils_backward": (i32, [S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


EXPORTED = ["hils_abi_version", "hils_attend", "hils_attend_selected", "hils_backward", "hils_decode",
            "hils_decode_ex", "hils_decode_static", "hils_device_status", "hils_summarize_paged_ex", "hils_select", "hils_set_wait_limit",
            "hils_status_string", "hils_summarize", "hils_summarize_paged", "hils_workspace_size"]

DEFAULT_WAIT_LIMIT = 1 << 26  # HILS_DEFAULT_WAIT_LIMIT


def set_wait_limit(polls: int) -> int:
    """Polls of an ordinary bounded device wait before a tensor-core kernel gives up
    (process-wide; 0 gives up at once).  Returns the previous limit."""
    return int(lib().hils_set_wait_limit(int(polls)))


def device_status(ws, stream=None) -> int:
    """Reads and clears the error word of a workspace (hils_device_status)."""
    return int(lib().hils_device_status(_ptr(ws), _stream(stream)))


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HILS_BF16
    if t.dtype == torch.float32:
        return HILS_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _expect(t, shape, dtypes, name):
    """Raises unless tensor t has exactly this shape and one of these dtypes: the kernels
    read every tensor at the extent the shape implies."""
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {list(shape)}, got {list(t.shape)}")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} must be {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")


def _same_device(ref, *ts):
    for t in ts:
        if t is not None and t.device != ref.device:
            raise ValueError("every tensor must be on q's device")


def check_prefill_args(shape, q, k, v, landmark, out=None):
    """The prefill inputs against the shape: q [b,h,N,d]; k, v [b,g,N,d] and landmark
    [b,h,N//64,d] in q's dtype; out (if given) like q."""
    s = shape
    _expect(q, (s.batch, s.heads_q, s.seq_len, s.head_dim), (torch.bfloat16, torch.float32), "q")
    if _dt(q) != s.dtype:
        raise TypeError("q's dtype does not match the prepared shape")
    kv = (s.batch, s.heads_kv, s.seq_len, s.head_dim)
    _expect(k, kv, (q.dtype,), "k")
    _expect(v, kv, (q.dtype,), "v")
    if landmark is not None:
        _expect(landmark, (s.batch, s.heads_q, s.seq_len // s.chunk, s.head_dim), (q.dtype,), "landmark")
    if out is not None:
        _expect(out, q.shape, (q.dtype,), "out")
    _same_device(q, k, v, landmark, out)


def check_decode_args(shape, q, k_pages, v_pages, kbar_pages, hbias_pages, seq_lens, out=None, topk_idx=None):
    """The decode inputs against the shape: q [b,h,d]; k/v pages [P,g,64,d] in q's dtype;
    kbar pages [P,h,d] fp32 (or bf16, the compact cache); hbias pages [P,h] fp32; seq_lens
    [b] int32; topk_idx (if given) int32 with at least b*g*K entries; out (if given) like q."""
    s = shape
    _expect(q, (s.batch, s.heads_q, s.head_dim), (torch.bfloat16, torch.float32), "q")
    if _dt(q) != s.dtype:
        raise TypeError("q's dtype does not match the prepared shape")
    P = k_pages.shape[0] if k_pages.dim() == 4 else -1
    _expect(k_pages, (P, s.heads_kv, s.chunk, s.head_dim), (q.dtype,), "k_pages")
    _expect(v_pages, (P, s.heads_kv, s.chunk, s.head_dim), (q.dtype,), "v_pages")
    _expect(kbar_pages, (P, s.heads_q, s.head_dim), (torch.float32, torch.bfloat16), "kbar_pages")
    _expect(hbias_pages, (P, s.heads_q), (torch.float32,), "hbias_pages")
    _expect(seq_lens, (s.batch,), (torch.int32,), "seq_lens")
    if topk_idx is not None and (topk_idx.dtype != torch.int32 or topk_idx.numel() < s.batch * s.heads_kv * s.top_k):
        raise TypeError("topk_idx must be an int32 tensor of at least batch * heads_kv * top_k entries")
    if out is not None:
        _expect(out, q.shape, (q.dtype,), "out")
    _same_device(q, k_pages, v_pages, kbar_pages, hbias_pages, seq_lens, out, topk_idx)


def _check(st: int, where: str):
    if st != 0:
        raise HilsError(st, where)


def make_shape(batch, heads_q, heads_kv, head_dim, seq_len, top_k, dtype, chunk=64, scale=0.0, window=0):
    return Shape(batch, heads_q, heads_kv, head_dim, seq_len, chunk, top_k, float(scale or 0.0), dtype,
                 int(window or 0))


def workspace_size(shape: Shape, op: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().hils_workspace_size(ctypes.byref(shape), op, ctypes.byref(out)), "hils_workspace_size")
    return out.value


def new_workspace(shape: Shape, op: int, device) -> torch.Tensor:
    """Zero-filled workspace (the error word must start cleared)."""
    n = workspace_size(shape, op)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def summarize(k, landmark, scale=None, stream=None):
    """kbar [b,h,C,d] fp32, hbias [b,h,C] fp32 of every complete chunk."""
    b, g, n, d = k.shape
    h = landmark.shape[1]
    c = n // 64
    if landmark.shape != (b, h, c, d) or landmark.dtype != k.dtype:
        raise ValueError("landmark must be [b, h, seq_len // 64, d] with k's dtype")
    sh = make_shape(b, h, g, d, n, 0, _dt(k), scale=scale or 0.0)
    kbar = torch.empty((b, h, c, d), dtype=torch.float32, device=k.device)
    hb = torch.empty((b, h, c), dtype=torch.float32, device=k.device)
    _check(lib().hils_summarize(ctypes.byref(sh), _ptr(k), _ptr(landmark), _ptr(kbar), _ptr(hb),
                                _stream(stream)), "hils_summarize")
    return kbar, hb


def summarize_paged(k_pages, landmark_pages, page_ids, kbar_pages, hbias_pages, scale=None, stream=None):
    """Writes the summaries of the listed pages into kbar_pages (fp32, or bf16 for the
    compact cache) / hbias_pages (fp32)."""
    n_pages, g, chunk, d = k_pages.shape
    h = landmark_pages.shape[1]
    if page_ids.dtype != torch.int32:
        raise TypeError("page_ids must be int32")
    _expect(landmark_pages, (n_pages, h, d), (k_pages.dtype,), "landmark_pages")
    _expect(kbar_pages, (n_pages, h, d), (torch.float32, torch.bfloat16), "kbar_pages")
    _expect(hbias_pages, (n_pages, h), (torch.float32,), "hbias_pages")
    _same_device(k_pages, landmark_pages, page_ids, kbar_pages, hbias_pages)
    sh = make_shape(0, h, g, d, 0, 0, _dt(k_pages), chunk=chunk, scale=scale or 0.0)
    _check(lib().hils_summarize_paged_ex(ctypes.byref(sh), _ptr(k_pages), _ptr(landmark_pages), _ptr(page_ids),
                                         int(page_ids.numel()), int(n_pages), _ptr(kbar_pages), _dt(kbar_pages),
                                         _ptr(hbias_pages), _stream(stream)), "hils_summarize_paged_ex")


def select(q, kbar, hbias, top_k, heads_kv, scale=None, stream=None, with_scores=True, window=0, ws=None):
    """topk_idx [b,g,N,K] int32 and (optionally) topk_score [b,h,N,K] fp32; `ws`, if
    given, is the workspace whose error word the kernels report into."""
    b, h, n, d = q.shape
    sh = make_shape(b, h, heads_kv, d, n, top_k, _dt(q), scale=scale or 0.0, window=window)
    _expect(kbar, (b, h, n // 64, d), (torch.float32,), "kbar")
    _expect(hbias, (b, h, n // 64), (torch.float32,), "hbias")
    _same_device(q, kbar, hbias, ws)
    idx = torch.empty((b, heads_kv, n, top_k), dtype=torch.int32, device=q.device)
    sc = torch.empty((b, h, n, top_k), dtype=torch.float32, device=q.device) if with_scores else None
    if ws is None:
        ws = new_workspace(sh, OP_SELECT, q.device)
    _check(lib().hils_select(ctypes.byref(sh), _ptr(q), _ptr(kbar), _ptr(hbias), _ptr(idx), _ptr(sc),
                             _ptr(ws), ws.numel(), _stream(stream)), "hils_select")
    return idx, sc


class Prefill:
    """Reusable prefill call: holds the workspace for one shape."""

    def __init__(self, batch, heads_q, heads_kv, seq_len, head_dim, top_k, dtype, scale=None, device="cuda",
                 window=0):
        self.shape = make_shape(batch, heads_q, heads_kv, head_dim, seq_len, top_k,
                                HILS_BF16 if dtype in (torch.bfloat16, "bf16") else HILS_F32,
                                scale=scale or 0.0, window=window)
        self.ws = new_workspace(self.shape, OP_ATTEND, device)

    def __call__(self, q, k, v, landmark, out=None, topk_idx=None, stream=None, lse=None):
        s = self.shape
        check_prefill_args(s, q, k, v, landmark, out)
        _same_device(q, lse, topk_idx, self.ws)
        if out is None:
            out = torch.empty_like(q)
        if lse is not None and (lse.dtype != torch.float32 or lse.shape != q.shape[:3]):
            raise ValueError("lse must be fp32 [b, h, seq_len]")
        if topk_idx is not None and (topk_idx.dtype != torch.int32 or
                                     topk_idx.shape != (s.batch, s.heads_kv, s.seq_len, s.top_k)):
            raise ValueError("topk_idx must be int32 [b, heads_kv, seq_len, top_k]")
        _check(lib().hils_attend(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(landmark), _ptr(out),
                                 _ptr(lse), _ptr(topk_idx), _ptr(self.ws), self.ws.numel(), _stream(stream)),
               "hils_attend")
        return out

    def device_status(self, stream=None):
        return lib().hils_device_status(_ptr(self.ws), _stream(stream))


def attend(q, k, v, landmark, top_k, scale=None, stream=None, return_idx=False, q_score=None, window=0,
           return_lse=False):
    """HiLS prefill forward; returns out, then topk_idx and lse [b,h,N] (log Zhat)
    when asked.

    q_score: a separate scoring query (the Q-Cal interface): summaries, then
    hils_select with q_score, then hils_attend_selected with q.  window: 0 (the
    own-chunk local branch) or a multiple of 64 (a chunk-aligned sliding window)."""
    b, h, n, d = q.shape
    g = k.shape[1]
    lse = torch.empty((b, h, n), dtype=torch.float32, device=q.device) if return_lse else None
    if q_score is not None:
        if q_score.shape != q.shape or q_score.dtype != q.dtype:
            raise ValueError("q_score must match q's shape and dtype")
        kbar, hb = summarize(k, landmark, scale=scale, stream=stream)
        idx, sc = select(q_score, kbar, hb, top_k, g, scale=scale, stream=stream, window=window)
        out = attend_selected(q, k, v, idx, sc, scale=scale, stream=stream, window=window, lse=lse)
    else:
        call = Prefill(b, h, g, n, d, top_k, q.dtype, scale=scale, device=q.device, window=window)
        idx = torch.empty((b, g, n, top_k), dtype=torch.int32, device=q.device) if return_idx else None
        out = call(q, k, v, landmark, topk_idx=idx, stream=stream, lse=lse)
    res = (out,) + ((idx,) if return_idx else ()) + ((lse,) if return_lse else ())
    return res if len(res) > 1 else out


def attend_selected(q, k, v, topk_idx, topk_score, scale=None, out=None, ws=None, stream=None, window=0,
                    lse=None):
    """Attention + fusion for a given selection (topk_idx [b,g,N,K], topk_score [b,h,N,K]);
    lse, if given (fp32 [b,h,N]), receives log Zhat."""
    b, h, n, d = q.shape
    g = k.shape[1]
    K = topk_idx.shape[-1]
    sh = make_shape(b, h, g, d, n, K, _dt(q), scale=scale or 0.0, window=window)
    if topk_idx.dtype != torch.int32 or topk_score.dtype != torch.float32:
        raise TypeError("topk_idx must be int32 and topk_score fp32")
    if topk_idx.shape != (b, g, n, K) or topk_score.shape != (b, h, n, K):
        raise ValueError("topk_idx must be [b, heads_kv, N, K] and topk_score [b, heads_q, N, K]")
    if lse is not None and (lse.dtype != torch.float32 or lse.shape != (b, h, n)):
        raise ValueError("lse must be fp32 [b, h, N]")
    check_prefill_args(sh, q, k, v, None, out)
    _same_device(q, topk_idx, topk_score, lse, ws)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = new_workspace(sh, OP_ATTEND_SELECTED, q.device)
    _check(lib().hils_attend_selected(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(topk_idx),
                                      _ptr(topk_score), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                      _stream(stream)),
           "hils_attend_selected")
    return out


class Decode:
    """Reusable decode call for a paged cache of `max_chunks` chunks per sequence."""

    def __init__(self, batch, heads_q, heads_kv, head_dim, max_chunks, top_k, dtype, scale=None,
                 device="cuda", window=0):
        self.max_chunks = max_chunks
        self.shape = make_shape(batch, heads_q, heads_kv, head_dim, max_chunks * 64, top_k,
                                HILS_BF16 if dtype in (torch.bfloat16, "bf16") else HILS_F32,
                                scale=scale or 0.0, window=window)
        self.ws = new_workspace(self.shape, OP_DECODE, device)

    def __call__(self, q, k_pages, v_pages, kbar_pages, hbias_pages, block_table, seq_lens, out=None,
                 topk_idx=None, stream=None):
        s = self.shape
        if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
            raise TypeError("block_table and seq_lens must be int32")
        if block_table.shape != (s.batch, self.max_chunks):
            raise ValueError("block_table must be [batch, max_chunks]")
        check_decode_args(s, q, k_pages, v_pages, kbar_pages, hbias_pages, seq_lens, out, topk_idx)
        _same_device(q, block_table, self.ws)
        if out is None:
            out = torch.empty_like(q)
        _check(lib().hils_decode_ex(ctypes.byref(s), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(kbar_pages),
                                    _dt(kbar_pages), _ptr(hbias_pages), _ptr(block_table), self.max_chunks,
                                    _ptr(seq_lens), int(k_pages.shape[0]), _ptr(out), _ptr(topk_idx), _ptr(self.ws),
                                    self.ws.numel(), _stream(stream)), "hils_decode_ex")
        return out

    def device_status(self, stream=None):
        return lib().hils_device_status(_ptr(self.ws), _stream(stream))


def decode(q, k_pages, v_pages, kbar_pages, hbias_pages, block_table, seq_lens, top_k, scale=None,
           stream=None, return_idx=False, window=0):
    b, h, d = q.shape
    g = k_pages.shape[1]
    call = Decode(b, h, g, d, block_table.shape[1], top_k, q.dtype, scale=scale, device=q.device, window=window)
    idx = torch.empty((b, g, top_k), dtype=torch.int32, device=q.device) if return_idx else None
    out = call(q, k_pages, v_pages, kbar_pages, hbias_pages, block_table, seq_lens, topk_idx=idx,
               stream=stream)
    return (out, idx) if return_idx else out


DECODE_STATIC_SCRATCH_BYTES = 4 << 20


def decode_static(q, k_pages, v_pages, kbar_pages, hbias_pages, block_table, seq_lens, top_k,
                  scale=None, out=None, topk_idx=None, status_word=None, stream=None):
    """hils_decode_static: decode without a workspace (the library's own
    scratch array is used).  Calls on one device must not overlap in time."""
    b, h, d = q.shape
    g = k_pages.shape[1]
    max_chunks = block_table.shape[1]
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_table and seq_lens must be int32")
    if status_word is not None and (status_word.dtype != torch.int32 or status_word.numel() < 1):
        raise TypeError("status_word must be an int32 device tensor")
    # the entry point reads fp32 summaries only (it has no summary-dtype argument)
    if kbar_pages.dtype != torch.float32 or hbias_pages.dtype != torch.float32:
        raise TypeError("decode_static needs fp32 kbar_pages and hbias_pages (use decode() for a bf16 cache)")
    if kbar_pages.shape != (k_pages.shape[0], h, d) or hbias_pages.shape != (k_pages.shape[0], h):
        raise ValueError("kbar_pages must be [n_pages, heads_q, d] and hbias_pages [n_pages, heads_q]")
    if topk_idx is not None and (topk_idx.dtype != torch.int32 or topk_idx.numel() < b * g * top_k):
        raise TypeError("topk_idx must be an int32 tensor of at least batch * heads_kv * top_k entries")
    for t in (q, k_pages, v_pages, kbar_pages, hbias_pages, block_table, seq_lens, topk_idx, status_word, out):
        if t is not None and t.device != q.device:
            raise ValueError("every tensor must be on q's device")
    sh = make_shape(b, h, g, d, max_chunks * 64, top_k, _dt(q), scale=scale or 0.0)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().hils_decode_static(ctypes.byref(sh), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(kbar_pages),
                                    _ptr(hbias_pages), _ptr(block_table), max_chunks, _ptr(seq_lens),
                                    int(k_pages.shape[0]), _ptr(out), _ptr(topk_idx), _ptr(status_word),
                                    _stream(stream)), "hils_decode_static")
    return out


def backward(q, k, v, landmark, out, lse, topk_idx, topk_score, dout, scale=None, window=0, stream=None,
             ws=None):
    """hils_backward: fp32 (dq, dk, dv, dlandmark) for the forward that produced out,
    lse (log Zhat), topk_idx and topk_score on these bf16 inputs."""
    b, h, n, d = q.shape
    g = k.shape[1]
    K = topk_idx.shape[-1]
    if q.dtype != torch.bfloat16:
        raise TypeError("hils_backward takes bf16 inputs")
    for t in (k, v, landmark, out, dout):
        if t.dtype != torch.bfloat16:
            raise TypeError("q, k, v, landmark, out and dout must be bf16")
    if out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("out and dout must have q's shape")
    if lse.dtype != torch.float32 or lse.shape != (b, h, n):
        raise ValueError("lse must be fp32 [b, h, N]")
    if topk_idx.dtype != torch.int32 or topk_idx.shape != (b, g, n, K):
        raise ValueError("topk_idx must be int32 [b, heads_kv, N, K]")
    if topk_score.dtype != torch.float32 or topk_score.shape != (b, h, n, K):
        raise ValueError("topk_score must be fp32 [b, heads_q, N, K]")
    sh = make_shape(b, h, g, d, n, K, HILS_BF16, scale=scale or 0.0, window=window)
    check_prefill_args(sh, q, k, v, landmark, out)
    _same_device(q, lse, topk_idx, topk_score, dout, ws)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty((b, h, n, d), **f32)
    dk = torch.empty((b, g, n, d), **f32)
    dv = torch.empty((b, g, n, d), **f32)
    dl = torch.zeros(landmark.shape, **f32)
    if ws is None:
        ws = new_workspace(sh, OP_BACKWARD, q.device)
    _check(lib().hils_backward(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(landmark), _ptr(out), _ptr(lse),
                               _ptr(topk_idx), _ptr(topk_score), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(dl), _ptr(ws), ws.numel(), _stream(stream)), "hils_backward")
    return dq, dk, dv, dl

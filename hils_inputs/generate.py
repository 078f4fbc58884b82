"""Seeded synthetic workloads for HiLS-Attention (no method arithmetic here).

Recipe (shared by tests, smoke and bench):

* Prefill: a ``torch.Generator`` seeded with ``seed`` draws, in this order,
  Q [b,h,N,d], K [b,g,N,d], V [b,g,N,d] as ``qkv_std * N(0,1)`` and the
  landmark queries L [b,h,C,d] (C = N // chunk complete chunks) as N(0,1).
  Values are drawn in fp32 and rounded once to the requested dtype
  (round-to-nearest-even for bf16).
* Needles (prefill): a second CPU generator seeded with ``seed + 1`` picks, per
  (batch, query head), ``needles`` distinct chunks c in [0, C-1), a target query
  i uniformly in the later positions [(c+1)*chunk, N) and a slot j in the chunk.
  The key at c*chunk + j of that head's KV head is overwritten with
  4 * q_i / |q_i| (q_i taken after rounding, the result rounded again).
* Decode: q [b,h,d], K/V pages [P,g,chunk,d], landmark pages [P,h,d] are drawn
  in that order; a permutation of the P pages (seeded CPU generator, seed + 1)
  scatters each sequence's chunks over the pool through block_table [b,C_max]
  (-1 where unused).  One needle per (batch, query head): a chunk before the
  query's own chunk, a slot in it, and key = 4 * q / |q|.

Sizes follow the workloads named in CONFIGS.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import torch

# The synthetic workloads (shapes, distributions, needle counts).
CONFIGS = {
    "tiny_fp32": dict(batch=1, heads_q=2, heads_kv=2, seq_len=1024, head_dim=64,
                      chunk=64, top_k=4, dtype="f32", qkv_std=1.0, needles=0),
    "prefill_345m": dict(batch=4, heads_q=16, heads_kv=16, seq_len=8192, head_dim=64,
                         chunk=64, top_k=16, dtype="bf16", qkv_std=1.0, needles=8),
    "prefill_7b_gqa": dict(batch=1, heads_q=32, heads_kv=8, seq_len=32768, head_dim=128,
                           chunk=64, top_k=32, dtype="bf16", qkv_std=0.5, needles=8),
    "train_16k": dict(batch=2, heads_q=16, heads_kv=16, seq_len=16384, head_dim=128,
                      chunk=64, top_k=16, dtype="bf16", qkv_std=1.0, needles=0),
    "decode_32k": dict(batch=8, heads_q=16, heads_kv=16, seq_len=32768, head_dim=64,
                       chunk=64, top_k=16, dtype="bf16"),
    "decode_128k": dict(batch=8, heads_q=16, heads_kv=16, seq_len=131072, head_dim=64,
                        chunk=64, top_k=16, dtype="bf16"),
    "decode_512k": dict(batch=8, heads_q=16, heads_kv=16, seq_len=524288, head_dim=64,
                        chunk=64, top_k=16, dtype="bf16"),
    # the longer contexts the pages extrapolate decode to: about 34 GB of K/V pages each
    "decode_1m": dict(batch=8, heads_q=16, heads_kv=16, seq_len=1048576, head_dim=64,
                      chunk=64, top_k=16, dtype="bf16"),
    "decode_4m": dict(batch=2, heads_q=16, heads_kv=16, seq_len=4194304, head_dim=64,
                      chunk=64, top_k=16, dtype="bf16"),
}

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _randn(shape, gen, device, std, dtype, slab_elems=1 << 28):
    """std * N(0,1) drawn in fp32 then rounded to dtype; large tensors in slabs."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    pos = 0
    while pos < n:
        m = min(slab_elems, n - pos)
        x = torch.randn(m, generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        flat[pos:pos + m] = x.to(dtype)
        pos += m
    return out


@dataclasses.dataclass
class PrefillInputs:
    q: torch.Tensor          # [b, h, N, d]
    k: torch.Tensor          # [b, g, N, d]
    v: torch.Tensor          # [b, g, N, d]
    landmark: torch.Tensor   # [b, h, C, d]
    chunk: int
    top_k: int
    needles: List[tuple]     # (b, h, c, j, i)

    @property
    def shape(self):
        b, h, n, d = self.q.shape
        return dict(batch=b, heads_q=h, heads_kv=self.k.shape[1], seq_len=n,
                    head_dim=d, chunk=self.chunk, top_k=self.top_k)


def prefill_inputs(batch, heads_q, heads_kv, seq_len, head_dim, chunk=64, top_k=16,
                   dtype="bf16", qkv_std=1.0, needles=0, seed=0, device="cpu",
                   **_ignored) -> PrefillInputs:
    dt = _DT[dtype] if isinstance(dtype, str) else dtype
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    n_chunks = seq_len // chunk
    q = _randn((batch, heads_q, seq_len, head_dim), gen, device, qkv_std, dt)
    k = _randn((batch, heads_kv, seq_len, head_dim), gen, device, qkv_std, dt)
    v = _randn((batch, heads_kv, seq_len, head_dim), gen, device, qkv_std, dt)
    lm = _randn((batch, heads_q, n_chunks, head_dim), gen, device, 1.0, dt)
    planted = []
    if needles > 0 and n_chunks >= 2:
        cg = torch.Generator(device="cpu")
        cg.manual_seed(seed + 1)
        group = heads_q // heads_kv
        rows_b, rows_h, rows_c, rows_j, rows_i = [], [], [], [], []
        for bi in range(batch):
            for hi in range(heads_q):
                n = min(needles, n_chunks - 1)
                cs = torch.randperm(n_chunks - 1, generator=cg)[:n].tolist()
                for c in cs:
                    lo = (c + 1) * chunk
                    i = lo + int(torch.randint(0, seq_len - lo, (1,), generator=cg))
                    j = int(torch.randint(0, chunk, (1,), generator=cg))
                    rows_b.append(bi); rows_h.append(hi); rows_c.append(c)
                    rows_j.append(j); rows_i.append(i)
        tb = torch.tensor(rows_b, device=device)
        th = torch.tensor(rows_h, device=device)
        ti = torch.tensor(rows_i, device=device)
        tpos = torch.tensor([c * chunk + j for c, j in zip(rows_c, rows_j)], device=device)
        qrows = q[tb, th, ti].float()
        nk = (4.0 * qrows / qrows.norm(dim=-1, keepdim=True)).to(dt)
        k[tb, th // group, tpos] = nk
        planted = list(zip(rows_b, rows_h, rows_c, rows_j, rows_i))
    return PrefillInputs(q, k, v, lm, chunk, top_k, planted)


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor              # [b, h, d]
    k_pages: torch.Tensor        # [P, g, B, d]
    v_pages: torch.Tensor        # [P, g, B, d]
    landmark_pages: torch.Tensor  # [P, h, d]
    block_table: torch.Tensor    # [b, C_max] int32, -1 where unused
    seq_lens: torch.Tensor       # [b] int32
    chunk: int
    top_k: int
    needles: List[tuple]         # (b, h, c, j)

    @property
    def max_chunks(self):
        return self.block_table.shape[1]


def decode_inputs(batch, heads_q, heads_kv, seq_len, head_dim, chunk=64, top_k=16,
                  dtype="bf16", seed=0, device="cpu", seq_lens: Optional[Sequence[int]] = None,
                  spare_pages=0, qkv_std=1.0, **_ignored) -> DecodeInputs:
    dt = _DT[dtype] if isinstance(dtype, str) else dtype
    if seq_lens is None:
        seq_lens = [seq_len] * batch
    seq_lens = [int(s) for s in seq_lens]
    pages_per = [max(1, math.ceil(s / chunk)) for s in seq_lens]
    c_max = max(pages_per)
    n_pages = sum(pages_per) + spare_pages
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _randn((batch, heads_q, head_dim), gen, device, qkv_std, dt)
    kp = _randn((n_pages, heads_kv, chunk, head_dim), gen, device, qkv_std, dt)
    vp = _randn((n_pages, heads_kv, chunk, head_dim), gen, device, qkv_std, dt)
    lp = _randn((n_pages, heads_q, head_dim), gen, device, 1.0, dt)
    cg = torch.Generator(device="cpu")
    cg.manual_seed(seed + 1)
    perm = torch.randperm(n_pages, generator=cg)
    bt = torch.full((batch, c_max), -1, dtype=torch.int32)
    off = 0
    for bi, npg in enumerate(pages_per):
        bt[bi, :npg] = perm[off:off + npg].to(torch.int32)
        off += npg
    planted = []
    group = heads_q // heads_kv
    for bi in range(batch):
        own = (seq_lens[bi] - 1) // chunk if seq_lens[bi] > 0 else 0
        for hi in range(heads_q):
            if own < 1:
                continue
            c = int(torch.randint(0, own, (1,), generator=cg))
            j = int(torch.randint(0, chunk, (1,), generator=cg))
            page = int(bt[bi, c])
            qr = q[bi, hi].float()
            kp[page, hi // group, j] = (4.0 * qr / qr.norm()).to(dt)
            planted.append((bi, hi, c, j))
    return DecodeInputs(q, kp, vp, lp, bt.to(device), torch.tensor(seq_lens, dtype=torch.int32,
                        device=device), chunk, top_k, planted)

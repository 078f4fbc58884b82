"""Benchmark: HiLS forward prefill (TFLOP/s) and paged decode (tok/s) on B200.

One step = one full prefill forward pass (summaries, scores + Top-K,
selected-chunk and own-chunk attention, fusion) of the 345M-shaped workload:
batch 4, 16 heads, N = 8192, d = 64, B = 64, Top-K = 16, bf16 inputs with
planted needles.  `value` is whole-job TFLOP/s of algorithmic FLOPs
(4*d*(K_eff*B + own keys) per query head, the selected-chunk and own-chunk
QK^T + PV work), device-timed with CUDA events, inputs resident in HBM, L2
flushed (256 MB write) between steps outside the timed events.

Decode is reported beside it (tok/s at 32K/128K/512K, CUDA-graph replay).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs an independent replica (no collective on
the data path); rank 0 prints one JSON line with the max time over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from hils_inputs import CONFIGS, decode_inputs, prefill_inputs  # noqa: E402

PREFILL = CONFIGS["prefill_345m"]
METRIC = "HiLS fwd prefill TFLOP/s + decode tok/s; % of roofline on 1 B200"


def algorithmic_flops(batch, heads_q, seq_len, head_dim, top_k, chunk=64):
    i = np.arange(seq_len)
    keff = np.minimum(top_k, i // chunk)
    keys = keff * chunk + (i % chunk) + 1
    return float(4 * head_dim * keys.sum() * batch * heads_q)


def decode_bytes(cfg, summary_bytes=4):
    b, h, g, d, K = cfg["batch"], cfg["heads_q"], cfg["heads_kv"], cfg["head_dim"], cfg["top_k"]
    L = cfg["seq_len"]
    own = (L - 1) // 64
    keff = min(K, own)
    own_keys = L - own * 64
    kv = b * g * (keff * 64 + own_keys) * d * 2 * 2
    summ = b * own * h * (d * summary_bytes + 4)  # kbar (fp32 or bf16 cache) + fp32 H
    qo = b * h * d * 2 * 2
    return float(kv + summ + qo), float(kv)


# DRAM bytes (read + write) per launch of the prefill attention kernel at the bench size
# (attend_tc3_kernel for the 345M shape), from one ncu capture summarised under profiles/
# (attend_tc3_kernel_prefill_345m.md).  Reported only while the kernel's sources are the
# ones it was taken on.
ATTEND_TRAFFIC = {
    "sources": {"chunk_wise_hierarchical_b200/csrc/attend_tc3.cu":
                "c7a1d131b1c13ee793f69feff2448454ba899db1bba06b02660749024742bc2b",
                "chunk_wise_hierarchical_b200/csrc/tc_util.cuh":
                "ef2b1f54b29d8d04a25e377aec7307ed799b53c87ff99ab707d9d0d845134640",
                "chunk_wise_hierarchical_b200/csrc/common.cuh":
                "f19fe418aeaa91592e04d1c59c503e5fa51570749ec0ad3378b36b7762f2c5b4"},
    "bytes": 275178496 + 52989440,
}


def attend_traffic():
    import hashlib
    if ATTEND_TRAFFIC["bytes"] is None:
        return None
    for rel, digest in ATTEND_TRAFFIC["sources"].items():
        with open(os.path.join(ROOT, rel), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != digest:
                return None
    return ATTEND_TRAFFIC["bytes"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """Samples the SM clock and the throttle reasons while running (read-only queries).

    NVML is polled every ~2 ms from a thread, so that even a timed region of a few
    milliseconds gets several samples; the device is found by its UUID, so the reading
    is of this process's GPU whatever the visible-device mapping.  Without NVML it falls
    back to `nvidia-smi -lms 100`.
    """

    Q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    # NVML clocks-event reason bits, in the order of NAMES
    BITS = (0x8, 0x40, 0x20, 0x4)

    def __init__(self, index, period_s=0.002):
        self.index = index
        self.period = period_s
        self.proc = None
        self.thread = None
        self.stop = threading.Event()
        self.samples = []  # (sm MHz, max sm MHz, frozenset of active reasons)
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            u = str(torch.cuda.get_device_properties(self.index).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _nvml_sample(self, nv, h, mx):
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        self.samples.append((float(sm), mx, frozenset(n for n, bit in zip(self.NAMES, self.BITS) if r & bit)))

    def _nvml_loop(self, nv, h, mx):
        while not self.stop.is_set():
            try:
                self._nvml_sample(nv, h, mx)
            except Exception:
                return
            self.stop.wait(self.period)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._nvml_sample(nv, h, mx)  # one reading before the timed work starts
            self.source = "nvml"
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h, mx), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.samples = []
        try:
            # nvidia-smi numbers GPUs without regard to CUDA_VISIBLE_DEVICES: address the device by UUID
            try:
                u = str(torch.cuda.get_device_properties(self.index).uuid)
                dev_id = u if u.startswith("GPU-") else "GPU-" + u
            except Exception:
                dev_id = str(self.index)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", dev_id, f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            active = frozenset(n for n, v in zip(self.NAMES, parts[2:6]) if v.lower().startswith("active"))
            self.samples.append((sm, mx, active))

    def __exit__(self, *a):
        self.stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        sm = [x[0] for x in self.samples]
        mx = self.samples[-1][1] if self.samples else None
        reasons = set().union(*[x[2] for x in self.samples]) if self.samples else set()
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


def dist_setup(args=None, backend="nccl"):
    """One process per GPU under torchrun; returns (world size, rank, local rank)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        timeout = datetime.timedelta(seconds=300)
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group(backend, timeout=timeout)
    return ws, rank, local


def max_over_ranks(x, ws):
    """Max of a per-rank time over all ranks (every rank gets the result)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def job_tflops(ws, flops_per_replica, ms_max):
    """Whole-job throughput of ws replicas that each do flops_per_replica in (max) ms_max."""
    return ws * flops_per_replica / (ms_max * 1e-3) / 1e12


# ---------------------------------------------------------------------------- CPU baseline (oracle)
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(seconds_budget=20.0, threads=None, cfg_name="prefill_345m", inp=None, row_stride=1):
    """Times the fp64 oracle, as it stands, on a bounded sample of a prefill workload:
    (batch, KV group) slices, in order, until the time budget is spent, each with every
    row_stride-th query row.  The throughput is the algorithmic FLOPs of the rows done
    over the time taken.  threads: BLAS threads (None = every host core)."""
    from threadpoolctl import threadpool_limits

    from oracle import hils_oracle as O
    cfg = dict(CONFIGS[cfg_name])
    if inp is None:
        inp = prefill_inputs(seed=0, device="cpu", **cfg)
    n, grp = cfg["seq_len"], cfg["heads_q"] // cfg["heads_kv"]
    rows = np.arange(0, n, row_stride)
    keff = np.minimum(cfg["top_k"], rows // 64)
    head_flops = float(4 * cfg["head_dim"] * (keff * 64 + rows % 64 + 1).sum())
    full_flops = algorithmic_flops(cfg["batch"], cfg["heads_q"], n, cfg["head_dim"], cfg["top_k"])
    cores = threads or host_cores()
    t0 = time.perf_counter()
    flops, slices = 0.0, 0
    with threadpool_limits(limits=cores):
        for bi in range(cfg["batch"]):
            for gi in range(cfg["heads_kv"]):
                if slices and time.perf_counter() - t0 >= seconds_budget:
                    break
                hs = slice(gi * grp, (gi + 1) * grp)
                O.forward(inp.q[bi:bi + 1, hs], inp.k[bi:bi + 1, gi:gi + 1], inp.v[bi:bi + 1, gi:gi + 1],
                          inp.landmark[bi:bi + 1, hs], 64, cfg["top_k"], rows=None if row_stride == 1 else rows)
                flops += head_flops * grp
                slices += 1
    dt = time.perf_counter() - t0
    total = cfg["batch"] * cfg["heads_kv"]
    rows_txt = f"all {n} query rows" if row_stride == 1 else f"every {row_stride}th of {n} query rows"
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "seconds": round(dt, 2), "full_config_seconds_scaled": round(dt * full_flops / flops, 1),
            "sample": f"{cfg_name}: {slices} of {total} (batch, KV group) slices, {rows_txt} each "
                      f"(summaries, scores, Top-K, attention, fusion), {dt:.1f} s, fp64 numpy, "
                      f"BLAS on {cores} thread(s); full-config time scaled by algorithmic FLOPs"}


def cpu_decode_baseline(name, seconds_budget=10.0, threads=None):
    """The oracle's decode step on whole (sequence, KV head) slices of a decode workload
    (each slice drawn on its own, with the workload's shape), scaled by slice count to
    the whole batch (tokens/s)."""
    from threadpoolctl import threadpool_limits

    from oracle import hils_oracle as O
    cfg = dict(CONFIGS[name])
    grp = cfg["heads_q"] // cfg["heads_kv"]
    cores = threads or host_cores()
    spent, slices = 0.0, 0
    while slices == 0 or spent < seconds_budget:
        one = dict(cfg, batch=1, heads_q=grp, heads_kv=1)
        di = decode_inputs(seed=slices, device="cpu", **one)
        t0 = time.perf_counter()
        with threadpool_limits(limits=cores):
            O.decode(di.q, di.k_pages, di.v_pages, di.landmark_pages, di.block_table.numpy(),
                     di.seq_lens.numpy(), cfg["top_k"])
        spent += time.perf_counter() - t0
        slices += 1
        if slices >= cfg["batch"] * cfg["heads_kv"]:
            break
    total = cfg["batch"] * cfg["heads_kv"]
    step_s = spent * total / slices
    return {"tok_s": cfg["batch"] / step_s, "seconds": round(spent, 2), "full_step_seconds_scaled": round(step_s, 2),
            "cores": cores, "kind": "oracle",
            "sample": f"{name}: {slices} of {total} (sequence, KV head) slices of one decode step, each drawn "
                      f"alone with the workload's shape, scaled by slice count"}


def oracle_times(budget):
    """Oracle seconds beside the GPU time for every workload (each a bounded, stated sample)."""
    res = {}
    from threadpoolctl import threadpool_limits

    from oracle import hils_oracle as O
    cfg = CONFIGS["tiny_fp32"]
    inp = prefill_inputs(seed=0, device="cpu", **cfg)
    for cores in (1, None):
        t0 = time.perf_counter()
        with threadpool_limits(limits=cores or host_cores()):
            O.forward(inp.q, inp.k, inp.v, inp.landmark, 64, cfg["top_k"])
        res["tiny_fp32" + ("_1core" if cores == 1 else "")] = {
            "seconds": round(time.perf_counter() - t0, 3), "cores": cores or host_cores(), "sample": "full config"}
    res["prefill_7b_gqa"] = cpu_baseline(budget, cfg_name="prefill_7b_gqa", row_stride=16)
    for name in ("decode_32k", "decode_128k", "decode_512k"):
        res[name] = cpu_decode_baseline(name, budget / 2)
    return res


# ---------------------------------------------------------------------------- prefill (ours)
def run_prefill(args, ws_world, rank, local):
    import chunk_wise_hierarchical_b200 as hils
    dev = torch.device("cuda", local)
    cfg = PREFILL
    inp = prefill_inputs(seed=rank, device=dev, **cfg)
    q, k, v, lm = inp.q, inp.k, inp.v, inp.landmark
    b, h, n, d = q.shape
    g = k.shape[1]
    K = cfg["top_k"]
    out = torch.empty_like(q)
    sh = hils.make_shape(b, h, g, d, n, K, 1)
    C = n // 64
    kbar = torch.empty((b, h, C, d), dtype=torch.float32, device=dev)
    hb = torch.empty((b, h, C), dtype=torch.float32, device=dev)
    idx = torch.empty((b, g, n, K), dtype=torch.int32, device=dev)
    ssel = torch.empty((b, h, n, K), dtype=torch.float32, device=dev)
    ws_sel = hils.new_workspace(sh, hils.OP_ATTEND_SELECTED, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    flops = algorithmic_flops(b, h, n, d, K)

    def step(evs=None):
        # the three stages of hils_attend, called separately so the attention kernel can be timed
        if evs: evs[0].record(stream)
        kb, hbb = kbar, hb
        lib = hils.lib()
        import ctypes
        P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        st = ctypes.c_void_p(stream.cuda_stream)
        r = lib.hils_summarize(ctypes.byref(sh), P(k), P(lm), P(kb), P(hbb), st)
        if evs: evs[1].record(stream)
        r |= lib.hils_select(ctypes.byref(sh), P(q), P(kb), P(hbb), P(idx), P(ssel), P(ws_sel), ws_sel.numel(), st)
        if evs: evs[2].record(stream)
        r |= lib.hils_attend_selected(ctypes.byref(sh), P(q), P(k), P(v), P(idx), P(ssel), P(out), None,
                                      P(ws_sel), ws_sel.numel(), st)
        if evs: evs[3].record(stream)
        if r != 0:
            raise RuntimeError(f"HiLS call failed: {r}")

    for _ in range(args.warmup):
        step()
    barrier(ws_world)
    evsets = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with Clocks(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(evsets[i])
        barrier(ws_world)
    tot = [e[0].elapsed_time(e[3]) for e in evsets]
    att = [e[2].elapsed_time(e[3]) for e in evsets]
    summ = [e[0].elapsed_time(e[1]) for e in evsets]
    sel = [e[1].elapsed_time(e[2]) for e in evsets]
    ms_step = max_over_ranks(statistics.median(tot), ws_world)
    ms_att = statistics.median(att)
    recall = needle_recall(inp.needles, idx, h // g)

    # End to end through the public API with host buffers (pinned): every step uploads its
    # inputs and downloads its output inside the timed region.  Two buffer sets and three
    # streams (upload, compute, download) let step s+1's upload overlap step s's compute
    # and download, as a serving loop would; events guard every buffer's reuse.
    host = [t.cpu().pin_memory() for t in (q, k, v, lm)]
    host_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    call = hils.Prefill(b, h, g, n, d, K, torch.bfloat16, device=dev)
    bufs = [[torch.empty_like(t) for t in (q, k, v, lm)] for _ in range(2)]
    douts = [torch.empty_like(q) for _ in range(2)]
    up, comp, down = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n_steps):
        for st in range(n_steps):
            j = st % 2
            with torch.cuda.stream(up):
                if st >= 2:
                    up.wait_event(ev_comp[j])  # step st-2 has consumed this buffer set
                for dst, src in zip(bufs[j], host):
                    dst.copy_(src, non_blocking=True)
                ev_up[j].record(up)
            with torch.cuda.stream(comp):
                comp.wait_event(ev_up[j])
                if st >= 2:
                    comp.wait_event(ev_down[j])  # step st-2's output has been read back
                call(*bufs[j], out=douts[j], stream=comp)
                ev_comp[j].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(ev_comp[j])
                host_out[j].copy_(douts[j], non_blocking=True)
                ev_down[j].record(down)

    e2e_steps(max(2, args.warmup))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = args.steps
    e0.record(up)  # before the first upload
    e2e_steps(n_e2e)
    e1.record(down)  # after the last download, which follows every other step's work
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, ws_world)
    assert call.device_status() == 0
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = host_out[0].numel() * host_out[0].element_size()
    return dict(flops=flops, ms_step=ms_step, ms_att=ms_att, ms_summ=statistics.median(summ),
                ms_sel=statistics.median(sel), ms_e2e=ms_e2e, h2d=h2d, d2h=d2h, clocks=clk.summary(),
                launches_per_step=3, needle_recall=recall)


def needle_recall(needles, idx, group):
    """Diagnostic (not parity): the fraction of planted needles (b, h, c, j, i) whose
    target query i selected the needle's chunk c."""
    if not needles:
        return None
    t = torch.tensor([[b, h // group, i, c] for b, h, c, j, i in needles], device=idx.device)
    sel = idx[t[:, 0], t[:, 1], t[:, 2]]
    hit = (sel == t[:, 3:4]).any(dim=1)
    return {"hits": int(hit.sum()), "needles": len(needles), "fraction": round(float(hit.float().mean()), 4)}


def run_prefill_gqa(dev, steps=5, warmup=3, seq_len=None):
    """The 7B-shaped GQA prefill (b1 h32 g8 N32768 d128 K32): per-stage device times and
    TFLOP/s of the same algorithmic FLOP count, reported beside the headline step.
    seq_len shortens the sequence (a reduced case for profiling, not a bench line)."""
    import chunk_wise_hierarchical_b200 as hils
    cfg = dict(CONFIGS["prefill_7b_gqa"])
    if seq_len:
        cfg["seq_len"] = seq_len
    inp = prefill_inputs(seed=0, device=dev, **cfg)
    q, k, v, lm = inp.q, inp.k, inp.v, inp.landmark
    b, h, n, d = q.shape
    g = k.shape[1]
    K = cfg["top_k"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    times = []
    for it in range(warmup + steps):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record()
        kbar, hb = hils.summarize(k, lm)
        ev[1].record()
        idx, sc = hils.select(q, kbar, hb, K, g)
        ev[2].record()
        hils.attend_selected(q, k, v, idx, sc)
        ev[3].record()
        torch.cuda.synchronize()
        if it >= warmup:
            times.append([ev[i].elapsed_time(ev[i + 1]) for i in range(3)])
    med = [statistics.median(t[i] for t in times) for i in range(3)]
    flops = algorithmic_flops(b, h, n, d, K)
    return {"workload": f"prefill_7b_gqa: batch 1, 32 query heads / 8 KV heads, N {n}, d 128, top-k 32, bf16",
            "ms_per_step": round(sum(med), 4), "needle_recall": needle_recall(inp.needles, idx, h // g),
            "stage_ms": {"summarize": round(med[0], 4), "select": round(med[1], 4), "attend_selected": round(med[2], 4)},
            "tflops": round(flops / (sum(med) * 1e-3) / 1e12, 3),
            "attend_tflops": round(flops / (med[2] * 1e-3) / 1e12, 3),
            "timing": "CUDA events per stage, median of %d steps, L2 flushed between steps" % steps}


def run_training(dev, steps=5, warmup=3, seq_len=None):
    """The training workload (b2 h16 N16384 d128 K16, bf16): one forward (summaries,
    selection, attention with log Zhat) and one hils_backward per step, with dO ~ N(0,1).
    Backward algorithmic FLOPs = 2.5 x the forward's: per (query, key) pair the forward
    does 4d (QK^T, PV) and the backward 10d (QK^T and dO V^T recomputed, dV, dK, dQ)."""
    import chunk_wise_hierarchical_b200 as hils
    cfg = dict(CONFIGS["train_16k"])
    if seq_len:
        cfg["seq_len"] = seq_len
    inp = prefill_inputs(seed=0, device=dev, **cfg)
    q, k, v, lm = inp.q, inp.k, inp.v, inp.landmark
    b, h, n, d = q.shape
    g = k.shape[1]
    K = cfg["top_k"]
    dout = torch.randn(q.shape, device=dev, generator=torch.Generator(device=dev).manual_seed(1)).to(torch.bfloat16)
    lse = torch.empty((b, h, n), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    sh = hils.make_shape(b, h, g, d, n, K, 1)
    ws = hils.new_workspace(sh, hils.OP_BACKWARD, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    times = []
    for it in range(warmup + steps):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record()
        kbar, hb = hils.summarize(k, lm)
        idx, sc = hils.select(q, kbar, hb, K, g)
        hils.attend_selected(q, k, v, idx, sc, out=out, lse=lse)
        ev[1].record()
        hils.backward(q, k, v, lm, out, lse, idx, sc, dout, ws=ws)
        ev[2].record()
        torch.cuda.synchronize()
        if it >= warmup:
            times.append((ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])))
    assert hils.lib().hils_device_status(ctypes.c_void_p(ws.data_ptr()), None) == 0
    fwd = statistics.median(t[0] for t in times)
    bwd = statistics.median(t[1] for t in times)
    flops = algorithmic_flops(b, h, n, d, K)
    return {"workload": f"train_16k: batch 2, 16 heads, N {n}, d 128, top-k 16, bf16 N(0,1), dO N(0,1)",
            "forward_ms": round(fwd, 3), "backward_ms": round(bwd, 3),
            "forward_tflops": round(flops / (fwd * 1e-3) / 1e12, 2),
            "backward_tflops": round(2.5 * flops / (bwd * 1e-3) / 1e12, 2),
            "algorithmic_gflop": {"forward": round(flops / 1e9, 1), "backward": round(2.5 * flops / 1e9, 1)},
            "timing": "CUDA events, median of %d steps, L2 flushed between steps" % steps}


# ---------------------------------------------------------------------------- decode (ours)
def run_decode(name, n_caches, dev, reps=50):
    """Decode step time for the fp32 summary cache and for the compact bf16 one, on the
    same inputs: CUDA-graph replays rotating over n_caches independent caches."""
    import chunk_wise_hierarchical_b200 as hils
    cfg = CONFIGS[name]
    K = cfg["top_k"]
    caches = []
    for c in range(n_caches):
        di = decode_inputs(seed=100 + c, device=dev, **cfg)
        P, g, B, d = di.k_pages.shape
        h = di.landmark_pages.shape[1]
        ids = torch.arange(P, dtype=torch.int32, device=dev)
        kbars = {}
        for dt in (torch.float32, torch.bfloat16):
            kbar = torch.empty((P, h, d), dtype=dt, device=dev)
            hb = torch.empty((P, h), dtype=torch.float32, device=dev)
            hils.summarize_paged(di.k_pages, di.landmark_pages, ids, kbar, hb)
            kbars[dt] = (kbar, hb)
        call = hils.Decode(cfg["batch"], h, g, d, di.max_chunks, K, torch.bfloat16, device=dev)
        out = torch.empty_like(di.q)
        del di.landmark_pages
        caches.append((di, kbars, call, out))
    torch.cuda.synchronize()
    s = torch.cuda.Stream(device=dev)
    res = {}
    for dt, sbytes in ((torch.float32, 4), (torch.bfloat16, 2)):
        graphs = []
        with torch.cuda.stream(s):
            for (di, kbars, call, out) in caches:  # warm up outside capture
                call(di.q, di.k_pages, di.v_pages, *kbars[dt], di.block_table, di.seq_lens, out=out)
        torch.cuda.synchronize()
        for (di, kbars, call, out) in caches:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=s):
                call(di.q, di.k_pages, di.v_pages, *kbars[dt], di.block_table, di.seq_lens, out=out)
            graphs.append(gr)
        for gr in graphs:
            gr.replay()
        torch.cuda.synchronize()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        evs[0].record()
        for r in range(reps):
            graphs[r % len(graphs)].replay()
            evs[r + 1].record()
        torch.cuda.synchronize()
        ms = statistics.median(evs[r].elapsed_time(evs[r + 1]) for r in range(reps))
        for (di, kbars, call, out) in caches:
            assert call.device_status() == 0
        alg, kv_only = decode_bytes(cfg, sbytes)
        del graphs
        res[dt] = dict(ms=ms, tok_s=cfg["batch"] / (ms * 1e-3), gbs=alg / (ms * 1e-3) / 1e9, bytes=alg,
                       kv_bytes=kv_only, caches=n_caches, reps=reps)
    del caches
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    ws_world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    hbm, bf16_peak, bf16_sus, peak_src = load_peaks()
    dec = {}
    if not args.no_decode:
        for name in args.decode_configs.split(","):
            # three rotating caches (each larger than L2 from 128K up) keep every step's reads in
            # HBM; from 1M tokens on, one cache (about 34 GB) is far beyond L2 by itself
            big = CONFIGS[name]["batch"] * CONFIGS[name]["seq_len"] > (1 << 22)
            r = run_decode(name, 1 if big else 3, torch.device("cuda", local))
            dec[name] = r[torch.float32]
            dec[name + "_bf16_summaries"] = r[torch.bfloat16]
    if args.decode_only:
        if rank == 0:
            print(json.dumps({"decode": {k: {"us_per_step": round(r["ms"] * 1e3, 2),
                                             "tok_s": round(r["tok_s"], 1),
                                             "frac_hbm": round(r["gbs"] / hbm, 4)} for k, r in dec.items()}}))
        return
    pre = run_prefill(args, ws_world, rank, local)
    gqa = run_prefill_gqa(torch.device("cuda", local), seq_len=args.gqa_seq) if not args.no_gqa else None
    train = run_training(torch.device("cuda", local), seq_len=args.train_seq) if not args.no_train else None
    cpu = cpu1 = otimes = None
    if rank == 0 and ws_world == 1 and not args.no_cpu:
        cpu = cpu_baseline(args.cpu_seconds)                 # every host core
        cpu1 = cpu_baseline(args.cpu_seconds / 2, threads=1)  # one core
        otimes = oracle_times(args.cpu_seconds / 2)
    if ws_world > 1:
        torch.distributed.barrier()
    if rank != 0:
        torch.distributed.destroy_process_group()
        return
    flops = pre["flops"]
    value = job_tflops(ws_world, flops, pre["ms_step"])
    att_tflops = flops / (pre["ms_att"] * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": ws_world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(pre["ms_step"], 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "prefill_345m: batch 4, 16 heads (MHA), N 8192, d 64, chunk 64, top-k 16, "
                               "bf16 N(0,1) Q/K/V/landmarks, 8 needles per head",
                   "global_batch": PREFILL["batch"] * ws_world, "seq_len": PREFILL["seq_len"],
                   "parallelism": f"replicas x{ws_world}", "l2": "flushed (256 MB write) between steps",
                   "algorithmic_gflop_per_step": round(flops / 1e9, 3)},
        "stage_ms": {"summarize": round(pre["ms_summ"], 4), "select": round(pre["ms_sel"], 4),
                     "attend_selected": round(pre["ms_att"], 4)},
        "roofline": {"bound": "tensor", "kernel": "attend_selected (selected + own chunk attention, fusion)",
                     "achieved": round(att_tflops, 3), "peak": bf16_peak, "unit": "TFLOP/s",
                     "frac": round(att_tflops / bf16_peak, 5), "peak_source": f"{peak_src} bf16 burst",
                     "traffic": args.traffic if args.traffic is not None else attend_traffic()},
        "e2e": {"value": round(job_tflops(ws_world, flops, pre["ms_e2e"]), 4), "unit": "TFLOP/s",
                "ms_per_step": round(pre["ms_e2e"], 3), "h2d_bytes_per_step": pre["h2d"],
                "d2h_bytes_per_step": pre["d2h"],
                "timing": "public Prefill call; per step: upload Q/K/V/L from pinned host memory, compute, "
                          "download the output; two buffer sets on upload/compute/download streams overlap "
                          "consecutive steps"},
        "gpu_launches": pre["launches_per_step"] * args.steps,
        "clocks": pre["clocks"],
        "needle_recall": pre["needle_recall"],
        "timing": "CUDA-event median over the timed steps",
    }
    if gqa:
        line["prefill_7b_gqa"] = gqa
    if train:
        line["train_16k"] = train
    if dec:
        line["decode"] = {
            k: {"tok_s": round(r["tok_s"], 1), "us_per_step": round(r["ms"] * 1e3, 2),
                "alg_bytes": int(r["bytes"]), "kv_bytes": int(r["kv_bytes"]),
                "achieved_gbs": round(r["gbs"], 1), "frac_hbm": round(r["gbs"] / hbm, 4),
                "timing": f"CUDA-graph replay, 2 kernels per step, median of {r['reps']} steps rotating over "
                          f"{r['caches']} independent caches"}
            for k, r in dec.items()}
    if cpu:
        line["cpu_baseline"] = cpu
        line["cpu_baseline_1core"] = cpu1
        line["oracle_times"] = otimes
    print(json.dumps(line), flush=True)
    if ws_world > 1:
        torch.distributed.destroy_process_group()


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, bounded sample per step."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(per_step / 4)
    vals = [cpu_baseline(per_step) for _ in range(args.steps)]
    value = statistics.median(v["value"] for v in vals)
    flops = algorithmic_flops(PREFILL["batch"], PREFILL["heads_q"], PREFILL["seq_len"], PREFILL["head_dim"],
                              PREFILL["top_k"])
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        # each timed step is a bounded sample of the workload (see cpu_baseline.sample)
        "ms_per_step": round(statistics.median(v["seconds"] for v in vals) * 1e3, 1),
        "ms_per_full_step_extrapolated": round(flops / (value * 1e12) * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "prefill_345m: batch 4, 16 heads (MHA), N 8192, d 64, chunk 64, top-k 16",
                   "global_batch": PREFILL["batch"], "seq_len": PREFILL["seq_len"], "parallelism": "cpu oracle"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": vals[-1]["cores"], "kind": "oracle",
                         "sample": "each step: " + vals[-1]["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true", help="time only the decode configurations")
    ap.add_argument("--decode-configs", default="decode_32k,decode_128k,decode_512k,decode_1m,decode_4m")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-gqa", action="store_true", help="skip the 7B-shaped GQA prefill line")
    ap.add_argument("--gqa-seq", type=int, default=None,
                    help="shorter sequence for the GQA line (a reduced case for profiling)")
    ap.add_argument("--train-seq", type=int, default=None,
                    help="shorter sequence for the training line (a reduced case for profiling)")
    ap.add_argument("--no-train", action="store_true", help="skip the forward + backward training line")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the attention kernel from an ncu capture")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

Headline: causal prefill forward (B=4, H=16, L=4096, d=128, bf16) in TFLOP/s
(causal FLOPs counted as half: 4 * d * visible (query, key) pairs) and its
fraction of the measured dense bf16 tensor peak.  The same JSON line carries
the split-KV decode leg (B=64, Hq=32, Hkv=8, cache 32768 x 128, k_len ~
U[1024, 32768]) in HBM GB/s and, once available, the causal backward leg
(B=2, H=16, L=8192, d=128) in TFLOP/s.

Contract: ``python bench.py --gpus N --steps K --warmup W [--impl reference]``;
under torchrun each rank runs an independent replica of the workload (no
collective on the data path), the step time is the max over ranks and rank 0
prints one JSON line.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import signal
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "fwd attention TFLOP/s & % of BF16 tensor peak; decode KV-scan HBM GB/s"
FWD = dict(B=4, Hq=16, Hkv=16, L=4096, d=128, causal=True)
DEC = dict(B=64, Hq=32, Hkv=8, Lmax=32768, d=128, klo=1024)
BWD = dict(B=2, Hq=16, Hkv=16, L=8192, d=128, causal=True)
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2


def causal_pairs(Lq, Lk, causal, k_len=None):
    """Number of visible (query, key) pairs of one head."""
    kl = Lk if k_len is None else k_len
    if not causal:
        return Lq * kl
    off = Lk - Lq
    i = np.arange(Lq, dtype=np.int64)
    return int(np.clip(np.minimum(i + off + 1, kl), 0, None).sum())


def fwd_flops(c):
    return 4.0 * c["d"] * causal_pairs(c["L"], c["L"], c["causal"]) * c["B"] * c["Hq"]


def bwd_flops(c):
    return 10.0 * c["d"] * causal_pairs(c["L"], c["L"], c["causal"]) * c["B"] * c["Hq"]


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
         "source": "fallback peaks (MEASURED_PEAKS.json absent)"}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        p.update({k: float(m[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")})
        p["source"] = "measured peaks (MEASURED_PEAKS.json)"
    except Exception:
        pass
    return p


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.send_signal(signal.SIGTERM)
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k] == "Active"})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(rows[0][2]),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit()),
                "samples": len(rows), "reasons": reasons}


# ------------------------------------------------------------------ distributed plumbing


def dist_setup(n_gpus):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    import torch

    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    """Max of a host float over the ranks (NCCL on the GPU, gloo on the CPU)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ DRAM traffic of the kernels

TRAFFIC_TABLE = os.path.join(ROOT, "profiles", "traffic.json")


def kernel_sources_sha(files):
    """sha256 over the listed source files (relative to the repo root)."""
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def traffic_per_launch(kernel, algorithmic=None):
    """DRAM bytes (read + write) per launch from the committed ncu table, or
    None when there is no entry or the kernel's sources changed since.  When
    the capture ran a smaller case of the same kernel, its traffic is scaled by
    the ratio of algorithmic bytes (``algorithmic`` = this launch's)."""
    try:
        with open(TRAFFIC_TABLE) as f:
            t = json.load(f)[kernel]
        if kernel_sources_sha(t["sources"]) != t["sources_sha256"]:
            return None
        dram = float(t["dram_bytes_per_launch"])
        if algorithmic is not None and t.get("algorithmic_bytes_per_launch"):
            dram *= algorithmic / float(t["algorithmic_bytes_per_launch"])
        return dram
    except Exception:
        return None


# ------------------------------------------------------------------ legs


def l2_flush(flush_buf):
    """Evicts the kernels' data from L2: writes the first half of ``flush_buf``
    (larger than L2), then reads the second half, so that the write's dirty
    lines are written back here and not inside the next timed region."""
    import torch

    n = flush_buf.numel() // 2
    flush_buf[:n].fill_(1)
    torch.sum(flush_buf[n:])


def timed_loop(fn, steps, warmup, stream, flush_buf):
    """Runs fn() warmup + steps times; each timed call is bracketed by CUDA events
    on ``stream`` and preceded by an L2 flush.  Returns per-step ms list."""
    import torch

    for _ in range(warmup):
        l2_flush(flush_buf)
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for s, e in ev:
        l2_flush(flush_buf)
        s.record(stream)
        fn()
        e.record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in ev]


def fwd_leg(steps, warmup, world, flush):
    import torch

    import exact_io_aware_46_b200 as attn

    c = FWD
    dev = torch.device("cuda")
    q = synth.normal_bf16_device(synth.workload_seed(2, "q"), (c["B"], c["Hq"], c["L"], c["d"]), dev)
    k = synth.normal_bf16_device(synth.workload_seed(2, "k"), (c["B"], c["Hkv"], c["L"], c["d"]), dev)
    v = synth.normal_bf16_device(synth.workload_seed(2, "v"), (c["B"], c["Hkv"], c["L"], c["d"]), dev)
    O = torch.empty_like(q)
    lse = torch.empty((c["B"], c["Hq"], c["L"]), dtype=torch.float32, device=dev)
    ws = torch.zeros(attn.attn_fwd_workspace_size(c["B"], c["Hq"], c["Hkv"], c["L"], c["L"], c["d"]),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    call = lambda: attn.attn_fwd(q, k, v, causal=True, O=O, lse=lse, workspace=ws, stream=stream)
    barrier(world)
    ms = timed_loop(call, steps, warmup, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")

    # end to end: pinned host inputs -> device -> kernels -> host outputs, every step,
    # through the public API one sequence at a time so that the copies overlap: the
    # inputs of sequence b copy in on one stream while sequence b - 1 computes and
    # earlier outputs copy out on a third (the host link is full duplex)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    hL = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(c["B"])]
    ev_out = [torch.cuda.Event() for _ in range(c["B"])]

    def e2e_call():
        h2d_s.wait_stream(stream)  # nothing starts before the timed region does
        d2h_s.wait_stream(stream)
        for b in range(c["B"]):
            with torch.cuda.stream(h2d_s):
                q[b].copy_(hq[b], non_blocking=True)
                k[b].copy_(hk[b], non_blocking=True)
                v[b].copy_(hv[b], non_blocking=True)
                ev_in[b].record(h2d_s)
            stream.wait_event(ev_in[b])
            attn.attn_fwd(q[b:b + 1], k[b:b + 1], v[b:b + 1], causal=True, O=O[b:b + 1],
                          lse=lse[b:b + 1], workspace=ws, stream=stream)
            ev_out[b].record(stream)
            d2h_s.wait_event(ev_out[b])
            with torch.cuda.stream(d2h_s):
                hO[b].copy_(O[b], non_blocking=True)
                hL[b].copy_(lse[b], non_blocking=True)
        stream.wait_stream(d2h_s)  # the step ends when the last output is on the host

    barrier(world)
    ms_e2e = timed_loop(e2e_call, max(3, steps // 2), 3, stream, flush)
    torch.cuda.synchronize()
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = hO.numel() * hO.element_size() + hL.numel() * hL.element_size()
    # the same workload with a sliding window of 1024 keys (key tiles outside skipped)
    W = WINDOW
    call_w = lambda: attn.attn_fwd_sliding(q, k, v, W, O=O, lse=lse, workspace=ws, stream=stream)
    barrier(world)
    wms = timed_loop(call_w, steps, warmup, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    wflops = 4.0 * c["d"] * c["B"] * c["Hq"] * sum(min(i + 1, W) for i in range(c["L"]))
    # the same workload with E4M3 inputs: these tensors quantised per 128-row tile
    del hq, hk, hv, hO, hL
    q8, qs = synth.quantize_e4m3_tiles(q.float())
    k8, ks = synth.quantize_e4m3_tiles(k.float())
    v8, vs = synth.quantize_e4m3_tiles(v.float())
    del q, k, v
    torch.cuda.empty_cache()
    call_8 = lambda: attn.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=True, O=O, lse=lse,
                                       workspace=ws, stream=stream)
    barrier(world)
    fms = timed_loop(call_8, steps, warmup, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    del q8, k8, v8, qs, ks, vs, O, lse
    torch.cuda.empty_cache()
    # the same shape at d = 64
    shp64 = (c["B"], c["Hq"], c["L"], 64)
    q6, k6, v6 = (synth.normal_bf16_device(synth.workload_seed(2, t) ^ 64, shp64, dev)
                  for t in ("q", "k", "v"))
    O6 = torch.empty_like(q6)
    lse6 = torch.empty((c["B"], c["Hq"], c["L"]), dtype=torch.float32, device=dev)
    call_6 = lambda: attn.attn_fwd(q6, k6, v6, causal=True, O=O6, lse=lse6, workspace=ws,
                                   stream=stream)
    barrier(world)
    ms64 = timed_loop(call_6, steps, warmup, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    del q6, k6, v6, O6, lse6
    torch.cuda.empty_cache()
    return (ms, ms_e2e, h2d, d2h, varlen_leg(steps, warmup, world, flush), (W, wms, wflops),
            fms, ms64)


WINDOW = 1024


VARLEN = dict(n_seq=16, lo=256, hi=4096, H=16, d=128)


def varlen_leg(steps, warmup, world, flush):
    """Packed causal prefill: 16 sequences with seeded lengths ~ U[256, 4096] back to
    back, Hq = Hkv = 16, d = 128.  FLOPs count each sequence's visible pairs."""
    import torch

    import exact_io_aware_46_b200 as attn

    c = VARLEN
    dev = torch.device("cuda")
    lens = synth.uniform_int(synth.workload_seed(6, "klen"), c["n_seq"], c["lo"], c["hi"])
    total = int(np.sum(lens.astype(np.int64)))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    q = synth.normal_bf16_device(synth.workload_seed(6, "q"), (total, c["H"], c["d"]), dev)
    k = synth.normal_bf16_device(synth.workload_seed(6, "k"), (total, c["H"], c["d"]), dev)
    v = synth.normal_bf16_device(synth.workload_seed(6, "v"), (total, c["H"], c["d"]), dev)
    O = torch.empty_like(q)
    lse = torch.empty((c["H"], total), dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    mx = int(lens.max())
    call = lambda: attn.attn_fwd_varlen(q, k, v, cu, cu, mx, mx, causal=True, O=O, lse=lse,
                                        workspace=ws, stream=stream)
    barrier(world)
    ms = timed_loop(call, steps, warmup, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    flops = sum(4.0 * c["d"] * causal_pairs(int(L), int(L), True) * c["H"] for L in lens)
    return ms, flops, total


def decode_leg(steps, warmup, world, flush):
    import torch

    import exact_io_aware_46_b200 as attn

    c = DEC
    dev = torch.device("cuda")
    k_lens = synth.uniform_int(synth.workload_seed(4, "klen"), c["B"], c["klo"], c["Lmax"])
    q = synth.normal_bf16_device(synth.workload_seed(4, "q"), (c["B"], c["Hq"], 1, c["d"]), dev)
    kc = synth.normal_bf16_device(synth.workload_seed(4, "k"), (c["B"], c["Hkv"], c["Lmax"], c["d"]), dev)
    vc = synth.normal_bf16_device(synth.workload_seed(4, "v"), (c["B"], c["Hkv"], c["Lmax"], c["d"]), dev)
    kl = torch.from_numpy(k_lens).to(dev)
    O = torch.empty_like(q)
    lse = torch.empty((c["B"], c["Hq"]), dtype=torch.float32, device=dev)
    ws = torch.zeros(attn.attn_decode_workspace_size(c["B"], c["Hq"], c["Hkv"], c["Lmax"], c["d"]),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    call = lambda: attn.attn_fwd_splitkv_decode(q, kc, vc, kl, O=O, lse=lse, workspace=ws,
                                                stream=stream)
    barrier(world)
    ms = timed_loop(call, steps, warmup, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    kv_bytes = float(np.sum(k_lens.astype(np.int64))) * c["Hkv"] * c["d"] * 2 * 2
    # the same workload over a paged cache: 64-row pages in a seeded random order
    page = 64
    nb = c["Lmax"] // page
    order = torch.from_numpy(
        np.argsort(synth.uniform_u64(synth.workload_seed(4, "pages"), c["B"] * nb),
                   kind="stable")).to(dev)
    table = order.view(c["B"], nb).to(torch.int32).contiguous()

    def to_pages(cache):
        blocks = cache.view(c["B"], c["Hkv"], nb, page, c["d"]).permute(0, 2, 1, 3, 4)
        out = torch.empty((c["B"] * nb, c["Hkv"], page, c["d"]), dtype=cache.dtype, device=dev)
        out[order] = blocks.reshape(c["B"] * nb, c["Hkv"], page, c["d"])
        return out

    kp, vp = to_pages(kc), to_pages(vc)
    del kc, vc
    torch.cuda.empty_cache()
    call_p = lambda: attn.attn_fwd_splitkv_decode_paged(q, kp, vp, table, kl, O=O, lse=lse,
                                                        workspace=ws, stream=stream)
    barrier(world)
    pms = timed_loop(call_p, steps, warmup, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    del kp, vp
    torch.cuda.empty_cache()
    return ms, kv_bytes, k_lens, (page, pms)


LONG = dict(B=1, Hq=32, Hkv=8, L=16384, d=128, klo=8192)


def long_klen():
    """The padding variant's valid key length, uniform in [8192, 16384] (seeded)."""
    c = LONG
    return int(synth.uniform_int(synth.workload_seed(3, "klen"), c["B"], c["klo"], c["L"])[0])


def long_leg(steps, warmup, world, flush):
    """Long-context causal forward B1 Hq32 Hkv8 (GQA) L16384 d128, and the same
    with key padding (k_len ~ U[8192, 16384], seeded); FLOPs over visible pairs."""
    import torch

    import exact_io_aware_46_b200 as attn

    c = LONG
    dev = torch.device("cuda")
    q = synth.normal_bf16_device(synth.workload_seed(3, "q"), (c["B"], c["Hq"], c["L"], c["d"]), dev)
    k = synth.normal_bf16_device(synth.workload_seed(3, "k"), (c["B"], c["Hkv"], c["L"], c["d"]), dev)
    v = synth.normal_bf16_device(synth.workload_seed(3, "v"), (c["B"], c["Hkv"], c["L"], c["d"]), dev)
    O = torch.empty_like(q)
    lse = torch.empty((c["B"], c["Hq"], c["L"]), dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    kl = long_klen()
    k_lens = torch.full((c["B"],), kl, dtype=torch.int32, device=dev)
    calls = {name: (lambda kls=kls: attn.attn_fwd(q, k, v, causal=True, k_lens=kls, O=O,
                                                  lse=lse, workspace=ws, stream=stream))
             for name, kls in (("causal", None), ("padded", k_lens))}
    # the two variants alternate step by step, so that both see the same clocks (under a
    # sustained load the power cap lowers them over seconds: timed one after the other,
    # the second variant read ~8 % slower than the same kernel measured first)
    barrier(world)
    out = {name: [] for name in calls}
    for _ in range(warmup):
        for fn in calls.values():
            l2_flush(flush)
            fn()
    for _ in range(steps):
        for name, fn in calls.items():
            out[name] += timed_loop(fn, 1, 0, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    flops = {"causal": 4.0 * c["d"] * causal_pairs(c["L"], c["L"], True) * c["B"] * c["Hq"],
             "padded": 4.0 * c["d"] * causal_pairs(c["L"], c["L"], True, kl) * c["B"] * c["Hq"]}
    del q, k, v, O, lse
    torch.cuda.empty_cache()
    return out, flops, kl


RING = dict(world=4, B=1, Hq=32, Hkv=8, L=16384, d=128)


def ring_leg(steps, warmup, world, flush):
    """Ring attention's decomposition on one GPU: the long-context causal workload
    B1 Hq32 Hkv8 L16384 d128 split into 4 chunks of 4096; every emulated rank's
    ring steps (attn_fwd_merge on each visible chunk: the forward with the fold
    into the fp32 accumulator in its epilogue) run back to back, without the
    exchange (one GPU).  Also times the stand-alone attn_merge_partial on one
    chunk's rows (HBM-bound)."""
    import torch

    import exact_io_aware_46_b200 as attn
    from exact_io_aware_46_b200.ring import (bwd_chunk, fold_chunk, ring_steps, zigzag_chunks,
                                             zigzag_folds)

    c = RING
    W, Lc = c["world"], c["L"] // c["world"]
    dev = torch.device("cuda")
    q = synth.normal_bf16_device(synth.workload_seed(3, "q"), (c["B"], c["Hq"], c["L"], c["d"]), dev)
    k = synth.normal_bf16_device(synth.workload_seed(3, "k"), (c["B"], c["Hkv"], c["L"], c["d"]), dev)
    v = synth.normal_bf16_device(synth.workload_seed(3, "v"), (c["B"], c["Hkv"], c["L"], c["d"]), dev)
    qs = [q[:, :, r * Lc:(r + 1) * Lc].contiguous() for r in range(W)]
    ks = [k[:, :, r * Lc:(r + 1) * Lc].contiguous() for r in range(W)]
    vs = [v[:, :, r * Lc:(r + 1) * Lc].contiguous() for r in range(W)]
    Lz = c["L"] // (2 * W)  # zigzag: 2 * W chunks, rank r holds chunks r and 2W - 1 - r
    zq = [q[:, :, i * Lz:(i + 1) * Lz].contiguous() for i in range(2 * W)]
    zk = [k[:, :, i * Lz:(i + 1) * Lz].contiguous() for i in range(2 * W)]
    zv = [v[:, :, i * Lz:(i + 1) * Lz].contiguous() for i in range(2 * W)]
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    # the undivided sequence in one call, for comparison
    O1 = torch.empty_like(q)
    L1 = torch.empty((c["B"], c["Hq"], c["L"]), dtype=torch.float32, device=dev)
    whole = lambda: attn.attn_fwd(q, k, v, causal=True, O=O1, lse=L1, workspace=ws)
    barrier(world)
    wms = timed_loop(whole, steps, warmup, torch.cuda.current_stream(), flush)
    # the backward's decomposition: every rank's chunk pairs through attn_bwd, the
    # partial gradients summed in fp32 (stream launches), next to the undivided call
    dO = synth.normal_bf16_device(synth.workload_seed(3, "do"), tuple(q.shape), dev)
    bws = torch.zeros(attn.attn_bwd_workspace_size(c["B"], c["Hq"], c["Hkv"], Lc, Lc, c["d"]),
                      dtype=torch.uint8, device=dev)
    bws_whole = torch.zeros(attn.attn_bwd_workspace_size(c["B"], c["Hq"], c["Hkv"], c["L"],
                                                         c["L"], c["d"]),
                            dtype=torch.uint8, device=dev)
    os_ = [O1[:, :, r * Lc:(r + 1) * Lc].contiguous() for r in range(W)]
    ls_ = [L1[:, :, r * Lc:(r + 1) * Lc].contiguous() for r in range(W)]
    dos = [dO[:, :, r * Lc:(r + 1) * Lc].contiguous() for r in range(W)]
    dq_acc = [torch.empty_like(qs[0], dtype=torch.float32) for _ in range(W)]
    dk_acc = [torch.empty_like(ks[0], dtype=torch.float32) for _ in range(W)]
    dv_acc = [torch.empty_like(vs[0], dtype=torch.float32) for _ in range(W)]
    bplans = [ring_steps(r, W, True) for r in range(W)]

    def bwd_step():
        started = set()
        for r in range(W):
            first = True
            for _, src, kind in bplans[r]:
                part = bwd_chunk(qs[r], ks[src], vs[src], os_[r], dos[r], ls_[r], kind,
                                 workspace=bws)
                if part is None:
                    continue
                attn.attn_accumulate(part[0], dq_acc[r], init=first)
                first = False
                attn.attn_accumulate(part[1], dk_acc[src], init=src not in started)
                attn.attn_accumulate(part[2], dv_acc[src], init=src not in started)
                started.add(src)

    barrier(world)
    bms_ring = timed_loop(bwd_step, max(3, steps // 2), warmup, torch.cuda.current_stream(), flush)
    whole_b = lambda: attn.attn_bwd(q, k, v, O1, dO, L1, causal=True, workspace=bws_whole)
    bms_whole = timed_loop(whole_b, max(3, steps // 2), warmup, torch.cuda.current_stream(), flush)
    del q, k, v, O1, L1, dO, os_, ls_, dos, dq_acc, dk_acc, dv_acc, bws, bws_whole
    acc = [(torch.empty((c["B"], c["Hq"], Lc, c["d"]), dtype=torch.float32, device=dev),
            torch.empty((c["B"], c["Hq"], Lc), dtype=torch.float32, device=dev),
            torch.empty((c["B"], c["Hq"], Lc, c["d"]), dtype=torch.bfloat16, device=dev))
           for _ in range(W)]
    plans = [ring_steps(r, W, True) for r in range(W)]
    # the emulated ranks are independent: each rank's folds run in order on a
    # stream of its own (its own scheduler workspace), the ranks side by side
    rstreams = [torch.cuda.Stream() for _ in range(W)]
    rws = [torch.zeros(256, dtype=torch.uint8, device=dev) for _ in range(W)]

    def step():
        main = torch.cuda.current_stream()  # the capture stream while a graph records
        for r in range(W):
            rstreams[r].wait_stream(main)
            last = max(s for s, _, kind in plans[r] if kind != "skip")
            with torch.cuda.stream(rstreams[r]):
                for s, src, kind in plans[r]:
                    fold_chunk(qs[r], ks[src], vs[src], kind, acc[r][0], acc[r][1],
                               first=(s == 0), O_out=acc[r][2] if s == last else None,
                               workspace=rws[r])
        for r in range(W):
            main.wait_stream(rstreams[r])

    # one emulated step is ten launches with Python between them: capture it in a
    # CUDA graph so that the timed region holds the kernels back to back (first
    # run outside the capture, which also sets the kernels' attributes)
    step()
    torch.cuda.synchronize()
    run, launch = step, "stream"
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        run, launch = graph.replay, "cuda graph"
    except Exception as e:  # capture refused: time the plain launches instead
        launch = f"stream (graph capture failed: {type(e).__name__})"
        torch.cuda.synchronize()
    barrier(world)
    ms = timed_loop(run, steps, warmup, torch.cuda.current_stream(), flush)
    for w_ in rws:
        st = attn.attn_read_device_status(w_)
        if st[0] != attn.ATTN_OK:
            raise RuntimeError(f"device status {st}")
    flops = 4.0 * c["d"] * causal_pairs(c["L"], c["L"], True) * c["Hq"] * c["B"]
    n_fold = sum(1 for p in plans for _, _, kind in p if kind != "skip")

    # one rank's own kernels (what each GPU of a 4-GPU ring computes, the exchange
    # aside), contiguous chunks against the zigzag layout; the slowest rank sets
    # the step time
    def graphed(fn):
        fn()
        torch.cuda.synchronize()
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            return g.replay, g
        except Exception:
            torch.cuda.synchronize()
            return fn, None

    def contiguous_rank(r):
        last = max(s for s, _, kind in plans[r] if kind != "skip")
        for s, src, kind in plans[r]:
            fold_chunk(qs[r], ks[src], vs[src], kind, acc[r][0], acc[r][1], first=(s == 0),
                       O_out=acc[r][2] if s == last else None, workspace=ws)

    zacc = [[(torch.empty_like(zq[0], dtype=torch.float32),
              torch.empty(zq[0].shape[:-1], dtype=torch.float32, device=dev),
              torch.empty_like(zq[0])) for _ in range(2)] for _ in range(W)]
    zplans = [zigzag_folds(r, W) for r in range(W)]

    def zigzag_rank(r):
        # as ring_attn_fwd_zigzag runs them: per step, the folds into the early
        # chunk's accumulator on the main stream and into the late chunk's on a
        # side stream, joined before the next step's chunk would be swapped in
        mine = zigzag_chunks(r, W)
        main = torch.cuda.current_stream()  # the capture stream while a graph records
        for s in range(W):
            rstreams[1].wait_stream(main)
            for s_, src, qi, ki, kind, first, last in zplans[r]:
                if s_ != s:
                    continue
                ch = zigzag_chunks(src, W)[ki]
                a = zacc[r][qi]
                with torch.cuda.stream(rstreams[1] if qi == 1 else main):
                    fold_chunk(zq[mine[qi]], zk[ch], zv[ch], kind, a[0], a[1], first=first,
                               O_out=a[2] if last else None, workspace=rws[qi])
            main.wait_stream(rstreams[1])

    per_rank = {}
    graphs = []
    for name, fn in (("contiguous", contiguous_rank), ("zigzag", zigzag_rank)):
        t = []
        for r in range(W):
            run_r, g = graphed(lambda r=r: fn(r))
            graphs.append(g)
            t.append(float(np.mean(timed_loop(run_r, steps, warmup, torch.cuda.current_stream(),
                                              flush))))
        per_rank[name] = t
    n_zfold = sum(len(p) for p in zplans)
    for w_ in [ws] + rws:
        st = attn.attn_read_device_status(w_)
        if st[0] != attn.ATTN_OK:
            raise RuntimeError(f"device status {st}")
    del graphs, zq, zk, zv, zacc
    # the merge kernel alone: one chunk's rows folded into an accumulator
    Op = acc[0][2]
    lp = torch.zeros_like(acc[0][1])
    merge = lambda: attn.attn_merge_partial(Op, lp, acc[0][0], acc[0][1], init=False)
    mms = timed_loop(merge, steps, warmup, torch.cuda.current_stream(), flush)
    rows = Op.numel() // c["d"]
    mbytes = rows * (4 * c["d"] * 2 + 2 * c["d"] + 12)  # acc read + write, partial, LSEs
    del qs, ks, vs, acc
    torch.cuda.empty_cache()
    return ms, flops, n_fold, mms, mbytes, wms, launch, (bms_ring, bms_whole), (per_rank, n_zfold)


def bwd_leg(steps, warmup, world, flush):
    import torch

    import exact_io_aware_46_b200 as attn

    c = BWD
    dev = torch.device("cuda")
    shp_q = (c["B"], c["Hq"], c["L"], c["d"])
    shp_k = (c["B"], c["Hkv"], c["L"], c["d"])
    q = synth.normal_bf16_device(synth.workload_seed(5, "q"), shp_q, dev)
    k = synth.normal_bf16_device(synth.workload_seed(5, "k"), shp_k, dev)
    v = synth.normal_bf16_device(synth.workload_seed(5, "v"), shp_k, dev)
    do = synth.normal_bf16_device(synth.workload_seed(5, "do"), shp_q, dev)
    O, lse = attn.attn_fwd(q, k, v, causal=True)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.zeros(attn.attn_bwd_workspace_size(c["B"], c["Hq"], c["Hkv"], c["L"], c["L"], c["d"]),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    call = lambda: attn.attn_bwd(q, k, v, O, do, lse, causal=True, dQ=dq, dK=dk, dV=dv,
                                 workspace=ws, stream=stream)
    try:
        call()
    except attn.AttnError as e:
        if e.code == attn.ATTN_ERR_UNSUPPORTED:
            return None
        raise
    barrier(world)
    ms = timed_loop(call, steps, warmup, stream, flush)
    st = attn.attn_read_device_status(ws)
    if st[0] != attn.ATTN_OK:
        raise RuntimeError(f"device status {st}")
    del q, k, v, do, O, lse, dq, dk, dv, ws
    torch.cuda.empty_cache()
    # d = 64: the tiny workload's shape and a larger causal one
    d64 = {}
    for name, (B, H, L, causal) in (("tiny B1 H2 L256 d64, no mask", (1, 2, 256, False)),
                                    ("B4 H16 L4096 d64 causal", (4, 16, 4096, True))):
        shp = (B, H, L, 64)
        q, k, v, do = (synth.normal_bf16_device(synth.workload_seed(1, t) ^ L, shp, dev)
                       for t in ("q", "k", "v", "do"))
        O, lse = attn.attn_fwd(q, k, v, causal=causal)
        ws = torch.zeros(attn.attn_bwd_workspace_size(B, H, H, L, L, 64), dtype=torch.uint8,
                         device=dev)
        call = lambda: attn.attn_bwd(q, k, v, O, do, lse, causal=causal, workspace=ws,
                                     stream=stream)
        barrier(world)
        t = timed_loop(call, steps, warmup, stream, flush)
        st = attn.attn_read_device_status(ws)
        if st[0] != attn.ATTN_OK:
            raise RuntimeError(f"device status {st}")
        d64[name] = (t, 10.0 * 64 * causal_pairs(L, L, causal) * B * H)
        del q, k, v, do, O, lse, ws
    torch.cuda.empty_cache()
    return ms, d64


# ------------------------------------------------------------------ CPU baseline (oracle)
# The fp64 oracle, as it stands, on the host cores, on the workloads' own input
# values (each sampled head drawn at its counters in the same seeded streams the
# GPU legs use).  One sampling unit per workload, shared by the cpu_baseline
# entries and by the reference arm:
#   forward (B4 H16 L4096 d128, causal): unit u = query rows i = u mod 16,
#     u mod 16 + 16, ... (256 rows) of head u // 16 (a (b, h) index): 256 rows
#     per call keep every host core busy (the oracle runs its rows in parallel);
#   long context (B1 Hq32 Hkv8 L16384 d128, causal, with and without padding):
#     whole query heads, taken in order; the rate is FLOPs of the visible pairs
#     computed over time, so the heads not run are "scaled" by the per-head rate;
#   decode (B64 Hq32 Hkv8 d128, k_len ~ U[1024, 32768]): whole sequences (all 32
#     query heads over the sequence's k_len keys), bytes = its K and V rows;
#   backward (B2 H16 L8192 d128, causal): whole heads through oracle.bwd.


def _head(workload, tensor, shape, bh):
    return synth.normal_bf16_block(synth.workload_seed(workload, tensor), shape, bh)


_FWD_HEAD = {}


def oracle_fwd_unit(u):
    """Runs forward sampling unit ``u`` on the oracle; returns (seconds, FLOPs)."""
    import oracle

    c = FWD
    L, d, H = c["L"], c["d"], c["Hq"]
    shp = (c["B"], c["Hq"], L, d)
    h = (u // 16) % (c["B"] * H)
    if h not in _FWD_HEAD:  # the 16 units of a head share its inputs (drawn untimed)
        _FWD_HEAD.clear()
        bh = (h // H, h % H)
        _FWD_HEAD[h] = tuple(_head(2, x, shp, bh)[None, None] for x in ("q", "k", "v"))
    Q, K, V = _FWD_HEAD[h]
    rows = np.arange(u % 16, L, 16, dtype=np.int32)
    t0 = time.perf_counter()
    oracle.fwd(Q, K, V, 1 / math.sqrt(d), causal=True, rows=rows)
    dt = time.perf_counter() - t0
    return dt, 4.0 * d * float(np.sum(rows + 1))


def cpu_baseline_fwd(budget_s=10.0):
    import oracle

    t, fl, u = 0.0, 0.0, 0
    while t < budget_s and u < 4096:
        dt, f = oracle_fwd_unit(u)
        t += dt
        fl += f
        u += 1
    return {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{u} units of 256 query rows (rows = u mod 16 + 16 k of one (b, h) head, "
                      f"heads in order) of the causal B4 H16 L4096 d128 forward, fp64, "
                      f"{t:.1f} s of oracle time; the reference arm times the same units"}


def cpu_baseline_long(budget_s=8.0, padded=False):
    import oracle

    c = LONG
    L, d = c["L"], c["d"]
    G = c["Hq"] // c["Hkv"]
    kl = int(long_klen()) if padded else L
    t, fl, n = 0.0, 0.0, 0
    while t < budget_s and n < c["Hq"]:
        Q = _head(3, "q", (1, c["Hq"], L, d), (0, n))[None, None]
        K = _head(3, "k", (1, c["Hkv"], L, d), (0, n // G))[None, None]
        V = _head(3, "v", (1, c["Hkv"], L, d), (0, n // G))[None, None]
        t0 = time.perf_counter()
        oracle.fwd(Q, K, V, 1 / math.sqrt(d), causal=True,
                   k_lens=np.array([kl], dtype=np.int32) if padded else None)
        t += time.perf_counter() - t0
        fl += 4.0 * d * causal_pairs(L, L, True, kl)
        n += 1
    what = f", key padding k_len = {kl}" if padded else ""
    return {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{n} of {c['Hq']} query heads (whole heads, all {L} rows) of the causal "
                      f"B1 Hq32 Hkv8 L16384 d128 forward{what}, fp64, {t:.1f} s; scaled: the "
                      f"rate of these heads stands for all {c['Hq']}"}


def cpu_baseline_decode(k_lens, budget_s=3.0):
    import oracle

    c = DEC
    d, Hq, Hkv = c["d"], c["Hq"], c["Hkv"]
    t, nbytes, n = 0.0, 0.0, 0
    while t < budget_s and n < c["B"]:
        kl = int(k_lens[n])
        Q = _head(4, "q", (c["B"], Hq, 1, d), (n,))[None]
        # the sequence's cache rows [0, k_len) of every kv head
        shp = (c["B"], Hkv, c["Lmax"], d)
        K = np.stack([synth.normal_bf16_block(synth.workload_seed(4, "k"), shp, (n, h), first=kl)
                      for h in range(Hkv)])
        V = np.stack([synth.normal_bf16_block(synth.workload_seed(4, "v"), shp, (n, h), first=kl)
                      for h in range(Hkv)])
        t0 = time.perf_counter()
        oracle.fwd(Q, K[None], V[None], 1 / math.sqrt(d))
        t += time.perf_counter() - t0
        nbytes += 2.0 * Hkv * kl * d * 2
        n += 1
    return {"value": nbytes / t / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} of {c['B']} sequences (all {Hq} query heads over the sequence's "
                      f"k_len cache rows; {nbytes / 1e9:.3f} GB of K and V) of the split-KV decode "
                      f"B64 Hq32 Hkv8 d128, fp64, {t:.1f} s; the oracle computes one query row "
                      f"per head, so one host thread works"}


def cpu_baseline_bwd(budget_s=8.0):
    import oracle

    c = BWD
    L, d = c["L"], c["d"]
    shp = (c["B"], c["Hq"], L, d)
    t, fl, n = 0.0, 0.0, 0
    while t < budget_s and n < c["B"] * c["Hq"]:
        bh = (n // c["Hq"], n % c["Hq"])
        Q, K, V, dO = (_head(5, x, shp, bh)[None, None] for x in ("q", "k", "v", "do"))
        t0 = time.perf_counter()
        oracle.bwd(Q, K, V, dO, 1 / math.sqrt(d), causal=True)
        t += time.perf_counter() - t0
        fl += 10.0 * d * causal_pairs(L, L, True)
        n += 1
    return {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{n} of {c['B'] * c['Hq']} (b, h) heads (whole heads, all {L} rows: dQ, dK, "
                      f"dV) of the causal backward B2 H16 L8192 d128, fp64, {t:.1f} s; scaled: "
                      f"the rate of these heads stands for all"}


def reference_arm(args, rank, world):
    """--impl reference: the oracle, as it stands, on this machine's host cores: each
    step is the next forward sampling unit (the units of cpu_baseline_fwd)."""
    if rank != 0:
        return
    steps, warmup = args.steps, args.warmup
    import oracle

    times, flops = [], []
    for it in range(warmup + steps):
        dt, f = oracle_fwd_unit(it)
        if it >= warmup:
            times.append(dt)
            flops.append(f)
    val = sum(flops) / sum(times) / 1e12
    sample = ("each step: one unit of 256 query rows (rows = u mod 16 + 16 k of one (b, h) head) "
              "of the causal B4 H16 L4096 d128 forward, fp64 oracle (the units of the "
              "cpu_baseline entry)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "causal prefill forward B4 H16 L4096 d128 (sampled rows)"},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------ main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--legs", default="fwd,decode,bwd,long,ring",
                    help="comma list of fwd, decode, bwd, long, ring (subsets are for profiling "
                         "runs)")
    ap.add_argument("--decode-lmax", type=int, default=DEC["Lmax"],
                    help="smaller KV cache for profiling captures (k_len ~ U[1024, Lmax])")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        reference_arm(args, rank, world)
        return

    import torch

    import exact_io_aware_46_b200 as attn

    attn.lib()  # fail loudly if the CUDA library is missing
    rank, world, local = dist_setup(args.gpus)
    pk = peaks()
    flush = torch.zeros(2 * L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    legs = args.legs.split(",")
    out = {}

    gpu_idx = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]
                  if os.environ.get("CUDA_VISIBLE_DEVICES") else local)
    DEC["Lmax"] = args.decode_lmax
    with Clocks(gpu_idx) as clk:
        if "fwd" in legs:
            (ms, ms_e2e, h2d, d2h, (vms, vflops, vtotal),
             (W, wms, wflops), fms, ms64) = fwd_leg(args.steps, args.warmup, world, flush)
        if "decode" in legs:
            dms, kv_bytes, dec_klens, (page, pms) = decode_leg(args.steps, args.warmup, world,
                                                               flush)
        if "bwd" in legs:
            bms = bwd_leg(max(3, args.steps // 2), args.warmup, world, flush)
        else:
            bms = None
        lng = long_leg(args.steps, args.warmup, world, flush) if "long" in legs else None
        ring = ring_leg(args.steps, args.warmup, world, flush) if "ring" in legs else None
    clocks = clk.summary()
    if "fwd" not in legs:  # profiling runs of single legs: report what ran
        rep = {"legs": legs, "clocks": clocks}
        if "decode" in legs:
            rep["decode_ms"] = float(np.mean(dms))
            rep["decode_GBs"] = kv_bytes / (float(np.mean(dms)) * 1e-3) / 1e9
            rep["decode_paged_GBs"] = kv_bytes / (float(np.mean(pms)) * 1e-3) / 1e9
        if bms is not None:
            rep["bwd_ms"] = float(np.mean(bms[0]))
            rep["bwd_TFLOPs"] = bwd_flops(BWD) / (float(np.mean(bms[0])) * 1e-3) / 1e12
            rep["bwd_d64"] = {n: float(np.mean(t)) for n, (t, _) in bms[1].items()}
        if lng is not None:
            for name in ("causal", "padded"):
                rep[f"long_{name}_ms"] = float(np.mean(lng[0][name]))
                rep[f"long_{name}_TFLOPs"] = lng[1][name] / (float(np.mean(lng[0][name])) * 1e-3) / 1e12
        if ring is not None:
            rep["ring_ms"] = float(np.mean(ring[0]))
            rep["ring_TFLOPs"] = ring[1] / (float(np.mean(ring[0])) * 1e-3) / 1e12
            rep["merge_GBs"] = ring[4] / (float(np.mean(ring[3])) * 1e-3) / 1e9
            rep["ring_launch"] = ring[6]
            rep["ring_per_rank_ms"] = ring[8][0]
        if rank == 0:
            print(json.dumps(rep), flush=True)
        return

    flops = fwd_flops(FWD)
    t_step = max_over_ranks(float(np.mean(ms)), world)
    t_e2e = max_over_ranks(float(np.mean(ms_e2e)), world)
    value = world * flops / (t_step * 1e-3) / 1e12
    achieved = flops / (float(np.mean(ms)) * 1e-3) / 1e12
    # one persistent forward kernel per step: timed forward, e2e, sliding-window, 8-bit,
    # d = 64 and packed-prefill loops
    launches = (args.steps + FWD["B"] * max(3, args.steps // 2) + args.steps + args.steps
                + args.steps + args.steps)

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "causal prefill forward B4 H16 L4096 d128 (bf16 in, fp32 "
                               "accumulate, O bf16 + LSE fp32)",
                   "B": FWD["B"], "H": FWD["Hq"], "L": FWD["L"], "d": FWD["d"], "causal": True,
                   "flops_per_step": flops, "flop_count": "4*d*visible pairs (causal = half)",
                   "l2": "flushed before every timed call: 256 MB written, then another 256 MB "
                         "read so that the write's dirty lines drain before the timed region",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                     "traffic": traffic_per_launch("attn_fwd_impl::fwd_kernel<128>"),
                     "peak_source": f"{pk['source']}: burst bf16",
                     "kernel": "attn_fwd_impl::fwd_kernel<128>"},
        "e2e": {"value": world * flops / (t_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": t_e2e,
                "pipeline": "one attn_fwd per sequence; its inputs copy in, the previous "
                            "sequence computes and earlier outputs copy out on three streams"},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    t_v = max_over_ranks(float(np.mean(vms)), world)
    line["varlen"] = {
        "workload": f"packed causal prefill: {VARLEN['n_seq']} sequences with lengths "
                    f"~U[{VARLEN['lo']},{VARLEN['hi']}] back to back ({vtotal} tokens), "
                    f"Hq=Hkv={VARLEN['H']}, d={VARLEN['d']}",
        "value": world * vflops / (t_v * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": t_v,
        "flops_per_step": vflops,
    }
    t_w = max_over_ranks(float(np.mean(wms)), world)
    line["sliding_window"] = {
        "workload": f"the causal prefill forward B4 H16 L4096 d128 with a sliding window of {W} "
                    f"keys (FLOPs over visible pairs)",
        "value": world * wflops / (t_w * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": t_w,
        "flops_per_step": wflops,
    }
    t_8 = max_over_ranks(float(np.mean(fms)), world)
    ach8 = flops / (float(np.mean(fms)) * 1e-3) / 1e12
    peak8 = 2.0 * pk["bf16_tflops"]
    line["fp8"] = {
        "workload": "the causal prefill forward B4 H16 L4096 d128 with E4M3 Q, K, V (the same "
                    "tensors quantised with one scale per 128-row tile), O bf16 + LSE fp32",
        "value": world * flops / (t_8 * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": t_8,
        "flops_per_step": flops, "dtype": "e4m3 (fp32 accumulate)",
        "roofline": {"bound": "tensor", "achieved": ach8, "peak": peak8, "unit": "TFLOP/s",
                     "frac": ach8 / peak8,
                     "traffic": traffic_per_launch("attn_fwd_impl::fwd_kernel<128,MODE_FP8>"),
                     "peak_source": f"{pk['source']}: burst bf16 x 2 (the nominal 8-bit:bf16 "
                                    f"dense ratio, 4.5 : 2.25 PFLOP/s)",
                     "kernel": "attn_fwd_impl::fwd_kernel<128,MODE_FP8>"},
    }
    t_64 = max_over_ranks(float(np.mean(ms64)), world)
    fl64 = flops * 64 / FWD["d"]
    line["d64"] = {
        "workload": "the causal prefill forward B4 H16 L4096 at d = 64",
        "value": world * fl64 / (t_64 * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": t_64,
        "flops_per_step": fl64,
    }
    if "decode" in legs:
        t_d = max_over_ranks(float(np.mean(dms)), world)
        gbs = kv_bytes / (float(np.mean(dms)) * 1e-3) / 1e9
        line["decode"] = {
            "workload": f"split-KV decode B64 Hq32 Hkv8 d128, cache {DEC['Lmax']}, "
                        f"k_len~U[1024,{DEC['Lmax']}]",
            "value": world * kv_bytes / (t_d * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": t_d,
            "kv_bytes_per_step": kv_bytes,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "frac_of_8TBs": gbs / 8000.0,
                         "traffic": traffic_per_launch(
                             "attn_decode_impl::tc::split_kernel<128>", kv_bytes),
                         "kernel": "attn_decode_impl::tc::split_kernel<128> + combine"},
            "gpu_launches": 4 * args.steps,
        }
        t_p = max_over_ranks(float(np.mean(pms)), world)
        line["decode"]["paged"] = {
            "workload": f"the same decode over a cache of {page}-row pages in a seeded random "
                        f"order (block table [64, {DEC['Lmax'] // page}])",
            "value": world * kv_bytes / (t_p * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": t_p,
            "page_size": page,
        }
        line["gpu_launches"] += 4 * args.steps
    if bms is not None:
        bms, bd64 = bms
        bfl = bwd_flops(BWD)
        t_b = max_over_ranks(float(np.mean(bms)), world)
        ach = bfl / (float(np.mean(bms)) * 1e-3) / 1e12
        line["bwd"] = {
            "workload": "causal backward B2 H16 L8192 d128", "value": world * bfl / (t_b * 1e-3) / 1e12,
            "unit": "TFLOP/s", "ms_per_step": t_b, "flops_per_step": bfl,
            "roofline": {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                         "traffic": traffic_per_launch("attn_bwd_impl::bwd_main_kernel<128>")},
            "d64": {name: {"ms_per_step": max_over_ranks(float(np.mean(t)), world),
                           "value": world * fl / (max_over_ranks(float(np.mean(t)), world) * 1e-3)
                           / 1e12, "unit": "TFLOP/s", "flops_per_step": fl}
                    for name, (t, fl) in bd64.items()},
        }
        line["gpu_launches"] += 3 * max(3, args.steps // 2) + 3 * 2 * max(3, args.steps // 2)
    if lng is not None:
        lms, lflops, kl = lng
        entry = {}
        for name, what in (("causal", "causal"),
                           ("padded", f"causal with key padding: k_len = {kl} (drawn from "
                                      f"U[{LONG['klo']}, {LONG['L']}])")):
            t_l = max_over_ranks(float(np.mean(lms[name])), world)
            ach = lflops[name] / (float(np.mean(lms[name])) * 1e-3) / 1e12
            entry[name] = {
                "workload": f"long-context forward B1 Hq32 Hkv8 (GQA) L16384 d128, {what}; "
                            f"FLOPs = 4 d x visible pairs",
                "value": world * lflops[name] / (t_l * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": t_l, "flops_per_step": lflops[name],
                "roofline": {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                             "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                             "traffic": traffic_per_launch("attn_fwd_impl::fwd_kernel<128>:long"),
                             "kernel": "attn_fwd_impl::fwd_kernel<128>"}}
        line["long_context"] = entry
        line["gpu_launches"] += 2 * args.steps
    if ring is not None:
        rms, rflops, n_fold, mms, mbytes, wholems, rlaunch, (rbms, wbms), (prank, n_zfold) = ring
        t_r = max_over_ranks(float(np.mean(rms)), world)
        gbs = mbytes / (float(np.mean(mms)) * 1e-3) / 1e9
        line["ring"] = {
            "workload": f"ring attention's decomposition of the causal B1 Hq32 Hkv8 L16384 d128 "
                        f"forward into {RING['world']} chunks, every rank's steps run on this "
                        f"GPU (one attn_fwd_merge per visible chunk, each rank's folds in "
                        f"order on a stream of its own, the ranks side by side; no exchange: "
                        f"one GPU)",
            "value": world * rflops / (t_r * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": t_r, "flops_per_step": rflops, "chunk_folds_per_step": n_fold,
            "launch": rlaunch,
            "per_rank": {
                "what": "each rank's own folds timed alone on this GPU (CUDA graph): the "
                        "compute of one step of a 4-GPU ring, exchange aside; the slowest "
                        "rank sets the step time; zigzag: per step the folds into the two "
                        "query chunks on two streams, as ring_attn_fwd_zigzag runs them",
                "contiguous_ms": prank["contiguous"], "contiguous_max_ms": max(prank["contiguous"]),
                "zigzag_ms": prank["zigzag"], "zigzag_max_ms": max(prank["zigzag"]),
                "zigzag_TFLOPs_per_gpu_modelled": rflops / RING["world"]
                / (max(prank["zigzag"]) * 1e-3) / 1e12},
            "backward": {
                "workload": "the same decomposition for the backward: attn_bwd per visible "
                            "chunk pair from the whole-sequence O and LSE, partial gradients "
                            "summed in fp32 with attn_accumulate (stream launches)",
                "value": world * 2.5 * rflops / (max_over_ranks(float(np.mean(rbms)), world)
                                                 * 1e-3) / 1e12,
                "unit": "TFLOP/s", "ms_per_step": max_over_ranks(float(np.mean(rbms)), world),
                "undivided_ms": float(np.mean(wbms)),
                "undivided_TFLOPs": 2.5 * rflops / (float(np.mean(wbms)) * 1e-3) / 1e12},
            "undivided_ms": float(np.mean(wholems)),
            "undivided_TFLOPs": rflops / (float(np.mean(wholems)) * 1e-3) / 1e12,
            "merge": {"kernel": "attn_merge_impl::merge_kernel", "rows": RING["B"] * RING["Hq"]
                      * (RING["L"] // RING["world"]), "ms": float(np.mean(mms)),
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"],
                                   "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                                   "traffic": traffic_per_launch("attn_merge_impl::merge_kernel")}},
        }
        # backward: per visible chunk pair 3 bwd kernels + 3 sums; the undivided call 3
        line["gpu_launches"] += (n_fold * args.steps + 2 * args.steps
                                 + (6 * n_fold + 3) * max(3, args.steps // 2)
                                 + (n_fold + n_zfold) * args.steps)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_fwd()
        if lng is not None:
            line["long_context"]["causal"]["cpu_baseline"] = cpu_baseline_long()
            line["long_context"]["padded"]["cpu_baseline"] = cpu_baseline_long(padded=True)
        if "decode" in legs:
            line["decode"]["cpu_baseline"] = cpu_baseline_decode(dec_klens)
        if bms is not None:
            line["bwd"]["cpu_baseline"] = cpu_baseline_bwd()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

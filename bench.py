#!/usr/bin/env python
"""Benchmark of attention over a head-split KV cache on B200.

Default workload: Llama-3-8B-shaped GQA decode at 128K context (32 layers,
32 query / 8 KV heads, head_dim 128, bf16, 50% retrieval KV heads, S=64 sinks +
R=256 recent), batch 1.  One step = one decode token through all 32 layers,
one fused launch per layer (``duo_decode_step``): the token's K/V is appended
(page row / ring slot) and the query attends (split-K retrieval heads,
streaming heads, log-sum-exp merge by the last split).  The chunked pre-fill
(32K prompt, 4K chunks, tcgen05 tensor cores) is measured in the same run and
reported under "prefill", and the other decode configurations under "configs"
(the same step at batch 4; Llama-2-7B-shaped MHA at 32K; 4-bit KV at 1M tokens,
one layer; a paged batch of 8 sequences of mixed lengths), each with its own
roofline and clock samples.  ``--extra`` adds one rank of a sequence-sharded
decode and pre-fill on a 4-bit cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl duo|reference]

Under torchrun every rank runs its own replica on its own GPU with distinct
sequences (weak scaling, no data-path collective); timing is the max over
ranks of CUDA-event time.  ``--impl reference`` times the fp64 CPU oracle on a
bounded sample of the same workload instead.
"""

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from head_split_kv_decode_b200 import binding as B  # noqa: E402
from head_split_kv_decode_b200 import synth  # noqa: E402

METRIC = "decode attn HBM GB/s (% of 8 TB/s) at 128K ctx; prefill attn TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- util


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def replica_batch_ids(rank, batch):
    """Sequences one rank's replica decodes: rank r owns batch rows
    [r*batch, (r+1)*batch) of the synthetic stream, so no two ranks repeat work."""
    return [rank * batch + b for b in range(batch)]


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank timings (ms) across the process group."""
    if world == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def aggregate_rate(bytes_per_rank_step, world, steps, max_ms):
    """Whole-job GB/s: the bytes every rank processed in `steps` steps over the
    slowest rank's time."""
    return world * bytes_per_rank_step * steps / (max_ms * 1e-3) / 1e9


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- decode


# DRAM traffic of one fused decode launch (dram__bytes_read.sum +
# dram__bytes_write.sum) from an ncu capture of one layer of a workload, and
# that launch's algorithmic bytes, per cache type: bf16 from the 128K batch-1
# GQA workload (4 retrieval + 4 streaming KV heads, context 131076); int4 from
# the 1M GQA workload (2 retrieval + 6 streaming KV heads).  The ratio scales
# to the benchmark's launches; it is reported only while the kernel's sources
# hash as they did when the counters were taken (otherwise traffic is null).
DECODE_TRAFFIC_SOURCES = ("decode_mma.cu", "decode_finish.cuh", "common.cuh", "kernels.h",
                          "quant_int4.cuh")
DECODE_TRAFFIC = {
    # fused step, Llama-3-8B-shaped GQA, 128K, batch 1, one layer
    "bf16": {"sha256": "72fc0ba15249c58de89e634ce90f414aba1fb1a82678080280855fd71d386b41",
             "dram_bytes": 269190144 + 3686656, "algorithmic_bytes": 269120512},
    # 4-bit fused step, Llama-3-8B-shaped GQA, 1M, batch 1, one layer
    "int4": {"sha256": "72fc0ba15249c58de89e634ce90f414aba1fb1a82678080280855fd71d386b41",
             "dram_bytes": 285927680 + 3641088, "algorithmic_bytes": 285495496},
}


def decode_traffic(kv_dtype, bytes_per_launch):
    """ncu DRAM bytes per launch scaled to this launch size, or None if the
    kernel changed since the capture (or none was taken)."""
    ref = DECODE_TRAFFIC.get(kv_dtype)
    if not ref or ref["sha256"] is None:
        return None
    h = hashlib.sha256()
    for name in DECODE_TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "head_split_kv_decode_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != ref["sha256"]:
        return None
    return ref["dram_bytes"] / ref["algorithmic_bytes"] * bytes_per_launch


def hbm_roofline(achieved_gbs, avg_launch_ms, bytes_per_launch, kernel, peaks, peak_kind,
                 traffic=None):
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": achieved_gbs, "peak": peak, "unit": "GB/s",
            "frac": achieved_gbs / peak, "traffic": traffic, "kernel": kernel,
            "avg_launch_ms": avg_launch_ms, "bytes_per_launch": bytes_per_launch,
            "peak_kind": peak_kind}


def decode_bytes_per_layer(w, batch, n, n_ret, n_str):
    """Algorithmic bytes of one decode-attention launch (visible KV + Q + O)."""
    per_tok = 4 * w.head_dim if w.kv_dtype != "int4" else 2 * (w.head_dim // 2 + 4)
    io = 2 if w.kv_dtype != "f32" else 4
    kv = batch * (n_ret * n + n_str * min(n, w.S + w.R)) * per_tok
    qo = 2 * batch * w.n_q_heads * w.head_dim * io
    return kv + qo


def append_bytes(w, batch):
    io = 2 if w.kv_dtype != "f32" else 4
    return 2 * batch * w.n_kv_heads * w.head_dim * io


def fill_cache(cache, w, mask, b_ids, chunk=8192):
    """Pre-fill every layer with the workload's context through duo_append_kv."""
    dt = synth.io_dtype(w)
    for layer in range(w.layers):
        for p0 in range(0, w.context, chunk):
            pos = range(p0, min(w.context, p0 + chunk))
            k = synth.history(w, layer, "k", b_ids, pos, device="cuda", mask_row=mask[layer]).to(dt)
            v = synth.history(w, layer, "v", b_ids, pos, device="cuda", mask_row=mask[layer]).to(dt)
            cache.append(layer, k.contiguous(), v.contiguous())
        torch.cuda.synchronize()


def decode_inputs(w, mask, b_ids, first, count):
    """Per layer: q [count, B, Hq, d], k/v [count, B, 1, Hkv, d] for decode steps."""
    dt = synth.io_dtype(w)
    qs, ks, vs = [], [], []
    pos = range(first, first + count)
    for layer in range(w.layers):
        q = synth.queries(w, layer, b_ids, pos, device="cuda").to(dt)        # [B, T, Hq, d]
        k = synth.history(w, layer, "k", b_ids, pos, device="cuda", mask_row=mask[layer]).to(dt)
        v = synth.history(w, layer, "v", b_ids, pos, device="cuda", mask_row=mask[layer]).to(dt)
        qs.append(q.permute(1, 0, 2, 3).contiguous())
        ks.append(k.permute(1, 0, 2, 3).unsqueeze(2).contiguous())
        vs.append(v.permute(1, 0, 2, 3).unsqueeze(2).contiguous())
    return qs, ks, vs


def run_decode(args, w, batch, rank, world, peaks, peak_kind, clock_gpu):
    from head_split_kv_decode_b200.cache import DuoCache

    K, W = args.steps, args.warmup
    mask = synth.workload_mask(w)
    b_ids = replica_batch_ids(rank, batch)
    total_steps = W + 2 * K
    cache = DuoCache(w.layers, batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.kv_dtype,
                     w.context + total_steps + 1, mask, w.S, w.R)
    t0 = time.time()
    fill_cache(cache, w, mask, b_ids)
    fill_s = time.time() - t0
    qs, ks, vs = decode_inputs(w, mask, b_ids, w.context, total_steps)
    outs = [torch.empty(batch, w.n_q_heads, w.head_dim, dtype=synth.io_dtype(w), device="cuda")
            for _ in range(w.layers)]
    lib = B.lib()
    h = cache.handle
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    ws, wsb = cache.ws_ptr, cache.ws_bytes
    n_ret = [int(mask[layer].sum()) for layer in range(w.layers)]
    n_str = [w.n_kv_heads - r for r in n_ret]
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K * w.layers)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K * w.layers)]

    # bf16 and 4-bit head_dim-128 caches decode each layer in one fused launch
    # (duo_decode_step: append + attend); other caches append, then attend.
    fused = w.kv_dtype in ("bf16", "int4") and w.head_dim == 128

    # The fused path's timed region holds nothing but its decode launches, back
    # to back (programmatic dependent launch overlaps each one's set-up with
    # the previous one's tail), so its average launch duration is the region's
    # time over the launch count; an event between two launches would break
    # that overlap.  The unfused path brackets each attention launch with
    # events to separate it from the append before it.
    def step(s, timed_idx=None):
        for layer in range(w.layers):
            kp, vp = ks[layer][s].data_ptr(), vs[layer][s].data_ptr()
            if not fused:
                st = lib.duo_append_kv(h, layer, kp, vp, 1, sh)
                if st:
                    raise B.DuoError(st, "duo_append_kv")
            if timed_idx is not None and not fused:
                ev_s[timed_idx * w.layers + layer].record(stream)
            if fused:
                st = lib.duo_decode_step(h, layer, qs[layer][s].data_ptr(), kp, vp,
                                         outs[layer].data_ptr(), 0.0, ws, wsb, sh)
            else:
                st = lib.duo_decode_attn(h, layer, qs[layer][s].data_ptr(), outs[layer].data_ptr(),
                                         0.0, ws, wsb, sh)
            if st:
                raise B.DuoError(st, "duo_decode_step" if fused else "duo_decode_attn")
            if timed_idx is not None and not fused:
                ev_e[timed_idx * w.layers + layer].record(stream)

    for s in range(W):
        step(s)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    n_first = cache.seq_len(0) + 1
    splits = cache.decode_splits(0)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(clock_gpu) as clk:
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(K):
            step(W + i, timed_idx=i)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end)
    if fused:
        kern_ms = [ms / (K * w.layers)] * (K * w.layers)
    else:
        kern_ms = [a.elapsed_time(b) for a, b in zip(ev_s, ev_e)]
    if B.duo_poll_device_error() != 0:
        raise RuntimeError("a bounded device wait gave up during the benchmark")

    step_bytes = 0
    launch_bytes = []
    for i in range(K):
        n = n_first + i
        for layer in range(w.layers):
            lb = decode_bytes_per_layer(w, batch, n, n_ret[layer], n_str[layer])
            # the fused launch also reads the new K/V and writes them to the cache
            launch_bytes.append(lb + (append_bytes(w, batch) if fused else 0))
            step_bytes += lb + append_bytes(w, batch)
    step_bytes /= K

    # ---- end to end through the public API: each step copies that token's
    # q/k/v for every layer in from one pinned host buffer, runs the layers,
    # and copies every layer's output back to pinned host memory.
    nq, nk = qs[0][0].numel(), ks[0][0].numel()
    per_layer = nq + 2 * nk
    host_in = torch.empty((K, w.layers, per_layer), dtype=qs[0].dtype).pin_memory()
    for layer in range(w.layers):
        host_in[:, layer, :nq] = qs[layer][W + K:W + 2 * K].reshape(K, nq).cpu()
        host_in[:, layer, nq:nq + nk] = ks[layer][W + K:W + 2 * K].reshape(K, nk).cpu()
        host_in[:, layer, nq + nk:] = vs[layer][W + K:W + 2 * K].reshape(K, nk).cpu()
    dev_in = torch.empty((w.layers, per_layer), dtype=host_in.dtype, device="cuda")
    dev_out = torch.empty((w.layers,) + tuple(outs[0].shape), dtype=outs[0].dtype, device="cuda")
    host_out = torch.empty((K,) + tuple(dev_out.shape), dtype=dev_out.dtype).pin_memory()
    esz = host_in.element_size()
    qp = [dev_in[layer].data_ptr() for layer in range(w.layers)]
    kp = [p + nq * esz for p in qp]
    vp = [p + (nq + nk) * esz for p in qp]
    op = [dev_out[layer].data_ptr() for layer in range(w.layers)]
    h2d = host_in[0].numel() * esz
    d2h = dev_out.numel() * dev_out.element_size()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        dev_in.copy_(host_in[i], non_blocking=True)
        for layer in range(w.layers):
            if fused:
                B.duo_decode_step(h, layer, qp[layer], kp[layer], vp[layer], op[layer], 0.0, ws,
                                  wsb, sh)
            else:
                B.duo_append_kv(h, layer, kp[layer], vp[layer], 1, sh)
                B.duo_decode_attn(h, layer, qp[layer], op[layer], 0.0, ws, wsb, sh)
        host_out[i].copy_(dev_out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, "cuda")

    avg_kern_ms = sum(kern_ms) / len(kern_ms)
    avg_launch_bytes = sum(launch_bytes) / len(launch_bytes)
    achieved = avg_launch_bytes / (avg_kern_ms * 1e-3) / 1e9
    res = {
        "ms_per_step": ms / K,
        "value": aggregate_rate(step_bytes, world, K, ms),
        "e2e_value": aggregate_rate(step_bytes, world, K, e2e_ms),
        "h2d": h2d, "d2h": d2h,
        "step_bytes": step_bytes,
        "kernel": {"name": ("decode_mma_kernel %s (fused append + attention)" if fused else
                            "decode_mma_kernel %s") % w.kv_dtype,
                   "avg_ms": avg_kern_ms, "launches": len(kern_ms),
                   "bytes_per_launch": avg_launch_bytes, "achieved_gbs": achieved},
        "splits": splits,
        "fill_s": fill_s,
        "clocks": clk.summary(),
        "context": n_first,
        "gpu_launches": K * w.layers * (1 if fused else 2),
        "fused": fused,
        "roofline": hbm_roofline(achieved, avg_kern_ms, avg_launch_bytes,
                                 ("decode_mma_kernel %s (fused append + attention)" if fused else
                                  "decode_mma_kernel %s") % w.kv_dtype, peaks, peak_kind,
                                 decode_traffic(w.kv_dtype, avg_launch_bytes) if fused else None),
    }
    del cache
    torch.cuda.empty_cache()
    return res


def run_paged_mixed(args, w, rank, world, peaks, peak_kind, clock_gpu):
    """Decode of a mixed-length batch on the paged layout: every row (one
    sequence, w.row_lengths tokens of context) takes one fused step per layer,
    all rows in one launch, each at its own position."""
    from head_split_kv_decode_b200.cache import DuoCache

    K, Wm = min(args.steps, w.steps), args.warmup
    lens = list(w.row_lengths)
    B_ = len(lens)
    mask = synth.workload_mask(w)
    b_ids = replica_batch_ids(rank, B_)  # distinct sequences on every rank
    total_steps = Wm + K
    pool = sum((n + total_steps + 1 + B.PAGE_TOKENS - 1) // B.PAGE_TOKENS for n in lens)
    cache = DuoCache(w.layers, B_, w.n_q_heads, w.n_kv_heads, w.head_dim, "bf16",
                     max(lens) + total_steps + 1, mask, w.S, w.R, pool_blocks=pool)
    dt = torch.bfloat16
    t0 = time.time()
    for layer in range(w.layers):
        for r, n in enumerate(lens):
            for p0 in range(0, n, 16384):
                pos = range(p0, min(n, p0 + 16384))
                k = synth.history(w, layer, "k", [b_ids[r]], pos, device="cuda", mask_row=mask[layer])
                v = synth.history(w, layer, "v", [b_ids[r]], pos, device="cuda", mask_row=mask[layer])
                cache.append_rows(layer, [r], k.to(dt).contiguous(), v.to(dt).contiguous())
        torch.cuda.synchronize()
    fill_s = time.time() - t0
    # per layer and step: q [B, Hq, d], k/v [B, Hkv, d], row r at position lens[r] + step
    qs, ks, vs = [], [], []
    for layer in range(w.layers):
        qr, kr, vr = [], [], []
        for r, n in enumerate(lens):
            pos = range(n, n + total_steps)
            qr.append(synth.queries(w, layer, [b_ids[r]], pos, device="cuda")[0])
            kr.append(synth.history(w, layer, "k", [b_ids[r]], pos, device="cuda", mask_row=mask[layer])[0])
            vr.append(synth.history(w, layer, "v", [b_ids[r]], pos, device="cuda", mask_row=mask[layer])[0])
        qs.append(torch.stack(qr, 1).to(dt).contiguous())  # [steps, B, Hq, d]
        ks.append(torch.stack(kr, 1).to(dt).contiguous())
        vs.append(torch.stack(vr, 1).to(dt).contiguous())
    out = torch.empty(B_, w.n_q_heads, w.head_dim, dtype=dt, device="cuda")
    lib = B.lib()
    h, sh = cache.handle, torch.cuda.current_stream().cuda_stream
    ws, wsb = cache.ws_ptr, cache.ws_bytes

    def step(s):
        for layer in range(w.layers):
            st = lib.duo_decode_step(h, layer, qs[layer][s].data_ptr(), ks[layer][s].data_ptr(),
                                     vs[layer][s].data_ptr(), out.data_ptr(), 0.0, ws, wsb, sh)
            if st:
                raise B.DuoError(st, "duo_decode_step")

    for s in range(Wm):
        step(s)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(clock_gpu) as clk:
        torch.cuda.synchronize()
        e0.record()
        for i in range(K):
            step(Wm + i)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks([ms], world, "cuda")[0]
    if B.duo_poll_device_error() != 0:
        raise RuntimeError("a bounded device wait gave up during the benchmark")
    n_ret = [int(mask[layer].sum()) for layer in range(w.layers)]
    step_bytes = 0
    for i in range(K):
        for layer in range(w.layers):
            for n in lens:
                step_bytes += decode_bytes_per_layer(w, 1, n + Wm + i + 1, n_ret[layer],
                                                     w.n_kv_heads - n_ret[layer])
                step_bytes += append_bytes(w, 1)
    step_bytes /= K
    launches = K * w.layers
    res = {"workload": w.name, "row_lengths": lens, "pool_blocks": pool,
           "value": aggregate_rate(step_bytes, world, K, ms), "unit": "GB/s",
           "ms_per_step": ms / K, "kernel_avg_launch_ms": ms / launches,
           "bytes_per_launch": step_bytes / w.layers, "gpu_launches": launches,
           "decode_splits": cache.decode_splits(0), "fill_s": fill_s}
    res["kernel_achieved_gbs"] = res["bytes_per_launch"] / (res["kernel_avg_launch_ms"] * 1e-3) / 1e9
    res["frac"] = res["kernel_achieved_gbs"] / peaks["hbm_gbs"]
    res["roofline"] = hbm_roofline(res["kernel_achieved_gbs"], res["kernel_avg_launch_ms"],
                                   res["bytes_per_launch"],
                                   "decode_mma_kernel bf16 paged (fused append + attention)",
                                   peaks, peak_kind)
    res["clocks"] = clk.summary()
    del cache
    torch.cuda.empty_cache()
    return res


def run_shard_rank(args, w, world_emulated, rank, peaks):
    """One rank's share of a sequence-sharded decode: the sequence of
    w.context * world_emulated tokens is split into world_emulated shards; this
    measures rank 0 (the first w.context positions, and the streaming heads) —
    per layer one partial decode and the merge of world_emulated partials.  The
    exchange of the partials between GPUs is not part of it."""
    from head_split_kv_decode_b200.cache import DuoCache, merge_partials
    from head_split_kv_decode_b200 import shard

    K_, Wm = min(args.steps, 16), args.warmup
    total = w.context * world_emulated
    lo, hi = shard.shard_ranges(total, world_emulated)[0]
    mask = synth.workload_mask(w)
    dt = torch.bfloat16
    cache = DuoCache(w.layers, 1, w.n_q_heads, w.n_kv_heads, w.head_dim, "bf16", hi - lo, mask,
                     w.S, w.R)
    cache.set_retrieval_shard(lo, hi)
    zeros = torch.zeros(1, 65536, w.n_kv_heads, w.head_dim, dtype=dt, device="cuda")
    b_ids = [rank]
    for layer in range(w.layers):
        for p0 in range(0, hi, 16384):  # this shard's positions: real values
            pos = range(p0, p0 + 16384)
            k = synth.history(w, layer, "k", b_ids, pos, device="cuda", mask_row=mask[layer])
            v = synth.history(w, layer, "v", b_ids, pos, device="cuda", mask_row=mask[layer])
            cache.append(layer, k.to(dt).contiguous(), v.to(dt).contiguous())
        for p0 in range(hi, total, 65536):  # the other shards' positions only pass through
            cache.append(layer, zeros, zeros)  # the streaming window
        torch.cuda.synchronize()
    q = [synth.queries(w, layer, b_ids, [total - 1], device="cuda")[:, 0].to(dt).contiguous()
         for layer in range(w.layers)]
    o_all = torch.full((world_emulated, 1, w.n_q_heads, w.head_dim), 0.0, device="cuda")
    lse_all = torch.full((world_emulated, 1, w.n_q_heads), -float("inf"), device="cuda")
    out = torch.empty(1, w.n_q_heads, w.head_dim, dtype=dt, device="cuda")

    def step():
        for layer in range(w.layers):
            cache.decode_partial(layer, q[layer], o_all[0], lse_all[0], owns_streaming=True)
            merge_partials(o_all, lse_all, out)

    for _ in range(Wm):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K_):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / K_
    n_ret = [int(mask[layer].sum()) for layer in range(w.layers)]
    step_bytes = sum(decode_bytes_per_layer(w, 1, hi - lo, n_ret[l], 0) +
                     (w.n_kv_heads - n_ret[l]) * min(total, w.S + w.R) * 4 * w.head_dim * 2
                     for l in range(w.layers))
    res = {"workload": "%s: rank 0 of %d shards of a %d-token sequence (partial decode + merge of "
                       "%d partials per layer; the exchange between GPUs not included)"
                       % (w.name, world_emulated, total, world_emulated),
           "value": step_bytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
           "ms_per_layer": ms / w.layers, "gpu_launches": 2 * w.layers,
           "frac": step_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del cache
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- prefill


def prefill_tile_flops(w, C, c0, retrieval, tile=128):
    """Tile-counted flops of one chunk for one query head (4*d per visited
    128x128 tile element pair), matching the kernel's tile visits."""
    n_q_tiles = C // tile
    total = 0
    for qt in range(n_q_tiles):
        q_lo = c0 + qt * tile
        q_hi = q_lo + tile - 1
        if retrieval:
            keys = q_hi + 1
            total += math.ceil(keys / tile) * tile
        else:
            vis = set()
            for kt in range(math.ceil((q_hi + 1) / tile)):
                k_lo, k_hi = kt * tile, kt * tile + tile - 1
                if k_lo < w.S or k_hi > q_lo - w.R:
                    vis.add(kt)
            total += len(vis) * tile
    return 4 * w.head_dim * tile * total


def prefill_exact_flops(w, C, c0, retrieval):
    total = 0
    for i in range(c0, c0 + C):
        total += (i + 1) if retrieval else min(i + 1, w.S + max(0, min(w.R, i + 1 - w.S)))
    return 4 * w.head_dim * total


def run_prefill(args, w, rank, world, peaks, kv_dtype="bf16"):
    """One layer's prompt in chunks: attend, then append.  kv_dtype "int4"
    keeps the history in a 4-bit cache; each timed call then also expands the
    history it reads to bf16 (the launch before the tensor-core pass)."""
    from head_split_kv_decode_b200.cache import DuoCache

    mask = synth.workload_mask(w)[:1]
    C = w.chunk
    n_chunks = w.context // C
    cache = DuoCache(1, 1, w.n_q_heads, w.n_kv_heads, w.head_dim, kv_dtype, w.context, mask, w.S,
                     w.R)
    pws, pwsb = cache._prefill_ws()
    dt = torch.bfloat16
    b_ids = [rank]
    pos = range(w.context)
    K = synth.history(w, 0, "k", b_ids, pos, device="cuda").to(dt)
    V = synth.history(w, 0, "v", b_ids, pos, device="cuda").to(dt)
    Q = synth.queries(w, 0, b_ids, pos, device="cuda").to(dt)
    chunks = [(Q[:, c * C:(c + 1) * C].contiguous(), K[:, c * C:(c + 1) * C].contiguous(),
               V[:, c * C:(c + 1) * C].contiguous()) for c in range(n_chunks)]
    out = torch.empty_like(chunks[0][0])
    lib = B.lib()
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def one_prompt(events=None):
        cache.reset()
        for c, (q, k, v) in enumerate(chunks):
            if events is not None:
                events[c][0].record(stream)
            st = lib.duo_prefill_attn(cache.handle, 0, q.data_ptr(), k.data_ptr(), v.data_ptr(), C,
                                      out.data_ptr(), 0.0, pws, pwsb, sh)
            if st:
                raise B.DuoError(st, "duo_prefill_attn")
            if events is not None:
                events[c][1].record(stream)
            st = lib.duo_append_kv(cache.handle, 0, k.data_ptr(), v.data_ptr(), C, sh)
            if st:
                raise B.DuoError(st, "duo_append_kv")

    for _ in range(max(1, args.warmup)):
        one_prompt()
    torch.cuda.synchronize()
    reps = max(1, min(args.steps, 8))
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_chunks)]
           for _ in range(reps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for r in range(reps):
        one_prompt(evs[r])
    e1.record(stream)
    torch.cuda.synchronize()
    if B.duo_poll_device_error() != 0:
        raise RuntimeError("a bounded device wait gave up during pre-fill")
    attn_ms = sum(a.elapsed_time(b) for rep in evs for a, b in rep) / reps
    n_ret = int(mask[0].sum())
    G = w.group
    tile_fl = exact_fl = 0
    for c in range(n_chunks):
        for kvh in range(w.n_kv_heads):
            ret = bool(mask[0, kvh])
            tile_fl += G * prefill_tile_flops(w, C, c * C, ret)
            exact_fl += G * prefill_exact_flops(w, C, c * C, ret)
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tflops = tile_fl / (attn_ms * 1e-3) / 1e12
    del cache
    torch.cuda.empty_cache()
    return {
        "metric": "prefill attn TFLOP/s (tile-counted, 128x128 tiles)",
        "kv_dtype": kv_dtype,
        "value": tflops,
        "unit": "TFLOP/s",
        "exact_tflops": exact_fl / (attn_ms * 1e-3) / 1e12,
        "ms_per_layer": attn_ms,
        "ms_per_prompt_incl_append": e0.elapsed_time(e1) / reps,
        "workload": w.name,
        "retrieval_kv_heads": n_ret,
        "tile_flops_per_layer": tile_fl,
        "exact_flops_per_layer": exact_fl,
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "traffic": None},
        "gpu_launches": reps * n_chunks * (3 if kv_dtype == "int4" else 2),
    }


# --------------------------------------------------------------------------- oracle


def oracle_decode_sample(w, batch, n, mask_row):
    """Inputs for the CPU oracle: one decode step of layer 0 at context n for one
    retrieval and one streaming KV head of batch row 0 (generated untimed)."""
    ret = [h for h in range(w.n_kv_heads) if mask_row[h]][:1]
    strm = [h for h in range(w.n_kv_heads) if not mask_row[h]][:1]
    heads = ret + strm
    dt = synth.io_dtype(w)
    k = synth.history(w, 0, "k", [0], range(n), heads=heads, mask_row=mask_row).to(dt).double().numpy()
    v = synth.history(w, 0, "v", [0], range(n), heads=heads, mask_row=mask_row).to(dt).double().numpy()
    qh = [hq for h in heads for hq in range(h * w.group, (h + 1) * w.group)]
    q = synth.queries(w, 0, [0], [n - 1], heads=qh).to(dt).double().numpy()[:, 0]
    sub_mask = [1] * len(ret) + [0] * len(strm)
    per_tok = 4 * w.head_dim
    nbytes = (len(ret) * n + len(strm) * min(n, w.S + w.R)) * per_tok + \
        2 * len(qh) * w.head_dim * 2
    return (q, k, v, sub_mask), nbytes, "layer 0, one decode step at context %d, batch row 0, " \
        "KV heads %s (retrieval) + %s (streaming)" % (n, ret, strm)


def time_oracle(sample, w):
    from oracle import attention as OA
    q, k, v, sub_mask = sample
    t = time.perf_counter()
    OA.decode_reference(q, k, v, sub_mask, w.S, w.R)
    return time.perf_counter() - t


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline(w, batch):
    mask = synth.workload_mask(w)
    sample, nbytes, desc = oracle_decode_sample(w, batch, w.context + 1, mask[0])
    reps, secs = 0, 0.0
    while secs < 10.0 or reps < 2:
        secs += time_oracle(sample, w)
        reps += 1
    return {"value": reps * nbytes / secs / 1e9, "unit": "GB/s", "cores": cpu_cores(),
            "kind": "oracle",
            "sample": desc + "; numpy fp64, repeated %d times (%.1f s)" % (reps, secs)}


def reference_arm(args, w, batch):
    world, rank, _ = dist_info()
    if rank != 0:
        return 0
    mask = synth.workload_mask(w)
    sample, nbytes, desc = oracle_decode_sample(w, batch, w.context + 1, mask[0])
    for _ in range(args.warmup):
        time_oracle(sample, w)
    secs = [time_oracle(sample, w) for _ in range(args.steps)]
    total = sum(secs)
    value = nbytes * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, batch, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, batch, n_gpus):
    return {"workload": w.name, "batch": batch, "context": w.context, "layers": w.layers,
            "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "S": w.S, "R": w.R, "retrieval_frac": w.retrieval_frac,
            "l2": "inputs larger than L2 (every step streams each layer's KV cache from HBM)",
            "parallelism": "replicas x%d" % n_gpus}


# --------------------------------------------------------------------------- main


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["duo", "reference"], default="duo")
    ap.add_argument("--workload", default="llama3_8b_gqa_128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--layers", type=int, default=0,
                    help="decode only the first N layers of the workload (a small case for "
                         "profiling; 0 = all layers)")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--extra", action="store_true",
                    help="also time one rank of a sequence-sharded decode and pre-fill on a "
                         "4-bit cache")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the headline workload (and pre-fill), not the other "
                         "decode configurations")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        w = dataclasses.replace(w, layers=min(args.layers, w.layers))
    if args.impl == "reference":
        return reference_arm(args, w, args.batch)

    world, rank, local = dist_info()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    B.lib()
    peaks, peak_kind = load_peaks()
    clock_gpu = local
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x for x in vis.split(",") if x.strip()]
        if local < len(ids) and ids[local].strip().isdigit():
            clock_gpu = int(ids[local])

    res = run_decode(args, w, args.batch, rank, world, peaks, peak_kind, clock_gpu)

    def decode_entry(wx, rx, note=None):
        e = {"workload": wx.name, "batch": rx.get("batch", 1), "context": rx["context"],
             "layers": wx.layers, "value": rx["value"], "unit": "GB/s",
             "ms_per_step": rx["ms_per_step"], "roofline": rx["roofline"],
             "clocks": rx["clocks"], "decode_splits": rx["splits"],
             "gpu_launches": rx["gpu_launches"]}
        if note:
            e["note"] = note
        return e

    # The other decode configurations, each timed like the headline (the
    # same step function, its own clock samples and roofline).
    configs = {}
    if not args.headline_only and not args.layers:
        r4 = run_decode(args, w, 4, rank, world, peaks, peak_kind, clock_gpu)
        r4["batch"] = 4
        configs["llama3_8b_gqa_128k_b4"] = decode_entry(w, r4)
        wm = synth.WORKLOADS["llama2_7b_mha_32k"]
        configs["llama2_7b_mha_32k"] = decode_entry(
            wm, run_decode(args, wm, 1, rank, world, peaks, peak_kind, clock_gpu))
        wq = dataclasses.replace(synth.WORKLOADS["llama3_8b_gqa_int4_1m"], layers=1)
        configs["llama3_8b_gqa_int4_1m"] = decode_entry(
            wq, run_decode(args, wq, 1, rank, world, peaks, peak_kind, clock_gpu),
            note="one layer of the 32-layer workload (layer 0's head mask), its 1M-token "
                 "4-bit cache re-read every step (285 MB per launch, larger than L2); "
                 "a 32-layer step is 32 such launches")
        configs["llama3_8b_gqa_paged_mixed"] = run_paged_mixed(
            args, synth.WORKLOADS["llama3_8b_gqa_paged_mixed"], rank, world, peaks, peak_kind,
            clock_gpu)
    extra = {}
    if args.extra:
        extra["sequence_sharded_1m_rank0_of_8"] = run_shard_rank(args, w, 8, rank, peaks)
        pq = run_prefill(args, synth.WORKLOADS["llama3_8b_gqa_prefill_32k"], rank, world, peaks,
                         kv_dtype="int4")
        extra["prefill_int4_cache"] = {k: pq[k] for k in ("value", "unit", "exact_tflops",
                                                            "ms_per_layer", "kv_dtype")}
        extra["prefill_int4_cache"]["frac"] = pq["roofline"]["frac"]
    prefill = None
    if not args.no_prefill:
        try:
            prefill = run_prefill(args, synth.WORKLOADS["llama3_8b_gqa_prefill_32k"], rank, world, peaks)
            prefill["roofline"]["peak_kind"] = peak_kind
        except B.DuoError as e:
            prefill = {"unavailable": str(e)}

    if world > 1:
        torch.distributed.barrier()
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return 0
    kern = res["kernel"]
    line = {
        "metric": METRIC,
        "value": res["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(w, args.batch, world),
        "pct_of_8tbs": 100.0 * res["value"] / world / 8000.0,
        "roofline": res["roofline"],
        "e2e": {"value": res["e2e_value"], "unit": "GB/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": res["gpu_launches"] + (prefill or {}).get("gpu_launches", 0),
        "clocks": res["clocks"],
        "decode_splits": res["splits"],
        "prefill": prefill,
        "configs": configs,
    }
    line.update(extra)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.batch)
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

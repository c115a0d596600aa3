"""Throughput of the paged-attention hot path on B200.

One step = one decode iteration of the Llama-3-8B-shaped GQA batch (256
sequences, 32 q / 8 kv heads, head_dim 128, bf16, 16-token blocks, lengths
uniform in [128, 4096], shuffled physical blocks): slot mapping of the new
token of every sequence, the scatter of its K/V and split-KV paged decode in
one launch (pa_append_decode), then the log-sum-exp combine — all through
libpa.so's C ABI.

Printed (rank 0, one JSON line): the decode KV bandwidth over the whole step
(GB/s of algorithmic K/V bytes), decode tokens/s, the roofline of the decode launch,
the prefill-chunk TFLOP/s of the 8 x 512-token chunk workload, an end-to-end
figure through the C ABI with host buffers, clocks seen during the timed
region, the CPU oracle as a baseline, and (single GPU) secondary figures: the
same decode step over an FP8 pool, a mixed batch (decode rows and prefill
chunks in one launch, against the same work as two calls), copy-on-write
block copies and swap bandwidth to / from pinned host memory.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 launch with torch.distributed.run; every rank decodes its own batch
(weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "paged decode KV GB/s (% of HBM peak) and decode tokens/s; prefill-chunk TFLOP/s"
WORKLOAD = ("llama3_8b_gqa_decode: 256 seqs, 32 q / 8 kv heads, head_dim 128, bf16, "
            "block_size 16, lengths U[128,4096], shuffled block tables, +1 appended token/seq")
PROFILE = os.path.join(ROOT, "profiles", "decode_kernel_llama3_8b_gqa_decode.md")
KERNEL_SOURCES = [os.path.join(ROOT, "paged_kv_cache_397_b200", "csrc", f)
                  for f in ("decode.cuh", "ptx.cuh")]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# per-launch CUDA events around every EVENT_EVERY-th step of the timed region
EVENT_EVERY = 8


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kv_bytes_per_launch: float):
    """DRAM bytes per decode launch from the committed ncu summary, scaled to
    this launch by K/V bytes, or None if the kernel changed since the capture."""
    if not os.path.exists(PROFILE):
        return None
    text = open(PROFILE).read()
    m_hash = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_ratio = re.search(r"dram_bytes_per_algorithmic_byte:\s*([0-9.]+)", text)
    if not m_hash or not m_ratio or m_hash.group(1) != kernel_hash():
        return None
    return float(m_ratio.group(1)) * kv_bytes_per_launch


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        busy = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def setup_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time (all ranks call this in the same order)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank_step: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job GB/s: the bytes every rank processed over the slowest rank's time."""
    return world * bytes_per_rank_step * steps / (ms_max * 1e-3) / 1e9


class DecodeStep:
    """Device-resident inputs of one decode step and the C-ABI calls it makes.

    The per-step inputs (query, new K/V, block tables, context lengths,
    lengths) live in one staging buffer, each segment 256-byte aligned, so
    the end-to-end leg moves them with a single host-to-device copy from one
    pinned host buffer of the same layout; the device tensors are views.
    """

    def __init__(self, w, dev):
        import paged_kv_cache_397_b200 as pa
        self.pa = pa
        self.w = w
        self.dev = dev
        self.kc = w.key_cache.to(dev)
        self.vc = w.value_cache.to(dev)
        inputs = [w.query, w.new_key, w.new_value, w.block_tables, w.context_lens,
                  (w.context_lens + 1).to(torch.int32)]
        offs, total = [], 0
        for t in inputs:
            offs.append(total)
            total += -(-t.numel() * t.element_size() // 256) * 256
        self.h_stage = torch.zeros(total, dtype=torch.uint8).pin_memory()
        for t, o in zip(inputs, offs):
            n = t.numel() * t.element_size()
            self.h_stage[o:o + n].copy_(t.contiguous().view(-1).view(torch.uint8))
        self.d_stage = self.h_stage.to(dev)
        self._layout = [(o, t.numel() * t.element_size(), t.dtype, t.shape)
                        for t, o in zip(inputs, offs)]
        self.q, self.nk, self.nv, self.bt, self.ctx, self.lens = self._views(self.d_stage)
        self.out = torch.empty_like(self.q)
        self.max_len = int(w.context_lens.max()) + 1
        need = pa.pa_decode_workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads,
                                           w.head_dim, w.block_size, self.max_len)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        self.num_parts = math.ceil(self.max_len / pa.pa_decode_partition_tokens(
            w.num_seqs, w.num_kv_heads, w.block_size, self.max_len))
        self.launches_per_step = 1 + (1 if self.num_parts > 1 else 0)  # decode + combine
        total_tokens = int(self.lens.sum())
        self.kv_bytes = 2 * w.num_kv_heads * w.head_dim * 2 * total_tokens  # K and V, bf16
        self.h_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d_bytes = total  # the whole staging buffer (inputs + alignment padding)
        self.d2h_bytes = self.h_out.numel() * self.h_out.element_size()

    def _views(self, stage):
        return [stage[o:o + n].view(dt).view(shape) for o, n, dt, shape in self._layout]

    def _run(self, views, out):
        q, nk, nv, bt, ctx, _ = views
        self.pa.pa_append_decode(out, q, nk, nv, self.kc, self.vc, bt, ctx, self.max_len - 1,
                                 self.w.scale, workspace=self.ws)

    def step(self):
        # slot of each new token, scatter of its K/V, split-KV decode over the
        # grown sequences: one decode launch (+ the split-KV combine)
        self._run((self.q, self.nk, self.nv, self.bt, self.ctx, self.lens), self.out)

    def step_e2e(self):
        # one step after another: upload, kernels, download
        self.d_stage.copy_(self.h_stage, non_blocking=True)
        self.step()
        self.h_out.copy_(self.out, non_blocking=True)

    def init_pipeline(self):
        """A second set of device staging and output buffers and a copy stream,
        so that step i + 1's upload and step i's download overlap step i's
        kernels (every step still uploads its inputs and downloads its output)."""
        self.copy_stream = torch.cuda.Stream(device=self.dev)
        self.stages = [self.d_stage, torch.empty_like(self.d_stage)]
        self.stage_views = [self._views(b) for b in self.stages]
        self.outs = [self.out, torch.empty_like(self.out)]
        self.h_outs = [self.h_out, torch.empty_like(self.h_out).pin_memory()]
        self.uploaded = [torch.cuda.Event(), torch.cuda.Event()]
        self.computed = [torch.cuda.Event(), torch.cuda.Event()]

    def run_e2e_pipelined(self, steps, stream, start_event):
        """`steps` steps, double-buffered; the first upload waits for
        `start_event` and `stream` waits for the last download at the end.
        Copy stream order: upload 0, upload 1, download 0, upload 2,
        download 1, ...; an upload into a buffer pair comes after the
        download of the step that last used it (and that step's kernels)."""
        cs = self.copy_stream
        cs.wait_event(start_event)
        with torch.cuda.stream(cs):
            self.stages[0].copy_(self.h_stage, non_blocking=True)
        self.uploaded[0].record(cs)
        for i in range(steps):
            k = i % 2
            if i + 1 < steps:
                with torch.cuda.stream(cs):
                    self.stages[1 - k].copy_(self.h_stage, non_blocking=True)
                self.uploaded[1 - k].record(cs)
            stream.wait_event(self.uploaded[k])
            self._run(self.stage_views[k], self.outs[k])
            self.computed[k].record(stream)
            cs.wait_event(self.computed[k])
            with torch.cuda.stream(cs):
                self.h_outs[k].copy_(self.outs[k], non_blocking=True)
        stream.wait_stream(cs)


def time_e2e_pipelined(st, steps, stream):
    """CUDA-event time (ms total) of `steps` double-buffered end-to-end steps."""
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    st.run_e2e_pipelined(steps, stream, a)
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b)


def time_steps(fn, steps, stream):
    """CUDA-event time of `steps` calls of fn on `stream` (ms total)."""
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b)


def prefill_measure(dev, steps, warmup, block_size):
    import paged_kv_cache_397_b200 as pa
    p = synth.chunked_prefill(block_size=block_size)
    kc, vc = p.key_cache.to(dev), p.value_cache.to(dev)
    bt, cl, cu = p.block_tables.to(dev), p.ctx_lens.to(dev), p.cu_q_lens.to(dev)
    q = p.query.to(dev)
    nk, nv = p.new_key.to(dev), p.new_value.to(dev)
    slots = torch.empty(p.total_q, dtype=torch.int64, device=dev)
    pa.pa_slot_mapping(slots, bt, cl, p.block_size, cu_q_lens=cu)
    pa.pa_reshape_and_cache(nk, nv, kc, vc, slots)
    out = torch.empty_like(q)
    qmax, cmax = int(torch.diff(p.cu_q_lens).max()), int(p.ctx_lens.max())
    ws = torch.empty(pa.pa_prefill_workspace_size(p.head_dim), dtype=torch.uint8, device=dev)
    fn = lambda: pa.pa_prefill_chunk(out, q, kc, vc, bt, cu, cl, qmax, cmax, p.scale,
                                     workspace=ws)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ms = time_steps(fn, steps, torch.cuda.current_stream()) / steps
    flops = 0
    for c, n in zip(p.ctx_lens.tolist(), torch.diff(p.cu_q_lens).tolist()):
        flops += 4 * p.head_dim * p.num_q_heads * (n * c + n * (n + 1) // 2)
    return {"workload": p.name, "block_size": block_size, "ms": ms,
            "tflops": flops / ms / 1e9, "causal_flop": flops}


def fp8_decode_measure(dev, steps, warmup, hbm_peak):
    """The same GQA decode step over an FP8 (E4M3) pool: the new token of
    every sequence quantized and written, then the FP8 decode, in one launch
    (pa_append_decode_fp8) plus the split-KV combine.  GB/s of FP8 K/V bytes
    read."""
    import paged_kv_cache_397_b200 as pa
    w = synth.llama3_8b_gqa_decode_fp8()
    kc, vc, bt = w.key_cache.to(dev), w.value_cache.to(dev), w.block_tables.to(dev)
    ctx = w.context_lens.to(dev)
    lens = (w.context_lens + 1).to(dev)
    q, nk, nv = w.query.to(dev), w.new_key.to(dev), w.new_value.to(dev)
    out = torch.empty_like(q)
    max_len = int(lens.max())
    need = pa.pa_decode_workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                       w.block_size, max_len)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)

    def step():
        pa.pa_append_decode_fp8(out, q, nk, nv, kc, vc, bt, ctx, max_len - 1, w.scale,
                                w.kv_scale, w.kv_scale, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ms = time_steps(step, steps, torch.cuda.current_stream()) / steps
    kv = 2 * w.num_kv_heads * w.head_dim * int(lens.sum())
    return {"workload": w.name, "ms_per_step": ms, "value": kv / ms / 1e6, "unit": "GB/s",
            "hbm_frac": kv / ms / 1e6 / hbm_peak, "decode_tokens_per_s": w.num_seqs / ms * 1e3,
            "kv_bytes_per_step": kv}


def mixed_measure(dev, steps, warmup):
    """One chunked-prefill scheduler step: 256 decode rows (GQA decode shape)
    and 4 prompt chunks of 512 rows over 8192 cached tokens, as one
    pa_mixed_attention launch and as two calls (pa_decode on the decode rows,
    then pa_prefill_chunk on the chunks) over the same device buffers."""
    import paged_kv_cache_397_b200 as pa
    p = synth.mixed_batch()
    kc, vc = p.key_cache.to(dev), p.value_cache.to(dev)
    bt, cl, cu = p.block_tables.to(dev), p.ctx_lens.to(dev), p.cu_q_lens.to(dev)
    q = p.query.to(dev)
    pa.pa_append(p.new_key.to(dev), p.new_value.to(dev), kc, vc, bt, cl, cu_q_lens=cu)
    out = torch.empty_like(q)
    nd = p.num_decode
    qlens = torch.diff(p.cu_q_lens)
    max_q, max_ctx = int(qlens[nd:].max()), int(p.ctx_lens.max())
    need = max(pa.pa_mixed_workspace_size(nd, p.num_q_heads, p.num_kv_heads, p.head_dim,
                                          p.block_size, max_ctx),
               pa.pa_decode_workspace_size(nd, p.num_q_heads, p.num_kv_heads, p.head_dim,
                                           p.block_size, max_ctx + 1))
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    r0 = int(p.cu_q_lens[nd])
    d_bt, d_lens = bt[:nd].contiguous(), (cl[:nd] + 1).contiguous()
    p_bt, p_cl, p_cu = bt[nd:].contiguous(), cl[nd:].contiguous(), (cu[nd:] - r0).contiguous()
    p_q, p_out, d_out = q[r0:].contiguous(), out[r0:], out[:nd]
    pws = torch.empty(pa.pa_prefill_workspace_size(p.head_dim), dtype=torch.uint8, device=dev)

    def mixed():
        pa.pa_mixed_attention(out, q, kc, vc, bt, cu, cl, nd, max_q, max_ctx, p.scale,
                              workspace=ws)

    def two_calls():
        pa.pa_decode(d_out, q[:nd], kc, vc, d_bt, d_lens, max_ctx + 1, p.scale, workspace=ws)
        pa.pa_prefill_chunk(p_out, p_q, kc, vc, p_bt, p_cu, p_cl, max_q, max_ctx, p.scale,
                            workspace=pws)

    ms = {"mixed": [], "two": []}
    for _ in range(2):  # alternate to cancel clock drift
        for name, fn in (("mixed", mixed), ("two", two_calls)):
            for _ in range(warmup):
                fn()
            torch.cuda.synchronize()
            ms[name].append(time_steps(fn, steps, torch.cuda.current_stream()) / steps)
    t_mixed, t_two = min(ms["mixed"]), min(ms["two"])
    kv = 2 * p.num_kv_heads * p.head_dim * 2 * int((p.ctx_lens[:nd] + 1).sum())
    flops = 0
    for c, n in zip(p.ctx_lens[nd:].tolist(), qlens[nd:].tolist()):
        flops += 4 * p.head_dim * p.num_q_heads * (n * c + n * (n + 1) // 2)
    return {"workload": p.name, "ms": t_mixed, "ms_two_calls": t_two,
            "speedup_vs_two_calls": t_two / t_mixed, "decode_kv_bytes": kv,
            "prefill_causal_flop": flops}


NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, the vendor figure the decode target is stated against


def _decode_leg(name, w, lens_list, dev, steps, hbm_peak, *, tables=None, caches=None,
                flush=None, prefix=None):
    """pa_decode over one workload's batch (automatic partitions).  Returns ms,
    GB/s of algorithmic K/V bytes (valid tokens only), fractions of the
    measured and nominal HBM bandwidth and decode tokens/s (one layer).  With
    `flush` (a device buffer larger than L2) every timed launch starts from a
    cold L2 and is timed alone with events on the launching stream.  With
    `prefix` = (device int32 block ids, tokens) the batch runs through
    pa_decode_shared_prefix instead."""
    import paged_kv_cache_397_b200 as pa
    kc, vc = (w.key_cache.to(dev), w.value_cache.to(dev)) if caches is None else caches
    bt = (w.block_tables if tables is None else tables).to(dev)
    lens = torch.tensor(lens_list, dtype=torch.int32, device=dev)
    q = w.query.to(dev)
    out = torch.empty_like(q)
    max_len = max(lens_list)
    need = pa.pa_decode_workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                       w.block_size, max_len)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    if prefix is None:
        fn = lambda: pa.pa_decode(out, q, kc, vc, bt, lens, max_len, w.scale, workspace=ws)
    else:
        fn = lambda: pa.pa_decode_shared_prefix(out, q, kc, vc, prefix[0], prefix[1], bt, lens,
                                                max_len, w.scale, workspace=ws)
    stream = torch.cuda.current_stream()
    for _ in range(5):
        fn()
    torch.cuda.synchronize()
    if flush is None:
        ms = time_steps(fn, steps, stream) / steps
    else:
        times = []
        for _ in range(steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
    esize = w.key_cache.element_size()
    kv = 2 * w.num_kv_heads * w.head_dim * esize * sum(lens_list)
    parts = math.ceil(max_len / pa.pa_decode_partition_tokens(w.num_seqs, w.num_kv_heads,
                                                              w.block_size, max_len))
    return {"workload": name, "ms": ms, "GBps": kv / ms / 1e6, "hbm_frac": kv / ms / 1e6 / hbm_peak,
            "hbm_frac_nominal": kv / ms / 1e6 / NOMINAL_HBM_GBS,
            "decode_tokens_per_s": w.num_seqs / ms * 1e3, "kv_bytes": kv,
            "partitions_per_longest_seq": parts, "l2": "cold (flushed)" if flush is not None
            else "inputs larger than L2"}


def decode_configs_measure(dev, steps, hbm_peak):
    """Decode throughput on the other decode workloads: the Llama-2-13B shape
    (fp16, 40 q = 40 kv heads, so one query head per KV head), the
    shared-prefix batch after its copy-on-write (logical and unique bytes,
    L2 cold and hot, through pa_decode and through pa_decode_shared_prefix,
    which reads each shared tile once per group of sequences), and the
    16 x 32768-token long-context batch (split-KV) at block sizes 16 and 32."""
    res = {}
    w = synth.llama2_13b_decode()
    res["llama2_13b_decode"] = _decode_leg(w.name, w, w.context_lens.tolist(), dev, steps,
                                           hbm_peak)
    del w
    torch.cuda.empty_cache()
    for B in (16, 32):
        w = synth.long_context_decode(block_size=B)
        res[f"long_context_decode_B{B}"] = _decode_leg(w.name, w, w.context_lens.tolist(), dev,
                                                       steps, hbm_peak)
        del w
        torch.cuda.empty_cache()
    # shared prefix: every sequence's last shared block is copied to a private
    # block (pa_copy_blocks; timed on its own under copy_blocks) and remapped
    import paged_kv_cache_397_b200 as pa
    w = synth.shared_prefix_cow()
    lens = w.context_lens.tolist()
    kc, vc = w.key_cache.to(dev), w.value_cache.to(dev)
    src = w.shared_blocks[w.cow_logical_block].repeat(w.num_seqs)
    pa.pa_copy_blocks(kc, vc, torch.stack([src, w.cow_dst_blocks], 1).to(torch.int64).to(dev))
    bt = w.block_tables.clone()
    bt[:, w.cow_logical_block] = w.cow_dst_blocks.to(torch.int32)
    # unique bytes: every physical block read once, valid tokens only
    valid = {}
    for s, L in enumerate(lens):
        for j in range(-(-L // w.block_size)):
            b = int(bt[s, j])
            valid[b] = max(valid.get(b, 0), min(w.block_size, L - j * w.block_size))
    unique = 2 * w.num_kv_heads * w.head_dim * 2 * sum(valid.values())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    # the 49 blocks every sequence still shares after the copy-on-write
    npre = w.cow_logical_block
    pre = (w.shared_blocks[:npre].to(torch.int32).to(dev), npre * w.block_size)
    for call, mode, fl, pf in (("", "cold", flush, None), ("", "hot", None, None),
                               ("_shared_prefix_call", "cold", flush, pre),
                               ("_shared_prefix_call", "hot", None, pre)):
        r = _decode_leg(w.name, w, lens, dev, steps, hbm_peak, tables=bt, caches=(kc, vc),
                        flush=fl, prefix=pf)
        r["call"] = "pa_decode_shared_prefix" if pf is not None else "pa_decode"
        r["l2"] = "cold (256 MB written between launches)" if fl is not None else \
            "hot (back-to-back launches; unique bytes fit the 126 MB L2 only in part)"
        r["logical_kv_bytes"] = r.pop("kv_bytes")
        r["logical_GBps"] = r.pop("GBps")
        r["unique_kv_bytes"] = unique
        r["unique_GBps"] = unique / r["ms"] / 1e6
        r["hbm_frac"] = r["unique_GBps"] / hbm_peak
        r["hbm_frac_nominal"] = r["unique_GBps"] / NOMINAL_HBM_GBS
        res[f"shared_prefix_cow_decode{call}_{mode}"] = r
    del flush
    torch.cuda.empty_cache()
    return res


def copy_and_swap_measure(dev, steps):
    """Copy-on-write of the shared-prefix workload (128 block pairs) and swap
    of 256 blocks of the GQA decode shape out to pinned host memory and back."""
    import paged_kv_cache_397_b200 as pa
    res = {}
    w = synth.shared_prefix_cow()
    kc, vc = w.key_cache.to(dev), w.value_cache.to(dev)
    src = w.shared_blocks[w.cow_logical_block].repeat(w.num_seqs)
    pairs = torch.stack([src, w.cow_dst_blocks], 1).to(torch.int64).to(dev)
    fn = lambda: pa.pa_copy_blocks(kc, vc, pairs)
    for _ in range(3):
        fn()
    ms = time_steps(fn, steps, torch.cuda.current_stream()) / steps
    moved = 2 * 2 * pairs.shape[0] * kc[0].numel() * kc.element_size()  # K+V, read+write
    res["copy_blocks"] = {"workload": w.name, "pairs": int(pairs.shape[0]), "us": ms * 1e3,
                          "GBps_read_plus_write": moved / ms / 1e6}
    del kc, vc
    shape = (256, 8, 16, 128)
    dk = torch.randn(shape, dtype=torch.float32, device=dev).to(torch.bfloat16)
    dv = torch.randn(shape, dtype=torch.float32, device=dev).to(torch.bfloat16)
    hk = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
    hv = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
    ident = torch.stack([torch.arange(256), torch.arange(256)], 1).to(torch.int64).to(dev)
    block_bytes = 2 * dk[0].numel() * dk.element_size()  # K + V
    for name, f in (("swap_out_d2h", lambda: pa.pa_swap_blocks(hk, hv, dk, dv, ident)),
                    ("swap_in_h2d", lambda: pa.pa_swap_blocks(dk, dv, hk, hv, ident))):
        for _ in range(3):
            f()
        ms = time_steps(f, max(3, steps // 4), torch.cuda.current_stream()) / max(3, steps // 4)
        res[name] = {"blocks": 256, "bytes": 256 * block_bytes, "us": ms * 1e3,
                     "GBps": 256 * block_bytes / ms / 1e6}
    return res


def cpu_baseline(w, budget_s=10.0):
    """The oracle, as it stands, on a seeded sample of the batch's sequences."""
    import threadpoolctl

    import oracle
    lens = (w.context_lens + 1).tolist()
    rng = np.random.default_rng(0)
    seqs = sorted(rng.choice(w.num_seqs, size=min(64, w.num_seqs), replace=False).tolist())
    # the appended token: written with the oracle's own slot arithmetic
    kcv = w.key_cache.view(torch.int16).numpy()
    vcv = w.value_cache.view(torch.int16).numpy()
    slots = oracle.logical_positions_to_slots(w.block_tables.numpy(), np.arange(w.num_seqs),
                                              w.context_lens.numpy(), w.block_size)
    used = sorted({int(b) for s in seqs for b in w.block_tables[s, :-(-lens[s] // 16)]})
    remap = {b: i for i, b in enumerate(used)}
    idx = torch.tensor(used)
    kc = w.key_cache.index_select(0, idx).double().numpy()
    vc = w.value_cache.index_select(0, idx).double().numpy()
    bt = np.full((len(seqs), w.block_tables.shape[1]), -1, dtype=np.int64)
    for r, s in enumerate(seqs):
        n = -(-lens[s] // 16)
        bt[r, :n] = [remap[int(b)] for b in w.block_tables[s, :n]]
    q = w.query[seqs].double().numpy()
    nk = w.new_key[seqs].double().numpy()
    nv = w.new_value[seqs].double().numpy()
    sub_slots = [remap[int(slots[s]) // 16] * 16 + int(slots[s]) % 16 for s in seqs]
    del kcv, vcv
    info = threadpoolctl.threadpool_info()
    threads = max([d.get("num_threads", 1) for d in info if d.get("user_api") == "blas"] or [1])
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.reshape_and_cache(kc, vc, nk, nv, sub_slots, 16)
        oracle.paged_decode(q, kc, vc, bt, [lens[s] for s in seqs], w.scale, w.num_kv_heads)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    kv = 2 * w.num_kv_heads * w.head_dim * 2 * sum(lens[s] for s in seqs) * reps
    return {"value": kv / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(seqs)} of {w.num_seqs} sequences (seeded), append + decode, "
                      f"fp64 NumPy oracle, {reps} passes in {dt:.1f} s"}


def run_reference(args):
    """--impl reference: the CPU oracle on bounded samples of the same workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import threadpoolctl

    import oracle
    w = synth.llama3_8b_gqa_decode()
    lens = (w.context_lens + 1).tolist()
    rng = np.random.default_rng(1)
    per_step = 8
    info = threadpoolctl.threadpool_info()
    threads = max([d.get("num_threads", 1) for d in info if d.get("user_api") == "blas"] or [1])

    def one_step(seqs):
        used = sorted({int(b) for s in seqs for b in w.block_tables[s, :-(-lens[s] // 16)]})
        remap = {b: i for i, b in enumerate(used)}
        idx = torch.tensor(used)
        kc = w.key_cache.index_select(0, idx).double().numpy()
        vc = w.value_cache.index_select(0, idx).double().numpy()
        bt = np.full((len(seqs), w.block_tables.shape[1]), -1, dtype=np.int64)
        for r, s in enumerate(seqs):
            n = -(-lens[s] // 16)
            bt[r, :n] = [remap[int(b)] for b in w.block_tables[s, :n]]
        q = w.query[seqs].double().numpy()
        t0 = time.perf_counter()
        sl = oracle.logical_positions_to_slots(bt, np.arange(len(seqs)),
                                               w.context_lens[seqs].numpy(), 16)
        oracle.reshape_and_cache(kc, vc, w.new_key[seqs].double().numpy(),
                                 w.new_value[seqs].double().numpy(), sl, 16)
        oracle.paged_decode(q, kc, vc, bt, [lens[s] for s in seqs], w.scale, w.num_kv_heads)
        return time.perf_counter() - t0, 2 * w.num_kv_heads * w.head_dim * 2 * sum(
            lens[s] for s in seqs)

    for _ in range(args.warmup):
        one_step(sorted(rng.choice(w.num_seqs, per_step, replace=False).tolist()))
    tot_t = tot_b = 0.0
    for _ in range(args.steps):
        t, b = one_step(sorted(rng.choice(w.num_seqs, per_step, replace=False).tolist()))
        tot_t += t
        tot_b += b
    value = tot_b / tot_t / 1e9
    sample = f"{per_step} of {w.num_seqs} sequences per step (seeded), append + decode"
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the FP8 decode, copy-on-write and swap measurements")
    ap.add_argument("--min-warmup-s", type=float, default=1.0,
                    help="keep warming up for at least this long so clocks settle")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return run_reference(args)

    world, rank, local = setup_dist()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import paged_kv_cache_397_b200 as pa
    pa.lib()

    w = synth.llama3_8b_gqa_decode()
    st = DecodeStep(w, dev)
    stream = torch.cuda.current_stream()
    hbm_peak, bf16_peak, peak_kind = peaks()

    # one step first: a device error (a bounded wait that gave up, a bad
    # table entry) stops the run here instead of after the timed region
    st.step()
    err = pa.pa_get_device_error()
    if err:
        raise RuntimeError(f"device error word {err:#x} after the first step")

    clocks = ClockSampler(local)
    clocks.start()
    # warm-up: at least W steps and at least --min-warmup-s under load
    t_end = time.time() + args.min_warmup_s
    n = 1
    while n < args.warmup or time.time() < t_end:
        st.step()
        n += 1
    torch.cuda.synchronize()

    # timed region: K full steps, plus per-launch events around every
    # EVENT_EVERY-th step (an event pair per step costs ~1 % of a 0.34 ms step)
    sampled = list(range(0, args.steps, EVENT_EVERY))
    ev = {i: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for i in sampled}
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        if i in ev:
            ev[i][0].record(stream)
            st.step()
            ev[i][1].record(stream)
        else:
            st.step()
    t_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_total = max_over_ranks(t_start.elapsed_time(t_stop), world)
    decode_ms = statistics.mean(a.elapsed_time(b) for a, b in ev.values())
    err = pa.pa_get_device_error()
    if err:
        raise RuntimeError(f"device error word {err:#x} during the timed region")

    ms_step = ms_total / args.steps
    value = job_throughput(st.kv_bytes, world, args.steps, ms_total)
    achieved = st.kv_bytes / (decode_ms * 1e-3) / 1e9
    traffic = profiled_traffic(st.kv_bytes)

    # end to end through the C ABI with host buffers (pinned), copies timed:
    # one step after another, then double-buffered (the reported value)
    for _ in range(3):
        st.step_e2e()
    torch.cuda.synchronize()
    e2e_steps = max(3, args.steps)  # as many steps as the device-timed region (same clock regime)
    barrier(world)
    e2e_serial_ms = max_over_ranks(time_steps(st.step_e2e, e2e_steps, stream),
                                   world) / e2e_steps
    st.init_pipeline()
    warm = torch.cuda.Event()
    warm.record(stream)
    st.run_e2e_pipelined(3, stream, warm)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(time_e2e_pipelined(st, e2e_steps, stream), world) / e2e_steps
    # every step downloaded the same result (the step is idempotent)
    if not (torch.equal(st.h_outs[0], st.outs[0].cpu()) and torch.equal(st.h_outs[1], st.h_outs[0])):
        raise RuntimeError("double-buffered end-to-end steps disagree with the device output")
    e2e_value = job_throughput(st.kv_bytes, world, 1, e2e_ms)
    e2e_serial = job_throughput(st.kv_bytes, world, 1, e2e_serial_ms)

    kv_bytes, launches = st.kv_bytes, st.launches_per_step * args.steps
    h2d, d2h = st.h2d_bytes, st.d2h_bytes
    prefill = None
    if not args.no_prefill:
        del st
        torch.cuda.empty_cache()
        prefill = []
        for B in (16, 32):
            r = prefill_measure(dev, steps=20, warmup=3, block_size=B)
            r["tensor_frac"] = r["tflops"] / bf16_peak
            r["peak_tflops"] = bf16_peak
            r["peak_kind"] = f"bf16 dense, {peak_kind} (burst)"
            prefill.append(r)

    secondary = None
    if world == 1 and not args.no_secondary:
        torch.cuda.empty_cache()
        secondary = {"fp8_decode": fp8_decode_measure(dev, steps=50, warmup=5,
                                                      hbm_peak=hbm_peak)}
        secondary["fp8_decode"]["hbm_frac_nominal"] = \
            secondary["fp8_decode"]["value"] / NOMINAL_HBM_GBS
        torch.cuda.empty_cache()
        secondary["mixed_batch"] = mixed_measure(dev, steps=20, warmup=3)
        torch.cuda.empty_cache()
        secondary["decode_configs"] = decode_configs_measure(dev, steps=20, hbm_peak=hbm_peak)
        torch.cuda.empty_cache()
        secondary.update(copy_and_swap_measure(dev, steps=50))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "kv_bytes_per_step_per_gpu": kv_bytes,
                       "l2": "inputs larger than L2 (2.2 GB of K/V read per step, 126 MB L2)",
                       "parallelism": f"replicas x{world} (each rank its own batch)"},
            "hbm_frac": value / world / hbm_peak,
            "hbm_frac_nominal": value / world / NOMINAL_HBM_GBS,
            "decode_tokens_per_s": world * w.num_seqs / (ms_step * 1e-3),
            "roofline": {"kernel": "pa_append_decode (decode_kernel with the fused append + "
                                   "decode_reduce_kernel)",
                         "bound": "hbm", "achieved": achieved, "peak": hbm_peak,
                         "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": traffic,
                         "frac_nominal": achieved / NOMINAL_HBM_GBS,
                         "peak_kind": f"hbm copy, {peak_kind}"},
            "prefill_chunk": prefill,
            "secondary": secondary,
            "e2e": {"value": e2e_value, "unit": "GB/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "mode": "double-buffered: step i+1's upload and step i's download run on a "
                            "copy stream during step i's kernels",
                    "serial": {"value": e2e_serial, "ms_per_step": e2e_serial_ms}},
            "gpu_launches": launches,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

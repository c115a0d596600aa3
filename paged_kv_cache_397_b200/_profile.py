"""Small, self-contained cases of the hot kernels for ncu captures.

    python -m paged_kv_cache_397_b200._profile decode  --seqs 32
    python -m paged_kv_cache_397_b200._profile decode-fp8 --seqs 64
    python -m paged_kv_cache_397_b200._profile prefill --seqs 4 [--block-size 16]
    python -m paged_kv_cache_397_b200._profile mixed --seqs 64
    python -m paged_kv_cache_397_b200._profile decode-llama2 --seqs 16
    python -m paged_kv_cache_397_b200._profile decode-long --seqs 2 [--block-size 16]
    python -m paged_kv_cache_397_b200._profile decode-cow [--shared-prefix]

Each case builds a scaled-down copy of a bench workload (same shapes, head
counts, length distribution and block shuffling; fewer sequences), runs the
kernel three times on cuda:0 and prints the launch's K/V bytes or FLOPs, so
per-launch counters can be scaled to the full-size launch.  The inputs stay a
few hundred MB on the device (above the 126 MB L2) so that a multi-pass
capture ends in seconds.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import paged_kv_cache_397_b200 as pa  # noqa: E402
import synth  # noqa: E402


def decode_case(seqs: int, reps: int = 3):
    """The bench's decode step (pa_append_decode) on a slice of its batch."""
    w = synth.llama3_8b_gqa_decode(num_seqs=seqs)
    d = torch.device("cuda:0")
    kc, vc, bt = w.key_cache.to(d), w.value_cache.to(d), w.block_tables.to(d)
    ctx = w.context_lens.to(d)
    lens = ctx + 1
    q, nk, nv = w.query.to(d), w.new_key.to(d), w.new_value.to(d)
    out = torch.empty_like(q)
    max_ctx = int(w.context_lens.max())
    for _ in range(reps):  # the same token rewritten into the same slot each time
        pa.pa_append_decode(out, q, nk, nv, kc, vc, bt, ctx, max_ctx, w.scale)
    torch.cuda.synchronize()
    kv = 2 * w.num_kv_heads * w.head_dim * 2 * int(lens.sum())
    print(f"decode case: {w.name}, K/V bytes per launch {kv}")


def decode_fp8_case(seqs: int, reps: int = 3):
    """The bench's FP8 decode step (pa_append_decode_fp8) on a slice of its batch."""
    w = synth.llama3_8b_gqa_decode_fp8(num_seqs=seqs)
    d = torch.device("cuda:0")
    kc, vc, bt = w.key_cache.to(d), w.value_cache.to(d), w.block_tables.to(d)
    ctx = w.context_lens.to(d)
    lens = ctx + 1
    q, nk, nv = w.query.to(d), w.new_key.to(d), w.new_value.to(d)
    out = torch.empty_like(q)
    max_ctx = int(w.context_lens.max())
    for _ in range(reps):  # the same token rewritten into the same slot each time
        pa.pa_append_decode_fp8(out, q, nk, nv, kc, vc, bt, ctx, max_ctx, w.scale, w.kv_scale,
                                w.kv_scale)
    torch.cuda.synchronize()
    kv = 2 * w.num_kv_heads * w.head_dim * int(lens.sum())
    print(f"decode-fp8 case: {w.name}, K/V bytes per launch {kv}")


def prefill_case(seqs: int, block_size: int, reps: int = 3):
    p = synth.chunked_prefill(num_seqs=seqs, block_size=block_size)
    d = torch.device("cuda:0")
    kc, vc = p.key_cache.to(d), p.value_cache.to(d)
    bt, cl, cu = p.block_tables.to(d), p.ctx_lens.to(d), p.cu_q_lens.to(d)
    q = p.query.to(d)
    out = torch.empty_like(q)
    qmax, cmax = int(torch.diff(p.cu_q_lens).max()), int(p.ctx_lens.max())
    ws = torch.empty(pa.pa_prefill_workspace_size(p.head_dim), dtype=torch.uint8, device=d)
    for _ in range(reps):
        pa.pa_prefill_chunk(out, q, kc, vc, bt, cu, cl, qmax, cmax, p.scale, workspace=ws)
    torch.cuda.synchronize()
    flops = sum(4 * p.head_dim * p.num_q_heads * (n * c + n * (n + 1) // 2)
                for c, n in zip(p.ctx_lens.tolist(), torch.diff(p.cu_q_lens).tolist()))
    print(f"prefill case: {p.name}, causal FLOP per launch {flops}")


def mixed_case(seqs: int, reps: int = 3):
    """`seqs` decode rows (GQA decode lengths) and one 512-row chunk over 8192
    cached tokens, as one pa_mixed_attention launch."""
    p = synth.mixed_batch(num_decode=seqs, num_prefill=1)
    d = torch.device("cuda:0")
    kc, vc = p.key_cache.to(d), p.value_cache.to(d)
    bt, cl, cu = p.block_tables.to(d), p.ctx_lens.to(d), p.cu_q_lens.to(d)
    q = p.query.to(d)
    pa.pa_append(p.new_key.to(d), p.new_value.to(d), kc, vc, bt, cl, cu_q_lens=cu)
    out = torch.empty_like(q)
    nd = p.num_decode
    qlens = torch.diff(p.cu_q_lens)
    max_q, max_ctx = int(qlens[nd:].max()), int(p.ctx_lens.max())
    for _ in range(reps):
        pa.pa_mixed_attention(out, q, kc, vc, bt, cu, cl, nd, max_q, max_ctx, p.scale)
    torch.cuda.synchronize()
    kv = 2 * p.num_kv_heads * p.head_dim * 2 * int((p.ctx_lens[:nd] + 1).sum())
    flops = sum(4 * p.head_dim * p.num_q_heads * (n * c + n * (n + 1) // 2)
                for c, n in zip(p.ctx_lens[nd:].tolist(), qlens[nd:].tolist()))
    print(f"mixed case: {p.name}, decode K/V bytes {kv}, prefill causal FLOP {flops}")


def _plain_decode(w, lens, d, reps, tables=None, caches=None):
    kc, vc = (w.key_cache.to(d), w.value_cache.to(d)) if caches is None else caches
    bt = (w.block_tables if tables is None else tables).to(d)
    ld = torch.tensor(lens, dtype=torch.int32, device=d)
    q = w.query.to(d)
    out = torch.empty_like(q)
    for _ in range(reps):
        pa.pa_decode(out, q, kc, vc, bt, ld, max(lens), w.scale)
    torch.cuda.synchronize()
    return 2 * w.num_kv_heads * w.head_dim * w.key_cache.element_size() * sum(lens)


def decode_llama2_case(seqs: int, reps: int = 3):
    """The Llama-2-13B-shaped decode (fp16, 40 q = 40 kv heads) on `seqs` sequences."""
    w = synth.llama2_13b_decode(num_seqs=seqs)
    kv = _plain_decode(w, w.context_lens.tolist(), torch.device("cuda:0"), reps)
    print(f"decode-llama2 case: {w.name}, K/V bytes per launch {kv}")


def decode_long_case(seqs: int, block_size: int, reps: int = 3):
    """The long-context split-KV decode (32768 tokens per sequence) on `seqs` sequences."""
    w = synth.long_context_decode(num_seqs=seqs, block_size=block_size)
    kv = _plain_decode(w, w.context_lens.tolist(), torch.device("cuda:0"), reps)
    print(f"decode-long case: {w.name}, K/V bytes per launch {kv}")


def decode_cow_case(reps: int = 3, shared_prefix: bool = False):
    """The shared-prefix batch (128 sequences) after its copy-on-write and
    remap, through pa_decode or (shared_prefix) pa_decode_shared_prefix."""
    w = synth.shared_prefix_cow()
    d = torch.device("cuda:0")
    kc, vc = w.key_cache.to(d), w.value_cache.to(d)
    src = w.shared_blocks[w.cow_logical_block].repeat(w.num_seqs)
    pa.pa_copy_blocks(kc, vc, torch.stack([src, w.cow_dst_blocks], 1).to(torch.int64).to(d))
    bt = w.block_tables.clone()
    bt[:, w.cow_logical_block] = w.cow_dst_blocks.to(torch.int32)
    if shared_prefix:
        lens = w.context_lens.tolist()
        npre = w.cow_logical_block
        ld = torch.tensor(lens, dtype=torch.int32, device=d)
        q = w.query.to(d)
        out = torch.empty_like(q)
        pre = w.shared_blocks[:npre].to(torch.int32).to(d)
        for _ in range(reps):
            pa.pa_decode_shared_prefix(out, q, kc, vc, pre, npre * w.block_size, bt.to(d), ld,
                                       max(lens), w.scale)
        torch.cuda.synchronize()
        kv = 2 * w.num_kv_heads * w.head_dim * 2 * sum(lens)
    else:
        kv = _plain_decode(w, w.context_lens.tolist(), d, reps, tables=bt, caches=(kc, vc))
    print(f"decode-cow case: {w.name}, logical K/V bytes per launch {kv}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["decode", "decode-fp8", "prefill", "mixed", "decode-llama2",
                                     "decode-long", "decode-cow"])
    ap.add_argument("--seqs", type=int, default=None)
    ap.add_argument("--block-size", type=int, default=16)
    ap.add_argument("--shared-prefix", action="store_true")
    a = ap.parse_args()
    pa.lib()
    if a.case == "decode":
        decode_case(a.seqs or 32)
    elif a.case == "decode-fp8":
        decode_fp8_case(a.seqs or 64)
    elif a.case == "mixed":
        mixed_case(a.seqs or 64)
    elif a.case == "decode-llama2":
        decode_llama2_case(a.seqs or 16)
    elif a.case == "decode-long":
        decode_long_case(a.seqs or 2, a.block_size)
    elif a.case == "decode-cow":
        decode_cow_case(shared_prefix=a.shared_prefix)
    else:
        prefill_case(a.seqs or 4, a.block_size)
    if pa.pa_get_device_error():
        raise SystemExit("device error word set")


if __name__ == "__main__":
    main()

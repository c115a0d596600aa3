"""Shared test plumbing: tolerances, device copies, oracle references on
sub-pools (so full-size workloads can be checked on sampled sequences)."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# max |gpu - oracle| for the output dtype (fp32 accumulation inside the kernels)
TOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}


def dev():
    return torch.device("cuda:0")


def to_dev(t):
    return None if t is None else t.to(dev())


def int16_view(t: torch.Tensor) -> np.ndarray:
    """numpy view of a CPU fp16/bf16 tensor's bits (writes go through)."""
    return t.view(torch.int16).numpy()


def oracle_append(w):
    """Oracle slot mapping + bit scatter of the appended token into the CPU caches
    (in place); returns the slots."""
    slots = oracle.logical_positions_to_slots(w.block_tables.numpy(), np.arange(w.num_seqs),
                                              w.context_lens.numpy(), w.block_size)
    oracle.reshape_and_cache(int16_view(w.key_cache), int16_view(w.value_cache),
                             int16_view(w.new_key), int16_view(w.new_value), slots, w.block_size)
    return slots


def sub_pool(key_cache, value_cache, block_tables, lens, seqs, block_size):
    """fp64 copies of only the blocks the chosen sequences read, with their
    tables renumbered into the small pool."""
    bt = block_tables.numpy() if isinstance(block_tables, torch.Tensor) else block_tables
    used = []
    for s in seqs:
        n = -(-int(lens[s]) // block_size)
        used.extend(int(b) for b in bt[s, :n])
    used = sorted(set(used))
    remap = {b: i for i, b in enumerate(used)}
    idx = torch.tensor(used, dtype=torch.int64)
    kc = key_cache.index_select(0, idx).double().numpy()
    vc = value_cache.index_select(0, idx).double().numpy()
    sbt = np.full((len(seqs), bt.shape[1]), -1, dtype=np.int64)
    for r, s in enumerate(seqs):
        n = -(-int(lens[s]) // block_size)
        sbt[r, :n] = [remap[int(b)] for b in bt[s, :n]]
    return kc, vc, sbt


def decode_reference(w, lens, seqs):
    """Oracle decode output (fp64) for the chosen sequences of a workload."""
    kc, vc, sbt = sub_pool(w.key_cache, w.value_cache, w.block_tables, lens, seqs, w.block_size)
    q = w.query[list(seqs)].double().numpy()
    return oracle.paged_decode(q, kc, vc, sbt, [int(lens[s]) for s in seqs], w.scale,
                               w.num_kv_heads)


def max_err(gpu: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu.double().cpu().numpy()
    assert np.all(np.isfinite(g)), "non-finite values in the GPU output"
    return float(np.abs(g - ref).max()) if ref.size else 0.0


def sample_seqs(n_total, k, seed, must=()):
    rng = np.random.default_rng(seed)
    pick = set(int(x) for x in must)
    pick.update(int(x) for x in rng.choice(n_total, size=min(k, n_total), replace=False))
    return sorted(pick)


def oracle_scatter_chunks(p):
    """Oracle slot mapping + bit scatter of every query row's own K/V of a
    chunk batch into the CPU caches (in place)."""
    cu = p.cu_q_lens.numpy()
    seq_of = np.repeat(np.arange(p.num_seqs), np.diff(cu))
    pos = np.concatenate([np.arange(c, c + n) for c, n in zip(p.ctx_lens.numpy(), np.diff(cu))])
    slots = oracle.logical_positions_to_slots(p.block_tables.numpy(), seq_of, pos, p.block_size)
    oracle.reshape_and_cache(int16_view(p.key_cache), int16_view(p.value_cache),
                             int16_view(p.new_key), int16_view(p.new_value), slots, p.block_size)


def chunk_reference(p, seqs=None, rows=None):
    """Oracle chunk attention (fp64) for the chosen sequences of a chunk batch,
    their query rows packed; returns (out, packed cu_q_lens)."""
    seqs = list(range(p.num_seqs)) if seqs is None else seqs
    lens = (p.ctx_lens + torch.diff(p.cu_q_lens)).tolist()
    kc, vc, sbt = sub_pool(p.key_cache, p.value_cache, p.block_tables, lens, seqs, p.block_size)
    cu = p.cu_q_lens.numpy()
    qs = [p.query[cu[s]:cu[s + 1]] for s in seqs]
    sub_cu = np.concatenate([[0], np.cumsum([len(x) for x in qs])])
    q = torch.cat(qs).double().numpy()
    ref = oracle.paged_prefill_chunk(q, kc, vc, sbt, sub_cu, [int(p.ctx_lens[s]) for s in seqs],
                                     p.scale, p.num_kv_heads, rows=rows)
    return ref, sub_cu

"""Python binding of libpa.so, the B200 (sm_100a) paged-attention library.

Argument marshalling only: every function takes torch CUDA tensors, checks
their dtype / shape / contiguity, derives the sizes the C ABI wants from the
shapes, and calls the ``extern "C"`` entry point of the same name in
``libpa.so`` (declared in ``include/pa.h``) on the current CUDA stream.  Every
step of the computation runs in the library's kernels; there is no CPU or
PyTorch fallback — if ``libpa.so`` is missing, every call raises.

Cited pages (by title and section): "vLLM PagedAttention Deep Dive: KV Cache
Memory Fragmentation, Chunked Prefill & Prefix Caching" ("PagedAttention
Mechanism", "Mechanics of Chunked Prefill"); "PagedAttention: KV cache as
virtual memory" ("Deep dive"); "PagedAttention: Why Static Batching Wastes Your
KV Cache" ("How does copy-on-write eliminate duplicate prompt KV cache?").
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "PAError", "lib", "lib_path", "EXPORTED_SYMBOLS", "pa_status_string", "pa_version",
    "pa_slot_mapping", "pa_reshape_and_cache", "pa_copy_blocks", "pa_decode_partition_tokens",
    "pa_decode_workspace_size", "pa_decode", "pa_decode_static_workspace",
    "pa_prefill_workspace_size", "pa_prefill_chunk",
    "pa_get_device_error", "pa_selftest_wait_timeout", "PA_STATIC_WORKSPACE_BYTES",
    "PA_OK", "PA_ERR_INVALID_ARG", "PA_ERR_UNSUPPORTED", "PA_ERR_WORKSPACE",
    "PA_ERR_OUT_OF_RANGE", "PA_ERR_CUDA", "PA_F16", "PA_BF16", "PA_FP8_E4M3",
    "pa_reshape_and_cache_fp8", "pa_decode_fp8", "pa_swap_blocks", "pa_append",
    "pa_mixed_workspace_size", "pa_mixed_attention", "pa_append_decode", "pa_append_decode_fp8",
    "pa_decode_shared_prefix",
    "BlockManager",
    "PA_DEVERR_SLOT_RANGE", "PA_DEVERR_BLOCK_RANGE", "PA_DEVERR_SEQ_RANGE",
    "PA_DEVERR_WAIT_TIMEOUT",
]

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE = 0, 1, 2, 3
PA_ERR_OUT_OF_RANGE, PA_ERR_CUDA = 4, 5
PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2
PA_DEVERR_SLOT_RANGE, PA_DEVERR_BLOCK_RANGE = 0x1, 0x2
PA_DEVERR_SEQ_RANGE, PA_DEVERR_WAIT_TIMEOUT = 0x4, 0x8

lib_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")

# name -> (restype, argtypes); mirrors include/pa.h
_i, _f, _p, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_SIGS = {
    "pa_status_string": (ctypes.c_char_p, [_i]),
    "pa_version": (_i, []),
    "pa_slot_mapping": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _p]),
    "pa_reshape_and_cache": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]),
    "pa_append": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p]),
    "pa_copy_blocks": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _p]),
    "pa_decode_partition_tokens": (_i, [_i, _i, _i, _i]),
    "pa_decode_workspace_size": (_i, [_i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_sz)]),
    "pa_decode": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                       _p, _sz, _p]),
    "pa_decode_static_workspace": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                                        _i, _i, _f, _i, _p]),
    "pa_reshape_and_cache_fp8": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _f, _i, _p]),
    "pa_swap_blocks": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p]),
    "pa_decode_fp8": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _f, _f,
                           _f, _i, _p, _sz, _p]),
    "pa_prefill_workspace_size": (_i, [_i, ctypes.POINTER(_sz)]),
    "pa_prefill_chunk": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                              _i, _f, _i, _p, _sz, _p]),
    "pa_append_decode": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                              _i, _i, _f, _i, _p, _sz, _p]),
    "pa_append_decode_fp8": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i,
                                  _i, _i, _i, _f, _f, _f, _i, _p, _sz, _p]),
    "pa_decode_shared_prefix": (_i, [_p, _p, _p, _p, _p, _i, _p, _p, _i, _i, _i, _i, _i, _i,
                                     _i, _i, _i, _f, _i, _p, _sz, _p]),
    "pa_mixed_workspace_size": (_i, [_i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_sz)]),
    "pa_mixed_attention": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i,
                                _i, _i, _i, _i, _f, _i, _p, _sz, _p]),
    "pa_get_device_error": (_i, [ctypes.POINTER(ctypes.c_uint), _p]),
    "pa_selftest_wait_timeout": (_i, [ctypes.c_uint64, _p, _p]),
    "pa_bm_create": (_i, [_i, _i, _i, ctypes.POINTER(_p)]),
    "pa_bm_destroy": (None, [_p]),
    "pa_bm_add_sequence": (_i, [_p, ctypes.c_int64, _p, _i, ctypes.POINTER(_i)]),
    "pa_bm_append": (_i, [_p, ctypes.c_int64, _p, _i]),
    "pa_bm_fork": (_i, [_p, ctypes.c_int64, ctypes.c_int64]),
    "pa_bm_free": (_i, [_p, ctypes.c_int64]),
    "pa_bm_block_table": (_i, [_p, ctypes.c_int64, _p, _i, ctypes.POINTER(_i)]),
    "pa_bm_slots": (_i, [_p, ctypes.c_int64, _i, _i, _p]),
    "pa_bm_take_copies": (_i, [_p, _p, _i]),
    "pa_bm_num_free_blocks": (_i, [_p]),
    "pa_bm_ref_count": (_i, [_p, _i]),
    "pa_bm_num_tokens": (_i, [_p, ctypes.c_int64]),
}
EXPORTED_SYMBOLS = tuple(_SIGS)

_LIB: Optional[ctypes.CDLL] = None


class PAError(RuntimeError):
    """A libpa call returned a non-OK pa_status."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {pa_status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load libpa.so (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(
                f"libpa.so not found at {lib_path}; build it with "
                "`python -m paged_kv_cache_397_b200._build` (there is no CPU fallback)")
        h = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = h
    return _LIB


def _check(fn: str, status: int) -> None:
    if status != PA_OK:
        raise PAError(fn, status)


def _dtype_code(t: torch.Tensor, allow_fp8: bool = False) -> int:
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if allow_fp8 and t.dtype == torch.uint8:
        return PA_FP8_E4M3
    raise ValueError(f"unsupported dtype {t.dtype}; expected float16 or bfloat16"
                     + (" or uint8 (E4M3 codes)" if allow_fp8 else ""))


def _check_device(t, name: str) -> None:
    """The library launches on the calling thread's current device, so a CUDA
    tensor argument must live there (another device's pointer would reach
    the kernel as a foreign address)."""
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device} but the current device is cuda:{cur}; "
                         "call under torch.cuda.device(...) of the tensors' device")


def _ptr(t, name: str, dtype=None, ndim=None) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    _check_device(t, name)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _cache_dims(key_cache, value_cache):
    if key_cache.shape != value_cache.shape or key_cache.dtype != value_cache.dtype:
        raise ValueError("key_cache and value_cache must match in shape and dtype")
    if key_cache.dim() != 4:
        raise ValueError("caches must be [num_blocks][num_kv_heads][block_size][head_dim]")
    return tuple(int(x) for x in key_cache.shape)


def pa_status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def pa_version() -> int:
    return lib().pa_version()


def pa_slot_mapping(slot_mapping, block_tables, ctx_lens, block_size, cu_q_lens=None,
                    stream=None):
    """int64 slot of each new token (see include/pa.h, pa_slot_mapping)."""
    S = int(ctx_lens.numel())
    if block_tables.dim() != 2 or block_tables.shape[0] != S:
        raise ValueError("block_tables must be [num_seqs][max_blocks_per_seq]")
    if cu_q_lens is not None and cu_q_lens.numel() != S + 1:
        raise ValueError("cu_q_lens must have num_seqs + 1 entries")
    _check("pa_slot_mapping", lib().pa_slot_mapping(
        _ptr(slot_mapping, "slot_mapping", torch.int64, 1),
        _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(cu_q_lens, "cu_q_lens", torch.int32, 1), _ptr(ctx_lens, "ctx_lens", torch.int32, 1),
        S, int(slot_mapping.numel()), int(block_tables.shape[1]), int(block_size),
        _stream(stream)))
    return slot_mapping


def pa_reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, stream=None):
    """Scatter new K/V rows ``[num_tokens][num_kv_heads][head_dim]`` into their slots."""
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if key.shape != value.shape or key.dim() != 3 or tuple(key.shape[1:]) != (hkv, d):
        raise ValueError("key/value must be [num_tokens][num_kv_heads][head_dim] like the cache")
    if key.dtype != key_cache.dtype or value.dtype != key_cache.dtype:
        raise ValueError("key/value dtype must match the cache")
    if slot_mapping.numel() != key.shape[0]:
        raise ValueError("slot_mapping needs one entry per token")
    _check("pa_reshape_and_cache", lib().pa_reshape_and_cache(
        _ptr(key, "key"), _ptr(value, "value"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(slot_mapping, "slot_mapping", torch.int64, 1),
        int(key.shape[0]), hkv, d, bs, nb, _dtype_code(key_cache), _stream(stream)))


def pa_append(key, value, key_cache, value_cache, block_tables, ctx_lens, cu_q_lens=None,
              slot_mapping=None, stream=None):
    """Slot mapping and K/V scatter of new tokens in one launch (include/pa.h)."""
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if key.shape != value.shape or key.dim() != 3 or tuple(key.shape[1:]) != (hkv, d):
        raise ValueError("key/value must be [num_tokens][num_kv_heads][head_dim] like the cache")
    if key.dtype != key_cache.dtype or value.dtype != key_cache.dtype:
        raise ValueError("key/value dtype must match the cache")
    S = int(ctx_lens.numel())
    if block_tables.dim() != 2 or block_tables.shape[0] != S:
        raise ValueError("block_tables must be [num_seqs][max_blocks_per_seq]")
    if cu_q_lens is not None and cu_q_lens.numel() != S + 1:
        raise ValueError("cu_q_lens must have num_seqs + 1 entries")
    if slot_mapping is not None and slot_mapping.numel() != key.shape[0]:
        raise ValueError("slot_mapping needs one entry per token")
    _check("pa_append", lib().pa_append(
        _ptr(key, "key"), _ptr(value, "value"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(cu_q_lens, "cu_q_lens", torch.int32, 1), _ptr(ctx_lens, "ctx_lens", torch.int32, 1),
        _ptr(slot_mapping, "slot_mapping", torch.int64, 1), S, int(key.shape[0]),
        int(block_tables.shape[1]), hkv, d, bs, nb, _dtype_code(key_cache), _stream(stream)))


def pa_copy_blocks(key_cache, value_cache, block_pairs, stream=None):
    """Copy whole physical blocks: ``cache[dst] = cache[src]`` for each (src, dst) pair."""
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if block_pairs.dim() != 2 or block_pairs.shape[1] != 2:
        raise ValueError("block_pairs must be int64 [num_pairs][2]")
    _check("pa_copy_blocks", lib().pa_copy_blocks(
        _ptr(key_cache, "key_cache"), _ptr(value_cache, "value_cache"),
        _ptr(block_pairs, "block_pairs", torch.int64, 2), int(block_pairs.shape[0]), hkv, d, bs,
        nb, _dtype_code(key_cache, allow_fp8=True), _stream(stream)))


def pa_reshape_and_cache_fp8(key, value, key_cache, value_cache, slot_mapping, k_scale,
                             v_scale, stream=None):
    """Scatter new fp16/bf16 K/V rows into FP8 (E4M3, uint8) caches (include/pa.h)."""
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if key_cache.dtype != torch.uint8:
        raise ValueError("FP8 caches are uint8 tensors of E4M3 codes")
    if key.shape != value.shape or key.dim() != 3 or tuple(key.shape[1:]) != (hkv, d):
        raise ValueError("key/value must be [num_tokens][num_kv_heads][head_dim] like the cache")
    if key.dtype != value.dtype:
        raise ValueError("key and value dtypes differ")
    if slot_mapping.numel() != key.shape[0]:
        raise ValueError("slot_mapping needs one entry per token")
    _check("pa_reshape_and_cache_fp8", lib().pa_reshape_and_cache_fp8(
        _ptr(key, "key"), _ptr(value, "value"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(slot_mapping, "slot_mapping", torch.int64, 1),
        int(key.shape[0]), hkv, d, bs, nb, float(k_scale), float(v_scale), _dtype_code(key),
        _stream(stream)))


def pa_decode_fp8(out, query, key_cache, value_cache, block_tables, seq_lens, max_seq_len,
                  scale, k_scale, v_scale, workspace=None, partition_tokens=0, stream=None):
    """Paged decode over FP8 (E4M3, uint8) caches; fp16/bf16 query and output."""
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if key_cache.dtype != torch.uint8:
        raise ValueError("FP8 caches are uint8 tensors of E4M3 codes")
    if query.dim() != 3 or query.shape[2] != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs][num_q_heads][head_dim]")
    if out.dtype != query.dtype:
        raise ValueError("out dtype must match the query")
    S, hq = int(query.shape[0]), int(query.shape[1])
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.numel() != S:
        raise ValueError("block_tables / seq_lens do not match the batch")
    need = pa_decode_workspace_size(S, hq, hkv, d, bs, max_seq_len, partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_decode_fp8", lib().pa_decode_fp8(
        _ptr(out, "out"), _ptr(query, "query"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(seq_lens, "seq_lens", torch.int32, 1), S, hq, hkv, d, bs, nb,
        int(block_tables.shape[1]), int(max_seq_len), int(partition_tokens), float(scale),
        float(k_scale), float(v_scale), _dtype_code(query), ws_ptr, ws_bytes, _stream(stream)))
    return out


def _pool_ptr(t, name):
    """A CUDA tensor, or a pinned CPU tensor (addressed by the GPU through UVA)."""
    if not isinstance(t, torch.Tensor) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor")
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    if t.is_cuda:
        _check_device(t, name)
    return t.data_ptr()


def pa_swap_blocks(dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, block_pairs,
                   stream=None):
    """Copy blocks pairs[i][0] of the src pool to pairs[i][1] of the dst pool (K and V);
    either pool may be pinned host memory (swap out / swap in)."""
    snb, hkv, bs, d = _cache_dims(src_key_cache, src_value_cache)
    dnb, hkv2, bs2, d2 = _cache_dims(dst_key_cache, dst_value_cache)
    if (hkv, bs, d) != (hkv2, bs2, d2) or src_key_cache.dtype != dst_key_cache.dtype:
        raise ValueError("source and destination pools differ in block shape or dtype")
    if block_pairs.dim() != 2 or block_pairs.shape[1] != 2:
        raise ValueError("block_pairs must be int64 [num_pairs][2]")
    _check("pa_swap_blocks", lib().pa_swap_blocks(
        _pool_ptr(dst_key_cache, "dst_key_cache"), _pool_ptr(dst_value_cache, "dst_value_cache"),
        _pool_ptr(src_key_cache, "src_key_cache"), _pool_ptr(src_value_cache, "src_value_cache"),
        _ptr(block_pairs, "block_pairs", torch.int64, 2), int(block_pairs.shape[0]), hkv, d, bs,
        snb, dnb, _dtype_code(src_key_cache, allow_fp8=True), _stream(stream)))


def pa_decode_partition_tokens(num_seqs, num_kv_heads, block_size, max_seq_len) -> int:
    return int(lib().pa_decode_partition_tokens(num_seqs, num_kv_heads, block_size, max_seq_len))


def pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                             max_seq_len, partition_tokens=0) -> int:
    n = ctypes.c_size_t(0)
    _check("pa_decode_workspace_size", lib().pa_decode_workspace_size(
        int(num_seqs), int(num_q_heads), int(num_kv_heads), int(head_dim), int(block_size),
        int(max_seq_len), int(partition_tokens), ctypes.byref(n)))
    return int(n.value)


def pa_decode(out, query, key_cache, value_cache, block_tables, seq_lens, max_seq_len, scale,
              workspace=None, partition_tokens=0, stream=None):
    """Paged decode attention: one query row per sequence (see include/pa.h, pa_decode).

    ``workspace`` is a CUDA byte tensor of at least ``pa_decode_workspace_size``
    bytes; when None the binding allocates one with torch.
    """
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if query.dim() != 3 or query.shape[2] != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs][num_q_heads][head_dim]")
    if query.dtype != key_cache.dtype or out.dtype != key_cache.dtype:
        raise ValueError("query/out dtype must match the cache")
    S, hq = int(query.shape[0]), int(query.shape[1])
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.numel() != S:
        raise ValueError("block_tables / seq_lens do not match the batch")
    need = pa_decode_workspace_size(S, hq, hkv, d, bs, max_seq_len, partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_decode", lib().pa_decode(
        _ptr(out, "out"), _ptr(query, "query"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(seq_lens, "seq_lens", torch.int32, 1), S, hq, hkv, d, bs, nb,
        int(block_tables.shape[1]), int(max_seq_len), int(partition_tokens), float(scale),
        _dtype_code(key_cache), ws_ptr, ws_bytes, _stream(stream)))
    return out


def pa_append_decode(out, query, new_key, new_value, key_cache, value_cache, block_tables,
                     ctx_lens, max_ctx_len, scale, slot_mapping=None, workspace=None,
                     partition_tokens=0, stream=None):
    """One decode step in one launch: append each sequence's new token at
    position ctx_lens[s], then decode over ctx_lens + 1 tokens (include/pa.h,
    pa_append_decode).  ``workspace`` as for pa_decode with max_ctx_len + 1."""
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if query.dim() != 3 or query.shape[2] != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs][num_q_heads][head_dim]")
    if query.dtype != key_cache.dtype or out.dtype != key_cache.dtype:
        raise ValueError("query/out dtype must match the cache")
    S, hq = int(query.shape[0]), int(query.shape[1])
    if new_key.shape != (S, hkv, d) or new_value.shape != (S, hkv, d):
        raise ValueError("new_key/new_value must be [num_seqs][num_kv_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or ctx_lens.numel() != S:
        raise ValueError("block_tables / ctx_lens do not match the batch")
    need = pa_decode_workspace_size(S, hq, hkv, d, bs, int(max_ctx_len) + 1, partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    slot_ptr = _ptr(slot_mapping, "slot_mapping", torch.int64, 1) if slot_mapping is not None \
        else None
    _check("pa_append_decode", lib().pa_append_decode(
        _ptr(out, "out"), _ptr(query, "query"), _ptr(new_key, "new_key"),
        _ptr(new_value, "new_value"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(ctx_lens, "ctx_lens", torch.int32, 1), slot_ptr, S, hq, hkv, d, bs, nb,
        int(block_tables.shape[1]), int(max_ctx_len), int(partition_tokens), float(scale),
        _dtype_code(key_cache), ws_ptr, ws_bytes, _stream(stream)))
    return out


def pa_decode_shared_prefix(out, query, key_cache, value_cache, prefix_blocks, prefix_len,
                            block_tables, seq_lens, max_seq_len, scale, workspace=None,
                            partition_tokens=0, stream=None):
    """pa_decode for a batch whose sequences share a leading prefix stored in
    the physical blocks ``prefix_blocks`` (int32 CUDA tensor); the shared
    partitions are computed once per group of sequences (include/pa.h)."""
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if query.dim() != 3 or query.shape[2] != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs][num_q_heads][head_dim]")
    if query.dtype != key_cache.dtype or out.dtype != key_cache.dtype:
        raise ValueError("query/out dtype must match the cache")
    S, hq = int(query.shape[0]), int(query.shape[1])
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.numel() != S:
        raise ValueError("block_tables / seq_lens do not match the batch")
    if prefix_blocks.numel() * bs < int(prefix_len):
        raise ValueError("prefix_blocks holds fewer than prefix_len tokens")
    need = pa_decode_workspace_size(S, hq, hkv, d, bs, int(max_seq_len), partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_decode_shared_prefix", lib().pa_decode_shared_prefix(
        _ptr(out, "out"), _ptr(query, "query"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(prefix_blocks, "prefix_blocks", torch.int32, 1),
        int(prefix_len), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(seq_lens, "seq_lens", torch.int32, 1), S, hq, hkv, d, bs, nb,
        int(block_tables.shape[1]), int(max_seq_len), int(partition_tokens), float(scale),
        _dtype_code(key_cache), ws_ptr, ws_bytes, _stream(stream)))
    return out


def pa_append_decode_fp8(out, query, new_key, new_value, key_cache, value_cache, block_tables,
                         ctx_lens, max_ctx_len, scale, k_scale, v_scale, slot_mapping=None,
                         workspace=None, partition_tokens=0, stream=None):
    """pa_append_decode over FP8 (E4M3, uint8) caches: the new tokens are
    written as E4M3 codes of value / scale, then the decode runs over
    ctx_lens + 1 tokens, in one launch (include/pa.h, pa_append_decode_fp8)."""
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if key_cache.dtype != torch.uint8:
        raise ValueError("FP8 caches must be uint8 tensors of E4M3 codes")
    if query.dim() != 3 or query.shape[2] != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs][num_q_heads][head_dim]")
    if out.dtype != query.dtype or new_key.dtype != query.dtype or new_value.dtype != query.dtype:
        raise ValueError("out / new_key / new_value dtype must match the query")
    S, hq = int(query.shape[0]), int(query.shape[1])
    if new_key.shape != (S, hkv, d) or new_value.shape != (S, hkv, d):
        raise ValueError("new_key/new_value must be [num_seqs][num_kv_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or ctx_lens.numel() != S:
        raise ValueError("block_tables / ctx_lens do not match the batch")
    need = pa_decode_workspace_size(S, hq, hkv, d, bs, int(max_ctx_len) + 1, partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    slot_ptr = _ptr(slot_mapping, "slot_mapping", torch.int64, 1) if slot_mapping is not None \
        else None
    _check("pa_append_decode_fp8", lib().pa_append_decode_fp8(
        _ptr(out, "out"), _ptr(query, "query"), _ptr(new_key, "new_key"),
        _ptr(new_value, "new_value"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(ctx_lens, "ctx_lens", torch.int32, 1), slot_ptr, S, hq, hkv, d, bs, nb,
        int(block_tables.shape[1]), int(max_ctx_len), int(partition_tokens), float(scale),
        float(k_scale), float(v_scale), _dtype_code(query), ws_ptr, ws_bytes, _stream(stream)))
    return out


PA_STATIC_WORKSPACE_BYTES = 16 << 20


def pa_decode_static_workspace(out, query, key_cache, value_cache, block_tables, seq_lens,
                               max_seq_len, scale, partition_tokens=0, stream=None):
    """pa_decode with its scratch in the library's own per-device array.

    For callers that must not allocate device memory (see include/pa.h): no
    workspace argument, nothing allocated here or in the library.  Requests
    needing more than PA_STATIC_WORKSPACE_BYTES of scratch raise PAError
    (PA_ERR_WORKSPACE); concurrent calls on one device must be serialised.
    """
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if query.dim() != 3 or query.shape[2] != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs][num_q_heads][head_dim]")
    if query.dtype != key_cache.dtype or out.dtype != key_cache.dtype:
        raise ValueError("query/out dtype must match the cache")
    S, hq = int(query.shape[0]), int(query.shape[1])
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.numel() != S:
        raise ValueError("block_tables / seq_lens do not match the batch")
    _check("pa_decode_static_workspace", lib().pa_decode_static_workspace(
        _ptr(out, "out"), _ptr(query, "query"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(seq_lens, "seq_lens", torch.int32, 1), S, hq, hkv, d, bs, nb,
        int(block_tables.shape[1]), int(max_seq_len), int(partition_tokens), float(scale),
        _dtype_code(key_cache), _stream(stream)))
    return out


def pa_prefill_workspace_size(head_dim=128) -> int:
    n = ctypes.c_size_t(0)
    _check("pa_prefill_workspace_size",
           lib().pa_prefill_workspace_size(int(head_dim), ctypes.byref(n)))
    return int(n.value)


def pa_prefill_chunk(out, query, key_cache, value_cache, block_tables, cu_q_lens, ctx_lens,
                     max_q_len, max_ctx_len, scale, workspace=None, split_tail=True,
                     stream=None):
    """Causal chunked-prefill attention against the paged context (include/pa.h).

    ``workspace``: a CUDA byte tensor of at least ``pa_prefill_workspace_size``
    bytes; allocated with torch when None and ``split_tail``.  With
    ``split_tail=False`` no workspace is passed and no unit is split.
    """
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if query.dim() != 3 or query.shape[2] != d or out.shape != query.shape:
        raise ValueError("query/out must be [total_q][num_q_heads][head_dim]")
    if query.dtype != key_cache.dtype or out.dtype != key_cache.dtype:
        raise ValueError("query/out dtype must match the cache")
    S = int(ctx_lens.numel())
    if cu_q_lens.numel() != S + 1 or block_tables.dim() != 2 or block_tables.shape[0] != S:
        raise ValueError("cu_q_lens / block_tables do not match ctx_lens")
    if split_tail and workspace is None:
        workspace = torch.empty(pa_prefill_workspace_size(d), dtype=torch.uint8,
                                device=query.device)
    if not split_tail:
        workspace = None
    ws_ptr = _ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_prefill_chunk", lib().pa_prefill_chunk(
        _ptr(out, "out"), _ptr(query, "query"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(cu_q_lens, "cu_q_lens", torch.int32, 1), _ptr(ctx_lens, "ctx_lens", torch.int32, 1),
        S, int(query.shape[0]), int(max_q_len), int(max_ctx_len), int(query.shape[1]), hkv, d,
        bs, nb, int(block_tables.shape[1]), float(scale), _dtype_code(key_cache), ws_ptr,
        ws_bytes, _stream(stream)))
    return out


def pa_mixed_workspace_size(num_decode_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                            max_ctx_len, partition_tokens=0) -> int:
    n = ctypes.c_size_t(0)
    _check("pa_mixed_workspace_size", lib().pa_mixed_workspace_size(
        int(num_decode_seqs), int(num_q_heads), int(num_kv_heads), int(head_dim),
        int(block_size), int(max_ctx_len), int(partition_tokens), ctypes.byref(n)))
    return int(n.value)


def pa_mixed_attention(out, query, key_cache, value_cache, block_tables, cu_q_lens, ctx_lens,
                       num_decode_seqs, max_q_len, max_ctx_len, scale, workspace=None,
                       partition_tokens=0, stream=None):
    """Decode rows and prefill chunks in one launch (include/pa.h, pa_mixed_attention).

    The first ``num_decode_seqs`` sequences are decode rows (one query each,
    at row s); the rest are prefill chunks.  ``workspace`` is a CUDA byte
    tensor of at least ``pa_mixed_workspace_size`` bytes; allocated with
    torch when None.
    """
    nb, hkv, bs, d = _cache_dims(key_cache, value_cache)
    if query.dim() != 3 or query.shape[2] != d or out.shape != query.shape:
        raise ValueError("query/out must be [total_q][num_q_heads][head_dim]")
    if query.dtype != key_cache.dtype or out.dtype != key_cache.dtype:
        raise ValueError("query/out dtype must match the cache")
    S, hq = int(ctx_lens.numel()), int(query.shape[1])
    if cu_q_lens.numel() != S + 1 or block_tables.dim() != 2 or block_tables.shape[0] != S:
        raise ValueError("cu_q_lens / block_tables do not match ctx_lens")
    nd = int(num_decode_seqs)
    need = pa_mixed_workspace_size(nd, hq, hkv, d, bs, int(max_ctx_len), partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_mixed_attention", lib().pa_mixed_attention(
        _ptr(out, "out"), _ptr(query, "query"), _ptr(key_cache, "key_cache"),
        _ptr(value_cache, "value_cache"), _ptr(block_tables, "block_tables", torch.int32, 2),
        _ptr(cu_q_lens, "cu_q_lens", torch.int32, 1), _ptr(ctx_lens, "ctx_lens", torch.int32, 1),
        S, nd, int(query.shape[0]), int(max_q_len), int(max_ctx_len), hq, hkv, d, bs, nb,
        int(block_tables.shape[1]), int(partition_tokens), float(scale), _dtype_code(key_cache),
        ws_ptr, ws_bytes, _stream(stream)))
    return out


def pa_selftest_wait_timeout(limit_ns: int, waited_ns=None, stream=None) -> None:
    """Run the bounded-wait self-test kernel (include/pa.h): a wait with a
    limit of ``limit_ns`` on a barrier nothing arrives on, and a second wait
    of the same CTA that must give up with it.  ``waited_ns``: an int64 CUDA
    tensor of 2 elements receiving each wait's duration, or None."""
    ptr = _ptr(waited_ns, "waited_ns", torch.int64, 1) if waited_ns is not None else None
    if waited_ns is not None and waited_ns.numel() != 2:
        raise ValueError("waited_ns must hold 2 elements")
    _check("pa_selftest_wait_timeout",
           lib().pa_selftest_wait_timeout(int(limit_ns), ptr, _stream(stream)))


def pa_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    w = ctypes.c_uint(0)
    st = lib().pa_get_device_error(ctypes.byref(w), _stream(stream))
    if st not in (PA_OK, PA_ERR_OUT_OF_RANGE):
        raise PAError("pa_get_device_error", st)
    return int(w.value)


class BlockManager:
    """Handle on the library's host block manager (include/pa.h, pa_bm_*).

    Marshalling only: token ids in, block tables / slots / copy pairs out as
    numpy arrays.  ``add_sequence`` / ``append`` raise PAError with
    PA_ERR_OUT_OF_RANGE when the pool is exhausted (state unchanged).
    """

    def __init__(self, num_blocks: int, block_size: int, enable_prefix_caching: bool = True):
        import numpy as np  # local: the rest of the binding needs only torch
        self._np = np
        h = ctypes.c_void_p()
        _check("pa_bm_create", lib().pa_bm_create(int(num_blocks), int(block_size),
                                                   int(bool(enable_prefix_caching)),
                                                   ctypes.byref(h)))
        self._h = h
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _tokens(self, tokens):
        a = self._np.ascontiguousarray(tokens, dtype=self._np.int32)
        return a, a.ctypes.data_as(ctypes.c_void_p)

    def add_sequence(self, seq_id: int, tokens) -> int:
        a, ptr = self._tokens(tokens)
        cached = ctypes.c_int(0)
        _check("pa_bm_add_sequence", lib().pa_bm_add_sequence(self._h, int(seq_id), ptr, a.size,
                                                              ctypes.byref(cached)))
        return int(cached.value)

    def append(self, seq_id: int, tokens) -> None:
        a, ptr = self._tokens(tokens)
        _check("pa_bm_append", lib().pa_bm_append(self._h, int(seq_id), ptr, a.size))

    def fork(self, parent_id: int, child_id: int) -> None:
        _check("pa_bm_fork", lib().pa_bm_fork(self._h, int(parent_id), int(child_id)))

    def free(self, seq_id: int) -> None:
        _check("pa_bm_free", lib().pa_bm_free(self._h, int(seq_id)))

    def block_table(self, seq_id: int, capacity: int = None):
        n = ctypes.c_int(0)
        lib().pa_bm_block_table(self._h, int(seq_id), None, 0, ctypes.byref(n))
        cap = n.value if capacity is None else int(capacity)
        out = self._np.empty(cap, dtype=self._np.int32)
        _check("pa_bm_block_table", lib().pa_bm_block_table(
            self._h, int(seq_id), out.ctypes.data_as(ctypes.c_void_p), cap, ctypes.byref(n)))
        return out

    def slots(self, seq_id: int, start: int, count: int):
        out = self._np.empty(int(count), dtype=self._np.int64)
        _check("pa_bm_slots", lib().pa_bm_slots(self._h, int(seq_id), int(start), int(count),
                                                out.ctypes.data_as(ctypes.c_void_p)))
        return out

    def take_copies(self):
        n = -lib().pa_bm_take_copies(self._h, None, 0)
        n = max(n, 0)
        out = self._np.empty((n, 2), dtype=self._np.int64)
        got = lib().pa_bm_take_copies(self._h, out.ctypes.data_as(ctypes.c_void_p), n)
        if got < 0:
            raise RuntimeError("pa_bm_take_copies: capacity mismatch")
        return out[:got]

    @property
    def num_free_blocks(self) -> int:
        return int(lib().pa_bm_num_free_blocks(self._h))

    def ref_count(self, block: int) -> int:
        return int(lib().pa_bm_ref_count(self._h, int(block)))

    def num_tokens(self, seq_id: int) -> int:
        return int(lib().pa_bm_num_tokens(self._h, int(seq_id)))

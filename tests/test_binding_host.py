"""The Python binding's marshalling, without a GPU.

* The ctypes signature table agrees with every prototype in include/pa.h
  (parameter count and C types, return type), so no argument is passed with
  the wrong width.
* Every tensor wrapper, driven through a stand-in for libpa.so that records
  its arguments, passes exactly as many arguments as the C call takes, with
  the sizes derived from the tensor shapes.
* The current-device check refuses a tensor that lives on another device.
"""
import ctypes
import os
import re
import types

import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_P, _I = ctypes.c_void_p, ctypes.c_int
_C_TYPES = {
    "int": _I, "float": ctypes.c_float, "size_t": ctypes.c_size_t, "int64_t": ctypes.c_int64,
    "uint64_t": ctypes.c_uint64,
    "pa_dtype": _I, "pa_stream_t": _P, "pa_status": _I, "void": None,
    "const char *": ctypes.c_char_p, "int *": ctypes.POINTER(_I),
    "size_t *": ctypes.POINTER(ctypes.c_size_t), "unsigned int *": ctypes.POINTER(ctypes.c_uint),
    "pa_block_manager **": ctypes.POINTER(_P),
}


def _ctype(decl: str):
    t = re.sub(r"\s+", " ", decl.replace("*", " * ")).strip()
    t = re.sub(r"\bconst\b ", "", t) if t.startswith("const") and t != "const char *" else t
    t = t.replace("* *", "**")
    if t in _C_TYPES:
        return _C_TYPES[t]
    if t.endswith("*"):
        return _P  # any other data pointer (device or host buffer, handle)
    raise AssertionError(f"unmapped C type {decl!r}")


def _prototypes():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {}
    for ret, name, params in re.findall(
            r"([A-Za-z_][\w\s\*]*?)\s*\b(pa_[a-z0-9_]+)\s*\(([^()]*)\)\s*;", text):
        args = []
        params = params.strip()
        if params and params != "void":
            for p in params.split(","):
                p = p.strip()
                m = re.match(r"(.*?)(\w+)$", p)  # drop the parameter name
                args.append(_ctype(m.group(1)))
        protos[name] = (_ctype(ret.strip()), args)
    return protos


def test_signature_table_matches_the_header():
    protos = _prototypes()
    assert sorted(protos) == sorted(pa._SIGS)
    for name, (res, args) in pa._SIGS.items():
        want_res, want_args = protos[name]
        assert res == want_res, f"{name}: return type"
        assert len(args) == len(want_args), f"{name}: {len(args)} args, header has {len(want_args)}"
        for i, (got, want) in enumerate(zip(args, want_args)):
            assert got == want, f"{name}: argument {i} is {got}, header says {want}"


class _RecordingLib:
    """Stands in for libpa.so: records each call and returns PA_OK (sizes
    written through pointers stay zero, so no workspace is allocated)."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name not in pa._SIGS:
            raise AttributeError(name)

        def call(*args):
            self.calls.append((name, args))
            return pa.PA_OK
        return call

    def last(self, name):
        got = [a for n, a in self.calls if n == name]
        assert got, f"{name} was not called"
        return got[-1]


@pytest.fixture
def rec(monkeypatch):
    lib = _RecordingLib()
    monkeypatch.setattr(pa, "lib", lambda: lib)
    real_ptr = pa._ptr

    def ptr(t, name, dtype=None, ndim=None):
        # the real checks, with CPU tensors standing in for device ones
        if t is None:
            return None
        assert isinstance(t, torch.Tensor) and t.is_contiguous(), name
        if dtype is not None:
            assert t.dtype == dtype, f"{name}: {t.dtype}"
        if ndim is not None:
            assert t.dim() == ndim, f"{name}: {t.dim()} dims"
        return t.data_ptr()
    assert real_ptr is not ptr
    monkeypatch.setattr(pa, "_ptr", ptr)
    monkeypatch.setattr(pa, "_pool_ptr", lambda t, name: t.data_ptr())
    monkeypatch.setattr(pa, "_stream", lambda s: 0)
    return lib


def _arity(lib, name):
    args = lib.last(name)
    assert len(args) == len(pa._SIGS[name][1]), f"{name}: {len(args)} arguments"
    return args


def test_every_wrapper_passes_the_c_arity_and_shape_sizes(rec):
    w = synth.random_decode(5, [3, 40, 17], dtype=torch.bfloat16, block_size=16, hq=8, hkv=2,
                            d=64)
    kc, vc, bt, ctx, q = w.key_cache, w.value_cache, w.block_tables, w.context_lens, w.query
    nb, hkv, B, D = kc.shape
    S, hq = q.shape[0], q.shape[1]
    width = bt.shape[1]
    out = torch.empty_like(q)
    slots = torch.zeros(S, dtype=torch.int64)

    pa.pa_slot_mapping(slots, bt, ctx, B)
    a = _arity(rec, "pa_slot_mapping")
    assert a[4:8] == (S, S, width, B)

    pa.pa_reshape_and_cache(w.new_key, w.new_value, kc, vc, slots)
    a = _arity(rec, "pa_reshape_and_cache")
    assert a[5:11] == (S, hkv, D, B, nb, pa.PA_BF16)

    pa.pa_append(w.new_key, w.new_value, kc, vc, bt, ctx)
    a = _arity(rec, "pa_append")
    assert a[8:16] == (S, S, width, hkv, D, B, nb, pa.PA_BF16)

    pairs = torch.tensor([[0, 1], [2, 3]], dtype=torch.int64)
    pa.pa_copy_blocks(kc, vc, pairs)
    a = _arity(rec, "pa_copy_blocks")
    assert a[3:9] == (2, hkv, D, B, nb, pa.PA_BF16)

    host_k, host_v = torch.empty(4, hkv, B, D, dtype=kc.dtype), torch.empty(4, hkv, B, D,
                                                                              dtype=kc.dtype)
    pa.pa_swap_blocks(host_k, host_v, kc, vc, pairs)
    a = _arity(rec, "pa_swap_blocks")
    assert a[5:12] == (2, hkv, D, B, nb, 4, pa.PA_BF16)

    pa.pa_decode(out, q, kc, vc, bt, ctx + 1, 41, 0.125, partition_tokens=32)
    a = _arity(rec, "pa_decode")
    assert a[6:16] == (S, hq, hkv, D, B, nb, width, 41, 32, 0.125)
    assert a[16] == pa.PA_BF16
    _arity(rec, "pa_decode_workspace_size")

    pa.pa_append_decode(out, q, w.new_key, w.new_value, kc, vc, bt, ctx, 40, 0.125,
                        slot_mapping=slots)
    a = _arity(rec, "pa_append_decode")
    assert a[9:18] == (S, hq, hkv, D, B, nb, width, 40, 0)

    pa.pa_decode_shared_prefix(out, q, kc, vc, bt[0, :1].contiguous(), 16, bt, ctx + 1, 41,
                               0.125, partition_tokens=16)
    a = _arity(rec, "pa_decode_shared_prefix")
    assert a[5] == 16 and a[8:18] == (S, hq, hkv, D, B, nb, width, 41, 16, 0.125)

    pa.pa_decode_static_workspace(out, q, kc, vc, bt, ctx + 1, 41, 0.125)
    a = _arity(rec, "pa_decode_static_workspace")
    assert a[6:15] == (S, hq, hkv, D, B, nb, width, 41, 0)

    kc8 = torch.zeros(kc.shape, dtype=torch.uint8)
    vc8 = torch.zeros(kc.shape, dtype=torch.uint8)
    pa.pa_reshape_and_cache_fp8(w.new_key, w.new_value, kc8, vc8, slots, 0.5, 0.25)
    a = _arity(rec, "pa_reshape_and_cache_fp8")
    assert a[5:13] == (S, hkv, D, B, nb, 0.5, 0.25, pa.PA_BF16)

    pa.pa_decode_fp8(out, q, kc8, vc8, bt, ctx + 1, 41, 0.125, 0.5, 0.25)
    a = _arity(rec, "pa_decode_fp8")
    assert a[6:18] == (S, hq, hkv, D, B, nb, width, 41, 0, 0.125, 0.5, 0.25)

    pa.pa_append_decode_fp8(out, q, w.new_key, w.new_value, kc8, vc8, bt, ctx, 40, 0.125, 0.5,
                            0.25, slot_mapping=slots)
    a = _arity(rec, "pa_append_decode_fp8")
    assert a[9:22] == (S, hq, hkv, D, B, nb, width, 40, 0, 0.125, 0.5, 0.25, pa.PA_BF16)

    p = synth.chunked_prefill(seed=1, block_size=16, hq=4, hkv=2, d=128, ctx_lens=[5, 0],
                              q_lens=[7, 3], dtype=torch.float16)
    pout = torch.empty_like(p.query)
    pnb = p.key_cache.shape[0]
    pw = p.block_tables.shape[1]
    pa.pa_prefill_chunk(pout, p.query, p.key_cache, p.value_cache, p.block_tables, p.cu_q_lens,
                        p.ctx_lens, 7, 5, 0.1)
    a = _arity(rec, "pa_prefill_chunk")
    assert a[7:18] == (2, 10, 7, 5, 4, 2, 128, 16, pnb, pw, 0.1)
    assert a[18] == pa.PA_F16
    _arity(rec, "pa_prefill_workspace_size")

    pa.pa_mixed_attention(pout, p.query, p.key_cache, p.value_cache, p.block_tables, p.cu_q_lens,
                          p.ctx_lens, 1, 7, 5, 0.1)
    a = _arity(rec, "pa_mixed_attention")
    assert a[7:19] == (2, 1, 10, 7, 5, 4, 2, 128, 16, pnb, pw, 0)
    _arity(rec, "pa_mixed_workspace_size")

    assert pa.pa_get_device_error() == 0
    _arity(rec, "pa_get_device_error")

    pa.pa_selftest_wait_timeout(1_000_000)
    a = _arity(rec, "pa_selftest_wait_timeout")
    assert a[0] == 1_000_000 and a[1] is None

    host_only = {"pa_status_string", "pa_version", "pa_decode_partition_tokens"}
    called = {n for n, _ in rec.calls}
    untested = [n for n in pa._SIGS if n not in called and n not in host_only
                and not n.startswith("pa_bm_")]
    assert not untested, f"wrappers not driven: {untested}"


def test_current_device_check(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    pa._check_device(types.SimpleNamespace(device=torch.device("cuda", 0)), "x")
    with pytest.raises(ValueError, match="current device is cuda:0"):
        pa._check_device(types.SimpleNamespace(device=torch.device("cuda", 1)), "x")

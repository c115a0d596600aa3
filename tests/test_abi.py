"""The C ABI library loads on a CPU-only machine, exports every symbol that
include/pa.h declares, and rejects bad host arguments before launching."""
import ctypes
import os
import re
import subprocess

import pytest

import paged_kv_cache_397_b200 as pa
from paged_kv_cache_397_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return pa.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("pa_reshape_and_cache", "pa_decode", "pa_prefill_chunk", "pa_copy_blocks",
              "pa_decode_workspace_size", "pa_slot_mapping", "pa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.lib_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (pa_[a-z0-9_]+)\b", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    assert sorted(pa.EXPORTED_SYMBOLS) == _declared()
    assert "pa_bm_create" in _declared()
    for n in _declared():
        assert hasattr(lib, n)


def test_status_strings(lib):
    assert pa.pa_status_string(0) == "PA_OK"
    assert pa.pa_status_string(pa.PA_ERR_WORKSPACE) == "PA_ERR_WORKSPACE"
    assert pa.pa_status_string(99) == "PA_ERR_UNKNOWN"
    assert pa.pa_version() >> 16 == 1


def test_workspace_size_is_host_only(lib):
    # single partition -> no workspace; long context -> partials for every partition
    assert pa.pa_decode_workspace_size(4, 4, 4, 64, 16, 65, partition_tokens=128) == 0
    n = pa.pa_decode_workspace_size(16, 32, 8, 128, 16, 32768, partition_tokens=512)
    assert n >= 16 * 32 * 64 * (128 + 2) * 4
    pt = pa.pa_decode_partition_tokens(256, 8, 16, 4097)
    assert pt % 16 == 0 and pt >= 256
    assert pa.pa_decode_partition_tokens(1, 1, 32, 10) % 32 == 0
    with pytest.raises(pa.PAError):
        pa.pa_decode_workspace_size(4, 0, 4, 64, 16, 65)
    # prefill: counters + two waves (148 SMs without a GPU) of 256-row fp32 partials
    assert pa.pa_prefill_workspace_size(128) == 256 + 1024 + 2 * 148 * 256 * 130 * 4
    # mixed batches: no decode rows -> none; decode rows -> the queue counter
    # block (+ slack), plus partials once they span several partitions
    assert pa.pa_mixed_workspace_size(0, 8, 2, 128, 16, 100) == 0
    assert pa.pa_mixed_workspace_size(4, 8, 2, 128, 16, 100, partition_tokens=256) == 512
    assert pa.pa_mixed_workspace_size(4, 8, 2, 128, 16, 4000, partition_tokens=256) == \
        512 + 4 * 8 * 16 * (128 + 2) * 4
    # automatic partitions of a mixed batch are at most 1024 tokens (pa_decode
    # would take 2048 for this batch)
    assert pa.pa_decode_partition_tokens(256, 8, 16, 4096) == 2048
    assert pa.pa_mixed_workspace_size(256, 32, 8, 128, 16, 4095) == 512 + 256 * 32 * 4 * 130 * 4
    # a requested partition longer than every sequence is one partition (its
    # rounding to whole blocks does not overflow)
    assert pa.pa_decode_workspace_size(4, 4, 4, 64, 16, 5000, partition_tokens=2**31 - 1) == 0
    assert pa.pa_mixed_workspace_size(4, 8, 2, 128, 16, 100, partition_tokens=2**31 - 1) == 512
    with pytest.raises(pa.PAError):
        pa.pa_mixed_workspace_size(4, 8, 2, 128, 16, 2**31 - 1)  # decode rows see ctx + 1


P = ctypes.c_void_p
FAKE = P(0x100000)  # never dereferenced: every call below fails validation first


def test_decode_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, sl=FAKE, S=4, hq=8, hkv=2, d=128,
                 bs=16, nb=64, mb=8, maxl=100, pt=0, scale=0.1, dt=pa.PA_BF16, ws=None,
                 wsb=0, st=None)
        a.update(kw)
        return lib.pa_decode(a["out"], a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["S"],
                             a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["mb"], a["maxl"],
                             a["pt"], a["scale"], a["dt"], a["ws"], a["wsb"], a["st"])

    assert call(out=None) == pa.PA_ERR_INVALID_ARG
    assert call(hq=6, hkv=4) == pa.PA_ERR_INVALID_ARG           # Hq % Hkv != 0
    assert call(maxl=8 * 16 + 1) == pa.PA_ERR_INVALID_ARG       # longer than the table
    assert call(q=P(0x100004)) == pa.PA_ERR_INVALID_ARG         # misaligned
    assert call(dt=7) == pa.PA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert call(bs=8, mb=64) == pa.PA_ERR_UNSUPPORTED
    assert call(d=96) == pa.PA_ERR_UNSUPPORTED
    assert call(hq=34, hkv=1) == pa.PA_ERR_UNSUPPORTED          # group > 16
    assert call(maxl=128, pt=16) == pa.PA_ERR_WORKSPACE         # 8 partitions, no workspace
    # a length near INT_MAX: over 65535 partitions, refused without overflowing
    assert call(maxl=2**31 - 10, mb=2**27) == pa.PA_ERR_INVALID_ARG
    assert call(S=0) == pa.PA_OK                                # empty batch: nothing to do


def test_prefill_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cu=FAKE, cl=FAKE, S=2, tq=64,
                 mq=32, mc=100, hq=8, hkv=2, d=128, bs=16, nb=64, mb=16, scale=0.1,
                 dt=pa.PA_BF16, ws=None, wsb=0, st=None)
        a.update(kw)
        return lib.pa_prefill_chunk(a["out"], a["q"], a["kc"], a["vc"], a["bt"], a["cu"],
                                    a["cl"], a["S"], a["tq"], a["mq"], a["mc"], a["hq"],
                                    a["hkv"], a["d"], a["bs"], a["nb"], a["mb"], a["scale"],
                                    a["dt"], a["ws"], a["wsb"], a["st"])

    assert call(cu=None) == pa.PA_ERR_INVALID_ARG
    assert call(mc=16 * 16) == pa.PA_ERR_INVALID_ARG            # context fills the table
    assert call(hq=3, hkv=2) == pa.PA_ERR_INVALID_ARG
    assert call(d=96) == pa.PA_ERR_UNSUPPORTED                   # head_dim 64 or 128
    assert call(bs=64, mb=4) == pa.PA_ERR_UNSUPPORTED
    assert call(tq=0) == pa.PA_OK


def test_mixed_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cu=FAKE, cl=FAKE, S=6, nd=4,
                 tq=68, mq=32, mc=100, hq=8, hkv=2, d=128, bs=16, nb=64, mb=16, pt=0,
                 scale=0.1, dt=pa.PA_BF16, ws=None, wsb=0, st=None)
        a.update(kw)
        return lib.pa_mixed_attention(a["out"], a["q"], a["kc"], a["vc"], a["bt"], a["cu"],
                                      a["cl"], a["S"], a["nd"], a["tq"], a["mq"], a["mc"],
                                      a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["mb"],
                                      a["pt"], a["scale"], a["dt"], a["ws"], a["wsb"], a["st"])

    assert call(nd=7) == pa.PA_ERR_INVALID_ARG                  # more decode rows than seqs
    assert call(tq=3) == pa.PA_ERR_INVALID_ARG                  # fewer rows than decode seqs
    assert call(cu=None) == pa.PA_ERR_INVALID_ARG
    assert call(mc=16 * 16) == pa.PA_ERR_INVALID_ARG            # ctx + 1 does not fit the table
    assert call(mc=2**31 - 1, mb=2**27) == pa.PA_ERR_INVALID_ARG  # ctx + 1 is not an int
    assert call(hq=3, hkv=2) == pa.PA_ERR_INVALID_ARG
    assert call(q=P(0x100004)) == pa.PA_ERR_INVALID_ARG         # misaligned
    assert call(d=64) == pa.PA_ERR_UNSUPPORTED
    assert call(hq=34, hkv=2) == pa.PA_ERR_UNSUPPORTED          # group 17
    assert call(bs=64, mb=4) == pa.PA_ERR_UNSUPPORTED
    # decode rows long enough to split need a workspace
    assert call(mc=4000, mb=256, pt=256) == pa.PA_ERR_WORKSPACE
    assert call(tq=0, nd=0) == pa.PA_OK
    assert call(S=0, nd=0) == pa.PA_OK


def test_append_decode_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, nk=FAKE, nv=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE,
                 sm=None, S=4, hq=8, hkv=2, d=128, bs=16, nb=64, mb=8, mc=100, pt=0,
                 scale=0.1, dt=pa.PA_BF16, ws=None, wsb=0, st=None)
        a.update(kw)
        return lib.pa_append_decode(a["out"], a["q"], a["nk"], a["nv"], a["kc"], a["vc"],
                                    a["bt"], a["cl"], a["sm"], a["S"], a["hq"], a["hkv"],
                                    a["d"], a["bs"], a["nb"], a["mb"], a["mc"], a["pt"],
                                    a["scale"], a["dt"], a["ws"], a["wsb"], a["st"])

    assert call(nk=None) == pa.PA_ERR_INVALID_ARG
    assert call(nv=P(0x100008)) == pa.PA_ERR_INVALID_ARG          # misaligned
    assert call(mc=8 * 16) == pa.PA_ERR_INVALID_ARG               # ctx + 1 does not fit
    assert call(mc=-1) == pa.PA_ERR_INVALID_ARG
    assert call(mc=2**31 - 1, mb=2**27) == pa.PA_ERR_INVALID_ARG  # ctx + 1 is not an int
    assert call(dt=pa.PA_FP8_E4M3) == pa.PA_ERR_INVALID_ARG       # fp16 / bf16 only
    assert call(bs=8, mb=64) == pa.PA_ERR_UNSUPPORTED
    assert call(S=0) == pa.PA_OK


def test_decode_shared_prefix_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, pb=FAKE, pl=32, bt=FAKE, sl=FAKE, S=4,
                 hq=8, hkv=2, d=128, bs=16, nb=64, mb=8, ml=100, pt=0, scale=0.1, dt=pa.PA_BF16,
                 ws=None, wsb=0, st=None)
        a.update(kw)
        return lib.pa_decode_shared_prefix(a["out"], a["q"], a["kc"], a["vc"], a["pb"], a["pl"],
                                           a["bt"], a["sl"], a["S"], a["hq"], a["hkv"], a["d"],
                                           a["bs"], a["nb"], a["mb"], a["ml"], a["pt"],
                                           a["scale"], a["dt"], a["ws"], a["wsb"], a["st"])

    assert call(pl=-16) == pa.PA_ERR_INVALID_ARG
    assert call(pl=24) == pa.PA_ERR_INVALID_ARG            # not a multiple of block_size
    assert call(pl=112) == pa.PA_ERR_INVALID_ARG           # beyond max_seq_len
    assert call(pb=None) == pa.PA_ERR_INVALID_ARG
    assert call(ml=8 * 16 + 1) == pa.PA_ERR_INVALID_ARG    # as pa_decode
    assert call(S=0) == pa.PA_OK


def test_append_decode_fp8_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, nk=FAKE, nv=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE,
                 sm=None, S=4, hq=8, hkv=2, d=128, bs=16, nb=64, mb=8, mc=100, pt=0,
                 scale=0.1, ks=0.5, vs=0.25, dt=pa.PA_BF16, ws=None, wsb=0, st=None)
        a.update(kw)
        return lib.pa_append_decode_fp8(a["out"], a["q"], a["nk"], a["nv"], a["kc"], a["vc"],
                                        a["bt"], a["cl"], a["sm"], a["S"], a["hq"], a["hkv"],
                                        a["d"], a["bs"], a["nb"], a["mb"], a["mc"], a["pt"],
                                        a["scale"], a["ks"], a["vs"], a["dt"], a["ws"],
                                        a["wsb"], a["st"])

    assert call(nk=None) == pa.PA_ERR_INVALID_ARG
    assert call(nv=P(0x100008)) == pa.PA_ERR_INVALID_ARG          # misaligned
    assert call(mc=8 * 16) == pa.PA_ERR_INVALID_ARG               # ctx + 1 does not fit
    assert call(mc=-1) == pa.PA_ERR_INVALID_ARG
    assert call(ks=0.0) == pa.PA_ERR_INVALID_ARG                  # scales positive, finite
    assert call(vs=float("inf")) == pa.PA_ERR_INVALID_ARG
    assert call(dt=pa.PA_FP8_E4M3) == pa.PA_ERR_INVALID_ARG       # query type fp16 / bf16
    assert call(d=64) == pa.PA_ERR_UNSUPPORTED                    # head_dim 128 only
    assert call(S=0) == pa.PA_OK


def test_cache_ops_reject_bad_arguments(lib):
    assert lib.pa_reshape_and_cache(None, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 16, 8, 1,
                                    None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 8, 8, 1,
                                    None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 128, 16, 8, 1,
                                    None) == pa.PA_OK
    assert lib.pa_copy_blocks(FAKE, None, FAKE, 3, 2, 128, 16, 8, 1, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 0, 2, 128, 16, 8, 1, None) == pa.PA_OK
    assert lib.pa_slot_mapping(FAKE, FAKE, None, FAKE, 3, 4, 8, 16, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_slot_mapping(FAKE, FAKE, None, FAKE, 3, 0, 8, 16, None) == pa.PA_OK


def test_binding_refuses_cpu_tensors(lib):
    import torch
    kc = torch.zeros(4, 2, 16, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        pa.pa_copy_blocks(kc, kc.clone(), torch.zeros(1, 2, dtype=torch.int64))


def test_wait_timeout_selftest_rejects_bad_limits(lib):
    # limits outside 1 us .. 100 ms and a misaligned output are refused before any launch
    for limit in (0, 999, 100_000_001, 2**63):
        assert lib.pa_selftest_wait_timeout(limit, None, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_selftest_wait_timeout(1_000_000, ctypes.c_void_p(12), None) == \
        pa.PA_ERR_INVALID_ARG

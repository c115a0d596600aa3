"""The device-side failure path, exercised without breaking anything.

Every mbarrier wait in the library's kernels is bounded.  When one runs out,
the kernel records PA_DEVERR_WAIT_TIMEOUT in the device error word, raises its
CTA's abort word so that the CTA's other roles stop waiting at once, drains
its own copies in flight and returns.  pa_selftest_wait_timeout runs exactly
that on barriers nothing ever arrives on (a 1 ms limit for the first role, the
normal 4 s limit for the second, which must follow the abort word instead).
The test then checks that the host sees the error, that the context is still
usable (a decode afterwards matches the oracle with a clean error word), and
that the whole episode took milliseconds, not seconds.
"""
import time

import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth
from helpers import TOL, decode_reference, dev, max_err, to_dev

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_survives():
    pa.pa_get_device_error()
    waited = torch.full((2,), -1, dtype=torch.int64, device=dev())
    t0 = time.perf_counter()
    pa.pa_selftest_wait_timeout(1_000_000, waited)
    err = pa.pa_get_device_error()  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert err & pa.PA_DEVERR_WAIT_TIMEOUT
    w0, w1 = waited.tolist()
    assert 1_000_000 <= w0 < 100_000_000  # the first role waited out its 1 ms limit
    assert 0 <= w1 < 1_000_000_000  # the second gave up with it, far inside its 4 s limit
    assert elapsed < 2.0

    w = synth.random_decode(3, [1, 40, 300], dtype=torch.float16, hq=8, hkv=2, d=128,
                            append=False)
    lens = w.context_lens.tolist()
    out = torch.empty_like(w.query, device=dev())
    pa.pa_decode(out, to_dev(w.query), to_dev(w.key_cache), to_dev(w.value_cache),
                 to_dev(w.block_tables), to_dev(w.context_lens), max(lens), w.scale,
                 partition_tokens=64)
    assert pa.pa_get_device_error() == 0
    ref = decode_reference(w, lens, list(range(w.num_seqs)))
    assert max_err(out.cpu(), ref) <= TOL[w.dtype]


def test_wait_timeout_twice_in_a_row():
    # the abort word is per CTA and zeroed at its start: a second run behaves the same
    for _ in range(2):
        waited = torch.full((2,), -1, dtype=torch.int64, device=dev())
        pa.pa_selftest_wait_timeout(200_000, waited)
        assert pa.pa_get_device_error() & pa.PA_DEVERR_WAIT_TIMEOUT
        assert 200_000 <= waited[0].item() < 100_000_000
        assert 0 <= waited[1].item() < 1_000_000_000

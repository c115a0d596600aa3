"""FP8 (E4M3) KV cache: codec and paged decode — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use
this module; the CUDA library never does.

The pages name an FP8 KV cache as the way to halve bytes per block and raise
concurrency ("PagedAttention: KV cache as virtual memory", "Deep dive" and
"Interviewer follow-ups") but fix no format or scaling.  Readings taken:
  * the OCP 8-bit E4M3 encoding without infinities: 1 sign bit, 4 exponent
    bits (bias 7), 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6);
    S.1111.111 is NaN; the largest finite value is 448;
  * one fp32 scale per cache (k_scale, v_scale): a stored code represents
    code_value * scale;
  * writing a value x: q = fp32(x) / fp32(scale) in fp32 (IEEE division),
    then the nearest finite E4M3 value, ties to the even code, magnitudes
    above 448 saturate to 448, NaN stays NaN.

Pinned by ``tests/test_oracle_fp8.py`` (closed-form code values, torch's
float8_e4m3fn cast on the in-range domain, saturation and tie cases,
round trips).
"""
from __future__ import annotations

import numpy as np

from .paged_attention import paged_decode

__all__ = ["e4m3_value", "E4M3_TABLE", "e4m3_encode", "quantize", "paged_decode_fp8"]


def e4m3_value(code: int) -> float:
    """The real number an E4M3 code stands for (NaN for S.1111.111).

    The FP8 cache of "PagedAttention: KV cache as virtual memory", "Deep dive"
    names no format; this is the OCP E4M3 encoding read in the module header.
    """
    code = int(code) & 0xFF
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)

# non-negative finite codes 0x00..0x7E in increasing value order
_POS_VALUES = E4M3_TABLE[:0x7F]
_MAX = float(_POS_VALUES[-1])  # 448


def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 code of each float (ties to the even code, saturating).

    Writing into the FP8 cache of "PagedAttention: KV cache as virtual
    memory", "Deep dive"; the rounding rule is the reading in the module
    header (the pages fix none).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint8)
    flat_x = x.reshape(-1)
    flat_o = out.reshape(-1)
    mag = np.abs(flat_x)
    neg = np.signbit(flat_x)
    nan = np.isnan(flat_x)
    mag = np.where(nan, 0.0, np.minimum(mag, _MAX))
    # neighbours: the largest code value <= mag and the next one up
    hi = np.searchsorted(_POS_VALUES, mag, side="left")  # first value >= mag
    hi = np.minimum(hi, 0x7E)
    lo = np.where(_POS_VALUES[hi] > mag, hi - 1, hi)
    lo = np.maximum(lo, 0)
    d_lo = mag - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(neg, code | 0x80, code).astype(np.uint8)
    code = np.where(nan, np.uint8(0x7F), code)
    flat_o[:] = code
    return out


def quantize(x, scale: float) -> np.ndarray:
    """Codes of values x (any float array, exact in fp32) under a per-cache scale:
    fp32 division, then e4m3_encode.

    The per-cache scale is the module header's reading of the FP8 cache of
    "PagedAttention: KV cache as virtual memory", "Deep dive" and
    "Interviewer follow-ups".
    """
    q = np.asarray(x, dtype=np.float32) / np.float32(scale)
    return e4m3_encode(q.astype(np.float32))


def paged_decode_fp8(query, key_codes, value_codes, block_tables, seq_lens, scale, k_scale,
                     v_scale, num_kv_heads):
    """Paged decode over FP8 caches: the codes stand for code_value * scale;
    attention is then exactly the fp64 paged decode of those values.

    "PagedAttention: KV cache as virtual memory", "Interviewer follow-ups"
    (an FP8 KV cache halves the bytes per block; attention itself is
    unchanged), with the decode of "vLLM PagedAttention Deep Dive",
    "PagedAttention Mechanism".
    """
    kc = E4M3_TABLE[np.asarray(key_codes, dtype=np.uint8)] * float(np.float32(k_scale))
    vc = E4M3_TABLE[np.asarray(value_codes, dtype=np.uint8)] * float(np.float32(v_scale))
    return paged_decode(query, kc, vc, block_tables, seq_lens, scale, num_kv_heads)

"""8-bit floating-point KV cache (FP8 E4M3), oracle side.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline may use this module. It shares no code with the CUDA-side library.

The pages name KV-cache quantization as the next lever on a bandwidth-bound
path ("PagedAttention: The vLLM Paper", "Impact and Follow-Ups" and
"Limitations") but fix no format. Reading taken: the OCP 8-bit floating-point
format E4M3 (the variant without infinities), one scale per cache tensor:

  * a code is sign (1 bit), exponent e (4 bits, bias 7) and mantissa m (3 bits);
    e > 0: (-1)^s * 2^(e-7) * (1 + m/8); e = 0: (-1)^s * 2^-6 * m/8;
    e = 15 with m = 7 is NaN (codes 0x7F, 0xFF); the largest finite magnitude
    is 448 (code 0x7E);
  * storing x (a 16-bit key or value element) writes
    code = E4M3(float32(x) / float32(scale)), the division in float32 with
    round-to-nearest and the conversion rounding to the nearest code, ties to
    the even mantissa, magnitudes past 448 saturating to 448, the sign kept
    (also for results that round to zero);
  * reading a code gives decode(code) * scale; attention over the cache is the
    plain definition over those dequantized keys and values.
"""

import numpy as np

from oracle.attention import softmax_attention
from oracle.fpbits import bits_to_f64

MAX_E4M3 = 448.0


def decode_e4m3(code: int) -> float:
    """Value of one E4M3 code, from the format definition."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * 2.0 ** -6 * (m / 8.0)
    return sign * 2.0 ** (e - 7) * (1.0 + m / 8.0)


# the 127 non-negative finite magnitudes, code 0x00 .. 0x7E, in increasing order
_MAGNITUDES = [decode_e4m3(c) for c in range(0x7F)]


def encode_e4m3(x: float) -> int:
    """Nearest E4M3 code to ``x`` (ties to even mantissa, saturating, sign kept)."""
    x = float(x)
    if x != x:
        return 0x7F
    sign = 0x80 if (x < 0 or (x == 0 and np.signbit(x))) else 0x00
    a = abs(x)
    if a >= MAX_E4M3:
        return sign | 0x7E
    best = 0
    for c in range(1, 0x7F):
        da = abs(a - _MAGNITUDES[c])
        db = abs(a - _MAGNITUDES[best])
        if da < db or (da == db and c % 2 == 0 and best % 2 == 1):
            best = c
    return sign | best


def encode_e4m3_array(x) -> np.ndarray:
    """``encode_e4m3`` over an array: the two magnitudes around |x| by binary
    search, the nearer one taken, ties to the even code."""
    x = np.asarray(x, dtype=np.float64)
    mags = np.asarray(_MAGNITUDES)
    a = np.abs(x)
    hi = np.clip(np.searchsorted(mags, a), 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    dlo = np.abs(a - mags[lo])
    dhi = np.abs(a - mags[hi])
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= MAX_E4M3, 0x7E, pick)
    code = pick.astype(np.int64) | np.where(np.signbit(x), 0x80, 0x00)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def quantize(bits, dtype: str, scale: float) -> np.ndarray:
    """Codes of 16-bit elements (uint16 bit patterns of ``dtype``): divide by the
    scale in float32, then round to E4M3."""
    x = bits_to_f64(np.asarray(bits), dtype).astype(np.float32)
    with np.errstate(over="ignore"):     # a quotient past float32's range is inf: saturates
        q = (x / np.float32(scale)).astype(np.float32)
    return encode_e4m3_array(q)


def dequantize(codes, scale: float) -> np.ndarray:
    table = np.array([decode_e4m3(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)] * float(scale)


def reshape_and_cache_fp8(k_cache, v_cache, key, value, slot_mapping, block_size: int,
                          dtype: str, k_scale: float, v_scale: float):
    """Store token ``t``'s quantized keys/values ``[num_kv_heads, head_dim]`` at its
    slot of uint8 caches ``[num_blocks, num_kv_heads, block_size, head_dim]``;
    slots < 0 are skipped."""
    kq = quantize(key, dtype, k_scale)
    vq = quantize(value, dtype, v_scale)
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if slot < 0:
            continue
        block, offset = divmod(slot, block_size)
        k_cache[block, :, offset, :] = kq[t]
        v_cache[block, :, offset, :] = vq[t]


def paged_decode_fp8(q_bits, k_cache, v_cache, block_tables, context_lens, scale: float,
                     k_scale: float, v_scale: float, dtype: str, block_size: int = 16):
    """Decode attention over the dequantized paged cache: for sequence s and query
    head h, softmax(scale * K_s q) V_s with K_s, V_s the sequence's dequantized
    rows in logical order and query head h reading KV head h // G."""
    q = bits_to_f64(np.asarray(q_bits), dtype)
    B, hq, d = q.shape
    hkv = k_cache.shape[1]
    G = hq // hkv
    out = np.zeros((B, hq, d), np.float64)
    for s in range(B):
        n = int(context_lens[s])
        if n == 0:
            continue
        rows_k, rows_v = [], []
        for p in range(n):
            b = int(block_tables[s][p // block_size])
            rows_k.append(k_cache[b, :, p % block_size, :])
            rows_v.append(v_cache[b, :, p % block_size, :])
        K = dequantize(np.stack(rows_k), k_scale)    # [n, hkv, d]
        V = dequantize(np.stack(rows_v), v_scale)
        for h in range(hq):
            out[s, h] = softmax_attention(q[s, h], K[:, h // G], V[:, h // G], scale)
    return out

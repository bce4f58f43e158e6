"""FP8 (e4m3) KV cache with a per-tensor scale -- TEST INFRASTRUCTURE ONLY
(see the package docstring).

Sources (page title, section):
  * "从零构建LLM 推理引擎" (llminference.xinbetween.com), card "量化": decode
    speed is set by the bytes moved per token, so halving the bit width of
    every KV entry nearly halves decode latency; what remains is choosing where
    the error goes.
  * ursb.me Field Note "llm-inference-life", blurb: fp8 e4m3 versus e5m2.
  * "第三部分 · 推理系统与基础设施", chapter map 3.2 / 3.6: KV cache
    compression by quantisation; FP8 number formats.

Readings (the pages name the format, not its use):
  * Format: e4m3 -- 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
    exponent field 0 is subnormal (m/8 * 2^-6); no infinities; S.1111.111 is
    NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.
  * Scale: one float32 per pool (keys, values).  A cached entry is
    code = e4m3(x / scale) with x / scale taken in float32 (IEEE division),
    rounded to nearest, ties to even, saturated to +-448; the value it stands
    for is code * scale.  Q and the new K/V rows arrive in bf16.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """float64 value of every e4m3 byte (NaN codes give NaN).

    Source: ursb.me Field Note "llm-inference-life", blurb (fp8 e4m3); the
    bit layout is the format reading stated in this module's header.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.power(2.0, e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def e4m3_encode(x) -> np.ndarray:
    """Round float64 values (exact float32 values in practice) to e4m3 codes:
    nearest, ties to even, magnitudes above 448 saturate to 448.

    Source: as e4m3_decode; rounding and saturation are the readings stated
    in this module's header.
    """
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # quantisation step of the binade holding a: 2^(k-3) for a in [2^k, 2^(k+1)),
    # k >= -6; below 2^-6 (subnormals) the step is 2^-9
    with np.errstate(divide="ignore"):
        k = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    k = np.maximum(k, -6.0)
    step = np.power(2.0, k - 3.0)
    q = np.round(a / step) * step              # numpy rounds halves to even
    # a value rounded up into the next binade is still exact (q = 2^(k+1))
    e = np.floor(np.log2(np.where(q > 0, q, 1.0)))
    sub = q < 2.0 ** -6
    mant = np.where(sub, q / 2.0 ** -9, (q / np.power(2.0, e) - 1.0) * 8.0)
    expo = np.where(sub, 0, e + 7)
    code = (expo.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    code = np.where(q == 0, 0, code)
    return (code | np.where(sign, 0x80, 0)).astype(np.uint8)


def quantize(x, scale: float) -> np.ndarray:
    """Codes of x (bf16 / float32 values) for a pool with this scale: the
    float32 quotient x / scale, then e4m3_encode.

    Source: "从零构建LLM 推理引擎", card "量化" (fewer bits per KV entry); the per-pool scale is
    the reading stated in this module's header.
    """
    q = np.asarray(x, dtype=np.float32) / np.float32(scale)
    return e4m3_encode(q.astype(np.float64))


def dequantize(codes, scale: float) -> np.ndarray:
    """float64 values a pool of codes stands for.

    Source: "从零构建LLM 推理引擎", card "量化"; an entry stands for code * scale.
    """
    return e4m3_decode(codes) * float(np.float32(scale))

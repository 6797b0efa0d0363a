"""FP8 (e4m3) latent cache: the quantised form of the cached latent.

TEST INFRASTRUCTURE ONLY: imported by tests and ``bench.py``'s reference
legs; never by the product path.

Source: "DeepSeek-V3.2-Exp unboxing" (floratopia.github.io), the section on
the Indexer: the model code says deployment keeps the KV cache in fp8, and the
reference implementation imitates that precision by casting the cached
latent to fp8 and back to bf16 before using it.

Readings where the pages are silent:

* Format: e4m3 without infinities (largest finite 448, the fp8 type the
  tensor cores take as e4m3), rounding to nearest, ties to even, saturating at
  +-448.
* Scale: one float32 scale per cached token for its 512 latent values,
  ``s = max|x| / 448`` (``s = 1`` for an all-zero row), code ``e4m3(x / s)``;
  the 64 rope columns (k_pe) stay bf16. The pages print no scale layout.
* "Back to bf16": the dequantised value is ``bf16(code * s)``.
* Where this decides an integer (the fp8 code), it does so in float32, as a
  kernel would: ``s`` is the float32 quotient ``amax / 448`` and ``x / s`` the
  float32 (IEEE, correctly rounded) quotient; only then is the e4m3 rounding
  applied. The product ``code * s`` is rounded to float32 before bf16.
* Row layout in memory (the pages print none): one cached token is 656 bytes,
  ``[0, 512)`` the e4m3 codes of the latent in column order, ``[512, 640)``
  the 64 rope values as bf16 (little-endian), ``[640, 644)`` the float32
  scale, ``[644, 656)`` zero (rows stay 16-byte aligned); a page is 64 rows.
"""

from __future__ import annotations

import torch

D_LATENT = 512
D_ROPE = 64
ROW_BYTES = 656          # e4m3 codes 512 | bf16 rope 128 | f32 scale 4 | zero 12
ROPE_OFF, SCALE_OFF = 512, 640
E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6   # smallest normal 2^-6; subnormal spacing 2^-9
E4M3_MANT_BITS = 3


def e4m3_round(x: torch.Tensor) -> torch.Tensor:
    """Nearest e4m3 value to each element (ties to even), saturating at
    +-448, as float64. Written from the format: in the binade [2^e, 2^(e+1))
    with e >= -6 the spacing is 2^(e-3); below 2^-6 (subnormals) it is 2^-9,
    the same as the lowest normal binade."""
    xf = x.to(torch.float64)
    _, exp = torch.frexp(xf)                          # |x| = m * 2^exp, m in [0.5, 1): binade e = exp - 1
    e = torch.clamp(exp.to(torch.float64) - 1, min=E4M3_MIN_NORMAL_EXP)
    quantum = torch.pow(2.0, e - E4M3_MANT_BITS)
    r = torch.round(xf / quantum) * quantum          # torch.round: half to even
    return torch.clamp(r, -E4M3_MAX, E4M3_MAX)


def quantize_rows(latent: torch.Tensor):
    """Rows of ``latent`` [..., 512] (bf16 values) -> (codes as float64 values
    on the e4m3 grid, float32 scales [...])."""
    x32 = latent.to(torch.float32)
    amax = x32.abs().amax(-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))   # float32 quotient
    y32 = x32 / scale[..., None]                                            # float32 quotient
    return e4m3_round(y32), scale


def dequantize_rows(codes: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """``bf16(float32(code * s))``, as float64."""
    prod = codes.to(torch.float32) * scale.to(torch.float32)[..., None]
    return prod.to(torch.bfloat16).to(torch.float64)


def fp8_roundtrip_cache(cache: torch.Tensor) -> torch.Tensor:
    """The cache [pages, 64, 576] as an fp8-cache decode sees it: latent
    columns quantised per token and dequantised, rope columns unchanged;
    returned as bf16 so that ``oracle.mla_decode`` can consume it."""
    codes, scale = quantize_rows(cache[..., :D_LATENT])
    out = cache.clone()
    out[..., :D_LATENT] = dequantize_rows(codes, scale).to(cache.dtype)
    return out


def unpack_rows(raw: torch.Tensor):
    """Raw fp8-cache rows ``[..., 656]`` (uint8) -> (codes as float64 e4m3
    values [..., 512], float32 scales [...], bf16 rope [..., 64])."""
    raw = raw.contiguous()
    codes = raw[..., :D_LATENT].contiguous().view(torch.float8_e4m3fn).to(torch.float64)
    rope = raw[..., ROPE_OFF:SCALE_OFF].contiguous().view(torch.bfloat16)
    scale = raw[..., SCALE_OFF:SCALE_OFF + 4].contiguous().view(torch.float32)[..., 0]
    return codes, scale, rope


def dequantize_cache(raw: torch.Tensor) -> torch.Tensor:
    """An fp8 cache ``[pages, 64, 656]`` (uint8) as the bf16 cache ``[pages, 64,
    576]`` a decode over it computes with: latent ``bf16(float32(code * s))``,
    rope unchanged."""
    codes, scale, rope = unpack_rows(raw)
    out = torch.empty(raw.shape[:-1] + (D_LATENT + D_ROPE,), dtype=torch.bfloat16)
    out[..., :D_LATENT] = dequantize_rows(codes, scale).to(torch.bfloat16)
    out[..., D_LATENT:] = rope
    return out

"""Pins for the fp8 (e4m3) latent-cache oracle: its rounding against the
library's float8_e4m3fn cast (exhaustively on the grid, on random values and
on every tie), the per-token scale's closed forms, the error bound that three
mantissa bits allow, and what a decode over the quantised cache returns."""

import pytest
import torch

import oracle
from oracle import fp8_cache as f8

BF = torch.bfloat16


def _grid():
    """Every finite e4m3 value, from the library's decoding of all 256 codes."""
    v = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    return torch.unique(v[torch.isfinite(v)])


def test_grid_has_the_format_shape():
    g = _grid()
    assert g.numel() == 253  # 254 finite codes (+0 and -0 collapse), 2 NaN codes
    assert g.max() == 448.0 and g.min() == -448.0
    pos = g[g > 0]
    assert pos.min() == 2.0 ** -9          # smallest subnormal
    assert (pos == 2.0 ** -6).any()        # smallest normal


def test_grid_points_are_fixed_points():
    g = _grid()
    assert torch.equal(f8.e4m3_round(g), g)


def test_matches_library_cast_on_random_values():
    gen = torch.Generator().manual_seed(0)
    x = torch.cat([
        (torch.rand(200000, generator=gen, dtype=torch.float64) * 2 - 1) * 448,
        (torch.rand(200000, generator=gen, dtype=torch.float64) * 2 - 1) * 2.0 ** -5,   # subnormal range
        torch.randn(200000, generator=gen, dtype=torch.float64) * 3,
    ]).to(torch.float32)  # the oracle's inputs are float32 quotients
    lib = x.to(torch.float8_e4m3fn).to(torch.float64)
    assert torch.equal(f8.e4m3_round(x), lib)


def test_ties_go_to_even_like_the_library():
    g = _grid()
    mid = ((g[1:] + g[:-1]) / 2).to(torch.float32)
    mid = mid[mid.to(torch.float64) == (g[1:] + g[:-1]) / 2]   # exact midpoints only
    lib = mid.to(torch.float8_e4m3fn).to(torch.float64)
    assert torch.equal(f8.e4m3_round(mid), lib)
    # 2^-10 lies between 0 and 2^-9 and goes to 0; 3 * 2^-10 between 2^-9 and 2^-8 goes to 2^-8
    assert f8.e4m3_round(torch.tensor([2.0 ** -10, 3 * 2.0 ** -10])).tolist() == [0.0, 2.0 ** -8]


def test_saturates_beyond_the_largest_finite():
    x = torch.tensor([448.0, 449.0, 463.9, 500.0, 1e6, -1e6])
    assert f8.e4m3_round(x).tolist() == [448.0, 448.0, 448.0, 448.0, 448.0, -448.0]


def test_row_scale_closed_forms():
    # the largest element maps to +-448 exactly; a power-of-two amax gives an exact scale
    row = torch.zeros(2, 512)
    row[0, 7] = -3.5
    row[0, 100] = 1.0
    row[1, :] = 2.0 ** -3
    codes, scale = f8.quantize_rows(row.to(BF))
    assert codes[0, 7] == -448.0 and scale[0] == torch.tensor(3.5 / 448, dtype=torch.float32)
    assert scale[1] == 2.0 ** -3 / 448 and torch.all(codes[1] == 448.0)
    z_codes, z_scale = f8.quantize_rows(torch.zeros(3, 512, dtype=BF))
    assert torch.all(z_codes == 0) and torch.all(z_scale == 1.0)


def test_roundtrip_error_bound():
    """Three mantissa bits: half a step is at most 2^-4 of a normal value; in
    the subnormal range the step is s * 2^-9; the bf16 rounding of the
    product adds at most 2^-9 relative."""
    gen = torch.Generator().manual_seed(1)
    x = (torch.randn(64, 512, generator=gen) * torch.rand(64, 1, generator=gen) * 4).to(BF)
    codes, scale = f8.quantize_rows(x)
    dq = f8.dequantize_rows(codes, scale)
    xd = x.to(torch.float64)
    bound = (2.0 ** -4 + 2.0 ** -8) * xd.abs() + scale.to(torch.float64)[:, None] * 2.0 ** -9
    assert torch.all((dq - xd).abs() <= bound)
    # and the bound is not loose by orders of magnitude
    assert (dq - xd).abs().max() > 0.1 * bound.max()


def test_roundtrip_cache_changes_only_latent_columns():
    gen = torch.Generator().manual_seed(2)
    cache = torch.randn(3, 64, 576, generator=gen).to(BF)
    rt = f8.fp8_roundtrip_cache(cache)
    assert rt.dtype == BF and torch.equal(rt[..., 512:], cache[..., 512:])
    assert not torch.equal(rt[..., :512], cache[..., :512])


def test_decode_over_fp8_cache_single_key_returns_dequantised_latent():
    """A one-token context returns that token's latent: over the fp8 cache it is
    the dequantised latent, not the original one."""
    gen = torch.Generator().manual_seed(3)
    cache = torch.randn(1, 64, 576, generator=gen).to(BF)
    rt = f8.fp8_roundtrip_cache(cache)
    q = torch.randn(1, 1, 4, 576, generator=gen).to(BF)
    out, _ = oracle.mla_decode(q, rt, torch.zeros(1, 1, dtype=torch.int32), torch.tensor([1], dtype=torch.int32))
    assert torch.equal(out[0, 0], rt[0, 0, :512].to(torch.float64).expand(4, -1))


def test_row_layout_unpacks_a_hand_built_row():
    """A 656-byte row written byte by byte (struct, no tensor views): codes
    0x38 = 1, 0xB8 = -1, 0x01 = 2^-9 (smallest subnormal), 0x7E = 448 (largest),
    0x00 = 0; rope bf16 0x3FC0 = 1.5 and 0xC040 = -3; scale float32 2.0;
    twelve zero bytes. Dequantised: 2, -2, 2^-8, 896, 0; rope unchanged."""
    import struct

    codes = bytes([0x38, 0xB8, 0x01, 0x7E] + [0x00] * 508)
    rope = struct.pack("<64H", *([0x3FC0, 0xC040] * 32))
    row = codes + rope + struct.pack("<f", 2.0) + bytes(12)
    assert len(row) == f8.ROW_BYTES == 656
    raw = torch.tensor(list(row), dtype=torch.uint8).view(1, 1, 656)
    c, s, r = f8.unpack_rows(raw)
    assert c[0, 0, :5].tolist() == [1.0, -1.0, 2.0 ** -9, 448.0, 0.0]
    assert float(s[0, 0]) == 2.0
    assert r[0, 0, :2].to(torch.float64).tolist() == [1.5, -3.0]
    dq = f8.dequantize_cache(raw)
    assert dq.shape == (1, 1, 576) and dq.dtype == BF
    assert dq[0, 0, :5].to(torch.float64).tolist() == [2.0, -2.0, 2.0 ** -8, 896.0, 0.0]
    assert torch.equal(dq[0, 0, 512:], r[0, 0])


def test_dequantize_cache_matches_roundtrip_of_quantised_rows():
    """Packing quantize_rows' codes and scales into rows by hand and reading
    them back gives the same cache as fp8_roundtrip_cache."""
    import struct

    gen = torch.Generator().manual_seed(4)
    cache = (torch.randn(2, 64, 576, generator=gen) * 2).to(BF)
    codes, scale = f8.quantize_rows(cache[..., :512])
    code_bytes = codes.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
    rows = []
    for p in range(2):
        for t in range(64):
            rope = cache[p, t, 512:].view(torch.int16).to(torch.int32) & 0xFFFF
            rows.append(bytes(code_bytes[p, t].tolist()) + struct.pack("<64H", *rope.tolist())
                        + struct.pack("<f", float(scale[p, t])) + bytes(12))
    raw = torch.tensor(list(b"".join(rows)), dtype=torch.uint8).view(2, 64, 656)
    assert torch.equal(f8.dequantize_cache(raw), f8.fp8_roundtrip_cache(cache))

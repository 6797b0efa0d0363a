"""Pins for the cache-insert oracle (kv_norm RMSNorm, rotary pairs, paged
write): worked values computed by hand in bf16, exact special cases,
invariants, and the addressing of the decode oracle's row gather."""

import math

import pytest
import torch

import oracle
from oracle import decode as od

BF = torch.bfloat16


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(BF)


# ---------------------------------------------------------------- RMSNorm


def test_rms_norm_worked_example_cast_order():
    """x = (3, 4), weight 1.5, eps 0: rms = sqrt(12.5); x/rms = (0.848528...,
    1.131370...). In bf16 (8 significant bits) these round to 0.84765625
    (217/256) and 1.1328125 (145/128). Times 1.5: 1.271484375 -> 1.2734375
    (163/128) and 1.69921875 -> a tie between 217/128 and 218/128, which rounds
    to the even 218/128 = 1.703125. Multiplying the unrounded 1.131370 by 1.5
    instead would give 1.6953125, so the second value pins the page's order:
    cast the normalised row first, then multiply by the weight."""
    x = torch.tensor([3.0, 4.0], dtype=BF)
    w = torch.tensor([1.5, 1.5], dtype=BF)
    out = oracle.rms_norm(x, w, 0.0)
    assert out.tolist() == [1.2734375, 1.703125]


def test_rms_norm_constant_row_is_sign():
    """A row of equal magnitudes c has rms |c|: the normalised row is the sign,
    exactly, and the output is sign * weight."""
    x = torch.full((512,), -2.75, dtype=BF)
    x[::3] = 2.75
    w = _rand(512, 1)
    out = oracle.rms_norm(x, w, 0.0)
    assert torch.equal(out, torch.sign(x.double()) * w.double())


def test_rms_norm_unit_mean_square():
    """With weight 1 and eps 0 the normalised row has mean square 1, up to the
    bf16 rounding of each element (relative 2^-9)."""
    x = _rand((8, 512), 2)
    out = oracle.rms_norm(x, torch.ones(512, dtype=BF), 0.0)
    ms = (out * out).mean(-1)
    assert torch.all((ms - 1).abs() < 2 * 2.0 ** -9), ms


def test_rms_norm_rows_independent_and_scale_invariant():
    """Rows are normalised one by one (a row's result does not depend on the
    others), and scaling a row by a power of two changes nothing (eps 0)."""
    x = _rand((4, 512), 3)
    w = _rand(512, 4)
    both = oracle.rms_norm(x, w, 0.0)
    for i in range(4):
        assert torch.equal(both[i], oracle.rms_norm(x[i], w, 0.0))
        assert torch.equal(both[i], oracle.rms_norm((x[i].double() * 8).to(BF), w, 0.0))


def test_rms_norm_eps_keeps_zero_row_finite():
    out = oracle.rms_norm(torch.zeros(512, dtype=BF), torch.ones(512, dtype=BF), 1e-6)
    assert torch.equal(out, torch.zeros(512, dtype=torch.float64))


def test_rms_norm_eps_enters_under_the_root():
    """x = (1, 1), eps 3: rms = sqrt(1 + 3) = 2, so the row becomes (0.5, 0.5)
    exactly (eps added to the mean square, inside the square root)."""
    out = oracle.rms_norm(torch.tensor([1.0, 1.0], dtype=BF), torch.ones(2, dtype=BF), 3.0)
    assert out.tolist() == [0.5, 0.5]


# ---------------------------------------------------------------- rotary pairs


def _angles(p, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.rand(p, generator=g, dtype=torch.float64) * 2 * math.pi


def test_rope_zero_angle_is_identity():
    x = _rand(64, 5)
    out = oracle.rope_pairs(x, torch.ones(32), torch.zeros(32))
    assert torch.equal(out, x.double())


def test_rope_quarter_turn_pairs_consecutive_elements():
    """A quarter turn maps each consecutive pair (a, b) to (-b, a): with
    x = (1, 2, 0, ...) the result is (-2, 1, 0, ...). Rotating element 0 with
    element 32 (the split-halves convention) would leave element 1 alone."""
    x = torch.zeros(64, dtype=BF)
    x[0], x[1] = 1.0, 2.0
    out = oracle.rope_pairs(x, torch.zeros(32), torch.ones(32))
    want = torch.zeros(64, dtype=torch.float64)
    want[0], want[1] = -2.0, 1.0
    assert torch.equal(out, want)
    y = _rand(64, 6)
    out = oracle.rope_pairs(y, torch.zeros(32), torch.ones(32))
    assert torch.equal(out[0::2], -y.double()[1::2]) and torch.equal(out[1::2], y.double()[0::2])


def test_rope_half_turn_negates():
    y = _rand(64, 7)
    assert torch.equal(oracle.rope_pairs(y, -torch.ones(32), torch.zeros(32)), -y.double())


def test_rope_preserves_pair_norms_and_inverts():
    """A rotation keeps each pair's length (up to the bf16 rounding of the two
    outputs) and rotating back by -angle returns the input within two
    roundings."""
    y = _rand(64, 8)
    a = _angles(32, 9)
    c, s = torch.cos(a), torch.sin(a)
    r = oracle.rope_pairs(y, c, s)
    n_in = y.double()[0::2] ** 2 + y.double()[1::2] ** 2
    n_out = r[0::2] ** 2 + r[1::2] ** 2
    assert torch.all((n_out.sqrt() - n_in.sqrt()).abs() <= n_in.sqrt() * 2.0 ** -7)
    back = oracle.rope_pairs(r.to(BF), c, -s)
    assert torch.all((back - y.double()).abs() <= y.double().abs().max() * 2.0 ** -6)


def test_rope_composes_angles():
    """Rotating by a then by b equals rotating by a + b (within rounding): a
    wrong sign on either sine term breaks this for generic angles."""
    y = _rand(64, 10)
    a, b = _angles(32, 11), _angles(32, 12)
    two = oracle.rope_pairs(oracle.rope_pairs(y, torch.cos(a), torch.sin(a)).to(BF), torch.cos(b), torch.sin(b))
    one = oracle.rope_pairs(y, torch.cos(a + b), torch.sin(a + b))
    assert torch.all((two - one).abs() <= y.double().abs().max() * 2.0 ** -6)


# ---------------------------------------------------------------- paged write


def _setup(lens, seed, extra_pages=3):
    g = torch.Generator().manual_seed(seed)
    npg = [(L + 63) // 64 for L in lens]
    total = sum(npg) + extra_pages
    perm = torch.randperm(total, generator=g)
    bt = torch.full((len(lens), max(npg)), -1, dtype=torch.int32)
    k = 0
    for b, n in enumerate(npg):
        bt[b, :n] = perm[k:k + n].to(torch.int32)
        k += n
    cache = torch.randn(total, 64, 576, generator=g).to(BF)
    return cache, bt


def test_insert_then_gather_reads_back_in_order():
    """Insert every token of two sequences (lengths 70 and 129, pages
    shuffled): the decode oracle's gather of positions 0..L-1 reads back, in
    order, the normalised latent and the rotated rope key of exactly those
    tokens. This ties the write address (page = table[p // 64], row = p % 64)
    to the one decode reads."""
    lens = [70, 129]
    cache, bt = _setup(lens, 13)
    seq = torch.cat([torch.full((L,), b, dtype=torch.int32) for b, L in enumerate(lens)])
    pos = torch.cat([torch.arange(L, dtype=torch.int32) for L in lens])
    kv = _rand((len(seq), 576), 14)
    w = _rand(512, 15)
    a = torch.rand(256, 32, dtype=torch.float64, generator=torch.Generator().manual_seed(16)) * 6.3
    cos, sin = torch.cos(a).float(), torch.sin(a).float()
    out, skipped = oracle.cache_insert(cache, bt, seq, pos, kv, w, 1e-6, cos, sin)
    assert skipped == []
    n = 0
    for b, L in enumerate(lens):
        rows = od.gather_rows(out, bt[b], torch.arange(L))
        for t in range(L):
            assert torch.equal(rows[t, :512], oracle.rms_norm(kv[n, :512], w, 1e-6))
            assert torch.equal(rows[t, 512:], oracle.rope_pairs(kv[n, 512:], cos[t], sin[t]))
            n += 1


def test_insert_leaves_other_rows_and_skips_out_of_range():
    """Only the addressed rows change; a token whose sequence, position, page
    or table row is out of range writes nothing and is reported."""
    cache, bt = _setup([100], 17)
    bt[0, 1] = 10_000                                 # second page id out of range
    seq = torch.tensor([0, 0, 5, 0, 0], dtype=torch.int32)
    pos = torch.tensor([3, 70, 1, 300, 64], dtype=torch.int32)
    kv = _rand((5, 576), 18)
    cos, sin = torch.ones(128, 32), torch.zeros(128, 32)
    out, skipped = oracle.cache_insert(cache, bt, seq, pos, kv, torch.ones(512, dtype=BF), 1e-6, cos, sin)
    assert skipped == [1, 2, 3, 4]
    changed = (out != cache.double()).any(-1)
    assert changed.sum() == 1 and changed[int(bt[0, 0]), 3]


def test_insert_later_token_wins_on_same_row():
    cache, bt = _setup([10], 19)
    kv = _rand((2, 576), 20)
    seq = torch.zeros(2, dtype=torch.int32)
    pos = torch.tensor([4, 4], dtype=torch.int32)
    cos, sin = torch.ones(16, 32), torch.zeros(16, 32)
    w = torch.ones(512, dtype=BF)
    out, _ = oracle.cache_insert(cache, bt, seq, pos, kv, w, 1e-6, cos, sin)
    assert torch.equal(out[int(bt[0, 0]), 4, :512], oracle.rms_norm(kv[1, :512], w, 1e-6))
    assert torch.equal(out[int(bt[0, 0]), 4, 512:], kv[1, 512:].double())

"""Pins of the indexer oracle (oracle/indexer.py) against what the V3.2
page fixes and against the mathematics, independent of the oracle's own
code: the e4m3 code table written from the format, brute force with
pure-Python loops on tiny shapes, closed forms of the score, and top-k by
exhaustive ordering. Source: "DeepSeek-V3.2-Exp unboxing", the Indexer
section (the fp8_index signature, the weights passed as q_s, the shapes)."""

import itertools
import math
import random

import pytest
import torch

from oracle.indexer import index_scores, topk_positions


def _e4m3_value(code: int) -> float:
    """The e4m3 (fn) format written out: 1 sign bit, 4 exponent bits with
    bias 7, 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6);
    S.1111.111 is NaN; there are no infinities."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def test_e4m3_code_table_matches_the_format():
    """Every one of the 256 codes decodes (as the oracle's upcast does) to the
    value the format defines; 448 is the largest finite value."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    vals = codes.view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        want = _e4m3_value(c)
        got = float(vals[c])
        if math.isnan(want):
            assert math.isnan(got), c
        else:
            assert got == want, (c, got, want)
    finite = [abs(_e4m3_value(c)) for c in range(256) if not math.isnan(_e4m3_value(c))]
    assert max(finite) == 448.0


def _fp8(t):
    return t.to(torch.float8_e4m3fn)


def _rand_inputs(b, m, h, d, n, seed):
    g = torch.Generator().manual_seed(seed)
    q = _fp8(torch.randn(b, m, h, d, generator=g) * 2)
    k = _fp8(torch.randn(b, n, d, generator=g) * 2)
    q_s = torch.randn(b, m, h, generator=g)
    k_s = torch.rand(b, n, generator=g) + 0.1
    return q, q_s, k, k_s


def _py(x):
    return x.to(torch.float64).tolist()


def test_brute_force_loops():
    """The score by plain Python loops over (b, i, t, h, d) on a tiny case."""
    b, m, h, d, n = 2, 3, 4, 8, 5
    q, q_s, k, k_s = _rand_inputs(b, m, h, d, n, seed=1)
    Q, QS, K, KS = _py(q.to(torch.float32)), _py(q_s), _py(k.to(torch.float32)), _py(k_s)
    o = index_scores(q, q_s, k, k_s)
    for bb, i, t in itertools.product(range(b), range(m), range(n)):
        acc = 0.0
        for hh in range(h):
            dot = 0.0
            for dd in range(d):
                dot += Q[bb][i][hh][dd] * K[bb][t][dd]
            acc += QS[bb][i][hh] * (dot if dot > 0 else 0.0)
        want = KS[bb][t] * acc
        assert abs(float(o[bb, i, t]) - want) <= 1e-12 * (1 + abs(want)), (bb, i, t)


def test_page_shapes():
    """The shapes printed on the page: q [2,128,64,128], q_s [2,128,64],
    k [2,128,128], k_s [2,128] give o [2,128,128]."""
    q, q_s, k, k_s = _rand_inputs(2, 128, 64, 128, 128, seed=2)
    assert index_scores(q, q_s, k, k_s).shape == (2, 128, 128)


def test_one_hot_query_reads_one_key_column():
    """h = 1, q_s = 1, k_s = 1 and q = 2 e_j: the score of key t is
    relu(2 k[t, j]) — exact, since every term is an fp8 value times 2."""
    d, n = 16, 40
    g = torch.Generator().manual_seed(3)
    k = _fp8(torch.randn(1, n, d, generator=g))
    for j in (0, 7, 15):
        q = torch.zeros(1, 1, 1, d)
        q[0, 0, 0, j] = 2.0
        o = index_scores(_fp8(q), torch.ones(1, 1, 1), k, torch.ones(1, n))
        want = (2 * k[0, :, j].to(torch.float64)).clamp_min(0)
        assert torch.equal(o[0, 0], want)


def test_relu_zeroes_negative_dot_products():
    """Queries with non-positive entries against keys with non-negative
    entries: every dot product is <= 0, so every score is exactly 0 whatever
    the weights; flipping the query's sign makes every dot product >= 0 and
    the score becomes the plain weighted sum."""
    g = torch.Generator().manual_seed(4)
    q = _fp8(-torch.rand(1, 2, 3, 32, generator=g))
    k = _fp8(torch.rand(1, 9, 32, generator=g))
    q_s = torch.randn(1, 2, 3, generator=g)
    k_s = torch.rand(1, 9, generator=g) + 0.5
    assert torch.equal(index_scores(q, q_s, k, k_s), torch.zeros(1, 2, 9, dtype=torch.float64))
    qp = _fp8(-q.to(torch.float32))
    dots = qp.to(torch.float64)[0] @ k.to(torch.float64)[0].T                # [m, h, n]
    want = (dots * q_s.to(torch.float64)[0][..., None]).sum(1) * k_s.to(torch.float64)[0][None]
    assert torch.allclose(index_scores(qp, q_s, k, k_s)[0], want, rtol=1e-12, atol=0)


def test_weights_and_scales_are_linear():
    """Doubling q_s doubles the score; scaling k_s[t] by 4 scales column t by 4;
    negating one head's weight subtracts that head (exact powers of two)."""
    q, q_s, k, k_s = _rand_inputs(1, 2, 4, 32, 11, seed=5)
    base = index_scores(q, q_s, k, k_s)
    assert torch.equal(index_scores(q, 2 * q_s, k, k_s), 2 * base)
    ks4 = k_s.clone()
    ks4[0, 3] *= 4
    got = index_scores(q, q_s, k, ks4)
    assert torch.equal(got[..., 3], 4 * base[..., 3])
    assert torch.equal(torch.cat([got[..., :3], got[..., 4:]], -1), torch.cat([base[..., :3], base[..., 4:]], -1))
    # heads add up: the score with head 0 alone plus the score without head 0
    only0, without0 = q_s.clone(), q_s.clone()
    only0[..., 1:] = 0
    without0[..., 0] = 0
    parts = index_scores(q, only0, k, k_s) + index_scores(q, without0, k, k_s)
    assert torch.allclose(parts, base, rtol=1e-12, atol=1e-12)


def test_head_permutation_invariance():
    q, q_s, k, k_s = _rand_inputs(2, 2, 8, 16, 7, seed=6)
    perm = torch.randperm(8, generator=torch.Generator().manual_seed(0))
    a = index_scores(q, q_s, k, k_s)
    b = index_scores(q[:, :, perm], q_s[:, :, perm], k, k_s)
    assert torch.allclose(a, b, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- top-k


def _brute_topk(row, k, L):
    """Exhaustive: order positions by (-score, position), keep k, sort them."""
    items = sorted(range(L), key=lambda t: (-row[t], t))[:k]
    items = sorted(items)
    return items + [-1] * (k - len(items))


@pytest.mark.parametrize("n,k", [(1, 1), (5, 3), (64, 64), (100, 7), (300, 128), (40, 50)])
def test_topk_against_exhaustive_ordering(n, k):
    rnd = random.Random(n * 31 + k)
    rows = []
    for r in range(6):
        # few distinct values, so that ties at the cut are common
        rows.append([float(rnd.choice([-2.0, -0.5, 0.0, 0.25, 1.0, 3.0, rnd.uniform(-4, 4)])) for _ in range(n)])
    lens = [n, n // 2, 1, 0, max(n - 3, 0), n]
    got = topk_positions(torch.tensor(rows, dtype=torch.float32), k, torch.tensor(lens))
    for r in range(6):
        assert got[r].tolist() == _brute_topk(rows[r], k, lens[r]), r


def test_topk_ties_go_to_smaller_positions():
    s = torch.tensor([[1.0, 2.0, 2.0, 2.0, 0.5, 2.0]])
    assert topk_positions(s, 2).tolist() == [[1, 2]]
    assert topk_positions(s, 4).tolist() == [[1, 2, 3, 5]]
    # signed zeros are equal scores: the earlier position wins
    z = torch.tensor([[-0.0, 0.0, -1.0]])
    assert topk_positions(z, 1).tolist() == [[0]]


def test_topk_all_equal_and_short_rows():
    s = torch.full((2, 10), 0.75)
    assert topk_positions(s, 4).tolist() == [[0, 1, 2, 3]] * 2
    assert topk_positions(s, 12, torch.tensor([10, 3])).tolist() == [list(range(10)) + [-1, -1],
                                                                     [0, 1, 2] + [-1] * 9]

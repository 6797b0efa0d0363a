"""GPU parity of the latent-cache insert (``mla_cache_insert``) against the
float64 oracle.

Tolerance, from the arithmetic: the kernel computes the normaliser and the
rotation in float32, the oracle in float64; both round to bf16 at the same
two points (the normalised row, then its product with the weight). The
float32 values differ from the float64 ones by a few float32 ulps, so a bf16
rounding can land on the other side of a tie point: the normalised value may
differ by one bf16 ulp, which the weight product can turn into two ulps of
the output (relative 2^-6). The rotated pair is rounded once (one ulp, 2^-7
relative) plus float32 cancellation (2^-20 of the pair's magnitude). Nearly
every element is bit-identical; the test also requires that.
"""

import pytest
import torch

import oracle
from mla_latent_kv_26_b200.workloads import insert_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(libmla):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def run_insert(libmla, d, dev, eps=1e-6):
    from mla_latent_kv_26_b200.decoder import cache_insert

    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    cache_insert(g["kv"], g["weight"], g["cos"], g["sin"], g["seq_ids"], g["positions"], g["block_table"],
                 g["cache"], eps=eps, error_word=err)
    torch.cuda.synchronize(dev)
    return g["cache"].cpu(), int(err.item()) & 0xffffffff


def assert_rows(got, ref, where=""):
    """got, ref: [..., 576] float64 (bf16 values)."""
    lat_g, lat_r = got[..., :512], ref[..., :512]
    rope_g, rope_r = got[..., 512:], ref[..., 512:]
    d_lat = (lat_g - lat_r).abs()
    assert torch.all(d_lat <= lat_r.abs() * 2.0 ** -6), f"{where}: latent max diff {d_lat.max()}"
    mag = rope_r.abs().amax(-1, keepdim=True)
    d_rope = (rope_g - rope_r).abs()
    assert torch.all(d_rope <= rope_r.abs() * 2.0 ** -7 + mag * 2.0 ** -20), f"{where}: rope max diff {d_rope.max()}"
    exact = (got == ref).double().mean().item()
    assert exact >= 0.99, f"{where}: only {exact:.4f} of the elements are bit-identical"


def check_full(libmla, d, dev, eps=1e-6, where=""):
    got, err = run_insert(libmla, d, dev, eps)
    ref, skipped = oracle.cache_insert(d["cache"], d["block_table"], d["seq_ids"], d["positions"], d["kv"],
                                       d["weight"], eps, d["cos"], d["sin"])
    got = got.double()
    written = (ref != d["cache"].double()).any(-1)
    assert torch.equal(got[~written], ref[~written]), f"{where}: rows not addressed changed"
    assert_rows(got[written], ref[written], where)
    return err, skipped


@pytest.mark.parametrize("lens,new", [
    ([70, 129], [70, 129]),                 # prefill of two sequences, ragged last pages
    ([1, 64, 65, 200], [1, 64, 65, 200]),   # page-boundary lengths
    ([300, 5000, 77], [1, 1, 1]),           # one decode token each
    ([4000, 130], [17, 2]),                 # chunked prefill appending to a cache
])
def test_insert_parity(libmla, dev, lens, new):
    d = insert_inputs(lens=lens, new_tokens=new, seed=sum(lens))
    err, skipped = check_full(libmla, d, dev, where=f"{lens}/{new}")
    assert err == 0 and skipped == []


def test_insert_single_token_and_ragged_tail(libmla, dev):
    for n in (1, 15, 16, 17, 33):
        d = insert_inputs(lens=[n], new_tokens=[n], seed=100 + n)
        err, _ = check_full(libmla, d, dev, where=f"n{n}")
        assert err == 0


def test_insert_decode_batch_of_64(libmla, dev):
    lens = torch.randint(1024, 32768, (64,), generator=torch.Generator().manual_seed(7)).tolist()
    d = insert_inputs(lens=lens, new_tokens=[1] * 64, seed=8)
    err, _ = check_full(libmla, d, dev, where="decode64")
    assert err == 0


def test_insert_full_size_prefill_64x1024(libmla, dev):
    """The benchmark's insert workload: 64 sequences x 1,024 new tokens
    (positions 0..1023, seed 5), every row against the oracle."""
    d = insert_inputs(lens=[1024] * 64, new_tokens=[1024] * 64, seed=5)
    err, skipped = check_full(libmla, d, dev, where="prefill 64x1024")
    assert err == 0 and len(skipped) == 0


def test_insert_scale_extremes_and_zero_row(libmla, dev):
    """Rows scaled by 2^-56 and 2^+56 (the float32 sum of squares of 512
    N(0,1) values times 2^112 stays far below the float32 maximum 2^128), and
    an all-zero latent, which eps keeps at zero."""
    d = insert_inputs(lens=[8], new_tokens=[8], seed=9)
    kv = d["kv"].double()
    kv[1] *= 2.0 ** -56
    kv[2] *= 2.0 ** 56
    kv[3, :512] = 0
    d["kv"] = kv.to(torch.bfloat16)
    check_full(libmla, d, dev, where="extremes")
    check_full(libmla, d, dev, eps=0.5, where="eps 0.5")


def test_insert_bad_tokens_skipped_and_flagged(libmla, dev):
    d = insert_inputs(lens=[100, 200], new_tokens=[100, 200], seed=11)
    d["seq_ids"][3] = 2                           # no such sequence
    d["positions"][150] = -1                      # negative position
    d["positions"][151] = d["cos"].shape[0]       # beyond the tables
    d["block_table"][1, 2] = 10_000               # page id out of range: tokens 128..191 of sequence 1
    err, skipped = check_full(libmla, d, dev, where="bad tokens")
    assert err == 0x10 | 0x2
    assert len(skipped) == 3 + 64


def test_insert_then_decode_matches_oracle_chain(libmla, dev):
    """Fill two sequences' caches through the GPU insert, decode them on the
    GPU, and compare with the oracle's insert followed by the oracle's decode:
    the two steps agree on the cache layout end to end."""
    from mla_latent_kv_26_b200.decoder import MlaDecoder
    from test_parity import assert_parity  # tests/ is on sys.path under pytest

    lens = [700, 130]
    d = insert_inputs(lens=lens, new_tokens=lens, seed=13, kv_std=0.7)
    got, _ = run_insert(libmla, d, dev)
    ref, _ = oracle.cache_insert(d["cache"], d["block_table"], d["seq_ids"], d["positions"], d["kv"], d["weight"],
                                 1e-6, d["cos"], d["sin"])
    q = (torch.randn(2, 1, 128, 576, generator=torch.Generator().manual_seed(14)) * 0.5).to(torch.bfloat16)
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    dec = MlaDecoder(batch=2, q_len=1, num_heads=128, num_pages=d["num_pages"],
                     max_pages_per_seq=d["max_pages_per_seq"], device=dev)
    out, lse = dec(q.to(dev), got.to(dev), d["block_table"].to(dev), seq_lens.to(dev))
    # the oracle decodes the GPU-written cache (same bf16 values) and, as a
    # second check, its own insert's cache within the insert tolerance
    o_ref, l_ref = oracle.mla_decode(q, got, d["block_table"], seq_lens)
    assert_parity(out.double().cpu(), lse.double().cpu(), o_ref, l_ref, "insert->decode")
    o_own, _ = oracle.mla_decode(q, ref.to(torch.bfloat16), d["block_table"], seq_lens)
    assert (o_own - o_ref).abs().max() < 2e-2

"""GPU parity of the absorb / un-absorb projections (``mla_absorb_query``,
``mla_unabsorb_output``) against the float64 oracle, and of the whole chain
q -> absorb -> decode -> un-absorb against the oracle's unabsorbed attention.

Tolerance, from the arithmetic: the kernels accumulate bf16 products in fp32
(K = 128 or 512 terms) and round the result to bf16 once. The rounding costs
at most half a bf16 ulp (2^-9 relative; 2^-8 allowed); the fp32 sum's error
is below K * 2^-24 of the sum of the terms' magnitudes (2^-14 of it allowed).
The q_pe columns are copied and must be bit-identical.
"""

import pytest
import torch

import oracle
from mla_latent_kv_26_b200.workloads import absorb_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(libmla):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def _ref_absorb(q, wkv_b):
    """Oracle q_lat [T, H, 512] and the magnitude bound sum_d |q_d W_dj|."""
    w_uk = wkv_b[:, :128, :]
    ref = torch.stack([oracle.absorb_query(q[t, :, :128], w_uk) for t in range(q.shape[0])])
    mag = torch.stack([oracle.absorb_query(q[t, :, :128].abs(), w_uk.abs()) for t in range(q.shape[0])])
    return ref, mag


def _ref_unabsorb(o_lat, wkv_b):
    w_uv = wkv_b[:, 128:, :]
    ref = torch.stack([oracle.unabsorb_output(o_lat[t], w_uv) for t in range(o_lat.shape[0])])
    mag = torch.stack([oracle.unabsorb_output(o_lat[t].abs(), w_uv.abs()) for t in range(o_lat.shape[0])])
    return ref, mag


def _assert_close(got, ref, mag, where):
    err = (got.double() - ref).abs()
    bound = ref.abs() * 2.0 ** -8 + mag * 2.0 ** -14
    bad = err > bound
    assert not bad.any(), f"{where}: {int(bad.sum())} elements out of bound, max err {err.max():.3e}"


CASES = [(1, 128), (64, 128), (127, 16), (128, 40), (129, 128), (300, 1)]


@pytest.mark.parametrize("tokens,heads", CASES)
def test_absorb_query(dev, tokens, heads):
    from mla_latent_kv_26_b200.decoder import absorb_query

    d = absorb_inputs(tokens=tokens, heads=heads, seed=tokens + heads)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    got = absorb_query(d["q"].to(dev), d["wkv_b"].to(dev), error_word=err).cpu()
    assert int(err.item()) == 0
    ref, mag = _ref_absorb(d["q"], d["wkv_b"])
    _assert_close(got[..., :512], ref, mag, f"absorb T{tokens} H{heads}")
    assert torch.equal(got[..., 512:], d["q"][..., 128:]), "q_pe must pass through unchanged"


@pytest.mark.parametrize("tokens,heads", CASES)
def test_unabsorb_output(dev, tokens, heads):
    from mla_latent_kv_26_b200.decoder import unabsorb_output

    d = absorb_inputs(tokens=tokens, heads=heads, seed=7 * tokens + heads)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    got = unabsorb_output(d["o_lat"].to(dev), d["wkv_b"].to(dev), error_word=err).cpu()
    assert int(err.item()) == 0
    ref, mag = _ref_unabsorb(d["o_lat"], d["wkv_b"])
    _assert_close(got, ref, mag, f"unabsorb T{tokens} H{heads}")


def test_output_rows_outside_the_tokens_untouched(dev):
    """Token tiles are padded to 128 rows with zeros inside the kernel; rows of
    the output past T must not be written."""
    from mla_latent_kv_26_b200.decoder import absorb_query, unabsorb_output

    d = absorb_inputs(tokens=70, heads=8, seed=3)
    big = torch.full((80, 8, 576), 7.0, dtype=torch.bfloat16, device=dev)
    absorb_query(d["q"].to(dev), d["wkv_b"].to(dev), out=big[:70])
    assert torch.all(big[70:] == 7.0)
    big_o = torch.full((80, 8, 128), 7.0, dtype=torch.bfloat16, device=dev)
    unabsorb_output(d["o_lat"].to(dev), d["wkv_b"].to(dev), out=big_o[:70])
    assert torch.all(big_o[70:] == 7.0)


@pytest.mark.parametrize("heads,lens", [(128, [700, 65]), (16, [300, 1, 130])])
def test_chain_matches_unabsorbed_attention(dev, heads, lens):
    """q (192-wide heads) -> absorb -> latent decode -> un-absorb on the GPU
    against the oracle's unabsorbed attention (keys and values expanded per
    head from the latent cache, softmax over 192-wide dot products): the three
    kernels together compute standard attention."""
    from mla_latent_kv_26_b200.decoder import MlaDecoder, absorb_query, unabsorb_output
    from mla_latent_kv_26_b200.workloads import small

    B = len(lens)
    d = small(batch=B, heads=heads, lens=lens, seed=11, cache_std=0.5)
    a = absorb_inputs(tokens=B, heads=heads, seed=12, w_std=0.05)
    q_abs = absorb_query(a["q"].to(dev), a["wkv_b"].to(dev))
    dec = MlaDecoder(batch=B, q_len=1, num_heads=heads, num_pages=d["num_pages"],
                     max_pages_per_seq=d["max_pages_per_seq"], device=dev)
    o_lat, _ = dec(q_abs.view(B, 1, heads, 576), d["cache"].to(dev), d["block_table"].to(dev),
                   d["seq_lens"].to(dev))
    got = unabsorb_output(o_lat.view(B, heads, 512), a["wkv_b"].to(dev)).double().cpu()
    w_uk, w_uv = a["wkv_b"][:, :128, :], a["wkv_b"][:, 128:, :]
    for b, L in enumerate(lens):
        rows = oracle.gather_rows(d["cache"], d["block_table"][b], torch.arange(L))
        naive = oracle.unabsorbed_attention(a["q"][b, :, :128], a["q"][b, :, 128:], w_uk, w_uv, rows[:, :512],
                                            rows[:, 512:])
        rel = ((got[b] - naive).norm() / naive.norm()).item()
        assert rel < 1e-2, f"sequence {b} (L={L}): relative L2 error {rel:.3e}"

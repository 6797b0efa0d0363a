"""More GPU parity cases against the float64 oracle (same tolerances as
test_parity.py): the online softmax's rescaling paths, fully masked tiles,
odd head counts, three causal query tokens, non-default softmax scales and a
single long sequence split across every worker.

With random N(0,1) data the running row maximum rarely grows by more than
2^8 after the first tile, so the O-rescaling code (in both CTAs of a pair:
the rows a CTA owns and the rows its peer owns) would hardly run; the
"growing scores" inputs scale the rope columns (k_pe, which are not part of
V) of cached row t by 1 + t/100 (t = its position in the sequence), which
makes the scores' maximum grow through the whole sequence while the values
keep their N(0,1) scale.
"""

import pytest
import torch

import oracle
from mla_latent_kv_26_b200.workloads import small

from test_parity import assert_parity, run_gpu  # noqa: E402  (tests/ is on sys.path under pytest)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(libmla):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def _grow_scores(d, per=100.0):
    """Scale the rope columns of cached row t of every sequence by 1 + t/per
    (through the block table)."""
    cache = d["cache"].float()
    for b in range(d["batch"]):
        L = int(d["seq_lens"][b])
        for i in range((L + 63) // 64):
            page = int(d["block_table"][b, i])
            t = torch.arange(i * 64, i * 64 + 64, dtype=torch.float32)
            cache[page, :, 512:] *= (1.0 + t / per)[:, None]
    d["cache"] = cache.to(torch.bfloat16)
    return d


def _check(d, dev, num_sms=0, scale=None, where=""):
    kw = {} if scale is None else {"softmax_scale": scale}
    from mla_latent_kv_26_b200.decoder import decoder_for

    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    dec = decoder_for(d, num_sms=num_sms, device=dev, **kw)
    out, lse = dec(g["q"], g["cache"], g["block_table"], g["seq_lens"], g["indices"])
    st, bits = dec.error()
    assert st == 0 and bits == 0, (st, bits)
    okw = {} if scale is None else {"softmax_scale": scale}
    o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], causal=d["causal"],
                                     indices=d["indices"], **okw)
    assert_parity(out.double().cpu(), lse.double().cpu(), o_ref, l_ref, where)


@pytest.mark.parametrize("num_sms", [2, 0])
@pytest.mark.parametrize("heads", [128, 40])
def test_growing_scores_exercise_rescaling(dev, heads, num_sms):
    d = _grow_scores(small(batch=2, heads=heads, lens=[1200, 700], seed=41))
    _check(d, dev, num_sms, where=f"growing h{heads} sms{num_sms}")


def test_growing_scores_causal_pair(dev):
    d = _grow_scores(small(batch=2, heads=128, q_len=2, causal=True, lens=[900, 130], seed=43))
    _check(d, dev, where="growing causal")


@pytest.mark.parametrize("heads", [1, 8, 17, 33, 100, 127])
def test_odd_head_counts(dev, heads):
    d = small(batch=2, heads=heads, lens=[300, 65], seed=47 + heads, nan_tail=True)
    _check(d, dev, where=f"h{heads}")


def test_three_causal_query_tokens(dev):
    d = small(batch=3, heads=32, q_len=3, causal=True, lens=[3, 70, 200], seed=53)
    _check(d, dev, where="sq3")


def test_sparse_fully_masked_tiles(dev):
    """Index slots 0..63 and 128..191 are all -1: two tiles with no visible
    token, one of them the first (running max still -inf after it)."""
    d = small(batch=2, heads=128, lens=[3000, 800], topk=320, seed=59)
    d["indices"][:, :, 0:64] = -1
    d["indices"][:, :, 128:192] = -1
    _check(d, dev, where="masked tiles")


def test_sparse_topk_not_multiple_of_page(dev):
    d = small(batch=3, heads=64, q_len=2, lens=[5000, 200, 77], topk=150, seed=61)
    _check(d, dev, where="topk150")


@pytest.mark.parametrize("scale", [0.02, 0.15])
def test_non_default_softmax_scale(dev, scale):
    d = small(batch=2, heads=128, lens=[700, 1500], seed=67)
    _check(d, dev, scale=scale, where=f"scale {scale}")


def test_one_long_sequence_split_across_all_workers(dev):
    d = small(batch=1, heads=128, lens=[20000], seed=71)
    _check(d, dev, where="long split")

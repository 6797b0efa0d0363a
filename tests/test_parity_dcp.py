"""GPU parity of decode context parallelism on one GPU: N ranks emulated one
after another (each shard decoded by the library as its own launches; no
kernel waits on another), their results stacked as the all-gather would
deliver them, and merged by mla_merge; compared with the float64 oracle on
the un-sharded inputs. Also mla_merge alone against the oracle's LSE merge.

Tolerances: the decode's (rel L2 <= 5e-3, |err| <= 1e-2 + 2^-8 |x|, LSE
within 1e-3); each shard's output is rounded to bf16 before the merge, which
adds at most half a bf16 ulp of the shard outputs.
"""

import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(libmla):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def _parity(out, lse, o_ref, l_ref):
    out, lse = out.double().cpu(), lse.double().cpu()
    assert ((out - o_ref).abs() <= 1e-2 + 2.0 ** -8 * o_ref.abs()).all()
    if o_ref.norm() > 0:
        assert float((out - o_ref).norm() / o_ref.norm()) <= 5e-3
    fin = torch.isfinite(l_ref)
    assert torch.equal(torch.isfinite(lse), fin)
    if fin.any():
        assert float((lse[fin] - l_ref[fin]).abs().max()) <= 1e-3


def _emulated_dcp(d, cache, world, dev):
    """Every rank's shard decoded by the library one after another on one
    GPU, then merged by mla_merge."""
    from mla_latent_kv_26_b200.dcp import _library_decode, library_merge, shard_inputs

    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items() if k != "cache"}
    cache = cache.to(dev)
    outs, lses = [], []
    for r in range(world):
        shard = shard_inputs(g["block_table"], g["seq_lens"], world=world, rank=r, q_len=d["q_len"],
                             causal=d["causal"], indices=g["indices"])
        o, l = _library_decode(g["q"], cache, shard)
        outs.append(o)
        lses.append(l)
    out, lse = library_merge(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize(dev)
    return out, lse


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("case", ["dense", "causal", "sparse", "fp8"])
def test_dcp_emulated_ranks_match_oracle(libmla, dev, world, case):
    from mla_latent_kv_26_b200.workloads import make_fp8_cache, small

    if case == "dense":
        d = small(batch=4, heads=128, lens=[5000, 700, 1, 64], seed=31, nan_tail=True)
    elif case == "causal":
        d = small(batch=3, heads=128, q_len=2, causal=True, lens=[4097, 2, 130], seed=32)
    elif case == "sparse":
        d = small(batch=3, heads=128, lens=[9000, 300, 2100], topk=512, seed=33)
    else:
        d = small(batch=4, heads=128, lens=[6000, 129, 1, 700], seed=34)
    cache = make_fp8_cache(d, nan_tail=True) if case == "fp8" else d["cache"]
    out, lse = _emulated_dcp(d, cache, world, dev)
    ref_cache = oracle.dequantize_cache(cache) if case == "fp8" else d["cache"]
    o_ref, l_ref = oracle.mla_decode(d["q"], ref_cache, d["block_table"], d["seq_lens"], causal=d["causal"],
                                     indices=d["indices"])
    _parity(out, lse, o_ref, l_ref)


def test_dcp_full_size_workload_eight_ranks(libmla, dev):
    """The batch-64, 128-head, ragged 1k-32k workload sharded over 8 emulated
    ranks: every sequence of the merged result against the oracle's
    un-sharded decode."""
    from mla_latent_kv_26_b200.workloads import make_inputs

    d = make_inputs("C3")
    out, lse = _emulated_dcp(d, d["cache"], 8, dev)
    o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"])
    _parity(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("parts,rows", [(1, 5), (2, 1000), (4, 37), (8, 129)])
def test_merge_kernel_matches_oracle_lse_merge(libmla, dev, parts, rows):
    from mla_latent_kv_26_b200.dcp import library_merge

    g = torch.Generator().manual_seed(parts * 1000 + rows)
    po = torch.randn(parts, rows, 512, generator=g).to(torch.bfloat16)
    pl = torch.randn(parts, rows, generator=g) * 5
    pl[torch.rand(parts, rows, generator=g) < 0.2] = float("-inf")   # empty shards of some rows
    pl[:, 0] = float("-inf")                                          # a row empty everywhere
    out, lse = library_merge(po.to(dev), pl.to(dev))
    torch.cuda.synchronize(dev)
    o_ref, l_ref = oracle.lse_merge(po, pl)
    out, lse = out.double().cpu(), lse.double().cpu()
    assert torch.equal(out[0], torch.zeros_like(out[0])) and torch.isneginf(lse[0])
    assert ((out - o_ref).abs() <= 1e-5 + 2.0 ** -8 * o_ref.abs()).all()
    fin = torch.isfinite(l_ref)
    assert torch.equal(torch.isfinite(lse), fin)
    assert float((lse[fin] - l_ref[fin]).abs().max()) <= 1e-5

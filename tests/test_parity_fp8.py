"""GPU parity of the fp8 latent cache: mla_cache_insert_fp8 and
mla_decode_fp8, through the C ABI, against the float64 oracle.

Insert: the e4m3 codes are integers decided by floating point, so both sides
decide from the same bf16 latent (the GPU's own bf16 insert of the same
tokens): the codes and the float32 scale must equal oracle.quantize_rows of
those values bit for bit; k_pe must equal the bf16 insert's; the tail bytes
are zero; rows of other tokens are untouched.

Decode: caches drawn directly in the fp8 format (random codes and scales);
the oracle decodes oracle.dequantize_cache of the same bytes. Tolerances are
the decode's (rel L2 <= 5e-3, |err| <= 1e-2 + 2^-8 |x|, LSE within 1e-3).
"""

import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(libmla):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def _to(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def _assert_parity(out, lse, o_ref, l_ref, where):
    out, lse = out.double().cpu(), lse.double().cpu()
    err = (out - o_ref).abs()
    assert (err <= 1e-2 + 2.0 ** -8 * o_ref.abs()).all(), f"{where}: max abs {float(err.max()):.3e}"
    if o_ref.norm() > 0:
        rel = float((out - o_ref).norm() / o_ref.norm())
        assert rel <= 5e-3, f"{where}: rel L2 {rel:.3e}"
    fin = torch.isfinite(l_ref)
    assert torch.equal(torch.isfinite(lse), fin), where
    if fin.any():
        assert float((lse[fin] - l_ref[fin]).abs().max()) <= 1e-3, where


# ---------------------------------------------------------------- insert


@pytest.mark.parametrize("case", ["prefill", "decode-token", "zero-latent", "large-and-small", "prefill-64x1024"])
def test_fp8_insert_codes_bit_exact(libmla, dev, case):
    from mla_latent_kv_26_b200.decoder import cache_insert
    from mla_latent_kv_26_b200.workloads import insert_inputs

    if case == "prefill":
        d = insert_inputs(lens=[200, 70], new_tokens=[200, 70], seed=41)
    elif case == "decode-token":
        d = insert_inputs(lens=[300, 65, 1], new_tokens=[1, 1, 1], seed=42)
    elif case == "prefill-64x1024":
        d = insert_inputs(lens=[1024] * 64, new_tokens=[1024] * 64, seed=5)
    elif case == "zero-latent":
        d = insert_inputs(lens=[64], new_tokens=[64], seed=43)
        d["kv"][:5, :512] = 0
    else:
        d = insert_inputs(lens=[130], new_tokens=[130], seed=44, kv_std=3.0)
        d["kv"][::3] = (d["kv"][::3].float() * 2.0 ** 40).to(torch.bfloat16)
        d["kv"][1::3] = (d["kv"][1::3].float() * 2.0 ** -40).to(torch.bfloat16)
    g = _to(d, dev)
    eps = 1e-6
    # the bf16 insert gives the latent values both sides quantise
    bf = g["cache"].clone()
    cache_insert(g["kv"], g["weight"], g["cos"], g["sin"], g["seq_ids"], g["positions"], g["block_table"], bf, eps=eps)
    P = d["num_pages"]
    raw = torch.full((P, 64, 656), 0xA5, dtype=torch.uint8, device=dev)
    before = raw.clone()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    cache_insert(g["kv"], g["weight"], g["cos"], g["sin"], g["seq_ids"], g["positions"], g["block_table"], raw,
                 eps=eps, error_word=err)
    torch.cuda.synchronize(dev)
    assert int(err.item()) == 0
    bf, raw, before = bf.cpu(), raw.cpu(), before.cpu()
    written = torch.zeros(P, 64, dtype=torch.bool)
    for b, p in zip(d["seq_ids"].tolist(), d["positions"].tolist()):
        written[int(d["block_table"][b, p // 64]), p % 64] = True
    rows_bf = bf[written]                      # [n, 576]
    rows = raw[written]                        # [n, 656]
    codes, scale, rope = oracle.unpack_rows(rows)
    ref_codes, ref_scale = oracle.quantize_rows(rows_bf[:, :512])
    assert torch.equal(codes, ref_codes)
    assert torch.equal(scale, ref_scale.to(torch.float32))
    assert torch.equal(rope, rows_bf[:, 512:])
    assert torch.equal(rows[:, 644:], torch.zeros_like(rows[:, 644:]))
    assert torch.equal(raw[~written], before[~written])


# ---------------------------------------------------------------- decode


def _fp8_case(name):
    from mla_latent_kv_26_b200.workloads import make_fp8_cache, small

    if name == "dense":
        d = small(batch=4, heads=128, lens=[3000, 700, 64, 1], seed=51)
    elif name == "heads16":
        d = small(batch=3, heads=16, lens=[4097, 129, 5], seed=52)
    elif name == "causal":
        d = small(batch=3, heads=128, q_len=2, causal=True, lens=[2, 65, 4000], seed=53)
    elif name == "sparse":
        d = small(batch=2, heads=128, lens=[9000, 2100], topk=2048, seed=54)
    else:
        d = small(batch=2, heads=64, lens=[1000, 333], seed=55, q_std=10.0)
    return d, make_fp8_cache(d, nan_tail=True)


@pytest.mark.parametrize("name", ["dense", "heads16", "causal", "sparse", "large-q"])
@pytest.mark.parametrize("num_sms", [0, 2])
def test_fp8_decode_matches_oracle(libmla, dev, name, num_sms):
    from mla_latent_kv_26_b200.decoder import decoder_for

    d, raw = _fp8_case(name)
    g = _to(d, dev)
    dec = decoder_for(d, num_sms=num_sms, device=dev)
    out, lse = dec(g["q"], raw.to(dev), g["block_table"], g["seq_lens"], g["indices"])
    assert dec.error() == (0, 0)
    o_ref, l_ref = oracle.mla_decode(d["q"], oracle.dequantize_cache(raw), d["block_table"], d["seq_lens"],
                                     causal=d["causal"], indices=d["indices"])
    _assert_parity(out, lse, o_ref, l_ref, f"fp8 {name} sms{num_sms}")
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("key", ["C1", "C2", "C3", "C4", "C5"])
def test_fp8_decode_full_size_workload(libmla, dev, key):
    """The benchmark workloads at full size over an fp8 cache, in the
    benchmark's launch configuration (all SMs): every sequence of the batch
    against the oracle, the relative L2 error over the whole output."""
    from mla_latent_kv_26_b200.decoder import decoder_for
    from mla_latent_kv_26_b200.workloads import make_fp8_cache, make_inputs

    d = make_inputs(key)
    raw = make_fp8_cache(d)
    del d["cache"]
    g = _to(d, dev)
    dec = decoder_for(d, device=dev)
    out, lse = dec(g["q"], raw.to(dev), g["block_table"], g["seq_lens"], g["indices"])
    assert dec.error() == (0, 0)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    o_ref, l_ref = oracle.mla_decode(d["q"], oracle.dequantize_cache(raw), d["block_table"], d["seq_lens"],
                                     causal=d["causal"], indices=d["indices"])
    _assert_parity(out, lse, o_ref, l_ref, f"fp8 {key}")


def test_fp8_cuda_graph_replay_with_new_lengths(libmla, dev):
    """One captured step (plan, decode, combine over an fp8 cache) replayed
    after the device-side lengths were changed in place: the plan runs inside
    the graph, so the replay decodes the new lengths."""
    from mla_latent_kv_26_b200.decoder import decoder_for
    from mla_latent_kv_26_b200.workloads import make_fp8_cache, small

    d = small(batch=3, heads=128, lens=[3000, 300, 64], seed=57)
    raw = make_fp8_cache(d)
    g = _to(d, dev)
    cache = raw.to(dev)
    dec = decoder_for(d, device=dev)
    dec(g["q"], cache, g["block_table"], g["seq_lens"])
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            dec(g["q"], cache, g["block_table"], g["seq_lens"], stream=s)
    torch.cuda.current_stream(dev).wait_stream(s)
    # within each sequence's own pages: 3000 -> 3008 fills its last page,
    # 300 -> 1 and 64 -> 0 shorten
    new = torch.tensor([3008, 1, 0], dtype=torch.int32)
    g["seq_lens"].copy_(new.to(dev))
    graph.replay()
    torch.cuda.synchronize(dev)
    assert dec.error() == (0, 0)
    o_ref, l_ref = oracle.mla_decode(d["q"], oracle.dequantize_cache(raw), d["block_table"], new)
    _assert_parity(dec.out, dec.lse, o_ref, l_ref, "fp8 graph replay, new lengths")


def test_fp8_insert_then_decode_chain(libmla, dev):
    """Insert new tokens into an fp8 cache on the GPU, decode over it on the
    GPU; the oracle inserts into a bf16 cache, quantises and decodes."""
    from mla_latent_kv_26_b200.decoder import cache_insert, decoder_for
    from mla_latent_kv_26_b200.workloads import insert_inputs

    lens = [300, 64, 129]
    d = insert_inputs(lens=lens, new_tokens=lens, seed=61)
    g = _to(d, dev)
    raw = torch.zeros(d["num_pages"], 64, 656, dtype=torch.uint8, device=dev)
    cache_insert(g["kv"], g["weight"], g["cos"], g["sin"], g["seq_ids"], g["positions"], g["block_table"], raw)
    q = (torch.randn(len(lens), 1, 128, 576, generator=torch.Generator().manual_seed(62))).to(torch.bfloat16)
    seq = torch.tensor(lens, dtype=torch.int32)
    dec = decoder_for({"batch": len(lens), "q_len": 1, "heads": 128, "num_pages": d["num_pages"],
                       "max_pages_per_seq": d["max_pages_per_seq"], "topk": 0, "causal": False}, device=dev)
    out, lse = dec(q.to(dev), raw, g["block_table"], seq.to(dev))
    assert dec.error() == (0, 0)
    ref_cache, _ = oracle.cache_insert(d["cache"], d["block_table"], d["seq_ids"], d["positions"], d["kv"],
                                       d["weight"], 1e-6, d["cos"], d["sin"])
    o_ref, l_ref = oracle.mla_decode(q, oracle.fp8_roundtrip_cache(ref_cache.to(torch.bfloat16)), d["block_table"],
                                     seq)
    _assert_parity(out, lse, o_ref, l_ref, "fp8 insert -> decode")

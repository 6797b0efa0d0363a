"""GPU parity: libmla (through the C ABI) against the float64 oracle on the
same seeded inputs.

Tolerances (bf16 inputs, fp32 accumulation):
* relative L2 error of the whole output tensor <= 5e-3;
* elementwise |gpu - oracle| <= 1e-2 + 2^-8 |oracle|: a max-abs bound of 1e-2
  on the kernel's own error, on top of the rounding of the bf16 output itself
  (at most half a bf16 ulp, <= 2^-8 |x|), which every bf16 result carries;
* LSE: |gpu - oracle| <= 1e-3 where finite; -inf exactly where the oracle has
  no visible token.
"""

import math

import pytest
import torch

import oracle
from oracle.plan import split_plan

pytestmark = pytest.mark.gpu

REL_L2 = 5e-3
MAX_ABS = 1e-2
LSE_ABS = 1e-3


@pytest.fixture(scope="module")
def dev(libmla):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def _to(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def run_gpu(d, dev, num_sms=0):
    from mla_latent_kv_26_b200.decoder import decoder_for

    g = _to(d, dev)
    dec = decoder_for(d, num_sms=num_sms, device=dev)
    out, lse = dec(g["q"], g["cache"], g["block_table"], g["seq_lens"], g["indices"])
    st, bits = dec.error()
    return out.double().cpu(), lse.double().cpu(), st, bits, dec


def assert_parity(out, lse, o_ref, l_ref, where=""):
    err = (out - o_ref).abs()
    bound = MAX_ABS + (2.0 ** -8) * o_ref.abs()
    worst = (err - bound).max().item() if err.numel() else -1.0
    assert worst <= 0, f"{where}: elementwise error above 1e-2 + 2^-8|x| by {worst:.3e} (max abs {err.max():.3e})"
    nref = o_ref.norm().item()
    if nref > 0:
        rel = (out - o_ref).norm().item() / nref
        assert rel <= REL_L2, f"{where}: rel L2 {rel:.3e}"
    fin = torch.isfinite(l_ref)
    assert torch.equal(torch.isfinite(lse), fin), f"{where}: -inf pattern of LSE differs"
    assert torch.equal(torch.isneginf(lse), torch.isneginf(l_ref))
    if fin.any():
        le = (lse[fin] - l_ref[fin]).abs().max().item()
        assert le <= LSE_ABS, f"{where}: LSE abs error {le:.3e}"


def check_case(d, dev, num_sms=0, where=""):
    out, lse, st, bits, dec = run_gpu(d, dev, num_sms)
    assert st == 0 and bits == 0, (st, bits)
    o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], causal=d["causal"],
                                     indices=d["indices"])
    assert_parity(out, lse, o_ref, l_ref, where)
    return out, lse, dec


# ---------------------------------------------------------------- small shapes


DENSE = [
    (16, [256]), (16, [1, 63, 64, 65]), (32, [130, 7]), (64, [1000]), (128, [64]), (128, [1, 200, 65]),
    (128, [4100, 33]), (48, [129, 128, 127]),
]


@pytest.mark.parametrize("heads,lens", DENSE)
@pytest.mark.parametrize("num_sms", [2, 10, 0])
def test_dense_small(dev, heads, lens, num_sms):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=len(lens), heads=heads, lens=lens, seed=sum(lens) + heads)
    check_case(d, dev, num_sms, f"H{heads} {lens} sms{num_sms}")


@pytest.mark.parametrize("heads", [16, 128])
@pytest.mark.parametrize("lens", [[1, 2, 65, 300], [64, 4097]])
def test_causal_pair(dev, heads, lens):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=len(lens), heads=heads, q_len=2, causal=True, lens=lens, seed=7 + heads)
    check_case(d, dev, 0, f"causal H{heads} {lens}")
    check_case(d, dev, 2, f"causal H{heads} {lens} one worker")


@pytest.mark.parametrize("q_len,causal,lens", [(3, True, [65, 129, 1, 2, 700]), (4, False, [64, 193, 5]),
                                                (2, True, [1, 65, 4097, 3000])])
@pytest.mark.parametrize("num_sms", [0, 16, 14])
def test_query_token_groups(dev, q_len, causal, lens, num_sms):
    """Several query tokens per sequence: with enough workers the plan puts
    token g of every sequence in worker group g (16 SMs = 8 workers is the
    threshold for two tokens, 14 SMs stays ungrouped); lengths 64 k + 1 give
    the tokens different page counts under the causal mask."""
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=len(lens), heads=128, q_len=q_len, causal=causal, lens=lens, seed=40 + q_len)
    _, _, dec = check_case(d, dev, num_sms, f"Sq={q_len} causal={causal} sms{num_sms}")
    plan = dec.plan.view(torch.int32).cpu()
    assert plan[6].item() == oracle.plan.plan_groups(q_len=q_len, topk=0, num_pairs=dec.num_workers)


def test_non_causal_pair(dev):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=64, q_len=2, causal=False, lens=[100, 1], seed=9)
    check_case(d, dev, 0, "non-causal Sq=2")


@pytest.mark.parametrize("topk,lens", [(1, [50, 3]), (64, [5000, 64]), (100, [300, 7000]), (2048, [3000, 2100])])
def test_sparse(dev, topk, lens):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=len(lens), heads=128, lens=lens, topk=topk, seed=topk)
    check_case(d, dev, 0, f"sparse top{topk}")
    check_case(d, dev, 4, f"sparse top{topk} 2 workers")


def test_sparse_skips_minus_one(dev):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=3, heads=32, lens=[500, 90, 200], topk=150, seed=5)
    idx = d["indices"]
    idx[0, 0, ::3] = -1
    idx[2, 0, :] = -1                 # a row with nothing to attend to
    check_case(d, dev, 0, "sparse with -1")


def test_nan_tails_and_slack_pages_never_leak(dev):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=4, heads=128, lens=[70, 129, 1, 640], seed=11, nan_tail=True)
    out, lse, _ = check_case(d, dev, 0, "nan tails")
    assert torch.isfinite(out).all()


def test_empty_sequences_and_batch(dev):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=3, heads=64, lens=[0, 5, 0], seed=13)
    out, lse, _ = check_case(d, dev, 0, "empty sequences")
    assert torch.equal(out[0], torch.zeros_like(out[0])) and torch.isneginf(lse[0]).all()
    d0 = small(batch=1, heads=16, lens=[1], seed=1)
    from mla_latent_kv_26_b200.decoder import MlaDecoder

    dec = MlaDecoder(batch=0, q_len=1, num_heads=16, num_pages=1, max_pages_per_seq=1, device=dev)
    e = torch.empty(0, dtype=torch.int32, device=dev)
    dec(torch.empty(0, 1, 16, 576, dtype=torch.bfloat16, device=dev), d0["cache"].to(dev)[:1],
        torch.empty(0, 1, dtype=torch.int32, device=dev), e)
    assert dec.error() == (0, 0)


def test_split_invariance(dev):
    """One worker (no splits) vs many workers (most tasks split) agree with each
    other to bf16 rounding and both match the oracle."""
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=3, heads=128, lens=[3000, 1500, 64], seed=17)
    o1, l1, _ = check_case(d, dev, 2, "1 worker")
    o2, l2, dec = check_case(d, dev, 0, "all workers")
    assert dec.num_workers > 1
    assert ((o1 - o2).abs() <= 2.0 ** -7 * o1.abs().clamp_min(1.0)).all()
    assert (l1 - l2).abs().max() < 1e-4


def test_back_to_back_steps_with_changing_lengths(dev):
    """Steps on one decoder and one stream with no host synchronisation
    between them, the lengths (and so the plan and the split) changing every
    step. The plan, decode and combine are chained as programmatic
    dependents: a step's decode must read that step's plan, and must not
    overwrite the previous step's partials before its combine has merged
    them. Each step's result is copied on the same stream before the next
    step starts writing."""
    from mla_latent_kv_26_b200.workloads import small

    steps = [[3000, 700, 64, 1], [1, 5000, 200, 129], [4097, 2, 3000, 65], [0, 64, 1, 2000]] * 2
    cap = [max(col) for col in zip(*steps)]
    d = small(batch=4, heads=128, lens=cap, seed=71)
    g = _to(d, dev)
    dec = run_gpu(d, dev)[4]
    lens_dev = [torch.tensor(L, dtype=torch.int32, device=dev) for L in steps]
    torch.cuda.synchronize(dev)
    outs = []
    for sl in lens_dev:
        dec(g["q"], g["cache"], g["block_table"], sl)
        outs.append((dec.out.clone(), dec.lse.clone()))
    torch.cuda.synchronize(dev)
    assert dec.error() == (0, 0)
    for L, (o, l) in zip(steps, outs):
        o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"], torch.tensor(L, dtype=torch.int32))
        assert_parity(o.double().cpu(), l.double().cpu(), o_ref, l_ref, f"back-to-back {L}")


def test_deterministic(dev):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=128, lens=[5000, 77], seed=19)
    a = run_gpu(d, dev)
    b = run_gpu(d, dev)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_plan_matches_oracle_schedule(dev):
    from mla_latent_kv_26_b200.workloads import small

    for lens, Sq, causal, topk, sms in [([1024, 32768, 5000, 77, 0, 64], 1, False, 0, 10), ([4096, 600], 2, True, 0, 0),
                                         ([9000, 9000], 1, False, 2048, 6), ([65, 129, 1, 700], 3, True, 0, 0),
                                         ([4096, 600], 2, True, 0, 14)]:
        d = small(batch=len(lens), heads=128, q_len=Sq, causal=causal, lens=lens, topk=topk, seed=3)
        out, lse, st, bits, dec = run_gpu(d, dev, sms)
        plan = dec.plan.view(torch.int32).cpu()
        ref = split_plan(lens, q_len=Sq, causal=causal, topk=topk, max_pages_per_seq=d["max_pages_per_seq"],
                         num_pairs=dec.num_workers)
        T = len(ref["task_tokens"])
        assert plan[1].item() == T
        assert plan[2].item() == ref["quota"]
        assert plan[3].item() == ref["total_pages"]
        assert plan[4].item() == dec.num_workers
        assert plan[6].item() == ref["groups"] and plan[7].item() == ref["workers_per_group"]
        assert plan[8:8 + T + 1].tolist() == ref["prefix"]
        assert plan[9 + T:9 + 2 * T].tolist() == ref["task_tokens"]


def test_cuda_graph_capture(dev):
    from mla_latent_kv_26_b200.decoder import decoder_for
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=128, lens=[2000, 300], seed=23)
    g = _to(d, dev)
    dec = decoder_for(d, device=dev)
    dec(g["q"], g["cache"], g["block_table"], g["seq_lens"])
    ref = dec.out.clone()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        dec.out.zero_()
        with torch.cuda.graph(graph, stream=s):
            dec(g["q"], g["cache"], g["block_table"], g["seq_lens"], stream=s)
    torch.cuda.current_stream(dev).wait_stream(s)
    dec.out.zero_()
    graph.replay()
    torch.cuda.synchronize(dev)
    assert torch.equal(dec.out, ref)


# ---------------------------------------------------------------- device-side errors


def test_bad_page_id_is_skipped_and_flagged(dev):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=64, lens=[300, 200], seed=29)
    d["block_table"][0, 2] = 10 ** 6           # tokens 128..191 of sequence 0 point outside the cache
    out, lse, st, bits, _ = run_gpu(d, dev)
    from mla_latent_kv_26_b200.binding import MLA_DEVERR_PAGE_ID, MLA_ERR_DEVICE_BOUNDS

    assert st == MLA_ERR_DEVICE_BOUNDS and bits == MLA_DEVERR_PAGE_ID
    keep = [t for t in range(300) if not 128 <= t < 192]
    idx = torch.full((2, 1, 300), -1, dtype=torch.int32)
    idx[0, 0, :len(keep)] = torch.tensor(keep, dtype=torch.int32)
    idx[1, 0, :200] = torch.arange(200, dtype=torch.int32)
    o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"].clamp(max=d["num_pages"] - 1),
                                     d["seq_lens"], indices=idx)
    assert_parity(out, lse, o_ref, l_ref, "bad page")


def test_bad_length_is_flagged(dev):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=16, lens=[100, 64], seed=31)
    d["seq_lens"][1] = 64 * d["max_pages_per_seq"] + 1
    out, lse, st, bits, _ = run_gpu(d, dev)
    from mla_latent_kv_26_b200.binding import MLA_DEVERR_SEQ_LEN

    assert bits == MLA_DEVERR_SEQ_LEN
    assert torch.equal(out[1], torch.zeros_like(out[1])) and torch.isneginf(lse[1]).all()
    o_ref, l_ref = oracle.mla_decode(d["q"][:1], d["cache"], d["block_table"][:1], d["seq_lens"][:1])
    assert_parity(out[:1], lse[:1], o_ref, l_ref, "valid sequence next to a bad one")


def test_bad_sparse_index_is_skipped_and_flagged(dev):
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=1, heads=128, lens=[400], topk=70, seed=37)
    d["indices"][0, 0, 5] = 400            # == L: out of range
    d["indices"][0, 0, 6] = -7
    out, lse, st, bits, _ = run_gpu(d, dev)
    from mla_latent_kv_26_b200.binding import MLA_DEVERR_INDEX

    assert bits == MLA_DEVERR_INDEX
    idx = d["indices"].clone()
    idx[0, 0, 5] = -1
    idx[0, 0, 6] = -1
    o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], indices=idx)
    assert_parity(out, lse, o_ref, l_ref, "bad index")


# ---------------------------------------------------------------- full-size workloads


@pytest.mark.parametrize("key", ["C1", "C2", "C3", "C4", "C5"])
def test_full_size_workload(dev, key):
    """The benchmark workloads at full size in the benchmark's launch
    configuration (all SMs): every sequence of the batch against the oracle,
    element by element, with the relative L2 error taken over the whole
    output tensor."""
    from mla_latent_kv_26_b200.workloads import make_inputs

    d = make_inputs(key)
    out, lse, st, bits, dec = run_gpu(d, dev, 0)
    assert st == 0 and bits == 0
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], causal=d["causal"],
                                     indices=d["indices"])
    assert_parity(out, lse, o_ref, l_ref, key)


@pytest.mark.parametrize("q_std", [10.0, 20.0])
@pytest.mark.parametrize("heads", [128, 16])
def test_large_magnitude_queries(dev, q_std, heads):
    """Queries 10x and 20x the usual scale against an N(0, 1) cache: partial
    scores of each CTA half reach the hundreds, where the 23-bit block
    fixed-point exchange of partial scores is coarsest (its error per score is
    at most 2^-22 of the largest partial score of the row in the tile). Both
    the output and the LSE must stay within the usual tolerances."""
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=4, heads=heads, lens=[3000, 700, 64, 1], seed=int(q_std) + heads, q_std=q_std)
    check_case(d, dev, 0, f"q std {q_std} H{heads}")
    check_case(d, dev, 2, f"q std {q_std} H{heads} one worker")

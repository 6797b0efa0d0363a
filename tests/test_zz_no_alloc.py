"""The decode entry point that allocates nothing (mla_decode_noalloc).

Some callers cannot call cudaMalloc while they run (a caching allocator that
owns all device memory, or a host that forbids allocation while serving), so
this entry point keeps its scratch in a fixed array inside the library. Here
it is called through the C ABI three times in a row, on three different problems (the
last one too large for all workers' partials, so it runs on fewer), and
each result is compared with the allocating entry points (plan + decode +
combine with caller-provided buffers) within the parity tolerances used
elsewhere: relative L2 <= 5e-3, |a - b| <= 1e-2 + 2^-8 |b| elementwise, LSE
within 1e-3. This file is collected last on purpose.
"""

import pytest
import torch

pytestmark = pytest.mark.gpu


def _to(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def _close(out, lse, ref_out, ref_lse):
    a, b = out.double().cpu(), ref_out.double().cpu()
    assert ((a - b).abs() <= 1e-2 + 2.0 ** -8 * b.abs()).all()
    assert float((a - b).norm() / b.norm()) <= 5e-3
    la, lb = lse.double().cpu(), ref_lse.double().cpu()
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isfinite(la), fin)
    assert float((la[fin] - lb[fin]).abs().max()) <= 1e-3


def _noalloc(B, d, dev):
    g = _to(d, dev)
    desc = B.make_desc(batch=d["batch"], q_len=d["q_len"], num_heads=d["heads"], num_pages=d["num_pages"],
                       max_pages_per_seq=d["max_pages_per_seq"], topk=d["topk"], causal=d["causal"])
    out = torch.full((d["batch"], d["q_len"], d["heads"], 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((d["batch"], d["q_len"], d["heads"]), float("nan"), dtype=torch.float32, device=dev)
    st = B.mla_decode_noalloc(desc, g["seq_lens"], g["q"], g["cache"], g["block_table"], g["indices"], out, lse,
                              torch.cuda.current_stream(dev))
    assert st == B.MLA_OK, B.mla_status_string(st)
    torch.cuda.synchronize(dev)
    return out, lse


def test_noalloc_matches_allocating_path_twice(libmla):
    from mla_latent_kv_26_b200.decoder import decoder_for
    from mla_latent_kv_26_b200.workloads import small

    B = libmla
    dev = torch.device("cuda", torch.cuda.current_device())
    lens64 = [int(x) for x in torch.randint(1, 400, (64,), generator=torch.Generator().manual_seed(73))]
    problems = [
        small(batch=4, heads=128, lens=[5000, 64, 1, 2100], seed=71, nan_tail=True),
        small(batch=3, heads=16, q_len=2, causal=True, lens=[700, 2, 4097], seed=72),
        # 64 query tokens of 128 heads: the fixed scratch holds the partials of
        # only 63 workers, so this call runs on fewer workers than the device has
        small(batch=64, heads=128, lens=lens64, seed=73, nan_tail=True),
    ]
    for d in problems:   # calls in a row; each reuses the scratch the previous one left behind
        out, lse = _noalloc(B, d, dev)
        g = _to(d, dev)
        dec = decoder_for(d, device=dev)
        ref_out, ref_lse = dec(g["q"], g["cache"], g["block_table"], g["seq_lens"], g["indices"])
        torch.cuda.synchronize(dev)
        assert dec.error() == (0, 0)
        _close(out, lse, ref_out, ref_lse)


def test_noalloc_rejects_batches_beyond_its_scratch(libmla):
    B = libmla
    dev = torch.device("cuda", torch.cuda.current_device())
    # 400 query tokens of 128 heads need more split slots than the fixed scratch holds
    desc = B.make_desc(batch=400, q_len=1, num_heads=128, num_pages=1, max_pages_per_seq=1)
    one = torch.zeros(16, dtype=torch.int32, device=dev)
    st = B.mla_decode_noalloc(desc, one, one, one, one, None, one, one, torch.cuda.current_stream(dev))
    assert st == B.MLA_ERR_WORKSPACE_TOO_SMALL

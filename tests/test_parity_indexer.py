"""GPU parity of the sparse-attention indexer (mla_index_scores) and of the
exact top-k (mla_topk), through the C ABI, against the float64 oracle.

Scores: each product of two e4m3 values is exact in fp32; the GPU sums 128
of them on the tensor cores and h weighted ReLU terms in fp32. The bound is
|gpu - oracle| <= 2^-9 * mag, with mag the same score over absolute values
(k_s * sum_h |q_s| * sum_d |q k|): a few hundred fp32 roundings, with margin
for the tensor cores' internal accumulation order.

Top-k is integer index work decided by floating point, so both sides decide
on the same fp32 scores (the GPU's): the GPU positions must equal the
oracle's top-k of those scores bit for bit. Against the oracle's own float64
scores the selection is compared where it is unique: positions whose score
is clearly above the cut are chosen, clearly below are not.
"""

import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(libmla):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def gpu_scores(B, d, dev):
    q = d["q"].to(dev)
    q_s = d["q_s"].to(dev)
    k = d["k"].to(dev)
    k_s = d["k_s"].to(dev)
    out = torch.full((d["batch"], d["q_len"], d["num_keys"]), float("nan"), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    desc = B.make_index_desc(batch=d["batch"], q_len=d["q_len"], num_heads=d["heads"], num_keys=d["num_keys"])
    st = B.mla_index_scores(desc, q, q_s, k, k_s, out, err, torch.cuda.current_stream(dev))
    assert st == B.MLA_OK, B.mla_status_string(st)
    torch.cuda.synchronize(dev)
    assert int(err.item()) == 0
    return out.cpu()


def gpu_topk(B, scores, k, dev, lens=None):
    rows, n = scores.shape
    s = scores.contiguous().to(dev)
    out = torch.full((rows, k), -7, dtype=torch.int32, device=dev)
    vl = None if lens is None else torch.as_tensor(lens, dtype=torch.int32).to(dev)
    st = B.mla_topk(B.make_topk_desc(rows=rows, num_keys=n, k=k), s, vl, out, torch.cuda.current_stream(dev))
    assert st == B.MLA_OK, B.mla_status_string(st)
    torch.cuda.synchronize(dev)
    return out.cpu()


def assert_scores(got, d, batches=None):
    bs = list(range(d["batch"])) if batches is None else list(batches)
    sel = lambda t: t[bs]  # noqa: E731
    ref = oracle.index_scores(sel(d["q"]), sel(d["q_s"]), sel(d["k"]), sel(d["k_s"]))
    mag = oracle.index_scores(sel(d["q"]).to(torch.float32).abs(), sel(d["q_s"]).abs(),
                              sel(d["k"]).to(torch.float32).abs(), sel(d["k_s"]))
    g = got[bs].double()
    assert torch.isfinite(g).all()
    bad = (g - ref).abs() > 2.0 ** -9 * mag
    assert not bad.any(), f"{int(bad.sum())} scores off; worst {float(((g - ref).abs() / mag.clamp_min(1e-30)).max()):.3e}"
    return ref


SHAPES = [
    (2, 128, 64, 128),   # the shapes printed on the page
    (2, 3, 64, 300),     # ragged key tiles
    (1, 1, 16, 1),       # one key
    (3, 5, 32, 129),     # G = 8 queries per MMA: one partial group
    (1, 9, 64, 1000),    # G = 4: three groups, the last partial
    (2, 2, 128, 257),
    (1, 3, 256, 200),    # N = 256 heads, one query per MMA
    (4, 1, 64, 5000),    # decode-like: one query, many key tiles per CTA
]


@pytest.mark.parametrize("b,m,h,n", SHAPES)
def test_index_scores_match_oracle(libmla, dev, b, m, h, n):
    from mla_latent_kv_26_b200.workloads import indexer_inputs

    d = indexer_inputs(batch=b, q_len=m, heads=h, num_keys=n, seed=b * 1000 + m * 10 + h + n)
    assert_scores(gpu_scores(libmla, d, dev), d)


def test_index_scores_relu_and_sign_of_weights(libmla, dev):
    """Non-positive queries against non-negative keys: every score is exactly
    0 (the ReLU), whatever the sign of the weights."""
    from mla_latent_kv_26_b200.workloads import indexer_inputs

    d = indexer_inputs(batch=2, q_len=2, heads=32, num_keys=200, seed=5)
    d["q"] = (-(d["q"].to(torch.float32).abs())).to(torch.float8_e4m3fn)
    d["k"] = d["k"].to(torch.float32).abs().to(torch.float8_e4m3fn)
    got = gpu_scores(libmla, d, dev)
    assert torch.equal(got, torch.zeros_like(got))


# ---------------------------------------------------------------- top-k


def _tie_heavy(rows, n, seed):
    g = torch.Generator().manual_seed(seed)
    s = torch.randint(-3, 5, (rows, n), generator=g).float() * 0.5
    s[s == 0] = torch.where(torch.rand(int((s == 0).sum()), generator=g) < 0.5, -0.0, 0.0)
    return s


@pytest.mark.parametrize("rows,n,k", [(3, 1, 1), (4, 100, 7), (2, 16384, 2048), (2, 16385, 2048),
                                      (3, 40000, 2048), (2, 131072, 2048), (1, 131072, 1), (2, 1000, 1500),
                                      (1, 400000, 4096)])
@pytest.mark.parametrize("kind", ["normal", "ties"])
def test_topk_bit_exact(libmla, dev, rows, n, k, kind):
    g = torch.Generator().manual_seed(rows * 7 + n + k)
    s = torch.randn(rows, n, generator=g) if kind == "normal" else _tie_heavy(rows, n, n + k)
    got = gpu_topk(libmla, s, k, dev)
    assert torch.equal(got, oracle.topk_positions(s, k)), kind


def test_topk_valid_lengths(libmla, dev):
    g = torch.Generator().manual_seed(3)
    s = _tie_heavy(6, 50000, 9)
    s[1] = torch.randn(50000, generator=g)
    lens = [50000, 30000, 0, 5, 2048, 2049]
    got = gpu_topk(libmla, s, 2048, dev, lens)
    assert torch.equal(got, oracle.topk_positions(s, 2048, torch.tensor(lens)))


# ---------------------------------------------------------------- chain: indexer -> top-k -> sparse decode


def test_indexer_topk_sparse_decode_chain(libmla, dev):
    """Scores on the GPU, their top-k on the GPU (bit-exact against the oracle's
    top-k of the same scores, and the unique part of the selection against the
    oracle's float64 scores), then the sparse decode over those positions
    against the float64 decode oracle."""
    from mla_latent_kv_26_b200.decoder import decoder_for
    from mla_latent_kv_26_b200.workloads import indexer_inputs, small

    lens = [3000, 700, 2049, 64]
    B, K = len(lens), 512
    n = max(lens)
    d_idx = indexer_inputs(batch=B, q_len=1, heads=64, num_keys=n, seed=21)
    sc = gpu_scores(libmla, d_idx, dev)
    ref = assert_scores(sc, d_idx)
    idx = gpu_topk(libmla, sc.view(B, n), K, dev, lens)
    assert torch.equal(idx, oracle.topk_positions(sc.view(B, n), K, torch.tensor(lens)))
    for b, L in enumerate(lens):
        r = ref[b, 0, :L]
        chosen = set(int(t) for t in idx[b] if t >= 0)
        assert len(chosen) == min(K, L)
        if L > K:
            cut = torch.sort(r, descending=True).values[K - 1]
            tol = 2.0 ** -9 * float(r.abs().max())
            assert all(t in chosen for t in torch.nonzero(r > cut + tol).flatten().tolist())
            assert not any(t in chosen for t in torch.nonzero(r < cut - tol).flatten().tolist())
    d = small(batch=B, heads=128, lens=lens, topk=K, seed=22)
    d["indices"] = idx.view(B, 1, K)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    dec = decoder_for(d, device=dev)
    out, lse = dec(g["q"], g["cache"], g["block_table"], g["seq_lens"], g["indices"])
    assert dec.error() == (0, 0)
    o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], indices=d["indices"])
    o, l = out.double().cpu(), lse.double().cpu()
    assert ((o - o_ref).abs() <= 1e-2 + 2.0 ** -8 * o_ref.abs()).all()
    assert float((o - o_ref).norm() / o_ref.norm()) <= 5e-3
    assert float((l - l_ref).abs().max()) <= 1e-3


def test_indexer_full_size_sparse_shape(libmla, dev):
    """The sparse workload's shape: 16 sequences of 131072 keys, one query of
    64 index heads each, top-2048. Scores of two whole sequences against the
    oracle, the top-k of all 16 bit-exact on the GPU scores."""
    from mla_latent_kv_26_b200.workloads import indexer_inputs

    d = indexer_inputs(batch=16, q_len=1, heads=64, num_keys=131072, seed=8)
    sc = gpu_scores(libmla, d, dev)
    assert_scores(sc, d, batches=[0, 15])
    idx = gpu_topk(libmla, sc.view(16, -1), 2048, dev)
    assert torch.equal(idx, oracle.topk_positions(sc.view(16, -1), 2048))

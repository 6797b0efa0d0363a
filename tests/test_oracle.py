"""Pins for the float64 oracle: each test checks it against something other than
itself — the unabsorbed attention path, exact special cases, closed forms, a
pure-Python brute force, and figures the pages print."""

import json
import math
import os

import pytest
import torch

import oracle
from oracle import decode as od
from oracle.plan import split_plan, task_token_counts

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _paged(rows: torch.Tensor, shuffle_seed=None):
    """Pack ``rows [L, 576]`` into a paged cache with one sequence."""
    L = rows.shape[0]
    npg = max((L + 63) // 64, 1)
    cache = torch.zeros(npg, 64, rows.shape[1], dtype=rows.dtype)
    flat = cache.view(npg * 64, -1)
    flat[:L] = rows
    bt = torch.arange(npg, dtype=torch.int64)
    if shuffle_seed is not None:
        g = torch.Generator().manual_seed(shuffle_seed)
        perm = torch.randperm(npg, generator=g)
        new_cache = torch.empty_like(cache)
        new_cache[perm] = cache          # logical page j lives at physical page perm[j]
        cache, bt = new_cache, perm
    return cache, bt[None]


# ---------------------------------------------------------------- (a) absorption


@pytest.mark.parametrize("H", [16, 128])
@pytest.mark.parametrize("L", [1, 63, 64, 65, 1000])
def test_absorbed_equals_unabsorbed(H, L):
    g = torch.Generator().manual_seed(1000 * H + L)
    w_uk = torch.randn(H, 128, 512, generator=g, dtype=torch.float64) / math.sqrt(512)
    w_uv = torch.randn(H, 128, 512, generator=g, dtype=torch.float64) / math.sqrt(512)
    q_nope = torch.randn(H, 128, generator=g, dtype=torch.float64)
    q_pe = torch.randn(H, 64, generator=g, dtype=torch.float64)
    c = torch.randn(L, 512, generator=g, dtype=torch.float64)
    kpe = torch.randn(L, 64, generator=g, dtype=torch.float64)

    naive = oracle.unabsorbed_attention(q_nope, q_pe, w_uk, w_uv, c, kpe)

    q_abs = torch.cat([oracle.absorb_query(q_nope, w_uk), q_pe], dim=-1)
    cache, bt = _paged(torch.cat([c, kpe], dim=-1), shuffle_seed=L)
    out, _ = oracle.mla_decode(q_abs[None, None], cache, bt, torch.tensor([L]))
    absorbed = oracle.unabsorb_output(out[0, 0], w_uv)
    rel = (absorbed - naive).norm() / naive.norm()
    assert rel < 1e-10, rel

    if L > 1:
        # the same comparison with a 1/sqrt(576) scale must fail: the pin sees the scale
        wrong, _ = oracle.mla_decode(q_abs[None, None], cache, bt, torch.tensor([L]),
                                     softmax_scale=1 / math.sqrt(576))
        rel_wrong = (oracle.unabsorb_output(wrong[0, 0], w_uv) - naive).norm() / naive.norm()
        assert rel_wrong > 1e-4


def test_default_scale_is_qk_head_width():
    assert oracle.QK_HEAD_DIM == 192
    assert oracle.DEFAULT_SOFTMAX_SCALE == 1.0 / math.sqrt(192)


# ---------------------------------------------------------------- (b) single key


@pytest.mark.parametrize("sparse", [False, True])
def test_single_key_returns_that_latent(sparse):
    g = torch.Generator().manual_seed(7)
    H = 16
    rows = torch.randn(40, 576, generator=g).to(torch.bfloat16)
    cache, bt = _paged(rows)
    q = torch.randn(1, 1, H, 576, generator=g).to(torch.bfloat16)
    if sparse:
        idx = torch.tensor([[[17, -1, -1]]])
        out, lse = oracle.mla_decode(q, cache, bt, torch.tensor([40]), indices=idx)
        key = 17
    else:
        out, lse = oracle.mla_decode(q, cache, bt, torch.tensor([1]))
        key = 0
    want = rows[key, :512].double()
    for h in range(H):
        assert torch.equal(out[0, 0, h], want)
        qh = q[0, 0, h].double().tolist()
        rk = rows[key].double().tolist()
        s0 = oracle.DEFAULT_SOFTMAX_SCALE * math.fsum(a * b for a, b in zip(qh, rk))
        assert abs(float(lse[0, 0, h]) - s0) <= 1e-12 * max(1.0, abs(s0))


# ---------------------------------------------------------------- (c) rows sum to 1


def test_probabilities_sum_to_one():
    g = torch.Generator().manual_seed(3)
    q = torch.randn(16, 576, generator=g, dtype=torch.float64) * 3
    rows = torch.randn(777, 576, generator=g, dtype=torch.float64)
    p, lse = oracle.attention_probs(oracle.scores(q, rows, oracle.DEFAULT_SOFTMAX_SCALE))
    assert (p >= 0).all()
    assert torch.allclose(p.sum(-1), torch.ones(16, dtype=torch.float64), atol=1e-12, rtol=0)
    assert torch.isfinite(lse).all()


# ---------------------------------------------------------------- (d) brute force


def _brute(q, cache, bt, lens, Sq, causal, scale, idx=None):
    """Independent pure-Python restatement on lists (loops, math.exp)."""
    ql, cl, btl, ll = q.double().tolist(), cache.double().tolist(), bt.tolist(), [int(x) for x in lens]
    B, _, H, _ = q.shape
    out = [[[[0.0] * 512 for _ in range(H)] for _ in range(Sq)] for _ in range(B)]
    lse = [[[-math.inf] * H for _ in range(Sq)] for _ in range(B)]
    for b in range(B):
        for i in range(Sq):
            if idx is not None:
                toks = [t for t in idx[b][i].tolist() if t >= 0]
            else:
                hi = ll[b] - Sq + i + 1 if causal else ll[b]
                toks = list(range(max(hi, 0)))
            if not toks:
                continue
            rows = [cl[btl[b][t // 64]][t % 64] for t in toks]
            for h in range(H):
                qv = ql[b][i][h]
                s = [scale * sum(qv[j] * r[j] for j in range(576)) for r in rows]
                m = max(s)
                e = [math.exp(x - m) for x in s]
                z = sum(e)
                lse[b][i][h] = m + math.log(z)
                o = out[b][i][h]
                for w, r in zip(e, rows):
                    pw = w / z
                    for j in range(512):
                        o[j] += pw * r[j]
    return torch.tensor(out, dtype=torch.float64), torch.tensor(lse, dtype=torch.float64)


BRUTE_CASES = [
    # (B, H, Sq, causal, lens)
    (1, 1, 1, False, [1]),
    (2, 2, 1, False, [2, 3]),
    (1, 2, 2, True, [63]),
    (3, 1, 1, False, [64, 65, 1]),
    (1, 16, 1, False, [65]),
    (2, 2, 2, False, [130, 5]),
    (2, 1, 2, True, [1, 130]),
]


@pytest.mark.parametrize("case", BRUTE_CASES)
def test_brute_force_tiny(case):
    from mla_latent_kv_26_b200.workloads import small

    B, H, Sq, causal, lens = case
    d = small(batch=B, heads=H, q_len=Sq, lens=lens, causal=causal, seed=len(lens) * 10 + H, nan_slack=False)
    out, lse = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], causal=causal)
    bo, bl = _brute(d["q"], d["cache"], d["block_table"], d["seq_lens"], Sq, causal, oracle.DEFAULT_SOFTMAX_SCALE)
    assert torch.allclose(out, bo, atol=1e-12, rtol=1e-12)
    fin = torch.isfinite(bl)
    assert torch.equal(fin, torch.isfinite(lse))
    assert torch.allclose(lse[fin], bl[fin], atol=1e-12, rtol=1e-12)


def test_brute_force_sparse_tiny():
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=2, lens=[100, 70], topk=9, seed=5, nan_slack=False)
    idx = d["indices"].clone()
    idx[1, 0, 3] = -1
    out, lse = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], indices=idx)
    bo, bl = _brute(d["q"], d["cache"], d["block_table"], d["seq_lens"], 1, False, oracle.DEFAULT_SOFTMAX_SCALE,
                    idx=idx)
    assert torch.allclose(out, bo, atol=1e-12, rtol=1e-12)
    assert torch.allclose(lse, bl, atol=1e-12, rtol=1e-12)


# ---------------------------------------------------------------- closed forms


def test_zero_query_gives_mean_and_log_count():
    g = torch.Generator().manual_seed(11)
    rows = torch.randn(150, 576, generator=g, dtype=torch.float64)
    cache, bt = _paged(rows, shuffle_seed=2)
    q = torch.zeros(1, 1, 4, 576, dtype=torch.float64)
    out, lse = oracle.mla_decode(q, cache, bt, torch.tensor([150]))
    assert torch.allclose(out[0, 0], rows[:, :512].mean(0).expand(4, -1), atol=1e-13, rtol=0)
    assert torch.allclose(lse[0, 0], torch.full((4,), math.log(150), dtype=torch.float64), atol=1e-13, rtol=0)


def test_identical_rows_return_the_row():
    g = torch.Generator().manual_seed(12)
    row = torch.randn(576, generator=g, dtype=torch.float64)
    rows = row.expand(99, -1).clone()
    cache, bt = _paged(rows)
    q = torch.randn(1, 1, 3, 576, generator=g, dtype=torch.float64)
    out, lse = oracle.mla_decode(q, cache, bt, torch.tensor([99]))
    assert torch.allclose(out[0, 0], row[:512].expand(3, -1), atol=1e-12, rtol=0)
    s = oracle.DEFAULT_SOFTMAX_SCALE * (q[0, 0] @ row)
    assert torch.allclose(lse[0, 0], s + math.log(99), atol=1e-12, rtol=0)


def test_dominant_key_wins():
    g = torch.Generator().manual_seed(13)
    rows = torch.randn(64, 576, generator=g, dtype=torch.float64)
    q = torch.randn(1, 1, 1, 576, generator=g, dtype=torch.float64)
    # raise key 20's score by 50 along q's direction
    qv = q[0, 0, 0]
    rows[20] += 50.0 / oracle.DEFAULT_SOFTMAX_SCALE * qv / (qv @ qv)
    cache, bt = _paged(rows)
    out, _ = oracle.mla_decode(q, cache, bt, torch.tensor([64]))
    assert torch.allclose(out[0, 0, 0], rows[20, :512], atol=1e-9, rtol=0)


def test_causal_first_row_equals_shorter_context():
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=4, q_len=2, lens=[130, 64], causal=True, seed=21, nan_slack=False)
    out2, lse2 = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], causal=True)
    q0 = d["q"][:, :1]
    out1, lse1 = oracle.mla_decode(q0, d["cache"], d["block_table"], d["seq_lens"] - 1)
    assert torch.equal(out2[:, 0], out1[:, 0]) and torch.equal(lse2[:, 0], lse1[:, 0])
    q1 = d["q"][:, 1:]
    out1b, lse1b = oracle.mla_decode(q1, d["cache"], d["block_table"], d["seq_lens"])
    assert torch.equal(out2[:, 1], out1b[:, 0]) and torch.equal(lse2[:, 1], lse1b[:, 0])


def test_sparse_with_every_index_equals_dense():
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=3, lens=[200, 77], seed=31, nan_slack=False)
    dense, dl = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"])
    g = torch.Generator().manual_seed(32)
    idx = torch.full((2, 1, 200), -1, dtype=torch.int32)
    for b, L in enumerate([200, 77]):
        idx[b, 0, :L] = torch.randperm(L, generator=g).to(torch.int32)
    sp, sl = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], indices=idx)
    assert torch.allclose(sp, dense, atol=1e-12, rtol=0) and torch.allclose(sl, dl, atol=1e-12, rtol=0)


def test_page_permutation_is_invisible():
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=3, heads=2, lens=[300, 64, 1], seed=41, nan_slack=False)
    out, lse = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"])
    g = torch.Generator().manual_seed(42)
    P = d["cache"].shape[0]
    perm = torch.randperm(P, generator=g)           # physical page p moves to perm[p]
    cache2 = torch.empty_like(d["cache"])
    cache2[perm] = d["cache"]
    bt = d["block_table"].clone().long()
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt)
    out2, lse2 = oracle.mla_decode(d["q"], cache2, bt2, d["seq_lens"])
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_empty_rows():
    from mla_latent_kv_26_b200.workloads import small

    d = small(batch=2, heads=2, q_len=2, lens=[0, 1], causal=True, seed=51, nan_slack=False)
    out, lse = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], causal=True)
    assert torch.equal(out[0], torch.zeros_like(out[0])) and torch.isinf(lse[0]).all() and (lse[0] < 0).all()
    assert torch.isinf(lse[1, 0]).all()                  # L=1, Sq=2: the first new token sees nothing
    assert torch.isfinite(lse[1, 1]).all()


# ---------------------------------------------------------------- a8: the LSE merge


@pytest.mark.parametrize("cuts", [[0, 1000], [0, 1, 1000], [0, 64, 128, 640, 999, 1000], [0, 0, 500, 1000]])
def test_lse_merge_over_a_partition_equals_whole(cuts):
    g = torch.Generator().manual_seed(61)
    rows = torch.randn(1000, 576, generator=g, dtype=torch.float64)
    cache, bt = _paged(rows)
    q = torch.randn(1, 1, 8, 576, generator=g, dtype=torch.float64) * 2
    whole, wl = oracle.mla_decode(q, cache, bt, torch.tensor([1000]))
    po, pl = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        idx = torch.arange(a, b, dtype=torch.int32)[None, None] if b > a else torch.full((1, 1, 1), -1)
        o, l = oracle.mla_decode(q, cache, bt, torch.tensor([1000]), indices=idx)
        po.append(o)
        pl.append(l)
    mo, ml = oracle.lse_merge(torch.stack(po), torch.stack(pl))
    assert torch.allclose(mo, whole, atol=1e-12, rtol=0)
    assert torch.allclose(ml, wl, atol=1e-12, rtol=0)


def test_lse_merge_two_scalars_by_hand():
    # exp-weights of two parts with lse 0 and ln 3: weights 1/4 and 3/4, merged lse ln 4
    po = torch.tensor([[[1.0] * 512], [[5.0] * 512]], dtype=torch.float64)
    pl = torch.tensor([[0.0], [math.log(3.0)]], dtype=torch.float64)
    o, l = oracle.lse_merge(po, pl)
    assert abs(float(l[0]) - math.log(4.0)) < 1e-15
    assert torch.allclose(o[0], torch.full((512,), 4.0, dtype=torch.float64), atol=1e-14, rtol=0)
    # an empty part weighs nothing; all empty gives 0 / -inf
    pl2 = torch.tensor([[-math.inf], [0.7]], dtype=torch.float64)
    o2, l2 = oracle.lse_merge(po, pl2)
    assert torch.equal(o2[0], po[1, 0]) and float(l2[0]) == 0.7
    o3, l3 = oracle.lse_merge(po, torch.full((2, 1), -math.inf, dtype=torch.float64))
    assert torch.equal(o3, torch.zeros_like(o3)) and math.isinf(float(l3[0]))


# ---------------------------------------------------------------- a1: the plan


@pytest.mark.parametrize("lens,Sq,causal,topk,P", [
    ([256], 1, False, 0, 74),
    ([4096] * 32, 1, False, 0, 74),
    ([1024, 32768, 5000, 77, 0, 64], 1, False, 0, 5),
    ([4096, 65536, 1], 2, True, 0, 7),
    ([131072] * 4, 1, False, 2048, 74),
    ([3, 5], 2, True, 0, 1),
    ([], 1, False, 0, 3),
    ([4096, 65536, 1, 65, 129, 700], 2, True, 0, 74),   # grouped: 2 x 37 workers
    ([5000, 64, 3, 9000], 3, True, 0, 74),              # grouped: 3 x 24, 2 idle
    ([5000, 64, 3, 9000], 2, False, 0, 74),             # grouped, not causal
    ([5000, 64], 9, True, 0, 74),                       # q_len 9: not grouped
    ([300, 3000], 2, True, 2048, 74),                   # sparse: not grouped
])
def test_plan_covers_every_page_once_within_quota(lens, Sq, causal, topk, P):
    maxp = max([(L + 63) // 64 for L in lens] + [1])
    plan = split_plan(lens, q_len=Sq, causal=causal, topk=topk, max_pages_per_seq=maxp, num_pairs=P)
    G, Wg = plan["groups"], plan["workers_per_group"]
    grouped = 2 <= Sq <= 8 and topk == 0 and P // Sq >= 4
    assert G == (Sq if grouped else 1) and Wg == P // G
    T = len(lens) * Sq
    # plan order: a permutation of the query rows; token-major when grouped
    assert sorted(plan["task_rows"]) == list(range(T))
    for u, r in enumerate(plan["task_rows"]):
        assert r == ((u % len(lens)) * Sq + u // len(lens) if grouped else u)
    covered = {}
    slots = set()
    for p, items in enumerate(plan["items"]):
        load = 0
        g = p // Wg if Wg else 0
        for (t, a, b, slot) in items:
            assert 0 <= a < b <= plan["task_pages"][t]
            assert g < G and g * (T // G) <= t < (g + 1) * (T // G)   # a worker stays in its group
            for pg in range(a, b):
                assert (t, pg) not in covered
                covered[(t, pg)] = p
            load += b - a
            assert slot == p + t and slot not in slots
            slots.add(slot)
        if items:
            assert load <= plan["quotas"][g]
    want = {(t, pg) for t, n in enumerate(plan["task_pages"]) for pg in range(n)}
    assert set(covered) == want
    assert plan["total_pages"] == len(want)
    # tokens per task from the definition, by brute force
    for t, n in enumerate(plan["task_tokens"]):
        b, i = divmod(plan["task_rows"][t], Sq)
        L = lens[b]
        exp = topk if topk else (max(L - Sq + i + 1, 0) if causal else L)
        assert n == exp
        assert plan["task_pages"][t] == -(-n // 64)
        assert plan["splits"][t] == len({covered[(t, pg)] for pg in range(plan["task_pages"][t])})
    if grouped and not causal:
        # every token of a sequence reads the same pages: worker j of every
        # group gets the same (sequence, page range) items
        B = len(lens)
        for j in range(Wg):
            seen = [[(plan["task_rows"][t] // Sq, a, b) for (t, a, b, _) in plan["items"][g * Wg + j]]
                    for g in range(G)]
            assert all(s == seen[0] for s in seen)


def test_plan_flags_out_of_range_lengths():
    counts, bad = task_token_counts([10, 99999, -1], q_len=1, causal=False, topk=0, max_pages_per_seq=2)
    assert bad and counts == [10, 0, 0]
    counts, bad = task_token_counts([128], q_len=1, causal=False, topk=0, max_pages_per_seq=2)
    assert not bad and counts == [128]


# ---------------------------------------------------------------- printed figures


def test_page_printed_cost_figures():
    with open(os.path.join(GOLDEN, "v2lite_mla_costs.json")) as f:
        gold = json.load(f)
    mla = gold["cached_values_per_token_mla"]
    assert oracle.D_LATENT == mla["parts"][0] and oracle.D_ROPE == mla["parts"][1]
    assert oracle.D_QK == mla["value"] == 576
    assert sum(gold["cached_values_per_token_mha"]["parts"]) == gold["cached_values_per_token_mha"]["value"]
    parts = gold["qk_width_parts"]
    assert oracle.QK_HEAD_DIM == parts["nope"] + parts["rope"]
    assert gold["q_proj_heads_by_width"]["heads"] * oracle.QK_HEAD_DIM == gold["q_proj_heads_by_width"]["total"]
    H, ctx = 16, 8192
    kvb = gold["kv_b_proj_per_head"]["value"]
    decompress = ctx * oracle.D_LATENT * (H * kvb)
    assert decompress == math.prod(gold["decompress_macs_ctx8192"]["factors"])
    assert f"{decompress / 1e9:.1f}G" == gold["decompress_macs_ctx8192"]["value_printed"]
    attention = ctx * H * (oracle.QK_HEAD_DIM + parts["v"])
    assert f"{attention / 1e6:.1f}M" == gold["attention_macs_ctx8192"]["value_printed"]
    assert round(decompress / attention, -2) == gold["decompress_over_attention"]["value_printed"]
    assert round(2048 / oracle.D_QK, 1) == gold["latent_vs_hidden_ratio"]["value_printed"]
    assert round(gold["cached_values_per_token_mha"]["value"] / oracle.D_QK, 1) == \
        gold["mha_vs_mla_cache_ratio"]["value_printed"]

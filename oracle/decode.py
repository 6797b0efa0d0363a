"""Float64 CPU definition of MLA decode over a paged latent cache.

TEST INFRASTRUCTURE ONLY: imported by tests, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` leg of ``bench.py``; never by the product path.

Every step is written the plain way: gather the visible cache rows, form all
scores, take the normaliser and the probabilities, sum. No splitting, no
online softmax, no blocking. Library matmuls are the only building blocks.

Notation follows "深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA"
(absorbed branch): ``kv_cache`` holds the 512-wide normalised latent ``c``,
``pe_cache`` the 64-wide rotated key ``k_pe``; here both sit side by side in
one 576-wide row of a paged cache ``cache[page, slot, 0:576]``.
"""

from __future__ import annotations

import math

import torch

# "深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA", the ModelArgs block:
# kv_lora_rank = 512, qk_rope_head_dim = 64, qk_nope_head_dim = 128.
D_LATENT = 512
D_ROPE = 64
D_QK = D_LATENT + D_ROPE  # 576 values cached per token
QK_NOPE_HEAD_DIM = 128
V_HEAD_DIM = 128
# "DeepSeek-V2-Lite 模型结构详解", section "为什么 Q/K 是 192 维而 V 只有 128 维":
# a query/key head is 128 content + 64 position dimensions.
QK_HEAD_DIM = QK_NOPE_HEAD_DIM + D_ROPE  # 192
# The scale divides by sqrt of the query/key head width (beaiera.top abstract on
# the √d_k factor; the V3 walkthrough multiplies scores by ``softmax_scale``).
DEFAULT_SOFTMAX_SCALE = 1.0 / math.sqrt(QK_HEAD_DIM)
# Tokens per cache page. Paging is an interface choice; the pages keep one
# contiguous cache per sequence, which is the special case of an identity
# block table.
PAGE_SIZE = 64


def _f64(x) -> torch.Tensor:
    """Any tensor-like (bf16/fp32/int) to a float64 CPU tensor (bf16 upcasts exactly)."""
    if not isinstance(x, torch.Tensor):
        x = torch.as_tensor(x)
    return x.detach().to("cpu").to(torch.float64)


def visible_tokens(seq_len: int, q_len: int, qi: int, causal: bool, indices_row=None) -> torch.Tensor:
    """Logical cache positions that query token ``qi`` of a sequence may attend to.

    * sparse (``indices_row`` given): the listed positions, skipping entries < 0
      ("DeepSeek-V3.2-Exp unboxing", section on the Indexer: attention is
      restricted to the top-k selected tokens);
    * dense causal: ``t <= seq_len - q_len + qi`` — ``seq_len`` counts the
      ``q_len`` new tokens too, and each new token sees itself and what came
      before it (V3 walkthrough, section "Transformer": upper-triangular -inf
      mask when more than one token is processed);
    * dense: every ``t < seq_len``.
    """
    if indices_row is not None:
        idx = torch.as_tensor(indices_row).to(torch.int64).reshape(-1)
        return idx[idx >= 0]
    if causal:
        n = seq_len - q_len + qi + 1
    else:
        n = seq_len
    return torch.arange(max(n, 0), dtype=torch.int64)


def gather_rows(cache, block_table_row, tokens: torch.Tensor) -> torch.Tensor:
    """Rows ``cache[block_table_row[t // 64], t % 64, :]`` for each logical token ``t``, as float64."""
    bt = torch.as_tensor(block_table_row).to(torch.int64)
    pages = bt[tokens // PAGE_SIZE]
    slots = tokens % PAGE_SIZE
    return _f64(cache[pages, slots])


def scores(q_heads: torch.Tensor, rows: torch.Tensor, softmax_scale: float) -> torch.Tensor:
    """``s[h, t] = scale * (q_lat[h] · c_t + q_pe[h] · k_pe_t)`` — the two-term score of the
    absorbed branch (V3 walkthrough, section "MLA", "优化实现")."""
    latent = q_heads[:, :D_LATENT] @ rows[:, :D_LATENT].T
    rope = q_heads[:, D_LATENT:D_QK] @ rows[:, D_LATENT:D_QK].T
    return softmax_scale * (latent + rope)


def attention_probs(s: torch.Tensor):
    """Softmax over the last axis with its log-normaliser.

    ``M = max_t s_t``, ``lse = M + ln Σ_t exp(s_t - M)``, ``p_t = exp(s_t - lse)``.
    An empty row gives ``lse = -inf`` and no probabilities.
    """
    if s.shape[-1] == 0:
        return s.clone(), torch.full(s.shape[:-1], -math.inf, dtype=torch.float64)
    m = s.max(dim=-1).values
    lse = m + torch.log(torch.exp(s - m[..., None]).sum(dim=-1))
    p = torch.exp(s - lse[..., None])
    return p, lse


def mla_decode(q, cache, block_table, seq_lens, *, causal: bool = False,
               softmax_scale: float = DEFAULT_SOFTMAX_SCALE, indices=None, batches=None):
    """Latent-space MLA decode, the plain definition.

    Arguments (any dtype; upcast to float64):

    * ``q``            ``[B, Sq, H, 576]`` absorbed queries ``q_lat ‖ q_pe``
    * ``cache``        ``[num_pages, 64, 576]`` paged latent cache ``c ‖ k_pe``
    * ``block_table``  ``[B, max_pages_per_seq]`` page ids
    * ``seq_lens``     ``[B]`` cached tokens per sequence, including the Sq new ones
    * ``indices``      ``[B, Sq, topk]`` logical positions (sparse) or None (dense)
    * ``batches``      optional iterable of batch indices to compute (others stay 0 / -inf)

    Returns ``out [B, Sq, H, 512]`` and ``lse [B, Sq, H]`` (natural log), float64.
    For each (b, i): T = visible tokens, rows = cache rows of T,
    ``out = softmax(s) · rows[:, :512]`` — the latent PV of the absorbed branch
    (V3 walkthrough, section "MLA": ``einsum("bsht,btc->bshc", scores, kv_cache)``).
    """
    B, Sq, H, D = q.shape
    assert D == D_QK, "absorbed queries are 576 wide"
    lens = torch.as_tensor(seq_lens).to(torch.int64)
    out = torch.zeros(B, Sq, H, D_LATENT, dtype=torch.float64)
    lse = torch.full((B, Sq, H), -math.inf, dtype=torch.float64)
    for b in (range(B) if batches is None else batches):
        for i in range(Sq):
            idx_row = None if indices is None else indices[b, i]
            T = visible_tokens(int(lens[b]), Sq, i, causal, idx_row)
            if T.numel() == 0:
                continue
            rows = gather_rows(cache, block_table[b], T)
            s = scores(_f64(q[b, i]), rows, softmax_scale)
            p, l = attention_probs(s)
            out[b, i] = p @ rows[:, :D_LATENT]
            lse[b, i] = l
    return out, lse


def lse_merge(part_out, part_lse):
    """Merge softmax results computed over disjoint token sets.

    ``part_out [S, ..., 512]`` holds each part's normalised output, ``part_lse [S, ...]``
    its log-normaliser. With ``lse = ln Σ_i exp(lse_i)`` the merged output is
    ``Σ_i exp(lse_i - lse) · out_i`` — the softmax over the union written in
    terms of the parts. Parts with ``lse_i = -inf`` (no tokens) weigh zero; if
    every part is empty the result is 0 with ``lse = -inf``.
    """
    po = _f64(part_out)
    pl = _f64(part_lse)
    m = pl.max(dim=0).values
    finite = torch.isfinite(m)
    m_safe = torch.where(finite, m, torch.zeros_like(m))
    tot = torch.exp(pl - m_safe[None]).sum(dim=0)
    lse = torch.where(finite, m_safe + torch.log(tot), torch.full_like(m, -math.inf))
    w = torch.where(finite[None], torch.exp(pl - torch.where(finite, lse, torch.zeros_like(lse))[None]),
                    torch.zeros_like(pl))
    out = (w[..., None] * po).sum(dim=0)
    return out, lse


# ---------------------------------------------------------------------------
# The unabsorbed path and the absorption maps, used to pin the absorbed form.
# "深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA": wkv_b viewed as
# [H, 256, 512]; rows [:128] expand the latent into per-head keys (W_UK), rows
# [-128:] into per-head values (W_UV).
# ---------------------------------------------------------------------------

def absorb_query(q_nope, w_uk):
    """``q_lat[h, c] = Σ_d q_nope[h, d] · W_UK[h, d, c]`` (einsum "bshd,hdc->bshc")."""
    return torch.einsum("hd,hdc->hc", _f64(q_nope), _f64(w_uk))


def unabsorb_output(o_lat, w_uv):
    """``o[h, d] = Σ_c W_UV[h, d, c] · o_lat[h, c]`` (einsum "bshc,hdc->bshd")."""
    return torch.einsum("hc,hdc->hd", _f64(o_lat), _f64(w_uv))


def unabsorbed_attention(q_nope, q_pe, w_uk, w_uv, c_kv, k_pe):
    """Standard per-head attention after expanding the latent (the "naive" branch).

    ``k_t[h] = [W_UK[h] c_t ; k_pe_t]`` (192-d, k_pe shared by all heads),
    ``v_t[h] = W_UV[h] c_t`` (128-d), ``o[h] = softmax(q[h]·k[h] / sqrt(192)) · v[h]``,
    the scale taken from the width of the expanded query/key.
    """
    qn, qp = _f64(q_nope), _f64(q_pe)
    wk, wv = _f64(w_uk), _f64(w_uv)
    c, kp = _f64(c_kv), _f64(k_pe)
    H = qn.shape[0]
    k_nope = torch.einsum("hdc,tc->htd", wk, c)                      # [H, T, 128]
    k = torch.cat([k_nope, kp[None].expand(H, -1, -1)], dim=-1)     # [H, T, 192]
    v = torch.einsum("hdc,tc->htd", wv, c)                           # [H, T, 128]
    qf = torch.cat([qn, qp], dim=-1)                                 # [H, 192]
    s = torch.einsum("hd,htd->ht", qf, k) / math.sqrt(qf.shape[-1])
    p, _ = attention_probs(s)
    return torch.einsum("ht,htd->hd", p, v)

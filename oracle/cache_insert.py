"""CPU definition of the latent-cache insert: kv_norm (RMSNorm) of the
512-wide latent, rotary embedding of the 64-wide rope key, and the write of
both into the token's row of the paged cache.

TEST INFRASTRUCTURE ONLY: imported by tests and ``bench.py``'s reference
legs; never by the product path.

Sources (cited by page title and section):

* "深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA": the projection
  ``wkv_a(x)`` is split into the 512-wide latent ``kv`` and the 64-wide
  ``k_pe``; ``k_pe`` gets the rotary embedding ``apply_rotary_emb(k_pe,
  freqs_cis)``; the absorbed branch stores ``kv_norm(kv)`` in ``kv_cache`` and
  ``k_pe`` in ``pe_cache`` at the tokens' positions.
* "DeepSeek-V2-Lite 模型结构详解", section "四、RMSNorm": each row is divided by
  ``rms = sqrt(mean(x^2) + eps)`` and multiplied by ``weight``; rows are
  independent; sub-section "精度：半精度也在 float32 里算": the sum of squares
  and the division run in float32, the normalised row is cast back to the
  input dtype and then multiplied by ``weight``.

Readings where the pages are silent:

* ``apply_rotary_emb``'s body and the frequency table are not on the pages.
  The plainest reading, used here: consecutive pairs ``(x[2i], x[2i+1])`` are
  one complex number, multiplied by the table's unit complex number for the
  token's position and pair, ``(cos a, sin a)``; the caller supplies the
  ``cos``/``sin`` tables (their frequencies are a model setting). Computed in
  float32-or-better and cast back to bf16, like the normalised latent.
* ``eps`` is a parameter (its value is not printed).

Floating point: the normaliser and the rotation are computed in float64
here; the two casts the page prescribes (normalised row -> bf16, product with
the bf16 weight -> bf16) are applied, so a GPU result in float32 agrees to
within one bf16 rounding step.
"""

from __future__ import annotations

import torch

D_LATENT = 512
D_ROPE = 64
PAGE_SIZE = 64


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16).to(torch.float64)


def rms_norm(x: torch.Tensor, weight: torch.Tensor, eps: float) -> torch.Tensor:
    """Rows of ``x`` [..., D] (bf16 values) -> ``weight * bf16(x / rms)`` rounded
    to bf16, returned as float64. ("V2-Lite", section "四、RMSNorm".)"""
    xf = x.to(torch.float64)
    rms = torch.sqrt((xf * xf).mean(-1, keepdim=True) + eps)
    return _bf16(weight.to(torch.float64) * _bf16(xf / rms))


def rope_pairs(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    """Rotate consecutive pairs of ``x`` [..., 2P] by the angles whose cosines
    and sines are ``cos``/``sin`` [..., P]; result rounded to bf16, as float64."""
    xf = x.to(torch.float64)
    a, b = xf[..., 0::2], xf[..., 1::2]
    c, s = cos.to(torch.float64), sin.to(torch.float64)
    out = torch.empty_like(xf)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return _bf16(out)


def cache_insert(cache: torch.Tensor, block_table: torch.Tensor, seq_ids: torch.Tensor, positions: torch.Tensor,
                 kv: torch.Tensor, weight: torch.Tensor, eps: float, cos: torch.Tensor, sin: torch.Tensor):
    """Return a float64 copy of ``cache`` [pages, 64, 576] with token n
    (sequence ``seq_ids[n]``, position ``positions[n]``) written into row
    ``positions[n] % 64`` of page ``block_table[seq, positions[n] // 64]``:
    columns 0..511 = rms_norm(kv[n, :512]), 512..575 = rope(kv[n, 512:]) with
    the tables' row ``positions[n]``. Tokens whose page or table row is out of
    range are skipped (the second value lists them). Written one token at a
    time, in order (a later token at the same row wins)."""
    out = cache.to(torch.float64).clone()
    skipped = []
    num_pages = cache.shape[0]
    for n in range(kv.shape[0]):
        b, p = int(seq_ids[n]), int(positions[n])
        if not (0 <= b < block_table.shape[0]) or not (0 <= p < block_table.shape[1] * PAGE_SIZE) or \
                p >= cos.shape[0]:
            skipped.append(n)
            continue
        page = int(block_table[b, p // PAGE_SIZE])
        if not (0 <= page < num_pages):
            skipped.append(n)
            continue
        row = p % PAGE_SIZE
        out[page, row, :D_LATENT] = rms_norm(kv[n, :D_LATENT], weight, eps)
        out[page, row, D_LATENT:] = rope_pairs(kv[n, D_LATENT:], cos[p], sin[p])
    return out, skipped

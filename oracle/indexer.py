"""Float64 CPU definition of the sparse-attention indexer and its top-k.

TEST INFRASTRUCTURE ONLY: imported by tests, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` leg of ``bench.py``; never by the product path.

Source: "DeepSeek-V3.2-Exp unboxing" (floratopia.github.io), the section on
the Indexer and its ``fp8_index`` TileLang kernel. What the page fixes:

* the indexer scores the cached keys of every sequence for every query token
  and the highest-scoring ones are kept (a top-k of token positions) for the
  attention that follows;
* the scoring call is ``fp8_index(q, q_s, k, k_s) -> o`` with
  ``q [b, m, h, d]`` fp8, ``q_s [b, m, h]`` float32, ``k [b, n, d]`` fp8,
  ``k_s [b, n]`` float32 and ``o [b, m, n]`` float32; the model passes its
  per-head ``weights`` as ``q_s`` and the fp8 key cache's per-token scales as
  ``k_s``;
* the shapes seen at run time: ``q [2, 128, 64, 128]``, ``k [2, 128, 128]``
  (b = 2, m = 128 query tokens, h = 64 index heads, d = 128, n = 128 keys).

What the page does not print (the kernel body), and the reading taken here:
the score of key ``t`` for query ``(b, i)`` is the per-head dot product of
the fp8 values, passed through a ReLU, weighted by ``q_s`` and summed over
heads, then multiplied by the key's scale:

    o[b, i, t] = k_s[b, t] * sum_h q_s[b, i, h] * max(0, sum_d q[b, i, h, d] * k[b, t, d])

(``k_s`` is a positive scale, so applying it inside or outside the ReLU is
the same). Top-k: among positions ``t < valid_len`` of a row, the ``k``
largest scores, ties broken towards the smaller position; the selected
positions are returned in increasing order, padded with -1 when fewer than
``k`` are eligible (-1 is what the sparse decode skips).

The arithmetic of both functions is pinned in tests/test_oracle_indexer.py
(pure-Python brute force, closed forms, the e4m3 code table); the ReLU and
the head weighting themselves are a reading of the page, not something it
prints, so the formula as a whole is "parity unpinned" against the page.
"""

from __future__ import annotations

import torch

D_INDEX = 128  # index head width d seen on the page


def _f64(x) -> torch.Tensor:
    """Any tensor (fp8 / bf16 / fp32 / int) to a float64 CPU tensor; fp8 and bf16 upcast exactly."""
    if not isinstance(x, torch.Tensor):
        x = torch.as_tensor(x)
    x = x.detach().to("cpu")
    if x.dtype in (torch.float8_e4m3fn, torch.float8_e5m2):
        x = x.to(torch.float32)  # exact: every fp8 value is a float32 value
    return x.to(torch.float64)


def index_scores(q, q_s, k, k_s) -> torch.Tensor:
    """``o[b, i, t] = k_s[b, t] * sum_h q_s[b, i, h] * relu(q[b, i, h, :] . k[b, t, :])``.

    ``q [b, m, h, d]``, ``q_s [b, m, h]``, ``k [b, n, d]``, ``k_s [b, n]``; returns ``o [b, m, n]`` float64.
    """
    qf, qsf, kf, ksf = _f64(q), _f64(q_s), _f64(k), _f64(k_s)
    logits = torch.einsum("bmhd,bnd->bmhn", qf, kf)          # per-head dot products
    weighted = torch.einsum("bmhn,bmh->bmn", logits.clamp_min(0.0), qsf)
    return weighted * ksf[:, None, :]


def topk_positions(scores, k: int, valid_lens=None) -> torch.Tensor:
    """Top-``k`` positions of each row of ``scores [rows, n]`` (any float dtype).

    Row ``r`` considers positions ``t < valid_lens[r]`` (all ``n`` when
    ``valid_lens`` is None). Order: larger score first, equal scores by
    smaller position (a stable descending sort). Returns int32 ``[rows, k]``:
    the chosen positions in increasing order, then -1 for missing ones.
    """
    s = torch.as_tensor(scores)
    rows, n = s.shape
    out = torch.full((rows, k), -1, dtype=torch.int32)
    for r in range(rows):
        L = n if valid_lens is None else max(0, min(n, int(valid_lens[r])))
        if L == 0 or k == 0:
            continue
        vals = s[r, :L].to(torch.float64)  # -0.0 and +0.0 compare equal, as floats do
        order = torch.sort(vals, descending=True, stable=True).indices[:k]
        chosen = torch.sort(order).values.to(torch.int32)
        out[r, :chosen.numel()] = chosen
    return out

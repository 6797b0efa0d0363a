"""Seeded synthetic inputs for MLA latent-KV decode.

This module only draws inputs; it holds none of the decode arithmetic, so both
the CUDA path (through the tests and ``bench.py``) and the float64 oracle can
consume what it makes. Nothing here is a dataset: the shapes follow the
DeepSeek-V2-Lite (16 heads) and V3 (128 heads) attention dimensions — a
512-wide latent plus a 64-wide RoPE key per cached token ("DeepSeek-V2-Lite
模型结构详解", section "五、MLA：注意力"; "深度解读DeepSeek：源码解读 DeepSeek-V3",
section "MLA") — with random values.

Draw order for one workload, all from one ``torch.Generator``:
lengths → block table → cache pages → queries → sparse indices.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

PAGE = 64
D_QK = 576
D_LATENT = 512


@dataclasses.dataclass(frozen=True)
class Workload:
    key: str
    name: str
    batch: int
    q_len: int
    heads: int
    len_lo: int
    len_hi: int
    topk: int = 0
    causal: bool = False
    q_std: float = 1.0
    cache_std: float = 1.0
    seed: int = 0
    contiguous: bool = False

    @property
    def sparse(self) -> bool:
        return self.topk > 0


WORKLOADS = {
    "C1": Workload("C1", "v2lite-b1-h16-len256-contiguous", 1, 1, 16, 256, 256, seed=0, contiguous=True),
    "C2": Workload("C2", "v2lite-b32-h16-len4096-paged", 32, 1, 16, 4096, 4096, seed=1),
    "C3": Workload("C3", "v3-b64-h128-len1k-32k-ragged", 64, 1, 128, 1024, 32768, cache_std=0.5, seed=2),
    "C4": Workload("C4", "v3-mtp-b32-sq2-h128-len4k-64k-causal", 32, 2, 128, 4096, 65536, causal=True, seed=3),
    "C5": Workload("C5", "v32-sparse-b16-h128-len128k-top2048", 16, 1, 128, 131072, 131072, topk=2048, seed=4),
}


def make_inputs(w: Workload | str, *, seed: Optional[int] = None, lens: Optional[Sequence[int]] = None,
                slack_pages: int = 4, nan_slack: bool = True, nan_tail: bool = False,
                shuffle: Optional[bool] = None, chunk_pages: int = 512) -> dict:
    """Draw one workload's inputs on the CPU.

    * ``lens``: explicit per-sequence lengths (overrides the workload's range).
    * ``slack_pages``: extra physical pages no sequence owns; filled with NaN
      when ``nan_slack`` so that reading a wrong page poisons the result.
    * ``nan_tail``: fill the unused slots of each sequence's last page with NaN
      (they sit inside owned pages and must be masked, never summed).
    * ``shuffle``: random physical page order (default: not for contiguous workloads).

    Returns a dict with ``q [B,Sq,H,576] bf16``, ``cache [P,64,576] bf16``,
    ``block_table [B,maxp] int32`` (-1 past each sequence's pages),
    ``seq_lens [B] int32``, ``indices [B,Sq,topk] int32`` or None, and the
    workload fields.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    B = w.batch
    if lens is not None:
        seq_lens = torch.as_tensor(list(lens), dtype=torch.int64)
        assert seq_lens.numel() == B
    elif w.len_lo == w.len_hi:
        seq_lens = torch.full((B,), w.len_lo, dtype=torch.int64)
    else:
        seq_lens = torch.randint(w.len_lo, w.len_hi + 1, (B,), generator=g, dtype=torch.int64)
    pages_per_seq = (seq_lens + PAGE - 1) // PAGE
    used = int(pages_per_seq.sum())
    num_pages = max(used + slack_pages, 1)
    maxp = max(int(pages_per_seq.max()) if B > 0 else 0, 1)

    do_shuffle = (not w.contiguous) if shuffle is None else shuffle
    order = torch.randperm(used, generator=g) if do_shuffle else torch.arange(used)
    block_table = torch.full((B, maxp), -1, dtype=torch.int32)
    pos = 0
    for b in range(B):
        n = int(pages_per_seq[b])
        block_table[b, :n] = order[pos:pos + n].to(torch.int32)
        pos += n

    cache = torch.empty((num_pages, PAGE, D_QK), dtype=torch.bfloat16)
    for p0 in range(0, used, chunk_pages):
        p1 = min(p0 + chunk_pages, used)
        blk = torch.randn((p1 - p0, PAGE, D_QK), generator=g, dtype=torch.float32)
        if w.cache_std != 1.0:
            blk.mul_(w.cache_std)
        cache[p0:p1] = blk.to(torch.bfloat16)
    if used < num_pages:
        cache[used:] = float("nan") if nan_slack else 0.0
    if nan_tail:
        for b in range(B):
            L = int(seq_lens[b])
            if L % PAGE and L > 0:
                last = int(block_table[b, (L - 1) // PAGE])
                cache[last, L % PAGE:] = float("nan")

    q = torch.randn((B, w.q_len, w.heads, D_QK), generator=g, dtype=torch.float32)
    if w.q_std != 1.0:
        q.mul_(w.q_std)
    q = q.to(torch.bfloat16)

    indices = None
    if w.topk > 0:
        indices = torch.empty((B, w.q_len, w.topk), dtype=torch.int32)
        for b in range(B):
            for i in range(w.q_len):
                L = int(seq_lens[b])
                perm = torch.randperm(L, generator=g)[: w.topk]
                row = torch.full((w.topk,), -1, dtype=torch.int32)
                row[: perm.numel()] = perm.to(torch.int32)
                indices[b, i] = row

    return {
        "workload": w,
        "q": q,
        "cache": cache,
        "block_table": block_table,
        "seq_lens": seq_lens.to(torch.int32),
        "indices": indices,
        "batch": B,
        "q_len": w.q_len,
        "heads": w.heads,
        "topk": w.topk,
        "causal": w.causal,
        "num_pages": num_pages,
        "max_pages_per_seq": maxp,
    }


def small(key: str = "t", *, batch: int, heads: int, q_len: int = 1, lens: Sequence[int], topk: int = 0,
          causal: bool = False, seed: int = 0, q_std: float = 1.0, cache_std: float = 1.0,
          **kw) -> dict:
    """A custom (usually small) workload with explicit lengths."""
    w = Workload(key, f"custom-b{batch}-h{heads}-sq{q_len}", batch, q_len, heads, min(lens), max(lens), topk=topk,
                 causal=causal, q_std=q_std, cache_std=cache_std, seed=seed)
    return make_inputs(w, lens=lens, **kw)



def insert_inputs(*, lens: Sequence[int], new_tokens: Sequence[int], seed: int = 0, kv_std: float = 1.0,
                  rope_base: float = 10000.0, slack_pages: int = 2) -> dict:
    """Inputs of a latent-cache insert: sequence b already holds
    ``lens[b] - new_tokens[b]`` tokens and appends ``new_tokens[b]`` more at
    positions ``lens[b] - new_tokens[b] .. lens[b] - 1`` (a prefill chunk when
    that is the whole sequence, one decode token when it is 1).

    Draw order, from one generator: page permutation -> prior cache contents ->
    new rows ``kv`` [N, 576] (N(0, kv_std)) -> kv_norm weight (N(1, 0.1^2)).
    ``cos``/``sin`` [max(lens), 32] are the RoPE tables of the caller at angle
    ``pos * rope_base ** (-i / 32)`` for pair i (the usual RoPE frequency
    ladder; the method takes any table)."""
    g = torch.Generator().manual_seed(seed)
    lens = [int(x) for x in lens]
    new_tokens = [int(x) for x in new_tokens]
    npg = [max((L + PAGE - 1) // PAGE, 1) for L in lens]
    maxp = max(npg) if npg else 1
    num_pages = sum(npg) + slack_pages
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    bt = torch.full((len(lens), maxp), -1, dtype=torch.int32)
    k = 0
    for b, n in enumerate(npg):
        bt[b, :n] = perm[k:k + n]
        k += n
    cache = torch.randn(num_pages, PAGE, D_QK, generator=g).to(torch.bfloat16)
    seq_ids = torch.cat([torch.full((n,), b, dtype=torch.int32) for b, n in enumerate(new_tokens)])
    positions = torch.cat([torch.arange(L - n, L, dtype=torch.int32) for L, n in zip(lens, new_tokens)])
    kv = (torch.randn(len(seq_ids), D_QK, generator=g) * kv_std).to(torch.bfloat16)
    weight = (1.0 + 0.1 * torch.randn(D_LATENT, generator=g)).to(torch.bfloat16)
    max_pos = max(lens) if lens else 1
    inv_freq = rope_base ** (-torch.arange(32, dtype=torch.float64) / 32.0)
    ang = torch.arange(max_pos, dtype=torch.float64)[:, None] * inv_freq[None, :]
    return {
        "kv": kv, "weight": weight, "cos": torch.cos(ang).float(), "sin": torch.sin(ang).float(),
        "seq_ids": seq_ids, "positions": positions, "block_table": bt, "cache": cache,
        "batch": len(lens), "num_pages": num_pages, "max_pages_per_seq": maxp, "lens": lens,
    }


def absorb_inputs(*, tokens: int, heads: int, seed: int = 0, w_std: float = 0.05, o_std: float = 0.3) -> dict:
    """Inputs of the absorb / un-absorb projections for T = ``tokens`` query
    tokens: q [T, H, 192] ~ N(0, 1) (q_nope || q_pe), wkv_b [H, 256, 512] ~
    N(0, w_std^2) (rows 0-127 of a head: W_UK, 128-255: W_UV, as the model's
    kv up-projection viewed per head), o_lat [T, H, 512] ~ N(0, o_std^2).
    Draw order: q -> wkv_b -> o_lat."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(tokens, heads, 192, generator=g).to(torch.bfloat16)
    wkv_b = (torch.randn(heads, 256, 512, generator=g) * w_std).to(torch.bfloat16)
    o_lat = (torch.randn(tokens, heads, 512, generator=g) * o_std).to(torch.bfloat16)
    return {"q": q, "wkv_b": wkv_b, "o_lat": o_lat, "tokens": tokens, "heads": heads}


def indexer_inputs(*, batch: int, q_len: int, heads: int, num_keys: int, seed: int = 0, code_std: float = 16.0,
                   chunk: int = 1 << 22) -> dict:
    """Inputs of the sparse-attention indexer ("DeepSeek-V3.2-Exp unboxing",
    the Indexer section: fp8 q [b, m, h, 128] with per-head weights q_s
    [b, m, h], fp8 keys k [b, n, 128] with per-key scales k_s [b, n]).

    Draw order, from one generator: q codes -> q_s -> k codes -> k_s. Codes
    are N(0, code_std^2) clipped to the e4m3 range and cast to e4m3 by the
    library; q_s ~ N(0, 1/h) (weights of either sign); k_s ~ U[0.5, 1.5) /
    code_std (positive scales)."""
    g = torch.Generator().manual_seed(seed)
    D = 128

    def codes(n_rows):
        out = torch.empty(n_rows, D, dtype=torch.float8_e4m3fn)
        for r0 in range(0, n_rows, max(1, chunk // D)):
            r1 = min(n_rows, r0 + max(1, chunk // D))
            out[r0:r1] = (torch.randn(r1 - r0, D, generator=g) * code_std).clamp(-448, 448).to(torch.float8_e4m3fn)
        return out

    q = codes(batch * q_len * heads).view(batch, q_len, heads, D)
    q_s = torch.randn(batch, q_len, heads, generator=g) / math.sqrt(heads)
    k = codes(batch * num_keys).view(batch, num_keys, D)
    k_s = (0.5 + torch.rand(batch, num_keys, generator=g)) / code_std
    return {"q": q, "q_s": q_s, "k": k, "k_s": k_s, "batch": batch, "q_len": q_len, "heads": heads,
            "num_keys": num_keys}


FP8_ROW_BYTES = 656  # e4m3 latent codes 512 | bf16 rope 128 | f32 scale 4 | zero 12


def make_fp8_cache(inp: dict, *, seed: Optional[int] = None, code_std: float = 64.0,
                   nan_tail: bool = False) -> torch.Tensor:
    """An fp8 latent cache ``[num_pages, 64, 656]`` (uint8 rows: 512 e4m3
    codes, 64 bf16 rope values, a float32 scale, 12 zero bytes) for the page
    layout of ``inp`` (a dict from :func:`make_inputs`), drawn directly — no
    quantisation: codes ~ N(0, code_std^2) clipped to the e4m3 range and cast
    by the library, scales ~ U[0.5, 1.5) * cache_std / code_std, rope ~
    N(0, cache_std^2) in bf16. Draw order from one generator (seed: the
    workload's + 1000): codes -> scales -> rope. Pages no sequence owns, and
    with ``nan_tail`` the unused rows of each sequence's last page, are NaN
    (codes 0x7F, NaN scale and rope)."""
    w = inp["workload"]
    g = torch.Generator().manual_seed((w.seed if seed is None else seed) + 1000)
    P = inp["num_pages"]
    raw = torch.zeros(P, PAGE, FP8_ROW_BYTES, dtype=torch.uint8)
    rows = raw.view(P * PAGE, FP8_ROW_BYTES)
    n = P * PAGE
    step = 1 << 14
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        codes = (torch.randn(r1 - r0, D_LATENT, generator=g) * code_std).clamp(-448, 448)
        rows[r0:r1, :D_LATENT] = codes.to(torch.float8_e4m3fn).view(torch.uint8)
    scales = (0.5 + torch.rand(n, generator=g)) * (w.cache_std / code_std)
    rows[:, 640:644] = scales.to(torch.float32).view(torch.uint8).view(n, 4)
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        rope = (torch.randn(r1 - r0, 64, generator=g) * w.cache_std).to(torch.bfloat16)
        rows[r0:r1, 512:640] = rope.view(torch.uint8).view(r1 - r0, 128)

    def poison(sel):
        sel[..., :D_LATENT] = 0x7F
        sel[..., 512:640] = torch.full(sel.shape[:-1] + (64,), float("nan"), dtype=torch.bfloat16).view(
            torch.uint8).view(sel.shape[:-1] + (128,))
        sel[..., 640:644] = torch.full(sel.shape[:-1] + (1,), float("nan")).view(torch.uint8).view(
            sel.shape[:-1] + (4,))

    used = int(sum((int(L) + PAGE - 1) // PAGE for L in inp["seq_lens"].tolist()))
    if used < P:
        poison(raw[used:])
    if nan_tail:
        bt = inp["block_table"]
        for b, L in enumerate(inp["seq_lens"].tolist()):
            if L % PAGE and L > 0:
                poison(raw[int(bt[b, (L - 1) // PAGE]), L % PAGE:])
    return raw

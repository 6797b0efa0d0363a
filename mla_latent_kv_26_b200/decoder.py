"""Torch-facing wrapper around the C ABI: owns the plan / workspace / output
buffers for one decode shape and issues the three library calls on a CUDA
stream. It checks tensor dtypes, shapes and devices and passes raw pointers;
all arithmetic happens in libmla's kernels.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class MlaDecoder:
    def __init__(self, *, batch: int, q_len: int, num_heads: int, num_pages: int, max_pages_per_seq: int,
                 topk: int = 0, causal: bool = False, softmax_scale: float = B.DEFAULT_SOFTMAX_SCALE,
                 num_sms: int = 0, device="cuda"):
        self.desc = B.make_desc(batch=batch, q_len=q_len, num_heads=num_heads, num_pages=num_pages,
                                max_pages_per_seq=max_pages_per_seq, topk=topk, causal=causal,
                                softmax_scale=softmax_scale, num_sms=num_sms)
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        with torch.cuda.device(self.device):
            self.plan_bytes = B.mla_plan_bytes(self.desc)
            self.workspace_bytes = B.mla_workspace_bytes(self.desc)
            self.num_workers = B.mla_num_workers(self.desc)
        if self.plan_bytes == 0 or self.workspace_bytes == 0:
            raise B.MlaError(B.MLA_ERR_INVALID_ARG, "descriptor rejected by the sizing queries")
        self.plan = torch.empty(self.plan_bytes, dtype=torch.uint8, device=self.device)
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)
        self.out = torch.empty(batch, q_len, num_heads, 512, dtype=torch.bfloat16, device=self.device)
        self.lse = torch.empty(batch, q_len, num_heads, dtype=torch.float32, device=self.device)

    def _stream(self, stream):
        return torch.cuda.current_stream(self.device) if stream is None else stream

    def _check(self, name, t, dtype, shape=None):
        if t.device != self.device or t.dtype != dtype or not t.is_contiguous():
            raise ValueError(f"{name}: need a contiguous {dtype} tensor on {self.device}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")

    def plan_step(self, seq_lens: torch.Tensor, stream=None) -> None:
        d = self.desc
        self._check("seq_lens", seq_lens, torch.int32, (d.batch,))
        B.check(B.mla_decode_plan(d, seq_lens, self.plan, self.plan_bytes, self._stream(stream)), "mla_decode_plan")

    def decode_step(self, q, kv_cache, block_table, seq_lens, indices: Optional[torch.Tensor] = None,
                    stream=None) -> None:
        """``kv_cache``: bf16 [pages, 64, 576], or uint8 [pages, 64, 656] for an
        fp8 latent cache (mla_decode_fp8)."""
        d = self.desc
        self._check("q", q, torch.bfloat16, (d.batch, d.q_len, d.num_heads, 576))
        fp8 = kv_cache.dtype == torch.uint8
        if fp8:
            self._check("kv_cache", kv_cache, torch.uint8, (d.num_pages, 64, 656))
        else:
            self._check("kv_cache", kv_cache, torch.bfloat16, (d.num_pages, 64, 576))
        self._check("block_table", block_table, torch.int32, (d.batch, d.max_pages_per_seq))
        self._check("seq_lens", seq_lens, torch.int32, (d.batch,))
        if d.topk > 0:
            self._check("indices", indices, torch.int32, (d.batch, d.q_len, d.topk))
        elif indices is not None:
            raise ValueError("indices given for a dense descriptor")
        fn = B.mla_decode_fp8 if fp8 else B.mla_decode
        B.check(fn(d, self.plan, q, kv_cache, block_table, seq_lens, indices, self.out, self.lse,
                   self.workspace, self.workspace_bytes, self._stream(stream)), "mla_decode")

    def combine_step(self, stream=None) -> None:
        B.check(B.mla_combine(self.desc, self.plan, self.workspace, self.workspace_bytes, self.out, self.lse,
                              self._stream(stream)), "mla_combine")

    def __call__(self, q, kv_cache, block_table, seq_lens, indices=None, stream=None):
        self.plan_step(seq_lens, stream)
        self.decode_step(q, kv_cache, block_table, seq_lens, indices, stream)
        self.combine_step(stream)
        return self.out, self.lse

    def error(self, stream=None):
        """(status, device error bits); synchronises the stream."""
        return B.mla_get_error(self.plan, self._stream(stream))


def decoder_for(inputs: dict, *, num_sms: int = 0, device="cuda", **kw) -> MlaDecoder:
    """An MlaDecoder sized for a dict made by ``workloads.make_inputs``."""
    return MlaDecoder(batch=inputs["batch"], q_len=inputs["q_len"], num_heads=inputs["heads"],
                      num_pages=inputs["num_pages"], max_pages_per_seq=inputs["max_pages_per_seq"],
                      topk=inputs["topk"], causal=inputs["causal"], num_sms=num_sms, device=device, **kw)


def cache_insert(kv: torch.Tensor, weight: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor, seq_ids: torch.Tensor,
                 positions: torch.Tensor, block_table: torch.Tensor, kv_cache: torch.Tensor, *, eps: float = 1e-6,
                 error_word: Optional[torch.Tensor] = None, stream=None) -> None:
    """kv_norm + RoPE of the new tokens' rows ``kv`` [N, 576], written in place
    into their rows of ``kv_cache`` [pages, 64, 576] bf16, or of an fp8 cache
    [pages, 64, 656] uint8 (mla_cache_insert_fp8), in one library kernel.
    ``error_word``: optional int32 [1] device tensor that collects the
    MLA_DEVERR bits of skipped tokens."""
    dev = kv_cache.device
    n = kv.shape[0] if kv.dim() == 2 else -1
    want = [("kv", kv, torch.bfloat16, (n, 576)), ("weight", weight, torch.bfloat16, (512,)),
            ("cos", cos, torch.float32, (cos.shape[0], 32)), ("sin", sin, torch.float32, tuple(cos.shape)),
            ("seq_ids", seq_ids, torch.int32, (n,)), ("positions", positions, torch.int32, (n,)),
            ("block_table", block_table, torch.int32, None),
            ("kv_cache", kv_cache, torch.uint8 if kv_cache.dtype == torch.uint8 else torch.bfloat16, None)]
    for name, t, dtype, shape in want:
        if t.device != dev or t.dtype != dtype or not t.is_contiguous():
            raise ValueError(f"{name}: need a contiguous {dtype} tensor on {dev}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    fp8 = kv_cache.dtype == torch.uint8
    if block_table.dim() != 2 or kv_cache.dim() != 3 or tuple(kv_cache.shape[1:]) != (64, 656 if fp8 else 576):
        raise ValueError("block_table must be [batch, max_pages_per_seq], kv_cache [pages, 64, 576] bf16 "
                         "or [pages, 64, 656] uint8")
    if error_word is not None and (error_word.device != dev or error_word.dtype != torch.int32):
        raise ValueError("error_word: need an int32 tensor on the cache's device")
    desc = B.make_insert_desc(num_tokens=n, batch=block_table.shape[0], max_pages_per_seq=max(block_table.shape[1], 1),
                              num_pages=kv_cache.shape[0], max_positions=cos.shape[0], eps=eps)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    with torch.cuda.device(dev):
        fn = B.mla_cache_insert_fp8 if fp8 else B.mla_cache_insert
        B.check(fn(desc, kv, weight, cos, sin, seq_ids, positions, block_table, kv_cache, error_word, s),
                "mla_cache_insert")


def _check_tensor(name, t, dtype, shape, dev):
    if t.device != dev or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: need a contiguous {dtype} tensor on {dev}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")


def absorb_query(q: torch.Tensor, wkv_b: torch.Tensor, out: Optional[torch.Tensor] = None, *,
                 error_word: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """q [T, H, 192] (q_nope || q_pe) and wkv_b [H, 256, 512] -> the decode
    query [T, H, 576] = (W_UK^T q_nope || q_pe), one library kernel."""
    T, H = q.shape[0], q.shape[1]
    dev = q.device
    _check_tensor("q", q, torch.bfloat16, (T, H, 192), dev)
    _check_tensor("wkv_b", wkv_b, torch.bfloat16, (H, 256, 512), dev)
    if out is None:
        out = torch.empty(T, H, 576, dtype=torch.bfloat16, device=dev)
    _check_tensor("out", out, torch.bfloat16, (T, H, 576), dev)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    with torch.cuda.device(dev):
        B.check(B.mla_absorb_query(B.make_absorb_desc(num_tokens=T, num_heads=H), q, wkv_b, out, error_word, s),
                "mla_absorb_query")
    return out


def unabsorb_output(o_lat: torch.Tensor, wkv_b: torch.Tensor, out: Optional[torch.Tensor] = None, *,
                    error_word: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """o_lat [T, H, 512] (the decode output) and wkv_b [H, 256, 512] -> the
    per-head values [T, H, 128] = W_UV o_lat, one library kernel."""
    T, H = o_lat.shape[0], o_lat.shape[1]
    dev = o_lat.device
    _check_tensor("o_lat", o_lat, torch.bfloat16, (T, H, 512), dev)
    _check_tensor("wkv_b", wkv_b, torch.bfloat16, (H, 256, 512), dev)
    if out is None:
        out = torch.empty(T, H, 128, dtype=torch.bfloat16, device=dev)
    _check_tensor("out", out, torch.bfloat16, (T, H, 128), dev)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    with torch.cuda.device(dev):
        B.check(B.mla_unabsorb_output(B.make_absorb_desc(num_tokens=T, num_heads=H), o_lat, wkv_b, out, error_word,
                                      s), "mla_unabsorb_output")
    return out

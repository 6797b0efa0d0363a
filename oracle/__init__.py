"""Reference oracle for MLA latent-KV decode — TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, CPU float64 restatement of what the decode
path computes. It exists so that tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` can check and time the CUDA path against
an independent definition. Nothing on the product path may import it; the
CUDA library shares no code, header, table or helper with it.

Sources (web pages on DeepSeek V2/V3 inference, cited by title and section):

* "深度解读DeepSeek：源码解读 DeepSeek-V3" (dtcms.com), section "MLA", the
  absorbed branch ("优化实现"): the score is the sum of a latent term
  ``q_nope_abs · kv_cache`` and a RoPE term ``q_pe · pe_cache`` times
  ``softmax_scale``; softmax is taken in float32 (here float64); the output is
  the probability-weighted sum of the same latent cache rows.
* "DeepSeek-V2-Lite 模型结构详解" (yangyangai.win), section "五、MLA：注意力",
  sub-sections "最关键的一问：解压的代价去哪了" (the two absorption identities)
  and "为什么 Q/K 是 192 维而 V 只有 128 维" (Q/K width 128 + 64 = 192, which
  fixes ``softmax_scale = 1/sqrt(192)``).
* "DeepSeek tag page" (beaiera.top), abstract on the √d_k factor.

Modules:

* :mod:`oracle.decode` — the attention definition (a2–a7), the LSE merge (a8)
  and the unabsorbed ("naive") path used to pin the absorbed one.
* :mod:`oracle.plan` — the split schedule (a1) written as a plain sequential
  definition of a balanced contiguous partition.
* :mod:`oracle.cache_insert` — the step before decode: kv_norm (RMSNorm) of the
  latent, the rotary embedding of the rope key, and the write into the token's
  row of the paged cache.
* :mod:`oracle.fp8_cache` — the fp8 (e4m3) form of the cached latent: per-token
  scale, e4m3 rounding, and the round trip back to bf16 that an fp8-cache
  decode sees.
* :mod:`oracle.indexer` — the sparse-attention indexer ("DeepSeek-V3.2-Exp
  unboxing", the Indexer section): fp8 index scores per (query, key) and the
  top-k positions that the sparse decode attends to.

Pins (tests/test_oracle.py): absorption equivalence against the unabsorbed
path, single-key exactness, probabilities summing to one, brute force with
pure-Python loops on tiny shapes, closed forms (zero query, identical rows,
a dominant key, causal pair vs shorter context, sparse-with-all-indices vs
dense, page permutation), the partition identity of the LSE merge, and the
page's printed cost figures (tests/golden/). Every function here is pinned.
"""

from .decode import (  # noqa: F401
    D_LATENT,
    D_ROPE,
    D_QK,
    PAGE_SIZE,
    QK_HEAD_DIM,
    DEFAULT_SOFTMAX_SCALE,
    visible_tokens,
    gather_rows,
    scores,
    attention_probs,
    mla_decode,
    lse_merge,
    absorb_query,
    unabsorb_output,
    unabsorbed_attention,
)
from .plan import split_plan  # noqa: F401
from .cache_insert import rms_norm, rope_pairs, cache_insert  # noqa: F401,E402
from .fp8_cache import (e4m3_round, quantize_rows, dequantize_rows, fp8_roundtrip_cache, unpack_rows,  # noqa: F401,E402
                        dequantize_cache)
from .indexer import index_scores, topk_positions  # noqa: F401,E402

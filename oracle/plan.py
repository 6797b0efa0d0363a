"""Plain definition of the split-KV schedule (hot-path step a1).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages never split a sequence: their decode reads the whole cache of each
sequence in one einsum ("深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA").
Splitting is how one GPU keeps every SM busy when a batch holds few, ragged,
long sequences; its result is exact because of the LSE merge (see
:func:`oracle.decode.lse_merge`). The schedule defined here is a balanced
contiguous partition:

1. A *task* is one query token of one sequence: ``t = b * q_len + i``. Its
   token count ``n_t`` is ``topk`` (sparse), ``L_b - q_len + i + 1`` (dense
   causal, clamped at 0) or ``L_b`` (dense). A length outside
   ``[0, max_pages_per_seq * 64]`` is an error: the task gets no tokens and
   the error flag is raised.
2. Each task covers ``ceil(n_t / 64)`` pages (tiles of 64 tokens, or of 64
   index slots in sparse mode). The tasks' pages are laid end to end in task
   order; ``prefix[t]`` is the first global page of task ``t``.
3. With ``P`` workers (CTA pairs) the quota is ``q = max(1, ceil(total / P))``
   and worker ``p`` takes global pages ``[p*q, min((p+1)*q, total))``.
4. Each (worker, task) overlap is one work item; its partial result goes to
   slot ``p + t``. A task covered by one worker is *unsplit*.
"""

from __future__ import annotations

PAGE_SIZE = 64


def task_token_counts(seq_lens, *, q_len: int, causal: bool, topk: int, max_pages_per_seq: int):
    """Per-task token counts (step 1) and whether any length was out of range."""
    counts = []
    bad = False
    cap = max_pages_per_seq * PAGE_SIZE
    for L in [int(x) for x in seq_lens]:
        ok = 0 <= L <= cap
        bad |= not ok
        for i in range(q_len):
            if not ok:
                n = 0
            elif topk > 0:
                n = topk
            elif causal:
                n = max(L - q_len + i + 1, 0)
            else:
                n = L
            counts.append(n)
    return counts, bad


def split_plan(seq_lens, *, q_len: int, causal: bool, topk: int, max_pages_per_seq: int, num_pairs: int):
    """The full schedule as plain Python lists (steps 1–4)."""
    counts, bad = task_token_counts(seq_lens, q_len=q_len, causal=causal, topk=topk,
                                    max_pages_per_seq=max_pages_per_seq)
    pages = [(n + PAGE_SIZE - 1) // PAGE_SIZE for n in counts]
    prefix = [0]
    for pg in pages:
        prefix.append(prefix[-1] + pg)
    total = prefix[-1]
    quota = max(1, -(-total // num_pairs)) if num_pairs > 0 else 0
    items = []
    splits = [0] * len(pages)
    for p in range(num_pairs):
        lo = p * quota
        hi = min(lo + quota, total)
        mine = []
        for t in range(len(pages)):
            a = max(lo, prefix[t])
            b = min(hi, prefix[t + 1])
            if a < b:
                mine.append((t, a - prefix[t], b - prefix[t], p + t))
                splits[t] += 1
        items.append(mine)
    return {
        "task_tokens": counts,
        "task_pages": pages,
        "prefix": prefix,
        "total_pages": total,
        "quota": quota,
        "items": items,
        "splits": splits,
        "bad_lengths": bad,
    }

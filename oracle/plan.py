"""Plain definition of the split-KV schedule (hot-path step a1).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages never split a sequence: their decode reads the whole cache of each
sequence in one einsum ("深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA").
Splitting is how one GPU keeps every SM busy when a batch holds few, ragged,
long sequences; its result is exact because of the LSE merge (see
:func:`oracle.decode.lse_merge`). The schedule defined here is a balanced
contiguous partition:

1. A *task* is one query token of one sequence: query row ``b * q_len + i``.
   Its token count ``n`` is ``topk`` (sparse), ``L_b - q_len + i + 1``
   (dense causal, clamped at 0) or ``L_b`` (dense). A length outside
   ``[0, max_pages_per_seq * 64]`` is an error: the task gets no tokens and
   the error flag is raised.
2. Each task covers ``ceil(n / 64)`` pages (tiles of 64 tokens, or of 64
   index slots in sparse mode).
3. Plan order and worker groups. With several dense query tokens per
   sequence (``2 <= q_len <= 8``, no top-k) and at least 4 workers per
   token, the workers form ``G = q_len`` equal groups of ``Wg = P // G``
   (the ``P mod G`` left over stay idle) and the plan order is token-major:
   position ``u`` holds token ``u // B`` of sequence ``u % B``, so group
   ``g`` owns positions ``[g B, (g + 1) B)``, i.e. token ``g`` of every
   sequence. Tokens of one sequence read the same pages; the groups walk
   them in step, so that a page fetched for one token is still in L2 for
   the others. Otherwise ``G = 1``, ``Wg = P`` and position ``u`` is query
   row ``u`` (``u = b * q_len + i``).
4. The tasks' pages are laid end to end in plan order; ``prefix[u]`` is the
   first global page of position ``u``. Group ``g`` holds global pages
   ``[prefix[g T/G], prefix[(g+1) T/G])``; its quota is
   ``q_g = max(1, ceil(pages_g / Wg))`` and its ``j``-th worker (worker
   ``g Wg + j``) takes the group's pages ``[j q_g, (j+1) q_g)``.
5. Each (worker, position) overlap is one work item; its partial result goes
   to slot ``worker + u``. A task covered by one worker is *unsplit*.
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


def plan_groups(*, q_len: int, topk: int, num_pairs: int) -> int:
    """Number of worker groups (step 3)."""
    if 2 <= q_len <= 8 and topk == 0 and num_pairs // q_len >= 4:
        return q_len
    return 1


def split_plan(seq_lens, *, q_len: int, causal: bool, topk: int, max_pages_per_seq: int, num_pairs: int):
    """The full schedule as plain Python lists (steps 1-5), in plan order."""
    counts, bad = task_token_counts(seq_lens, q_len=q_len, causal=causal, topk=topk,
                                    max_pages_per_seq=max_pages_per_seq)
    B = len(counts) // q_len if q_len > 0 else 0
    G = plan_groups(q_len=q_len, topk=topk, num_pairs=num_pairs)
    Wg = num_pairs // G if num_pairs > 0 else 0
    # query row of each plan position
    rows = [(u % B) * q_len + u // B for u in range(len(counts))] if G > 1 else list(range(len(counts)))
    tokens = [counts[r] for r in rows]
    pages = [(n + PAGE_SIZE - 1) // PAGE_SIZE for n in tokens]
    prefix = [0]
    for pg in pages:
        prefix.append(prefix[-1] + pg)
    total = prefix[-1]
    T = len(pages)
    TG = T // G if G > 0 else 0
    quotas = []
    for g in range(G):
        n_g = prefix[(g + 1) * TG] - prefix[g * TG]
        quotas.append(max(1, -(-n_g // Wg)) if Wg > 0 else 0)
    items = [[] for _ in range(num_pairs)]
    splits = [0] * T
    for g in range(G):
        base, end = prefix[g * TG], prefix[(g + 1) * TG]
        for j in range(Wg):
            w = g * Wg + j
            lo = base + j * quotas[g]
            hi = min(lo + quotas[g], end)
            for u in range(g * TG, (g + 1) * TG):
                a = max(lo, prefix[u])
                b = min(hi, prefix[u + 1])
                if a < b:
                    items[w].append((u, a - prefix[u], b - prefix[u], w + u))
                    splits[u] += 1
    return {
        "groups": G,
        "workers_per_group": Wg,
        "task_rows": rows,
        "task_tokens": tokens,
        "task_pages": pages,
        "prefix": prefix,
        "total_pages": total,
        "quota": quotas[0],
        "quotas": quotas,
        "items": items,
        "splits": splits,
        "bad_lengths": bad,
    }

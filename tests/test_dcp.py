"""Decode context parallelism on CPU (gloo ranks, no GPU): the sharding of
every sequence's pages over the ranks, the all-gather of the ranks' (out,
lse) and the LSE merge, checked against the un-sharded float64 oracle.

On the CPU each rank's shard is decoded by the oracle and merged by the
oracle's lse_merge (the library kernels run in the GPU tests of
test_parity_dcp.py); what is tested here is the host logic that the GPU path
shares: which pages each rank holds, their renumbering, the causal flag of
each rank, the remapping of sparse positions, and the gather. A rank that
leaves between steps is detected on the host: the survivor's gather raises.
"""

import os
import socket
import sys
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("q_len,causal", [(1, False), (2, True), (3, True), (2, False)])
def test_shard_bounds_partition_every_sequence(world, q_len, causal):
    from mla_latent_kv_26_b200.dcp import shard_bounds

    for L in list(range(0, 300)) + [4096, 4097, 32768, 65535]:
        runs = shard_bounds(L, world, q_len=q_len, causal=causal)
        P = (L + 63) // 64
        assert len(runs) == world
        assert runs[0][0] == 0 and runs[-1][1] == P
        for (a0, a1), (b0, b1) in zip(runs, runs[1:]):
            assert a0 <= a1 == b0 <= b1
        if causal and L >= q_len:
            # every token some query row cannot see (t > L - Sq) lies on the last rank
            assert runs[-1][0] * 64 <= L - q_len + 1


def _oracle_decode(q, cache, shard):
    import oracle

    o, l = oracle.mla_decode(q, cache, shard["block_table"], shard["seq_lens"], causal=shard["causal"],
                             indices=shard["indices"])
    return o.float(), l.float()


def _oracle_merge(po, pl):
    import oracle

    return oracle.lse_merge(po.double(), pl.double())


CASES = {
    "dense": dict(lens=[700, 64, 1, 5000, 0], q_len=1, causal=False, topk=0),
    "causal-pair": dict(lens=[129, 2, 65, 3000], q_len=2, causal=True, topk=0),
    "causal-three": dict(lens=[193, 3, 64, 4000], q_len=3, causal=True, topk=0),
    "sparse": dict(lens=[3000, 400, 2100], q_len=1, causal=False, topk=256),
}


def _case_inputs(name):
    sys.path.insert(0, ROOT)
    from mla_latent_kv_26_b200.workloads import small

    c = CASES[name]
    return small(batch=len(c["lens"]), heads=16, q_len=c["q_len"], causal=c["causal"], lens=c["lens"],
                 topk=c["topk"], seed=len(name))


def _rank_main(rank, world, port, name, q):
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        from mla_latent_kv_26_b200.dcp import dcp_decode

        d = _case_inputs(name)
        out, lse = dcp_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], world=world, rank=rank,
                              q_len=d["q_len"], causal=d["causal"], indices=d["indices"],
                              decode=_oracle_decode, merge=_oracle_merge)
        # by value (numpy): a tensor would travel as a file descriptor that the
        # parent fetches from this process, which may have exited by then
        q.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", sorted(CASES))
def test_dcp_gloo_ranks_match_unsharded_oracle(world, name):
    import oracle

    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    d = _case_inputs(name)
    o_ref, l_ref = oracle.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], causal=d["causal"],
                                     indices=d["indices"])
    for rank, out, lse in results:
        out, lse = torch.from_numpy(out), torch.from_numpy(lse)
        # each rank's partial travelled as float32: agreement to float32 rounding
        assert torch.allclose(out, o_ref, rtol=1e-5, atol=1e-5), (name, rank)
        fin = torch.isfinite(l_ref)
        assert torch.equal(torch.isfinite(lse), fin)
        assert torch.allclose(lse[fin], l_ref[fin], rtol=0, atol=1e-5), (name, rank)


def _leaving_rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    from datetime import timedelta

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=10))
    from mla_latent_kv_26_b200.dcp import dcp_decode

    d = _case_inputs("dense")
    kw = dict(world=world, rank=rank, q_len=1, causal=False, decode=_oracle_decode, merge=_oracle_merge)
    dcp_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], **kw)  # one step together
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()
        os._exit(0)  # leaves between steps, with no collective in flight
    time.sleep(1.0)
    t0 = time.time()
    try:
        dcp_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], **kw)
        q.put((rank, "no error"))
    except Exception as e:  # noqa: BLE001 - any failure of the collective is what is expected
        q.put((rank, f"raised after {time.time() - t0:.1f} s: {type(e).__name__}"))
    q.close()
    q.join_thread()
    os._exit(0)


def test_rank_leaving_between_steps_is_seen_by_the_survivor():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_leaving_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert got[1] == "left"
    assert got[0].startswith("raised"), got[0]

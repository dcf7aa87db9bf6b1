"""The multi-GPU partition (hybrid_sparse_attention_qsa_b200/shard.py), on CPU.

Prefill rows are sharded in zig-zag chunks and K, V and the pooled keys are all-gathered; decode
splits the batch.  Here two gloo ranks on CPU run the partition and the exchange, with the CPU
oracle standing in for the per-rank kernels: the gathered tensors must equal the unsharded ones
bit for bit, and the ranks' output rows, put back in order, must equal the single-process oracle's.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from hybrid_sparse_attention_qsa_b200 import inputs as I
from hybrid_sparse_attention_qsa_b200 import shard as S


@pytest.mark.parametrize("T,world", [(131072, 1), (131072, 2), (131072, 4), (131072, 8), (1048576, 8), (2048, 2)])
def test_zigzag_chunks_cover_every_row_once_and_balance_the_triangle(T, world):
    owned = [S.rank_chunks(T, world, r) for r in range(world)]
    rows = np.zeros(T, dtype=np.int64)
    for ranges in owned:
        for a, b in ranges:
            assert a % 4 == 0 and b % 4 == 0 and a < b
            rows[a:b] += 1
    assert np.all(rows == 1)
    if world > 1:
        sizes = {b - a for ranges in owned for a, b in ranges}
        assert sizes == {T // (2 * world)}
    cost = [S.causal_cost(r, k=512) for r in owned]
    pairs = [c["index_pairs"] for c in cost]
    toks = [c["attended_tokens"] for c in cost]
    # the indexer's triangle splits exactly evenly; the attention (flat past 2048 tokens; the rank
    # holding the first chunk gets the cheap first rows) leaves the busiest rank within 1% of the mean
    assert max(pairs) == min(pairs)
    assert max(toks) <= 1.01 * sum(toks) / world
    total = S.causal_cost([(0, T)], k=512)
    assert sum(pairs) == total["index_pairs"] and sum(toks) == total["attended_tokens"]


def test_zigzag_rejects_unaligned_lengths():
    with pytest.raises(ValueError):
        S.zigzag_chunks(1000, 2)        # 1000 is not a multiple of 2 * 2 * 4
    with pytest.raises(ValueError):
        S.zigzag_chunks(4096, 0)


@pytest.mark.parametrize("B,world", [(32, 1), (32, 2), (32, 8), (5, 2), (3, 4)])
def test_decode_batch_ranges(B, world):
    got = [S.batch_range(B, world, r) for r in range(world)]
    assert got[0][0] == 0 and got[-1][1] == B
    assert all(got[i][1] == got[i + 1][0] for i in range(world - 1))
    sizes = [b - a for a, b in got]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


W = I.WORKLOADS["prefill_32k"].with_(T=512, Hq=4, Hkv=2, D=32, k=24, seed=5)


def _rank(rank, world, port, q):
    import oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = I.make_prefill(W, "cpu")            # the job's inputs; this rank keeps only its rows
        ranges = S.rank_chunks(W.T, world, rank)
        mine = {n: [x[n][:, a:b].contiguous() for a, b in ranges] for n in x}
        # per-rank pooling of its own indexer keys (the oracle in place of the pooling kernel)
        kp_local = [I.from_bits(O.pool_block_keys(I.bits(c), pos0=a)) for (a, _), c in zip(ranges, mine["ki"])]
        kfull = torch.empty_like(x["k"])
        vfull = torch.empty_like(x["v"])
        kpfull = torch.empty(W.B, W.T // 4, W.Di, dtype=torch.bfloat16)
        S.allgather_rows(kp_local, kpfull, W.T // 4, world, rank)
        S.allgather_rows(mine["k"], kfull, W.T, world, rank)
        S.allgather_rows(mine["v"], vfull, W.T, world, rank)
        same = (torch.equal(kfull.view(torch.int16), x["k"].view(torch.int16))
                and torch.equal(vfull.view(torch.int16), x["v"].view(torch.int16))
                and np.array_equal(I.bits(kpfull), O.pool_block_keys(I.bits(x["ki"]))))
        # this rank's rows over the gathered tensors (the oracle in place of select + attention)
        outs = []
        for (a, b), qc, qic in zip(ranges, mine["q"], mine["qi"]):
            r = O.prefill_rows(I.bits(qc), I.bits(kfull), I.bits(vfull), I.bits(qic), I.bits(kpfull),
                               [(0, t) for t in range(b - a)], topk=W.k, q_pos0=a, nthreads=1)
            outs.append((a, b, r["out"], r["idx"]))
        q.put((rank, same, ranges, outs))
    finally:
        torch.distributed.destroy_process_group()


def test_sharded_prefill_two_gloo_ranks_equals_one_process():
    import oracle as O
    O.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    res = {r[0]: r for r in res}
    assert res[0][1] and res[1][1], "gathered K / V / kp differ from the unsharded tensors"
    assert res[0][2] == [(0, 128), (384, 512)] and res[1][2] == [(128, 256), (256, 384)]
    # the ranks' rows, in order, against one process over all rows
    x = I.make_prefill(W, "cpu")
    h = {n: I.bits(x[n]) for n in x}
    kp = O.pool_block_keys(h["ki"])
    ref = O.prefill_rows(h["q"], h["k"], h["v"], h["qi"], kp, [(0, t) for t in range(W.T)], topk=W.k)
    out = np.empty_like(ref["out"])
    idx = np.empty_like(ref["idx"])
    seen = np.zeros(W.T, dtype=bool)
    for r in (0, 1):
        for a, b, o, i in res[r][3]:
            out[a:b] = o
            idx[a:b] = i
            seen[a:b] = True
    assert seen.all()
    assert np.array_equal(idx, ref["idx"])
    assert np.array_equal(out, ref["out"])

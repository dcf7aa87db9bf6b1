"""Data-parallel partition of the QSA hot path over the ranks of a process group (one GPU each).

Prefill: every query row is independent once the full pooled keys kp, K and V are known, so the
rows are sharded.  The causal triangle makes later rows dearer (the indexer scores floor(t/4)
blocks for row t), so the sequence is cut into 2N equal chunks and rank r owns chunks r and
2N-1-r ("zig-zag"): each rank gets one early and one late chunk and the same share of the
triangle.  Each rank pools its own rows' indexer keys, one all-gather per tensor brings every
rank's K, V and kp chunks into full-length buffers on every rank, and the rank then selects and
attends for its own rows only.  Outputs stay row-sharded: rank r holds the output rows of its two
chunks.  No other exchange is needed.

Decode: sequences are independent, so the batch is split into contiguous ranges; there is no
collective at all.

This module holds the partition logic and the exchange (torch.distributed, NCCL on GPUs, gloo in
the CPU tests); the per-rank compute goes through the C ABI (``qsa``).  No TMA multicast and no
peer memory is involved: every kernel reads only its own GPU's buffers after the all-gather.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def zigzag_chunks(T: int, world: int, align: int = 4) -> list[tuple[int, int]]:
    """The 2*world equal chunks [start, end) of a T-row sequence.  T must be a multiple of
    2 * world * align (so that every chunk starts on a micro-block boundary and the chunks of all
    ranks have one size, as an all-gather needs)."""
    n = 2 * world
    if world < 1 or T % (n * align) != 0:
        raise ValueError(f"T = {T} is not a multiple of 2 * world * align = {n * align}")
    c = T // n
    return [(i * c, (i + 1) * c) for i in range(n)]


def rank_chunks(T: int, world: int, rank: int, align: int = 4) -> list[tuple[int, int]]:
    """Row ranges owned by `rank`: chunk `rank` and chunk 2*world-1-rank, in ascending order."""
    ch = zigzag_chunks(T, world, align)
    if world == 1:
        return [(0, T)]
    return [ch[rank], ch[2 * world - 1 - rank]]


def causal_cost(ranges: list[tuple[int, int]], k: int, blk: int = 4) -> dict:
    """Work of a set of query rows: indexer (query, block) pairs sum floor(t/blk) and attended
    tokens sum |S(t)| = blk * min(floor(t/blk), k) + t mod blk + 1."""
    pairs = 0
    toks = 0
    for a, b in ranges:
        t = torch.arange(a, b, dtype=torch.int64)
        pairs += int((t // blk).sum())
        toks += int((blk * torch.clamp(t // blk, max=k) + t % blk + 1).sum())
    return {"index_pairs": pairs, "attended_tokens": toks}


def batch_range(B: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous sequences [start, end) of the decode batch owned by `rank` (sizes differ by at
    most one)."""
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def _as_bytes(t: torch.Tensor) -> torch.Tensor:
    # bf16 bits travel as bytes: the same bytes on every backend (gloo has no bf16 reductions to
    # care about, and no arithmetic is done on them)
    return t.view(torch.uint8) if t.dtype != torch.uint8 else t


def allgather_rows(local: list[torch.Tensor], full: torch.Tensor, T_rows: int, world: int, rank: int,
                   group=None) -> torch.Tensor:
    """Fill full [B, T_rows, ...] with every rank's row chunks.  `local` holds this rank's two chunks
    (or its whole range when world == 1) as [B, C, ...] tensors in the order of rank_chunks; rows are
    in units of the tensor's own row (tokens for K/V, micro-blocks for kp).  Two all-gathers per
    batch element: the first chunks land in chunks 0..N-1, the second ones in chunks 2N-1..N."""
    if world == 1:
        full.copy_(local[0])
        return full
    C = T_rows // (2 * world)
    assert all(x.shape[1] == C for x in local), "every chunk holds T_rows / (2 * world) rows"
    B = full.shape[0]
    for b in range(B):
        first = [_as_bytes(full[b, i * C:(i + 1) * C]) for i in range(world)]
        second = [_as_bytes(full[b, (2 * world - 1 - i) * C:(2 * world - i) * C]) for i in range(world)]
        dist.all_gather(first, _as_bytes(local[0][b].contiguous()), group=group)
        dist.all_gather(second, _as_bytes(local[1][b].contiguous()), group=group)
    return full


class ShardedPrefill:
    """One rank's share of a row-sharded QSA prefill (B sequences of T tokens).

    Holds the full-length K, V and kp buffers the all-gathers fill and the rank's workspace; call
    ``step`` with this rank's input rows (one [B, C, ...] tensor per owned chunk)."""

    def __init__(self, B: int, T: int, Hq: int, Hkv: int, D: int, Hi: int, Di: int, topk: int, world: int,
                 rank: int, device, blk: int = 4, group=None):
        from . import qsa as Q
        self.Q = Q
        self.B, self.T, self.Hq, self.Hkv, self.D, self.Hi, self.Di = B, T, Hq, Hkv, D, Hi, Di
        self.k, self.blk, self.world, self.rank, self.group = topk, blk, world, rank, group
        self.ranges = rank_chunks(T, world, rank, blk)
        dev = torch.device(device)
        E = Q._empty   # torch.empty, with canary guards in debug mode
        self.kfull = E(B, T, Hkv, D, dtype=torch.bfloat16, device=dev, what="gathered k")
        self.vfull = E(B, T, Hkv, D, dtype=torch.bfloat16, device=dev, what="gathered v")
        self.kpfull = E(B, T // blk, Di, dtype=torch.bfloat16, device=dev, what="gathered kp")
        self.kp_local = [E(B, (b - a) // blk, Di, dtype=torch.bfloat16, device=dev, what="local kp")
                         for a, b in self.ranges]
        rows = max(b - a for a, b in self.ranges)
        ws = Q.qsa_workspace_size(Q.QSA_OP_SELECT_TOPK, B, rows, T // blk, topk, Hq, D)
        self.ws = E(ws, dtype=torch.uint8, device=dev, what="select workspace")
        aws = Q.qsa_attn_prefill_workspace_size(B, rows, T, Hq, Hkv, D, topk)
        self.attn_ws = E(max(aws, 16), dtype=torch.uint8, device=dev, what="attention workspace")
        self.idx = [E(B, b - a, topk, dtype=torch.int32, device=dev, what="idx") for a, b in self.ranges]
        self.out = [E(B, b - a, Hq, D, dtype=torch.bfloat16, device=dev, what="out") for a, b in self.ranges]
        self.lse = [E(B, b - a, Hq, dtype=torch.float32, device=dev, what="lse") for a, b in self.ranges]

    def pool_local(self, ki: list):
        """Pool this rank's indexer keys, each chunk at its own positions."""
        for (a, _), ki_c, kp_c in zip(self.ranges, ki, self.kp_local):
            self.Q.qsa_pool_block_keys(ki_c, kp_c, pos0=a)

    def exchange(self, k: list, v: list):
        """The one exchange step: every rank's kp, K and V chunks into the full-length buffers."""
        allgather_rows(self.kp_local, self.kpfull, self.T // self.blk, self.world, self.rank, self.group)
        allgather_rows(k, self.kfull, self.T, self.world, self.rank, self.group)
        allgather_rows(v, self.vfull, self.T, self.world, self.rank, self.group)

    def compute(self, q: list, qi: list, events=None):
        """Selection and attention of this rank's rows over the full buffers (local kernels only).
        With `events` (two CUDA events per chunk) the selection and attention are bracketed."""
        Q = self.Q
        for i, (a, _) in enumerate(self.ranges):
            Q.qsa_select_topk(self.k, qi=qi[i], kp=self.kpfull, q_pos0=a, idx=self.idx[i], workspace=self.ws)
            if events:
                events[2 * i].record()
            Q.qsa_sparse_attn_prefill(q[i], self.kfull, self.vfull, self.idx[i], q_pos0=a, out=self.out[i],
                                      lse=self.lse[i], workspace=self.attn_ws)
            if events:
                events[2 * i + 1].record()
        return self.out, self.lse, self.idx

    def step(self, q: list, k: list, v: list, qi: list, ki: list):
        """q/k/v/qi/ki: this rank's chunks ([B, C, ...] each, in the order of ``self.ranges``).
        Returns (out chunks, lse chunks, idx chunks) for this rank's rows."""
        self.pool_local(ki)
        self.exchange(k, v)
        return self.compute(q, qi)

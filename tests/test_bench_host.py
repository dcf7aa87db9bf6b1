"""Host logic of bench.py: the algorithmic work counts behind the roofline numbers, the launch
count, and the multi-rank timing reduction (world size 2 over gloo on CPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
from hybrid_sparse_attention_qsa_b200 import inputs as I


def test_tokens_attended_closed_form():
    S = bench.tokens_attended(20, 2)
    # t < 8: every earlier complete block plus the own block; later: 2 blocks + own block
    expect = [4 * min(t // 4, 2) + t % 4 + 1 for t in range(20)]
    assert S.tolist() == expect
    assert bench.tokens_attended(3000, 512).max() == 2048 + 4


def test_prefill_work_matches_the_workload_arithmetic():
    w = I.WORKLOADS["prefill_128k"]
    work = bench.prefill_work(w)
    # indexer: 2*Hi*Di = 512 flop per causally visible (query, block) pair
    pairs = sum(t // 4 for t in range(w.T))
    assert work["index_flops"] == 512 * pairs
    assert abs(work["index_flops"] - 1.10e12) / 1.10e12 < 0.01
    # gathered K/V: ~274 GB at 128K (4 bytes per element pair of K and V, 2 KV heads, D = 128)
    gathered = work["attn_bytes"] - w.T * w.Hq * w.D * 4
    assert abs(gathered - 274.1e9) / 274.1e9 < 0.01


def test_decode_work():
    w = I.WORKLOADS["decode_256k"]
    d = bench.decode_work(w)
    assert d["kp_bytes"] == 32 * 65535 * 64 * 2
    assert d["gathered"] == 32 * 2052 * 2 * 128 * 2 * 2
    assert abs(d["bytes"] - 335.9e6) / 335.9e6 < 0.01


def test_select_launch_count():
    w = I.WORKLOADS["prefill_128k"]
    nbk = w.T // 4
    # a workspace too small for the filtered path (under 4096 rows of lists): 164 chunks of 800
    # score rows -> 164 score + 164 top-k launches
    assert bench.select_launches(w, nbk * 4 * 800) == 328
    # the first chunk of a 1-row workspace holds rows 0..0: no candidate, no score launch
    tiny = w.with_(T=12)
    assert bench.select_launches(tiny, 3 * 4) == 12 + 12 - 4
    # the size the library asks for: the filtered path in one chunk, five launches
    from hybrid_sparse_attention_qsa_b200 import qsa as Q
    ws = Q.qsa_workspace_size(Q.QSA_OP_SELECT_TOPK, w.B, w.T, nbk, w.k, w.Hq, w.D)
    assert bench.select_launches(w, ws) == 5
    # short sequences stay on the materialised path
    short = w.with_(T=8192)
    ws = Q.qsa_workspace_size(Q.QSA_OP_SELECT_TOPK, 1, short.T, short.T // 4, short.k, 16, 128)
    assert bench.select_launches(short, ws) == 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.max_over_ranks(10.0 + rank, world, "cpu")
        bench.barrier(world)
        q.put((rank, mx))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_world_size_2_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 11.0, 1: 11.0}
    assert all(p.exitcode == 0 for p in procs)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON line with the keys
    the measurement contract names; runs without a GPU."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1", "--ref-rows", "4"], capture_output=True, text=True, timeout=240, cwd=root)
    assert out.returncode == 0, out.stderr[-500:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["config"]["workload"] == "prefill_128k"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0

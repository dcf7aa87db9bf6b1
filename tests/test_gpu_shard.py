"""The row-sharded prefill's per-rank compute on the GPU.

One GPU runs the two ranks of a world-size-2 partition one after the other; the all-gather is
stood in for by copying every rank's chunks into every rank's full-length buffers (the exchange
itself is covered by the two-rank gloo test in tests/test_shard.py).  The ranks' rows, put back
in order, must equal the unsharded prefill: the same pooled keys bit for bit, the same lists, and
bit-identical outputs wherever the lists agree.
"""
import numpy as np
import pytest
import torch

from hybrid_sparse_attention_qsa_b200 import inputs as I
from hybrid_sparse_attention_qsa_b200 import qsa as Q
from hybrid_sparse_attention_qsa_b200 import shard as S
from tests import harness as H

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("T,world", [(16384, 2), (20480, 4)])
def test_sharded_ranks_on_one_gpu_equal_the_unsharded_prefill(T, world):
    w = I.WORKLOADS["prefill_32k"].with_(T=T, seed=9 + world)
    x = I.make_prefill(w, DEV)
    full = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=w.k)
    parts = [S.ShardedPrefill(w.B, w.T, w.Hq, w.Hkv, w.D, w.Hi, w.Di, w.k, world, r, DEV) for r in range(world)]
    mine = [{n: [x[n][:, a:b].contiguous() for a, b in p.ranges] for n in x} for p in parts]
    for p, m in zip(parts, mine):
        p.pool_local(m["ki"])
    for p in parts:   # the all-gather, stood in for on one GPU
        for src, m in zip(parts, mine):
            for (a, b), kc, vc, kpc in zip(src.ranges, m["k"], m["v"], src.kp_local):
                p.kfull[:, a:b] = kc
                p.vfull[:, a:b] = vc
                p.kpfull[:, a // 4:b // 4] = kpc
    torch.cuda.synchronize()
    assert torch.equal(parts[0].kpfull, full["kp"])
    seen = np.zeros(T, dtype=bool)
    differ = 0
    for p, m in zip(parts, mine):
        out, lse, idx = p.compute(m["q"], m["qi"])
        torch.cuda.synchronize()
        assert Q.qsa_get_device_status() == Q.QSA_OK
        for (a, b), o, l, i in zip(p.ranges, out, lse, idx):
            seen[a:b] = True
            same = (i[0] == full["idx"][0, a:b]).all(dim=1)
            differ += int((~same).sum())
            rows = torch.nonzero(same).flatten()
            assert torch.equal(o[0, rows], full["out"][0, a:b][rows]), "outputs differ on identical lists"
            assert torch.equal(l[0, rows], full["lse"][0, a:b][rows])
            bad = torch.nonzero(~same).flatten().tolist()
            if bad:   # rows whose selection took another path (last-bit ties): the oracle's tie rule
                pos = [a + r for r in bad]
                h = {n: I.bits(x[n])[0] for n in ("q", "k", "v", "qi")}
                H.compare_prefill(i[0, bad].cpu().numpy(), I.bits(o[0, bad]), l[0, bad].cpu().numpy(), h["q"][pos],
                                  h["qi"][pos], h["k"], h["v"], I.bits(full["kp"])[0], pos, topk=w.k)
    assert seen.all()
    assert differ <= T // 1000


def test_zigzag_needs_aligned_chunks_on_the_gpu_path():
    with pytest.raises(ValueError):
        S.ShardedPrefill(1, 1000, 16, 2, 128, 4, 64, 512, 2, 0, DEV)

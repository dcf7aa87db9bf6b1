"""The allocation-free decode entry point, qsa_sparse_attn_decode_noalloc.

Some callers cannot allocate device memory for a workspace: code running while a stream is being
captured into a CUDA graph (cudaMalloc is not allowed there), plugins of inference engines whose
memory planner owns the whole device heap, and hosts with a fixed device budget.  This entry point
keeps the split-KV partials in the library's own per-GPU scratch array instead.  The tests call it
through the C ABI, twice in a row, and check it against the workspace entry point and the CPU
oracle: once where the splits merge inside thread-block clusters (the array is not used) and on
shapes where they merge through partials (the array holds them, and the second call reads what it
wrote over the first call's contents).  This file is collected last on purpose; it also passes
alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from hybrid_sparse_attention_qsa_b200 import inputs as I
from hybrid_sparse_attention_qsa_b200 import qsa as Q
from tests import harness as H
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(B, L, seqlens, k, seed, **shape):
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=seed, k=k, **shape)
    x = I.make_decode(w, DEV, seqlens=seqlens)
    kp = Q.qsa_pool_block_keys(x["ki"])
    idx = Q.qsa_select_topk(k, qi=x["qi"], kp=kp, seqlens=x["seqlens"])
    return x, kp, idx


def _twice_against_workspace_and_oracle(x, kp, idx, splits, k, merge):
    B, Hq, D = x["q"].shape
    Hkv = x["k"].shape[2]
    used = splits or Q.qsa_decode_default_splits(B, k)
    assert Q.qsa_decode_split_merge(B, Hq, Hkv, D, used) == merge
    ref_out, ref_lse = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=used)
    seqs = list(range(B))
    hb = {n: I.bits(x[n]) for n in ("q", "k", "v", "qi")}
    for call in range(2):
        out = torch.full_like(x["q"], float("nan"))
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=DEV)
        Q.qsa_sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=splits, out=out,
                                         lse=lse)
        torch.cuda.synchronize()
        assert Q.qsa_get_device_status() == Q.QSA_OK
        P.assert_outputs_close(I.bits(out), I.bits(ref_out))
        assert torch.allclose(lse, ref_lse, atol=1e-4, rtol=0), f"call {call}"
        H.compare_decode(idx.cpu().numpy(), I.bits(out), lse.cpu().numpy(), hb["q"], hb["k"], hb["v"], hb["qi"],
                         I.bits(kp), x["seqlens"].cpu().numpy(), seqs, topk=k)


def test_noalloc_decode_cluster_merge_twice():
    # 6 sequences x the default 8 splits: merged inside clusters, the scratch array is not touched
    x, kp, idx = _case(6, 12000, [12000, 9001, 4096, 2051, 777, 5], 256, 71)
    _twice_against_workspace_and_oracle(x, kp, idx, 0, 256, merge=1)


@pytest.mark.parametrize("B,splits", [(6, 12), (24, 7)])
def test_noalloc_decode_partials_in_scratch_twice(B, splits):
    # 12 splits (more than a cluster merges) or 24 x 7 = 168 items (more than one per SM): the
    # partials go through the scratch array and the merge kernel
    lens = [12000 - 11000 * i // B for i in range(B)]
    lens[-1] = 5
    x, kp, idx = _case(B, 12000, lens, 256, 72 + B)
    _twice_against_workspace_and_oracle(x, kp, idx, splits, 256, merge=2)


def test_noalloc_decode_model_shape_partials_twice():
    # 24 query heads over 2 KV heads at head dimension 256: merged through the scratch array
    x, kp, idx = _case(3, 9000, [9000, 4099, 2050], 128, 73, Hq=24, D=256)
    _twice_against_workspace_and_oracle(x, kp, idx, 4, 128, merge=2)


def test_noalloc_decode_rejects_splits_beyond_the_scratch_array():
    # 8 sequences x 16 heads x (128 + 2) floats = 66560 bytes a split: 63 splits fit in 4 MiB; 64
    # (no more than the 512 listed blocks, so the call would really use them) do not
    x, _, idx = _case(8, 3000, None, 512, 74)
    per_split = 8 * 16 * (128 + 2) * 4
    n = (4 << 20) // per_split + 1
    assert n == 64
    with pytest.raises(Q.QSAError) as e:
        Q.qsa_sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=n)
    assert e.value.status == Q.QSA_ERR_WORKSPACE_TOO_SMALL
    out = torch.empty_like(x["q"])
    Q.qsa_sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=n - 1, out=out)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK

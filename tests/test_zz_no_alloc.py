"""The allocation-free decode entry point, qsa_sparse_attn_decode_noalloc.

Callers that cannot allocate device memory (a stream being captured into a CUDA graph, an engine
plugin whose memory planner owns the device heap, a host with a fixed device budget) cannot pass a
workspace, so this entry point keeps the split-KV partials in the library's own per-GPU scratch
array.  The test checks, through the C ABI, that two calls in a row give the same answer as the
workspace entry point within the parity tolerance (the second call reuses the array as the first
left it).  This file is collected last on purpose; it also passes alone in a fresh process.
"""
import math

import numpy as np
import pytest
import torch

from hybrid_sparse_attention_qsa_b200 import inputs as I
from hybrid_sparse_attention_qsa_b200 import qsa as Q
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(B, L, seqlens, k, seed):
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=seed, k=k)
    x = I.make_decode(w, DEV, seqlens=seqlens)
    kp = Q.qsa_pool_block_keys(x["ki"])
    idx = Q.qsa_select_topk(k, qi=x["qi"], kp=kp, seqlens=x["seqlens"])
    return x, idx


@pytest.mark.parametrize("splits", [0, 5])
def test_noalloc_decode_matches_workspace_decode_twice(splits):
    x, idx = _case(6, 12000, [12000, 9001, 4096, 2051, 777, 5], 256, 71)
    ref_out, ref_lse = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=splits or 4)
    for _ in range(2):
        out = torch.full_like(x["q"], float("nan"))
        lse = torch.full((6, 16), float("nan"), dtype=torch.float32, device=DEV)
        Q.qsa_sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=splits, out=out,
                                         lse=lse)
        torch.cuda.synchronize()
        assert Q.qsa_get_device_status() == Q.QSA_OK
        P.assert_outputs_close(I.bits(out), I.bits(ref_out))
        assert torch.allclose(lse, ref_lse, atol=1e-4, rtol=0)


def test_noalloc_decode_rejects_splits_beyond_the_scratch_array():
    x, idx = _case(2, 3000, None, 64, 72)
    per_split = 2 * 16 * (128 + 2) * 4
    n = (4 << 20) // per_split + 1
    with pytest.raises(Q.QSAError) as e:
        Q.qsa_sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=n)
    assert e.value.status == Q.QSA_ERR_WORKSPACE_TOO_SMALL

"""GPU: the wide sparse-attention kernel (head dimension 256 and GQA groups of 9 to 16 heads: the
model shape of the pages, 24 query heads over 2 KV heads at head dimension 256) against the oracle.
Same bars as the main parity tests: exact selection up to the tie rule, bf16 outputs within the
max-abs / mean-abs tolerances, and the invariants (poisoned unselected K/V, decode split counts)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from hybrid_sparse_attention_qsa_b200 import inputs as I
from hybrid_sparse_attention_qsa_b200 import qsa as Q
from tests import harness as H
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _prefill(T, Hq, Hkv, D, seed, Hi=4):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    rb = lambda shape, d: (torch.randn(shape, generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16)
    return dict(q=rb((1, T, Hq, D), D), k=rb((1, T, Hkv, D), D), v=rb((1, T, Hkv, D), D),
                qi=rb((1, T, Hi, 64), 64), ki=rb((1, T, 64), 64))


@pytest.mark.parametrize("T,Hq,Hkv,D,k", [(2100, 24, 2, 256, 64), (1700, 8, 1, 256, 100), (2000, 24, 2, 128, 64),
                                          (1500, 16, 2, 256, 32), (300, 12, 1, 256, 512), (2600, 10, 1, 128, 40)])
def test_wide_attention_with_oracle_index_lists(T, Hq, Hkv, D, k):
    x = _prefill(T, Hq, Hkv, D, T + Hq + D)
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"])
    rows = list(range(T)) if T <= 400 else H.sample_rows(T, k, n_random=60, seed=D)
    ora = O.prefill_rows(h["q"], h["k"], h["v"], h["qi"], kp, [(0, t) for t in range(T)], topk=k)
    idx = torch.from_numpy(ora["idx"]).to(DEV).view(1, T, k)
    out, lse = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    got = I.bits(out)[0]
    P.assert_outputs_close(got[rows], ora["out"][rows])
    assert np.abs(lse.cpu().numpy()[0][rows] - ora["lse"][rows]).max() <= 1e-2


def test_model_shape_whole_layer_sampled_rows():
    """24 query heads, 2 KV heads, head dimension 256, the 4 x 64 indexer, k = 512 at 6000 tokens."""
    T, k = 6000, 512
    x = _prefill(T, 24, 2, 256, 2024)
    res = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=k)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"])
    assert np.array_equal(I.bits(res["kp"]), kp)
    rows = H.sample_rows(T, k, n_random=30, seed=7)
    st = H.compare_prefill(res["idx"].cpu().numpy()[0][rows], I.bits(res["out"])[0][rows],
                           res["lse"].cpu().numpy()[0][rows], h["q"][0][rows], h["qi"][0][rows], h["k"][0], h["v"][0],
                           kp[0], rows, topk=k)
    print("model shape:", st)


def test_wide_unselected_tokens_poisoned_with_nan_do_not_matter():
    T, k, q0 = 3000, 8, 2990
    x = _prefill(T, 24, 2, 256, 66)
    qc, qic = x["q"][:, q0:].contiguous(), x["qi"][:, q0:].contiguous()
    res = Q.prefill(qc, x["k"], x["v"], qic, x["ki"], topk=k, q_pos0=q0)
    idx = res["idx"].cpu().numpy()[0]
    used = np.zeros(T, bool)
    used[q0 // 4 * 4:] = True
    for b in np.unique(idx[idx >= 0]):
        used[4 * b:4 * b + 4] = True
    assert not used.all()
    k2, v2 = x["k"].clone(), x["v"].clone()
    bad = torch.from_numpy(~used).to(DEV)
    k2[0, bad] = float("nan")
    v2[0, bad] = float("nan")
    out2, lse2 = Q.qsa_sparse_attn_prefill(qc, k2, v2, res["idx"], q_pos0=q0)
    assert torch.equal(out2, res["out"]) and torch.equal(lse2, res["lse"])


def test_wide_decode_matches_oracle_and_is_split_invariant():
    B, L, k = 5, 9000, 512
    seqlens = [1, 9, 2053, 6000, 9000]
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=91, Hq=24, D=256)
    x = I.make_decode(w, DEV, seqlens=seqlens)
    kp = Q.qsa_pool_block_keys(x["ki"])
    outs = []
    for splits in (1, 3, 8):
        res = Q.decode(x["q"], x["k"], x["v"], x["qi"], kp, x["seqlens"], topk=k, num_splits=splits)
        torch.cuda.synchronize()
        assert Q.qsa_get_device_status() == Q.QSA_OK
        outs.append(res)
    h = {n: I.bits(x[n]) for n in ("q", "k", "v", "qi")}
    st = H.compare_decode(outs[0]["idx"].cpu().numpy(), I.bits(outs[0]["out"]), outs[0]["lse"].cpu().numpy(), h["q"],
                          h["k"], h["v"], h["qi"], I.bits(kp), np.array(seqlens), list(range(B)), topk=k)
    print("wide decode:", st)
    for r in outs[1:]:
        assert torch.equal(r["idx"], outs[0]["idx"])
        P.assert_outputs_close(I.bits(r["out"]), I.bits(outs[0]["out"]))

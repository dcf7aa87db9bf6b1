"""GPU: the decode selection with a thread-block cluster of CTAs per sequence against the
one-CTA-per-sequence top-k over the same scores, and against the oracle.

Both decode selections take the top-k of the same fp32 scores written by the decode score kernel
(qsa_index_score then qsa_select_topk from scores: one CTA per row; qsa_select_topk from qi/kp:
the cluster kernel when there are 2 or more SMs per sequence), so their index lists must be
identical; the oracle's lists agree under the tie rule."""
import numpy as np
import pytest
import torch

import oracle as O
from hybrid_sparse_attention_qsa_b200 import inputs as I
from hybrid_sparse_attention_qsa_b200 import qsa as Q
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(B, nbk, seed, Hi=4):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    qi = (torch.randn((B, Hi, 64), generator=g, device=DEV) * 0.125).to(torch.bfloat16)
    kp = (torch.randn((B, nbk, 64), generator=g, device=DEV) * 0.125).to(torch.bfloat16)
    return qi, kp


def _select(qi, kp, seqlens, k, cluster, **kw):
    """cluster=True: scores and top-k in one call (the cluster top-k for few sequences);
    cluster=False: the same scores materialised, then the one-CTA-per-row top-k."""
    if cluster:
        idx = Q.qsa_select_topk(k, qi=qi, kp=kp, seqlens=seqlens, **kw)
    else:
        sc = Q.qsa_index_score(qi, kp, seqlens=seqlens, **kw)
        idx = Q.qsa_select_topk(k, scores=sc, NBk=kp.shape[1], seqlens=seqlens)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    return idx.cpu().numpy()


def _oracle_rows(idx, qi, kp, seqlens, k, rows, head_w=None, mode=0):
    qh, kph = I.bits(qi), I.bits(kp)
    wh = None if head_w is None else head_w.cpu().numpy()
    ora, kth, srows, nb = [], [], {}, []
    for i, b in enumerate(rows):
        n = (int(seqlens[b]) - 1) // 4
        s = O.index_scores(qh[b], kph[b], n, head_w=wh, mode=mode)
        ri, rk = O.select_topk(s, k)
        ora.append(ri)
        kth.append(rk)
        srows[i] = s
        nb.append(n)
    got = idx[rows]
    assert P.check_index_rows(got, np.array(nb), k) == []
    res = P.compare_selection(got, np.array(ora), np.array(kth), lambda i: srows[i])
    assert res["bad"] == [], res["bad"][:3]


def test_cluster_equals_one_cta_on_the_256k_shape():
    """32 sequences of 262144 tokens (65536 blocks), k = 512: the bench's decode shape (clusters
    of 4 CTAs on 148 SMs)."""
    B, L, k = 32, 262144, 512
    qi, kp = _case(B, L // 4, 3)
    seqlens = torch.full((B,), L, dtype=torch.int32, device=DEV)
    one = _select(qi, kp, seqlens, k, cluster=False)
    two = _select(qi, kp, seqlens, k, cluster=True)
    assert np.array_equal(one, two)
    _oracle_rows(two, qi, kp, seqlens.cpu().numpy(), k, [0, 17, 31])


@pytest.mark.parametrize("B,k", [(1, 512), (7, 512), (5, 1000), (12, 64), (40, 1024), (9, 1)])
def test_cluster_equals_one_cta_with_ragged_lengths(B, k):
    """Lengths below k blocks, at the keep-every-block limit (6144 blocks), just above it, and
    long, with clusters of 8 (B <= 18), 3 (B = 40) and 2 CTAs; linear scores with head weights."""
    nbk = 70000
    qi, kp = _case(B, nbk, 100 + B)
    lens = [4 * nbk, 1, 5, 4 * k + 1, 4 * 6144 + 1, 4 * 6145 + 3, 100003, 4 * 40000 + 2, 4 * nbk - 1]
    seqlens = torch.tensor([lens[b % len(lens)] for b in range(B)], dtype=torch.int32, device=DEV)
    w = torch.linspace(0.5, 1.5, 4, device=DEV)
    one = _select(qi, kp, seqlens, k, cluster=False, head_w=w, mode=1)
    two = _select(qi, kp, seqlens, k, cluster=True, head_w=w, mode=1)
    assert np.array_equal(one, two)
    _oracle_rows(two, qi, kp, seqlens.cpu().numpy(), k, list(range(min(B, 9))), head_w=w, mode=1)


def test_long_rows_take_several_rounds_per_slice():
    """1M-token caches (262144 blocks): two sequences, clusters of 8, slices of 32768 scores, i.e.
    two rounds of loads per CTA; k = 1024 as in the 1M workload."""
    B, nbk, k = 2, 262144, 1024
    qi, kp = _case(B, nbk, 44)
    seqlens = torch.tensor([4 * nbk, 4 * 150001 + 3], dtype=torch.int32, device=DEV)
    one = _select(qi, kp, seqlens, k, cluster=False)
    two = _select(qi, kp, seqlens, k, cluster=True)
    assert np.array_equal(one, two)
    _oracle_rows(two, qi, kp, seqlens.cpu().numpy(), k, [0, 1])


def test_heavy_ties_go_to_the_lowest_blocks():
    """A zero query scores every block 0: the slices' lists overflow (long row) or together exceed
    the merged capacity (shorter row), and CTA 0 selects over the row in memory: blocks 0 .. k-1."""
    B, nbk, k = 4, 65536, 512
    qi, kp = _case(B, nbk, 21)
    qi[1] = 0
    qi[2] = 0
    seqlens = torch.tensor([4 * nbk, 4 * nbk, 4 * 20000 + 1, 4 * nbk - 7], dtype=torch.int32, device=DEV)
    one = _select(qi, kp, seqlens, k, cluster=False)
    two = _select(qi, kp, seqlens, k, cluster=True)
    assert np.array_equal(one, two)
    assert np.array_equal(two[1], np.arange(k, dtype=np.int32))
    assert np.array_equal(two[2], np.arange(k, dtype=np.int32))


def test_coarse_scores_with_ties_at_the_kth():
    """Scores on a coarse grid (the indexer keys quantised), so many blocks tie at the k-th score
    and the lower block indices must win among them."""
    B, nbk, k = 6, 65536, 512
    qi, kp = _case(B, nbk, 8)
    kp = (kp.float() * 8).round().div(8).to(torch.bfloat16)
    qi = (qi.float() * 4).round().div(4).to(torch.bfloat16)
    seqlens = torch.full((B,), 4 * nbk, dtype=torch.int32, device=DEV)
    one = _select(qi, kp, seqlens, k, cluster=False)
    two = _select(qi, kp, seqlens, k, cluster=True)
    assert np.array_equal(one, two)


# ------------------------------------------------------------------ split-KV merge inside a cluster
@pytest.mark.parametrize("B,L,k", [(32, 65536, 512), (3, 20000, 512), (12, 9001, 100)])
def test_cluster_split_merge_matches_the_merge_kernel_and_the_oracle(B, L, k):
    """With B * splits <= SMs the splits of a sequence run as a cluster and merge through
    distributed shared memory; with more items they write partials that a second kernel merges.
    Both (and one split) against each other and against the oracle's attention over the same
    index lists, with ragged lengths (the split holding the own block, empty splits)."""
    from tests import harness as H
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=B + L)
    lens = [L, L - 1, 4 * k + 3, 17, L - 100, 1]
    seqlens = [lens[b % len(lens)] for b in range(B)]
    x = I.make_decode(w, DEV, seqlens=seqlens)
    kp = Q.qsa_pool_block_keys(x["ki"])
    idx = Q.qsa_select_topk(k, qi=x["qi"], kp=kp, seqlens=x["seqlens"])
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    many = sms // B + 1   # B * many > SMs: partials + merge kernel
    assert Q.lib().qsa_decode_split_merge(B, 16, 2, 128, 2) == 1
    assert Q.lib().qsa_decode_split_merge(B, 16, 2, 128, many) == 2
    outs = {}
    for sp in (1, 2, max(2, min(8, sms // B)), many):
        o, l = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=sp)
        torch.cuda.synchronize()
        assert Q.qsa_get_device_status() == Q.QSA_OK
        outs[sp] = (I.bits(o), l.cpu().numpy())
    ref = outs[1]
    for sp, (o, l) in outs.items():
        P.assert_outputs_close(o, ref[0])
        assert np.allclose(l, ref[1], atol=1e-4), sp
    h = {n: I.bits(x[n]) for n in ("q", "k", "v", "qi")}
    seqs = list(range(min(B, 6)))
    sp = max(2, min(8, sms // B))
    st = H.compare_decode(idx.cpu().numpy()[seqs], outs[sp][0][seqs], outs[sp][1][seqs], h["q"], h["k"], h["v"],
                          h["qi"], I.bits(kp), np.array(seqlens), seqs, topk=k)
    print("cluster decode:", st)


def test_cluster_split_merge_one_kv_head_and_clusters_of_eight():
    """Hkv = 1 (8 query heads on one KV head) with 8 splits per sequence (clusters of 8 CTAs) and
    Hkv = 2 with 3 splits, against one split and the oracle."""
    from tests import harness as H
    for Hq, Hkv, B, splits in [(8, 1, 5, 8), (16, 2, 7, 3)]:
        w = I.WORKLOADS["decode_256k"].with_(B=B, T=12000, Hq=Hq, Hkv=Hkv, seed=Hq * 100 + B)
        seqlens = [12000, 9001, 4 * 300 + 2, 12000 - 3, 33, 6000, 7777][:B]
        x = I.make_decode(w, DEV, seqlens=seqlens)
        kp = Q.qsa_pool_block_keys(x["ki"])
        idx = Q.qsa_select_topk(256, qi=x["qi"], kp=kp, seqlens=x["seqlens"])
        assert Q.lib().qsa_decode_split_merge(B, Hq, Hkv, 128, splits) == 1
        o1, l1 = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=1)
        oc, lc = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=splits)
        torch.cuda.synchronize()
        assert Q.qsa_get_device_status() == Q.QSA_OK
        P.assert_outputs_close(I.bits(oc), I.bits(o1))
        assert torch.allclose(lc, l1, atol=1e-4)
        h = {n: I.bits(x[n]) for n in ("q", "k", "v", "qi")}
        H.compare_decode(idx.cpu().numpy(), I.bits(oc), lc.cpu().numpy(), h["q"], h["k"], h["v"], h["qi"], I.bits(kp),
                         np.array(seqlens), list(range(B)), topk=256)


def test_cluster_split_merge_reports_a_bad_length_and_finishes():
    """A sequence length of 0 (no query position) in a cluster launch: its items record
    INVALID_ARGUMENT and attend to nothing, every CTA still passes both cluster barriers, the
    other sequences are unaffected."""
    B, L, k = 6, 8000, 128
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=3)
    seqlens = [L, 5000, 0, L, 1, 7000]
    x = I.make_decode(w, DEV, seqlens=seqlens)
    kp = Q.qsa_pool_block_keys(x["ki"])
    good = torch.tensor([L, 5000, 1, L, 1, 7000], dtype=torch.int32, device=DEV)
    idx = Q.qsa_select_topk(k, qi=x["qi"], kp=kp, seqlens=good)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert Q.lib().qsa_decode_split_merge(B, 16, 2, 128, 4) == 1
    ref, _ = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], good, idx, num_splits=4)
    out, _ = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seqlens"], idx, num_splits=4)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_ERR_INVALID_ARGUMENT
    keep = [0, 1, 3, 4, 5]
    assert torch.equal(out[keep], ref[keep])
    assert torch.isfinite(out.float()).all()
    assert Q.qsa_get_device_status() == Q.QSA_OK



# ------------------------------------------------------------------ pooling folded into the selection
@pytest.mark.parametrize("rope", [None, dict(theta=10000.0), dict(theta=10000.0, yarn=dict(factor=4.0, orig_ctx=4096))])
def test_decode_select_pools_the_newest_block(rope):
    """qsa_decode_select = pooling of the block the new token completes (bit-exact with
    qsa_pool_block_keys) + the decode selection over the updated pooled keys (identical lists)."""
    B, L, k = 6, 30000, 512
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=55)
    seqlens = [L, L - 1, 4 * 5000, 4 * 5000 + 3, 8, 4 * 7000]   # multiples of 4 complete a block
    x = I.make_decode(w, DEV, seqlens=seqlens)
    theta = rope["theta"] if rope else 0.0
    yarn = rope.get("yarn") if rope else None
    kp_full = Q.qsa_pool_block_keys(x["ki"], rope_theta=theta, yarn=yarn)
    kp = kp_full.clone()
    done = [b for b, n in enumerate(seqlens) if n % 4 == 0]
    for b in done:
        kp[b, seqlens[b] // 4 - 1] = 0       # the block each completing token finishes: not yet pooled
    qi = x["qi"] if theta == 0 else Q.qsa_rope_index_queries(x["qi"], rope_theta=theta, seqlens=x["seqlens"],
                                                             yarn=yarn)
    ref = Q.qsa_select_topk(k, qi=qi, kp=kp_full, seqlens=x["seqlens"])
    got = Q.qsa_decode_select(k, qi=qi, kp=kp, ki=x["ki"], seqlens=x["seqlens"], rope_theta=theta, yarn=yarn)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert torch.equal(kp, kp_full)          # every completed block pooled, nothing else touched
    assert torch.equal(got, ref)


def test_many_sequences_take_one_cta_each():
    """80 sequences on 148 SMs: fewer than 2 SMs per sequence, so the decode selection runs one CTA
    per sequence (no cluster) and the split merge a merge kernel or one split; the pooling-folded
    entry point gives the same lists; the oracle agrees on sampled sequences."""
    B, L, k = 80, 24000, 256
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert sms // B < 2
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=80)
    seqlens = [L - (b * 37) % 5000 for b in range(B)]
    x = I.make_decode(w, DEV, seqlens=seqlens)
    kp_full = Q.qsa_pool_block_keys(x["ki"])
    one = _select(x["qi"], kp_full, x["seqlens"], k, cluster=False)
    two = _select(x["qi"], kp_full, x["seqlens"], k, cluster=True)
    assert np.array_equal(one, two)
    kp = kp_full.clone()
    for b, n in enumerate(seqlens):
        if n % 4 == 0:
            kp[b, n // 4 - 1] = 0
    got = Q.qsa_decode_select(k, qi=x["qi"], kp=kp, ki=x["ki"], seqlens=x["seqlens"])
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert torch.equal(kp, kp_full)
    assert np.array_equal(got.cpu().numpy(), two)
    _oracle_rows(two, x["qi"], kp_full, np.array(seqlens), k, [0, 17, 40, 79])
    out, lse = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seqlens"], got)
    ref, _ = Q.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seqlens"], got, num_splits=1)
    torch.cuda.synchronize()
    P.assert_outputs_close(I.bits(out), I.bits(ref))


def test_cluster_with_unaligned_score_rows():
    """NBk not a multiple of 4: every other sequence's score row starts off a 16-byte boundary, so
    the cluster kernel's sample and slice loads take their scalar form; lists still equal the
    one-CTA selection's and the oracle's."""
    B, nbk, k = 7, 65537, 512
    qi, kp = _case(B, nbk, 71)
    seqlens = torch.tensor([4 * nbk, 4 * nbk - 2, 4 * 40001 + 1, 4 * nbk, 30001, 4 * 6145, 4 * nbk - 5],
                           dtype=torch.int32, device=DEV)
    one = _select(qi, kp, seqlens, k, cluster=False)
    two = _select(qi, kp, seqlens, k, cluster=True)
    assert np.array_equal(one, two)
    _oracle_rows(two, qi, kp, seqlens.cpu().numpy(), k, [0, 1, 6])


def test_decode_select_cache_too_short_is_reported():
    """A length past the pooled-key cache (seqlens[b] / 4 > NBk) is an invalid argument recorded on
    the device; nothing is pooled for it and the other sequences are unaffected."""
    B, L, k = 3, 8000, 128
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=12)
    x = I.make_decode(w, DEV)
    kp_full = Q.qsa_pool_block_keys(x["ki"])
    good = torch.tensor([L, L, L - 4], dtype=torch.int32, device=DEV)
    ref = Q.qsa_select_topk(k, qi=x["qi"], kp=kp_full, seqlens=good)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    bad = torch.tensor([L, L + 400, L - 4], dtype=torch.int32, device=DEV)
    kp = kp_full.clone()
    got = Q.qsa_decode_select(k, qi=x["qi"], kp=kp, ki=x["ki"], seqlens=bad)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_ERR_INVALID_ARGUMENT
    assert torch.equal(kp, kp_full)
    assert torch.equal(got[[0, 2]], ref[[0, 2]])
    assert Q.qsa_get_device_status() == Q.QSA_OK

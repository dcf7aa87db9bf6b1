"""GPU parity: every step of the CUDA path, called through the C ABI, against the CPU oracle on the
same seeded inputs.  Bars: bit-exact for pooled keys and for index lists selected from the same
scores; the tie rule and bf16 output tolerances of tests/parity.py for the whole layer."""
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


def _randn_bf16(shape, scale, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * scale).to(torch.bfloat16)


def _status_ok():
    assert Q.qsa_get_device_status() == Q.QSA_OK


# ------------------------------------------------------------------------------------------ pooling
@pytest.mark.parametrize("B,L,Di", [(1, 4, 64), (2, 1037, 64), (3, 4096, 64), (1, 999, 32)])
def test_pool_bit_exact(B, L, Di):
    ki = _randn_bf16((B, L, Di), Di ** -0.5, L)
    kp = Q.qsa_pool_block_keys(ki)
    torch.cuda.synchronize()
    assert np.array_equal(I.bits(kp), O.pool_block_keys(I.bits(ki)))
    _status_ok()


def test_pool_with_rope_matches_oracle():
    ki = _randn_bf16((2, 4000, 64), 0.125, 7)
    for theta, pos0 in ((10000.0, 0), (500000.0, 123456)):
        kp = I.bits(Q.qsa_pool_block_keys(ki, rope_theta=theta, pos0=pos0))
        ref = O.pool_block_keys(I.bits(ki), rope_theta=theta, pos0=pos0)
        diff = np.abs(O.bf16_to_f64(kp) - O.bf16_to_f64(ref))
        # sin/cos differ from the host libm in the last double bit at most: a 1-ulp bf16 flip is
        # possible only at an exact rounding tie, which is vanishingly rare
        assert (kp != ref).mean() <= 1e-4
        assert np.all(diff <= np.maximum(np.abs(O.bf16_to_f64(ref)), 1e-30) * 2 ** -7)


def test_rope_queries_match_oracle():
    qi = _randn_bf16((2, 300, 4, 64), 0.125, 8)
    out = Q.qsa_rope_index_queries(qi, rope_theta=10000.0, q_pos0=77)
    x = I.bits(qi).reshape(-1, 4, 64)
    pos = np.tile(np.arange(300) + 77, 2)
    ref = O.rope_rows(x, pos, 10000.0).reshape(2, 300, 4, 64)
    assert (I.bits(out) != ref).mean() <= 1e-4
    seqlens = torch.tensor([5, 9000], dtype=torch.int32, device=DEV)
    qd = _randn_bf16((2, 4, 64), 0.125, 9)
    outd = Q.qsa_rope_index_queries(qd, rope_theta=10000.0, seqlens=seqlens)
    refd = O.rope_rows(I.bits(qd), np.array([4, 8999]), 10000.0)
    assert (I.bits(outd) != refd).mean() <= 1e-3


# ------------------------------------------------------------------------------------------ scores
@pytest.mark.parametrize("B,T,Hi,mode,weighted", [(1, 1000, 4, 0, False), (2, 777, 1, 0, False),
                                                  (1, 2500, 4, 1, True), (1, 9000, 4, 0, False),
                                                  (1, 3000, 8, 0, True), (1, 600, 2, 0, False)])
def test_index_score_prefill(B, T, Hi, mode, weighted):
    qi = _randn_bf16((B, T, Hi, 64), 0.125, T + Hi)
    ki = _randn_bf16((B, T, 64), 0.125, T + 1)
    kp = Q.qsa_pool_block_keys(ki)
    w = torch.linspace(0.5, 1.5, Hi, device=DEV) if weighted else None
    s = Q.qsa_index_score(qi, kp, head_w=w, mode=mode).cpu().numpy()
    qh, kph = I.bits(qi), I.bits(kp)
    wh = None if w is None else w.cpu().numpy()
    rows = H.sample_rows(T, 64, n_random=60) if T > 3000 else range(T)
    for b in range(B):
        for t in rows:
            nb = t // 4
            ref = O.index_scores(qh[b, t], kph[b], nb, head_w=wh, mode=mode)
            got = s[b, t, :nb]
            assert np.allclose(got, ref, rtol=1e-5, atol=2e-6), (b, t, np.abs(got - ref).max())
            assert np.all(np.isnan(s[b, t, nb:])), "entries past the candidates must be left untouched"
    _status_ok()


def test_index_score_chunked_window_and_offset():
    """Scores for a chunk of query rows at a position offset (chunked prefill)."""
    T, q0 = 3000, 1700
    qi = _randn_bf16((1, T - q0, 4, 64), 0.125, 31)
    ki = _randn_bf16((1, T, 64), 0.125, 32)
    kp = Q.qsa_pool_block_keys(ki)
    s = Q.qsa_index_score(qi, kp, q_pos0=q0).cpu().numpy()
    qh, kph = I.bits(qi), I.bits(kp)
    for t in range(0, T - q0, 37):
        nb = (q0 + t) // 4
        assert np.allclose(s[0, t, :nb], O.index_scores(qh[0, t], kph[0], nb), rtol=1e-5, atol=2e-6)


def test_index_score_decode():
    B, L = 5, 20001
    qi = _randn_bf16((B, 4, 64), 0.125, 41)
    ki = _randn_bf16((B, L, 64), 0.125, 42)
    kp = Q.qsa_pool_block_keys(ki)
    seqlens = torch.tensor([1, 5, 4096, 17777, 20001], dtype=torch.int32, device=DEV)
    s = Q.qsa_index_score(qi, kp, seqlens=seqlens).cpu().numpy()
    qh, kph = I.bits(qi), I.bits(kp)
    for b in range(B):
        nb = (int(seqlens[b]) - 1) // 4
        assert np.allclose(s[b, 0, :nb], O.index_scores(qh[b], kph[b], nb), rtol=1e-5, atol=2e-6)


# ------------------------------------------------------------------------------------------ top-k
def _topk_case(n_rows, pos0, k, levels, seed):
    """Score rows for query positions pos0 .. pos0+n_rows-1 (candidates floor(p/4)), with ties."""
    nbk = (pos0 + n_rows - 1) // 4
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((1, n_rows, max(nbk, 1))).astype(np.float32)
    if levels:
        s = (np.floor(s * levels) / levels).astype(np.float32)
    s = np.maximum(s, 0).astype(np.float32)
    return s, nbk


@pytest.mark.parametrize("n_rows,pos0,k,levels", [(200, 0, 64, 0), (300, 2000, 512, 0), (64, 40000, 512, 0),
                                                  (64, 40000, 512, 4), (100, 130000, 512, 16), (50, 9000, 1, 0),
                                                  (50, 9000, 1024, 2), (40, 262000, 1024, 0)])
def test_topk_bit_exact_from_scores(n_rows, pos0, k, levels):
    s, nbk = _topk_case(n_rows, pos0, k, levels, n_rows + k)
    st = torch.from_numpy(s).to(DEV)
    idx = Q.qsa_select_topk(k, scores=st, NBk=nbk, q_pos0=pos0).cpu().numpy()
    for r in range(n_rows):
        n = (pos0 + r) // 4
        ref, _ = O.select_topk(s[0, r, :n], k)
        assert np.array_equal(idx[0, r], ref), (r, n)
    _status_ok()


@pytest.mark.parametrize("n_rows,pos0,k,levels", [(1600, 60000, 512, 0), (1300, 40000, 512, 3), (1300, 9000, 64, 2),
                                                  (1200, 3000, 512, 0), (1200, 262000, 1024, 0)])
def test_topk_many_rows_bit_exact(n_rows, pos0, k, levels):
    """Enough rows for the warp-per-row kernel, including heavy ties (threshold retries and the
    in-memory fallback) and rows shorter than k."""
    s, nbk = _topk_case(n_rows, pos0, k, levels, n_rows * 7 + k)
    st = torch.from_numpy(s).to(DEV)
    idx = Q.qsa_select_topk(k, scores=st, NBk=nbk, q_pos0=pos0).cpu().numpy()
    for r in list(range(0, n_rows, 37)) + [n_rows - 1]:
        n = (pos0 + r) // 4
        ref, _ = O.select_topk(s[0, r, :n], k)
        assert np.array_equal(idx[0, r], ref), (r, n)
    _status_ok()


def test_topk_decode_rows_bit_exact():
    B, L, k = 6, 262144, 512
    nbk = L // 4
    rng = np.random.default_rng(5)
    s = np.maximum(rng.standard_normal((B, 1, nbk)), 0).astype(np.float32)
    s[3] = np.floor(s[3] * 3) / 3              # heavy ties
    seqlens = np.array([1, 3000, 65536, 200001, 262144, 262144], dtype=np.int32)
    idx = Q.qsa_select_topk(k, scores=torch.from_numpy(s).to(DEV), NBk=nbk,
                            seqlens=torch.from_numpy(seqlens).to(DEV)).cpu().numpy()
    for b in range(B):
        n = (int(seqlens[b]) - 1) // 4
        ref, _ = O.select_topk(s[b, 0, :n], k)
        assert np.array_equal(idx[b], ref), b


# ------------------------------------------------------------------------------------------ attention
def _small_prefill(T, Hq, Hkv, Hi, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    rb = lambda shape, d: (torch.randn(shape, generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16)
    return dict(q=rb((1, T, Hq, 128), 128), k=rb((1, T, Hkv, 128), 128), v=rb((1, T, Hkv, 128), 128),
                qi=rb((1, T, Hi, 64), 64), ki=rb((1, T, 64), 64))


@pytest.mark.parametrize("T,Hq,Hkv,k", [(2048, 1, 1, 64), (1500, 16, 2, 64), (3001, 8, 2, 100), (700, 4, 1, 3),
                                        (257, 2, 2, 512)])
def test_attention_with_oracle_index_lists(T, Hq, Hkv, k):
    x = _small_prefill(T, Hq, Hkv, 4, T + k)
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"])
    rows = list(range(T))
    ora = O.prefill_rows(h["q"], h["k"], h["v"], h["qi"], kp, [(0, t) for t in rows], topk=k)
    idx = torch.from_numpy(ora["idx"]).to(DEV).view(1, T, k)
    out, lse = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    P.assert_outputs_close(I.bits(out)[0], ora["out"])
    assert np.abs(lse.cpu().numpy()[0] - ora["lse"]).max() <= 1e-2
    _status_ok()


def test_whole_layer_tiny_workload_every_row():
    w = I.WORKLOADS["tiny"]
    x = I.make_prefill(w, DEV)
    res = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=w.k)
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"])
    assert np.array_equal(I.bits(res["kp"]), kp)
    rows = list(range(w.T))
    st = H.compare_prefill(res["idx"].cpu().numpy()[0], I.bits(res["out"])[0], res["lse"].cpu().numpy()[0],
                           h["q"][0], h["qi"][0], h["k"][0], h["v"][0], kp[0], rows, topk=w.k)
    print("tiny:", st)
    _status_ok()


def test_whole_layer_with_rope_and_batches():
    B, T, k, theta = 2, 1800, 40, 10000.0
    x = {n: torch.cat([_small_prefill(T, 16, 2, 4, 100 + b)[n] for b in range(B)]) for n in ("q", "k", "v", "qi", "ki")}
    res = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=k, rope_theta=theta)
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"], rope_theta=theta)
    for b in range(B):
        rows = H.sample_rows(T, k, n_random=40, seed=b)
        st = H.compare_prefill(res["idx"].cpu().numpy()[b][rows], I.bits(res["out"])[b][rows],
                               res["lse"].cpu().numpy()[b][rows], h["q"][b][rows], h["qi"][b][rows], h["k"][b],
                               h["v"][b], kp[b], rows, topk=k, rope_theta=theta)
        print("rope batch", b, st)


YARN = dict(factor=4.0, orig_ctx=262144, alpha=1.0, beta=32.0)


def test_pool_and_query_rope_with_yarn_match_oracle():
    ki = _randn_bf16((2, 4000, 64), 0.125, 71)
    for pos0 in (0, 700000):
        kp = I.bits(Q.qsa_pool_block_keys(ki, rope_theta=10000.0, pos0=pos0, yarn=YARN))
        ref = O.pool_block_keys(I.bits(ki), rope_theta=10000.0, pos0=pos0, yarn=YARN)
        diff = np.abs(O.bf16_to_f64(kp) - O.bf16_to_f64(ref))
        assert (kp != ref).mean() <= 1e-4
        assert np.all(diff <= np.maximum(np.abs(O.bf16_to_f64(ref)), 1e-30) * 2 ** -7)
    qi = _randn_bf16((2, 300, 4, 64), 0.125, 72)
    out = Q.qsa_rope_index_queries(qi, rope_theta=10000.0, q_pos0=900000, yarn=YARN)
    pos = np.tile(np.arange(300) + 900000, 2)
    ref = O.rope_rows(I.bits(qi).reshape(-1, 4, 64), pos, 10000.0, yarn=YARN).reshape(2, 300, 4, 64)
    assert (I.bits(out) != ref).mean() <= 1e-4
    seqlens = torch.tensor([5, 1048576], dtype=torch.int32, device=DEV)
    qd = _randn_bf16((2, 4, 64), 0.125, 73)
    outd = Q.qsa_rope_index_queries(qd, rope_theta=10000.0, seqlens=seqlens, yarn=dict(YARN, mscale=1.25))
    refd = O.rope_rows(I.bits(qd), np.array([4, 1048575]), 10000.0, yarn=dict(YARN, mscale=1.25))
    assert (I.bits(outd) != refd).mean() <= 1e-3
    _status_ok()


def test_whole_layer_with_yarn_rope():
    """Pooled keys and indexer queries rotated with YaRN-scaled frequencies at positions past the
    original context; the oracle gets its own YaRN-rotated keys and queries."""
    T, k, theta, q0 = 2600, 48, 10000.0, 300000
    x = _small_prefill(T, 16, 2, 4, 107)
    y = dict(factor=8.0, orig_ctx=65536)
    qrows = {n: x[n][:, 1000:].contiguous() for n in ("q", "qi")}
    # a window of rows 1000.. of a sequence whose first token sits at position q0
    res_kp = Q.qsa_pool_block_keys(x["ki"], rope_theta=theta, pos0=q0, yarn=y)
    qr = Q.qsa_rope_index_queries(qrows["qi"], rope_theta=theta, q_pos0=q0 + 1000, yarn=y)
    idx = Q.qsa_select_topk(k, qi=qr, kp=res_kp, q_pos0=1000)
    out, lse = Q.qsa_sparse_attn_prefill(qrows["q"], x["k"], x["v"], idx, q_pos0=1000)
    torch.cuda.synchronize()
    _status_ok()
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"], rope_theta=theta, pos0=q0, yarn=y)
    assert (I.bits(res_kp) != kp).mean() <= 1e-3
    rows = [r for r in H.sample_rows(T, k, n_random=30, seed=5) if r >= 1000]
    qi_rot = O.rope_rows(h["qi"][0][rows], np.array(rows) + q0, theta, yarn=y)
    sel = [r - 1000 for r in rows]
    st = H.compare_prefill(idx.cpu().numpy()[0][sel], I.bits(out)[0][sel], lse.cpu().numpy()[0][sel], h["q"][0][rows],
                           qi_rot, h["k"][0], h["v"][0], kp[0], rows, topk=k)
    print("yarn", st)


@pytest.mark.parametrize("q0", [1234, 1232])
def test_chunked_prefill_matches_full_prefill(q0):
    # The lists are the same bit for bit.  The query-tile attention groups rows 16 at a time from the
    # call's first row: with q0 a multiple of 16 the chunk's tiles are the full call's tiles and the
    # outputs are bit-identical; otherwise only the fp32 summation order differs.
    T, k = 2500, 64
    x = _small_prefill(T, 16, 2, 4, 55)
    full = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=k)
    part = Q.prefill(x["q"][:, q0:].contiguous(), x["k"], x["v"], x["qi"][:, q0:].contiguous(), x["ki"], topk=k,
                     q_pos0=q0)
    assert torch.equal(full["idx"][:, q0:], part["idx"])
    if q0 % 16 == 0:
        assert torch.equal(full["out"][:, q0:], part["out"])
    else:
        P.assert_outputs_close(I.bits(full["out"][:, q0:]), I.bits(part["out"]))


def test_unselected_tokens_poisoned_with_nan_do_not_matter():
    T, k, q0 = 3000, 8, 2990
    x = _small_prefill(T, 16, 2, 4, 66)
    qc, qic = x["q"][:, q0:].contiguous(), x["qi"][:, q0:].contiguous()
    res = Q.prefill(qc, x["k"], x["v"], qic, x["ki"], topk=k, q_pos0=q0)
    idx = res["idx"].cpu().numpy()[0]
    used = np.zeros(T, bool)
    used[q0 // 4 * 4:] = True                  # own blocks of the chunk's queries
    for b in np.unique(idx[idx >= 0]):
        used[4 * b:4 * b + 4] = True
    assert not used.all()
    k2, v2 = x["k"].clone(), x["v"].clone()
    bad = torch.from_numpy(~used).to(DEV)
    k2[0, bad] = float("nan")
    v2[0, bad] = float("nan")
    out2, lse2 = Q.qsa_sparse_attn_prefill(qc, k2, v2, res["idx"], q_pos0=q0)
    assert torch.equal(out2, res["out"]) and torch.equal(lse2, res["lse"])


def test_index_order_does_not_matter_on_gpu():
    T, k = 2000, 64
    x = _small_prefill(T, 16, 2, 4, 77)
    res = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=k)
    perm = torch.argsort(torch.rand(res["idx"].shape, device=DEV), dim=-1)
    idx2 = torch.gather(res["idx"], -1, perm).contiguous()
    out2, _ = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx2)
    P.assert_outputs_close(I.bits(out2), I.bits(res["out"]))


def test_out_of_range_index_is_skipped_and_reported():
    T, k = 400, 8
    x = _small_prefill(T, 16, 2, 4, 88)
    res = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=k)
    _status_ok()
    idx = res["idx"].clone()
    idx[0, 300, 0] = 1000          # beyond the causal range of row 300
    idx[0, 301, 1] = -7
    out, _ = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    assert Q.qsa_get_device_status() == Q.QSA_ERR_INVALID_ARGUMENT
    assert torch.isfinite(out.float()).all()
    _status_ok()


def test_bounded_wait_reports_timeout_and_context_survives():
    Q.qsa_wait_timeout_selftest(2_000_000)          # 2 ms
    assert Q.qsa_get_device_status() == Q.QSA_ERR_TIMEOUT
    _status_ok()
    ki = _randn_bf16((1, 64, 64), 0.1, 3)
    assert np.array_equal(I.bits(Q.qsa_pool_block_keys(ki)), O.pool_block_keys(I.bits(ki)))


# ------------------------------------------------------------------------------------------ decode
def _decode_inputs(B, L, seqlens, seed):
    w = I.WORKLOADS["decode_256k"].with_(B=B, T=L, seed=seed)
    return w, I.make_decode(w, DEV, seqlens=seqlens)


def test_decode_parity_every_sequence():
    B, L, k = 6, 20000, 512
    seqlens = [1, 7, 2049, 2052, 15001, 20000]
    w, x = _decode_inputs(B, L, seqlens, 11)
    kp = Q.qsa_pool_block_keys(x["ki"])
    res = Q.decode(x["q"], x["k"], x["v"], x["qi"], kp, x["seqlens"], topk=k)
    h = {n: I.bits(x[n]) for n in ("q", "k", "v", "qi")}
    st = H.compare_decode(res["idx"].cpu().numpy(), I.bits(res["out"]), res["lse"].cpu().numpy(), h["q"], h["k"],
                          h["v"], h["qi"], I.bits(kp), np.array(seqlens), list(range(B)), topk=k)
    print("decode:", st)
    _status_ok()


def test_decode_split_invariance_and_prefill_last_row():
    T, k = 4097, 256
    x = _small_prefill(T, 16, 2, 4, 99)
    full = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=k)
    seqlens = torch.tensor([T], dtype=torch.int32, device=DEV)
    outs = []
    for splits in (1, 3, 8):
        d = Q.decode(x["q"][:, T - 1].contiguous(), x["k"], x["v"], x["qi"][:, T - 1].contiguous(), full["kp"], seqlens,
                     topk=k, num_splits=splits)
        outs.append(d)
        assert torch.equal(d["idx"], outs[0]["idx"])
    # decode scores come from the warp-level MMA (mma.sync) pass over the pooled-key cache, prefill
    # scores from the tcgen05 kernel: the fp32 sums may differ in the last bit.  Both sides are held
    # to the oracle's tie rule for row T - 1 (a differing block must lie within the tie band of the
    # oracle's k-th score), and both outputs to the oracle re-run on each side's own list.
    h = {n: I.bits(x[n]) for n in ("q", "k", "v", "qi")}
    kp_h = I.bits(full["kp"])
    row = [T - 1]
    H.compare_prefill(full["idx"].cpu().numpy()[0][row], I.bits(full["out"])[0][row], full["lse"].cpu().numpy()[0][row],
                      h["q"][0][row], h["qi"][0][row], h["k"][0], h["v"][0], kp_h[0], row, topk=k)
    for d in outs:
        H.compare_decode(d["idx"].cpu().numpy(), I.bits(d["out"]), d["lse"].cpu().numpy(), h["q"][:, T - 1],
                         h["k"], h["v"], h["qi"][:, T - 1], kp_h, np.array([T]), [0], topk=k)
    # the two lists against each other under the same rule, and the outputs against each other
    ora = H.oracle_prefill_rows(h["q"][0][row], h["qi"][0][row], h["k"][0], h["v"][0], kp_h[0], row, topk=k)
    nb = (T - 1) // 4
    sel = P.compare_selection(outs[0]["idx"].cpu().numpy(), full["idx"].cpu().numpy()[0][row], ora["kth"],
                              lambda r: O.index_scores(h["qi"][0][T - 1], kp_h[0], nb))
    assert not sel["bad"], sel["bad"]
    for d in outs:
        P.assert_outputs_close(I.bits(d["out"])[0], I.bits(full["out"])[0, T - 1])
    P.assert_outputs_close(I.bits(outs[0]["out"]), I.bits(outs[2]["out"]))
    assert torch.allclose(outs[0]["lse"], outs[2]["lse"], atol=1e-4)


# ------------------------------------------------------------------------------------------ full sizes
def _full_prefill_check(name, n_random):
    w = I.WORKLOADS[name]
    x = I.make_prefill(w, DEV)
    res = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=w.k)
    torch.cuda.synchronize()
    _status_ok()
    rows = H.sample_rows(w.T, w.k, n_random=n_random, seed=w.seed)
    ri = torch.tensor(rows, device=DEV)
    kp = O.pool_block_keys(I.bits(x["ki"]))
    assert np.array_equal(I.bits(res["kp"]), kp)
    st = H.compare_prefill(res["idx"][0, ri].cpu().numpy(), I.bits(res["out"][0, ri]), res["lse"][0, ri].cpu().numpy(),
                           I.bits(x["q"][0, ri]), I.bits(x["qi"][0, ri]), I.bits(x["k"][0]), I.bits(x["v"][0]), kp[0],
                           rows, topk=w.k)
    print(name, st)
    return st


def test_full_size_prefill_32k_sampled_rows():
    _full_prefill_check("prefill_32k", 40)


def test_full_size_prefill_128k_sampled_rows():
    _full_prefill_check("prefill_128k", 40)


def test_full_size_prefill_1m_sampled_rows():
    _full_prefill_check("prefill_1m", 16)


def test_full_size_decode_256k_sampled_sequences():
    w = I.WORKLOADS["decode_256k"]
    x = I.make_decode(w, DEV)
    kp = Q.qsa_pool_block_keys(x["ki"])
    res = Q.decode(x["q"], x["k"], x["v"], x["qi"], kp, x["seqlens"], topk=w.k)
    torch.cuda.synchronize()
    _status_ok()
    seqs = [0, 13, 31]
    sel = torch.tensor(seqs, device=DEV)
    sub = {n: I.bits(x[n][sel]) for n in ("q", "k", "v", "qi")}
    kph = I.bits(kp[sel])
    st = H.compare_decode(res["idx"][sel].cpu().numpy(), I.bits(res["out"][sel]), res["lse"][sel].cpu().numpy(),
                          sub["q"], sub["k"], sub["v"], sub["qi"], kph, x["seqlens"][sel].cpu().numpy(),
                          list(range(len(seqs))), topk=w.k)
    print("decode_256k:", st)

"""The query-tile prefill attention (tcgen05, tiles of 16 rows over the union of their blocks),
called through the C ABI (qsa_sparse_attn_prefill_ws) and checked against the CPU oracle and
against the row-by-row kernel on the same inputs."""
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


@pytest.fixture(autouse=True)
def _tiles_forced():
    Q.qsa_set_attn_options(Q.QSA_ATTN_TILES)
    yield
    Q.qsa_set_attn_options(Q.QSA_ATTN_AUTO)


def _inputs(T, Hq, Hkv, seed, Tk=None):
    Tk = T if Tk is None else Tk
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    rb = lambda shape, d: (torch.randn(shape, generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16)
    return dict(q=rb((1, T, Hq, 128), 128), k=rb((1, Tk, Hkv, 128), 128), v=rb((1, Tk, Hkv, 128), 128),
                qi=rb((1, T, 4, 64), 64), ki=rb((1, Tk, 64), 64))


def _oracle_lists(x, k, q_pos0=0):
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"])
    T = x["q"].shape[1]
    ora = O.prefill_rows(h["q"], h["k"], h["v"], h["qi"], kp, [(0, t) for t in range(T)], topk=k, q_pos0=q_pos0)
    return ora, torch.from_numpy(ora["idx"]).to(DEV).view(1, T, k)


def _status_ok():
    assert Q.qsa_get_device_status() == Q.QSA_OK


@pytest.mark.parametrize("T,Hq,Hkv,k", [(2500, 16, 2, 64), (1000, 8, 1, 37), (300, 16, 2, 512), (4099, 16, 2, 256)])
def test_tiles_match_the_oracle_on_every_row(T, Hq, Hkv, k):
    x = _inputs(T, Hq, Hkv, T + k)
    ora, idx = _oracle_lists(x, k)
    out, lse = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    torch.cuda.synchronize()
    _status_ok()
    P.assert_outputs_close(I.bits(out)[0], ora["out"])
    assert np.abs(lse.cpu().numpy()[0] - ora["lse"]).max() <= 1e-2


def test_tiles_across_sequences_of_a_batch():
    # three sequences of a ragged length: tiles 0-69 belong to sequence 0, 70-139 to 1, 140-209 to 2,
    # the last tile of each holding 7 rows
    B, T, Hq, Hkv, k = 3, 1111, 16, 2, 64
    g = torch.Generator(device=DEV)
    g.manual_seed(11)
    rb = lambda shape, d: (torch.randn(shape, generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16)
    x = dict(q=rb((B, T, Hq, 128), 128), k=rb((B, T, Hkv, 128), 128), v=rb((B, T, Hkv, 128), 128),
             qi=rb((B, T, 4, 64), 64), ki=rb((B, T, 64), 64))
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"])
    ora = O.prefill_rows(h["q"], h["k"], h["v"], h["qi"], kp, [(b, t) for b in range(B) for t in range(T)], topk=k)
    idx = torch.from_numpy(ora["idx"]).to(DEV).view(B, T, k)
    out, lse = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    Q.qsa_set_attn_options(Q.QSA_ATTN_ROWS)
    o_rows, l_rows = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    torch.cuda.synchronize()
    _status_ok()
    P.assert_outputs_close(I.bits(out).reshape(B * T, Hq, 128), ora["out"])
    assert np.abs(lse.cpu().numpy().reshape(B * T, Hq) - ora["lse"]).max() <= 1e-2
    P.assert_outputs_close(I.bits(out), I.bits(o_rows))
    assert torch.allclose(lse, l_rows, atol=1e-4)


def test_tiles_at_an_offset_with_garbage_past_the_last_query():
    # rows 1234 .. 2233 of a 2400-token cache whose positions past the last query hold NaN: a tile's
    # last own block reaches past the last query, and those positions must not be read
    q0, Tq, Tk, k = 1234, 1000, 2400, 48
    full = _inputs(Tk, 16, 2, 91)
    x = dict(q=full["q"][:, q0:q0 + Tq].contiguous(), k=full["k"].clone(), v=full["v"].clone(),
             qi=full["qi"][:, q0:q0 + Tq].contiguous(), ki=full["ki"])
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"])
    ora = O.prefill_rows(h["q"], h["k"], h["v"], h["qi"], kp, [(0, t) for t in range(Tq)], topk=k, q_pos0=q0)
    idx = torch.from_numpy(ora["idx"]).to(DEV).view(1, Tq, k)
    x["k"][:, q0 + Tq:] = float("nan")
    x["v"][:, q0 + Tq:] = float("nan")
    out, lse = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx, q_pos0=q0)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.isfinite(out.float()).all()
    P.assert_outputs_close(I.bits(out)[0], ora["out"])


def test_tiles_equal_rows_and_ranges_of_tiles_are_bit_identical():
    T, k = 6000, 128
    x = _inputs(T, 16, 2, 5)
    kp = Q.qsa_pool_block_keys(x["ki"])
    idx = Q.qsa_select_topk(k, qi=x["qi"], kp=kp)
    Q.qsa_set_attn_options(Q.QSA_ATTN_ROWS)
    o_rows, l_rows = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    Q.qsa_set_attn_options(Q.QSA_ATTN_TILES)
    o_all, l_all = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    # a workspace for 7 tiles: the call walks the 375 tiles in ranges of 7
    tile_bytes = (16 * k + 16) * 8 + (k + 1) * 128 + 4
    ws = torch.empty(512 + 7 * tile_bytes, dtype=torch.uint8, device=DEV)
    o_rng, l_rng = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx, workspace=ws)
    torch.cuda.synchronize()
    _status_ok()
    P.assert_outputs_close(I.bits(o_all), I.bits(o_rows))
    assert torch.allclose(l_all, l_rows, atol=1e-4)
    assert torch.equal(o_rng, o_all) and torch.equal(l_rng, l_all)


def test_tiles_with_unsorted_and_padded_lists():
    T, k = 1200, 400        # rows before position 1600 have fewer than k candidates: -1 padding
    x = _inputs(T, 16, 2, 6)
    ora, idx = _oracle_lists(x, k)
    perm = torch.argsort(torch.rand(idx.shape, device=DEV), dim=-1)
    idx2 = torch.gather(idx, -1, perm).contiguous()      # -1 entries in the middle, any order
    out, _ = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx2)
    torch.cuda.synchronize()
    _status_ok()
    P.assert_outputs_close(I.bits(out)[0], ora["out"])


def test_tiles_with_k_1024():
    T, k = 5000, 1024
    x = _inputs(T, 16, 2, 7)
    ora, idx = _oracle_lists(x, k)
    out, lse = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    torch.cuda.synchronize()
    _status_ok()
    P.assert_outputs_close(I.bits(out)[0], ora["out"])


def test_tiles_skip_and_report_out_of_range_entries():
    T, k = 400, 8
    x = _inputs(T, 16, 2, 8)
    _, idx = _oracle_lists(x, k)
    idx = idx.clone()
    idx[0, 300, 0] = 1000          # beyond the causal range of row 300
    idx[0, 301, 1] = -7
    out, _ = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx)
    assert Q.qsa_get_device_status() == Q.QSA_ERR_INVALID_ARGUMENT
    assert torch.isfinite(out.float()).all()
    _status_ok()


def test_tiles_unselected_blocks_poisoned_with_nan_do_not_matter():
    # the last 37 rows of a 3000-token prefill (three tiles, the last one ragged): K/V positions no row
    # of the call attends hold NaN
    T, k, q0 = 3000, 16, 2963
    full = _inputs(T, 16, 2, 9)
    x = dict(q=full["q"][:, q0:].contiguous(), k=full["k"], v=full["v"], qi=full["qi"][:, q0:].contiguous(),
             ki=full["ki"])
    h = {n: I.bits(t) for n, t in x.items()}
    kp = O.pool_block_keys(h["ki"])
    ora = O.prefill_rows(h["q"], h["k"], h["v"], h["qi"], kp, [(0, t) for t in range(T - q0)], topk=k, q_pos0=q0)
    idx = torch.from_numpy(ora["idx"]).to(DEV).view(1, T - q0, k)
    out, lse = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx, q_pos0=q0)
    used = np.zeros(T, bool)
    ih = ora["idx"]
    for b in np.unique(ih[ih >= 0]):
        used[4 * b:4 * b + 4] = True
    used[q0 // 4 * 4:] = True               # own blocks of the call's rows
    assert not used.all()
    k2, v2 = x["k"].clone(), x["v"].clone()
    bad = torch.from_numpy(~used).to(DEV)
    k2[0, bad] = float("nan")
    v2[0, bad] = float("nan")
    out2, lse2 = Q.qsa_sparse_attn_prefill(x["q"], k2, v2, idx, q_pos0=q0)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(out2, out) and torch.equal(lse2, lse)


def test_forced_tiles_refuse_other_shapes_and_missing_workspace():
    x = _inputs(64, 16, 2, 10)
    idx = torch.full((1, 64, 4), -1, dtype=torch.int32, device=DEV)
    with pytest.raises(Q.QSAError) as e:
        Q.qsa_sparse_attn_prefill(x["q"][:, :, :12].contiguous(), x["k"], x["v"], idx)   # groups of 6
    assert e.value.status == Q.QSA_ERR_UNSUPPORTED
    with pytest.raises(Q.QSAError) as e:
        Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx, workspace=torch.empty(64, dtype=torch.uint8,
                                                                                      device=DEV))
    assert e.value.status == Q.QSA_ERR_WORKSPACE_TOO_SMALL


# ------------------------------------------------------------------------------------------ full sizes
def _full_prefill_tiles(name, n_random):
    # the whole layer at the benchmark sizes with the query-tile attention forced: sampled rows
    # against the oracle (lists and outputs), every row against the row-by-row kernel
    w = I.WORKLOADS[name]
    x = I.make_prefill(w, DEV)
    res = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=w.k)
    torch.cuda.synchronize()
    _status_ok()
    rows = H.sample_rows(w.T, w.k, n_random=n_random, seed=w.seed + 1)
    ri = torch.tensor(rows, device=DEV)
    kp = O.pool_block_keys(I.bits(x["ki"]))
    st = H.compare_prefill(res["idx"][0, ri].cpu().numpy(), I.bits(res["out"][0, ri]), res["lse"][0, ri].cpu().numpy(),
                           I.bits(x["q"][0, ri]), I.bits(x["qi"][0, ri]), I.bits(x["k"][0]), I.bits(x["v"][0]), kp[0],
                           rows, topk=w.k)
    Q.qsa_set_attn_options(Q.QSA_ATTN_ROWS)
    o_rows, l_rows = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], res["idx"])
    torch.cuda.synchronize()
    _status_ok()
    # tiles against rows on every row, on the device in chunks (the 1M outputs are 4.3 GB each)
    mx, tot = 0.0, 0.0
    a, b = res["out"].view(-1, 128), o_rows.view(-1, 128)
    for s in range(0, a.shape[0], 1 << 20):
        d = (a[s:s + (1 << 20)].float() - b[s:s + (1 << 20)].float()).abs()
        mx = max(mx, d.max().item())
        tot += d.sum().item()
    mean = tot / a.numel()
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS, (mx, mean)
    assert (res["lse"] - l_rows).abs().max().item() <= 1e-4
    print(name, "tiles", st, "vs rows max", mx, "mean", mean)


def test_tiles_full_size_32k_sampled_rows():
    _full_prefill_tiles("prefill_32k", 40)


def test_tiles_full_size_128k_sampled_rows():
    _full_prefill_tiles("prefill_128k", 40)


def test_tiles_full_size_1m_sampled_rows():
    _full_prefill_tiles("prefill_1m", 12)

"""GPU: the filtered selection (thresholds from sampled scores, candidate lists built by the
tensor-core score kernel, exact select over the lists, exact redo of failed rows) against the
materialised selection and the oracle.

Both prefill selections take the top-k of the same fp32 tensor-core scores, so their index lists
must be identical; rows redone by the fallback use CUDA-core scores and are held to the oracle's
tie rule instead."""
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
def _default_options():
    yield
    Q.qsa_set_select_options(Q.QSA_SELECT_AUTO, 0)


def _case(B, T, Hi, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    qi = (torch.randn((B, T, Hi, 64), generator=g, device=DEV) * 0.125).to(torch.bfloat16)
    ki = (torch.randn((B, T, 64), generator=g, device=DEV) * 0.125).to(torch.bfloat16)
    return qi, Q.qsa_pool_block_keys(ki)


def _select(path, rank, qi, kp, k, **kw):
    Q.qsa_set_select_options(path, rank)
    idx = Q.qsa_select_topk(k, qi=qi, kp=kp, **kw)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    return idx.cpu().numpy()


def _oracle_check(idx, qi, kp, rows, k, b=0, head_w=None, mode=0, q_pos0=0):
    """Index lists of `rows` against the oracle's selection under the tie rule."""
    qh, kph = I.bits(qi[b]), I.bits(kp[b])
    wh = None if head_w is None else head_w.cpu().numpy()
    ora, kth, srows = [], [], {}
    for i, t in enumerate(rows):
        n = (q_pos0 + t) // 4
        s = O.index_scores(qh[t], kph, n, head_w=wh, mode=mode)
        ri, rk = O.select_topk(s, k)
        ora.append(ri)
        kth.append(rk)
        srows[i] = s
    got = idx[b, rows]
    nb = np.array([(q_pos0 + t) // 4 for t in rows])
    assert P.check_index_rows(got, nb, k) == []
    res = P.compare_selection(got, np.array(ora), np.array(kth), lambda i: srows[i])
    assert res["bad"] == [], res["bad"][:3]
    return res


@pytest.mark.parametrize("B,T,Hi,k,mode,weighted", [(1, 16384, 4, 512, 0, False), (2, 12000, 4, 64, 0, False),
                                                    (1, 16384, 8, 512, 1, True), (1, 24000, 4, 1024, 0, True),
                                                    (1, 9000, 4, 1, 0, False)])
def test_filtered_equals_materialised(B, T, Hi, k, mode, weighted):
    qi, kp = _case(B, T, Hi, T + k)
    w = torch.linspace(0.5, 1.5, Hi, device=DEV) if weighted else None
    mat = _select(Q.QSA_SELECT_MATERIALISED, 0, qi, kp, k, head_w=w, mode=mode)
    fil = _select(Q.QSA_SELECT_FILTERED, 0, qi, kp, k, head_w=w, mode=mode)
    assert np.array_equal(mat, fil)
    rows = H.sample_rows(T, k, n_random=12, seed=T)
    _oracle_check(fil, qi, kp, rows, k, b=B - 1, head_w=w, mode=mode)


def test_filtered_equals_materialised_on_the_32k_workload():
    """The benchmark's own input recipe (boosted keys, 16 q / 2 KV heads, 4 x 64 indexer)."""
    w = I.WORKLOADS["prefill_32k"]
    x = I.make_prefill(w, DEV)
    kp = Q.qsa_pool_block_keys(x["ki"])
    mat = _select(Q.QSA_SELECT_MATERIALISED, 0, x["qi"], kp, w.k)
    fil = _select(Q.QSA_SELECT_FILTERED, 0, x["qi"], kp, w.k)
    auto = _select(Q.QSA_SELECT_AUTO, 0, x["qi"], kp, w.k)
    assert np.array_equal(mat, fil) and np.array_equal(fil, auto)


def test_filtered_in_chunks_with_offset():
    """A workspace that holds fewer rows than the call (several chunks, a ragged last one) and a
    window of rows that starts past position 0."""
    T, k, pos0 = 14000, 512, 6000
    qi, kp_full = _case(1, T + pos0, 4, 31)
    qi = qi[:, pos0:].contiguous()
    nbk = (pos0 + T - 1) // 4
    kp = kp_full[:, :nbk].contiguous()
    mat = _select(Q.QSA_SELECT_MATERIALISED, 0, qi, kp, k, q_pos0=pos0)
    rank = max(64, (5 * k + 31) // 32)
    ns = (nbk - 9) // 16 + 1
    per_row = ((ns + 3) // 4 * 4) * 4 + 12 + 32 * rank * 8
    ws = torch.empty(12 * 256 + 4 + 128 * nbk * 4 + 3000 * per_row, dtype=torch.uint8, device=DEV)
    fil = _select(Q.QSA_SELECT_FILTERED, 0, qi, kp, k, q_pos0=pos0, workspace=ws)
    assert np.array_equal(mat, fil)


@pytest.mark.parametrize("rank", [1, 1 << 20])
def test_every_row_redone_by_the_fallback(rank):
    """rank 1 puts the threshold at the largest sample (lists shorter than k); a huge rank puts it
    at the smallest (lists overflow).  Every long row is then redone exactly."""
    T, k = 14000, 256
    qi, kp = _case(1, T, 4, 77)
    fil = _select(Q.QSA_SELECT_FILTERED, rank, qi, kp, k)
    rows = H.sample_rows(T, k, n_random=10, seed=3) + [T - 1, T - 2]
    res = _oracle_check(fil, qi, kp, rows, k)
    assert len(res["exact"]) >= len(rows) - 2
    mat = _select(Q.QSA_SELECT_MATERIALISED, 0, qi, kp, k)
    assert (mat == fil).all(axis=1).mean() >= 0.99


def test_all_equal_scores_go_to_the_lowest_blocks():
    """Zero indexer queries make every score 0: lists overflow, the redo keeps blocks 0 .. k-1."""
    T, k = 13000, 512
    qi, kp = _case(1, T, 4, 5)
    qi[0, 9000:11000] = 0
    fil = _select(Q.QSA_SELECT_FILTERED, 0, qi, kp, k)
    assert np.array_equal(fil[0, 9000:11000], np.tile(np.arange(k, dtype=np.int32), (2000, 1)))
    mat = _select(Q.QSA_SELECT_MATERIALISED, 0, qi, kp, k)
    assert np.array_equal(mat, fil)


def test_unsupported_head_count_is_refused():
    qi, kp = _case(1, 3000, 2, 1)
    Q.qsa_set_select_options(Q.QSA_SELECT_FILTERED, 0)
    with pytest.raises(Q.QSAError):
        Q.qsa_select_topk(64, qi=qi, kp=kp)


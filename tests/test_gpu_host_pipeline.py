"""GPU: the host-to-host prefill (inputs in pinned host memory, copies overlapped with the kernels
in causal row chunks) returns exactly what the device path returns: the same kernels run on the
same data, only the transfers are scheduled around them."""
import pytest
import torch

from hybrid_sparse_attention_qsa_b200 import inputs as I
from hybrid_sparse_attention_qsa_b200 import qsa as Q

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _pinned(x):
    return {n: t.cpu().pin_memory() for n, t in x.items()}


@pytest.mark.parametrize("chunks,sel_chunks", [(1, 1), (3, 4), (8, 3), (8, 7), (0, 2)])
def test_prefill_host_matches_device_path(chunks, sel_chunks):
    """Attention in `chunks` row chunks (0: quarters, then halving), pooling and selection in
    `sel_chunks` (ragged ones too)."""
    w = I.WORKLOADS["prefill_32k"].with_(T=12002)
    x = I.make_prefill(w, DEV)
    ref = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=w.k)
    h = _pinned(x)
    got = Q.prefill_host(h["q"], h["k"], h["v"], h["qi"], h["ki"], topk=w.k, device=DEV, chunks=chunks,
                         sel_chunks=sel_chunks)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert torch.equal(got["idx"], ref["idx"])
    assert torch.equal(got["out"], ref["out"].cpu())
    assert torch.equal(got["lse"], ref["lse"])


def test_prefill_host_window_with_offset():
    """Query rows q0.. of a longer context: the chunks send keys and values only up to their end."""
    w = I.WORKLOADS["prefill_32k"].with_(T=9000)
    x = I.make_prefill(w, DEV)
    q0 = 3001
    xq = {n: (t[:, q0:].contiguous() if n in ("q", "qi") else t) for n, t in x.items()}
    ref = Q.prefill(xq["q"], xq["k"], xq["v"], xq["qi"], xq["ki"], topk=w.k, q_pos0=q0)
    h = _pinned(xq)
    got = Q.prefill_host(h["q"], h["k"], h["v"], h["qi"], h["ki"], topk=w.k, device=DEV, q_pos0=q0, chunks=5)
    torch.cuda.synchronize()
    assert torch.equal(got["idx"], ref["idx"])
    assert torch.equal(got["out"], ref["out"].cpu())


def test_prefill_host_two_sequences_single_chunk():
    w = I.WORKLOADS["tiny"].with_(B=2, T=3000, Hq=4)
    x = I.make_prefill(w, DEV)
    ref = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=w.k)
    h = _pinned(x)
    got = Q.prefill_host(h["q"], h["k"], h["v"], h["qi"], h["ki"], topk=w.k, device=DEV)
    torch.cuda.synchronize()
    assert torch.equal(got["out"], ref["out"].cpu())


@pytest.mark.parametrize("q0", [3000, 3001])
def test_prefill_host_window_with_rope_and_selection_chunks(q0):
    """Rotated indexer keys and queries, a window starting on a block boundary (selection in chunks)
    or inside a block (one selection call), against the device path."""
    w = I.WORKLOADS["prefill_32k"].with_(T=10000)
    x = I.make_prefill(w, DEV)
    xq = {n: (t[:, q0:].contiguous() if n in ("q", "qi") else t) for n, t in x.items()}
    ref = Q.prefill(xq["q"], xq["k"], xq["v"], xq["qi"], xq["ki"], topk=w.k, q_pos0=q0, rope_theta=10000.0)
    h = _pinned(xq)
    got = Q.prefill_host(h["q"], h["k"], h["v"], h["qi"], h["ki"], topk=w.k, device=DEV, q_pos0=q0, chunks=4,
                         sel_chunks=3, rope_theta=10000.0)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert torch.equal(got["idx"], ref["idx"])
    assert torch.equal(got["out"], ref["out"].cpu())


@pytest.mark.parametrize("path", [Q.QSA_ATTN_ROWS, Q.QSA_ATTN_TILES])
def test_prefill_host_with_each_attention_path(path):
    """The host pipeline with the row kernel over k and v, or the query tiles, forced: the same
    result as the device path under the same choice."""
    w = I.WORKLOADS["prefill_32k"].with_(T=9000)
    x = I.make_prefill(w, DEV)
    Q.qsa_set_attn_options(path)
    try:
        ref = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=w.k)
        h = _pinned(x)
        got = Q.prefill_host(h["q"], h["k"], h["v"], h["qi"], h["ki"], topk=w.k, device=DEV)
        torch.cuda.synchronize()
    finally:
        Q.qsa_set_attn_options(Q.QSA_ATTN_AUTO)
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert torch.equal(got["idx"], ref["idx"])
    assert torch.equal(got["out"], ref["out"].cpu())
    assert torch.equal(got["lse"], ref["lse"])

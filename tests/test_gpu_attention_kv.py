"""K and V interleaved by block (qsa_interleave_kv) and the row-by-row attention over them
(qsa_sparse_attn_prefill_kv, and the automatic path of qsa_sparse_attn_prefill_ws that uses it):
the layout against a PyTorch restatement, and the attention bit for bit against the kernel over k
and v as given (the same arithmetic on the same data, only each block's K and V arrive in one copy)."""
import math

import pytest
import torch

from hybrid_sparse_attention_qsa_b200 import qsa as Q

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) / math.sqrt(shape[-1])).to(torch.bfloat16)


def _lists(B, Tq, k, q_pos0, seed):
    # random ascending lists of distinct visible blocks, -1 padded (rows with fewer than k visible)
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    idx = torch.full((B, Tq, k), -1, dtype=torch.int32)
    for b in range(B):
        for t in range(Tq):
            nb = (q_pos0 + t) // 4
            sel = torch.randperm(nb, generator=g)[:k] if nb else torch.empty(0, dtype=torch.int64)
            sel, _ = torch.sort(sel)
            idx[b, t, :len(sel)] = sel.to(torch.int32)
    return idx.to(DEV)


@pytest.mark.parametrize("B,Tk,Hkv", [(1, 4099, 2), (2, 1001, 1), (3, 64, 2)])
def test_interleave_layout(B, Tk, Hkv):
    k, v = _rand((B, Tk, Hkv, 128), 1), _rand((B, Tk, Hkv, 128), 2)
    kv = Q.qsa_interleave_kv(k, v)
    torch.cuda.synchronize()
    nblk = (Tk + 3) // 4
    pad = nblk * 4 - Tk
    kp = torch.cat([k, torch.zeros(B, pad, Hkv, 128, dtype=k.dtype, device=DEV)], 1).view(B, nblk, 4, Hkv, 128)
    vp = torch.cat([v, torch.zeros(B, pad, Hkv, 128, dtype=v.dtype, device=DEV)], 1).view(B, nblk, 4, Hkv, 128)
    assert kv.shape == (B, nblk, 2, 4, Hkv, 128)
    assert torch.equal(kv[:, :, 0], kp) and torch.equal(kv[:, :, 1], vp)


def test_interleave_in_pieces_equals_whole():
    # ranges that start inside a block rewrite that block whole; the pieces make the same buffer
    B, Tk = 1, 3001
    k, v = _rand((B, Tk, 2, 128), 3), _rand((B, Tk, 2, 128), 4)
    whole = Q.qsa_interleave_kv(k, v)
    kv = torch.full_like(whole, float("nan"))
    for lo, hi in [(0, 5), (5, 1234), (1234, 1235), (1235, 3001)]:
        Q.qsa_interleave_kv(k, v, kv, pos_lo=lo, pos_hi=hi)
    torch.cuda.synchronize()
    assert torch.equal(kv, whole)


@pytest.mark.parametrize("B,T,q0,Hq,Hkv,k", [(1, 3000, 0, 16, 2, 64), (2, 1500, 0, 8, 1, 37), (1, 2000, 1233, 16, 2, 128),
                                             (1, 800, 0, 8, 2, 512), (2, 600, 4101, 8, 1, 1024)])
def test_attention_over_interleaved_kv_is_bit_identical(B, T, q0, Hq, Hkv, k):
    Tk = q0 + T
    q = _rand((B, T, Hq, 128), 5)
    kk, vv = _rand((B, Tk + 7, Hkv, 128), 6), _rand((B, Tk + 7, Hkv, 128), 7)
    # positions past the last query hold NaN: the own block of the last rows is fetched only up to
    # the query, and no later block is listed
    kk[:, Tk:] = float("nan")
    vv[:, Tk:] = float("nan")
    idx = _lists(B, T, k, q0, 8)
    ref_o, ref_l = Q.qsa_sparse_attn_prefill(q, kk, vv, idx, q_pos0=q0, tiles=False)
    kv = Q.qsa_interleave_kv(kk, vv, pos_hi=Tk)
    o, l = Q.qsa_sparse_attn_prefill_kv(q, kv, idx, Tk=Tk + 7, q_pos0=q0)
    Q.qsa_set_attn_options(Q.QSA_ATTN_AUTO)
    o2, l2 = Q.qsa_sparse_attn_prefill(q, kk, vv, idx, q_pos0=q0)   # the automatic path interleaves itself
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert torch.isfinite(ref_o.float()).all()
    assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
    assert torch.equal(o2, ref_o) and torch.equal(l2, ref_l)


def test_interleaved_attention_refuses_other_shapes():
    q = _rand((1, 64, 24, 256), 9)
    kk = _rand((1, 64, 2, 256), 10)
    idx = torch.full((1, 64, 4), -1, dtype=torch.int32, device=DEV)
    with pytest.raises(Q.QSAError) as e:
        Q.qsa_interleave_kv(kk, kk)
    assert e.value.status == Q.QSA_ERR_UNSUPPORTED
    kv = torch.zeros(1, 16, 2, 4, 2, 256, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(Q.QSAError) as e:
        Q.qsa_sparse_attn_prefill_kv(q, kv, idx, Tk=64)
    assert e.value.status == Q.QSA_ERR_UNSUPPORTED

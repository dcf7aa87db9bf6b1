"""Small runs of every kernel family through the Python binding, shared by the debug-build test.

``run_cases`` runs each family once on seeded inputs and returns the results on the host.  The
GPU test calls it in-process against the release library and in a child process whose environment
sets QSA_DEBUG=1 (the debug library, with device-side bounds checks and canary guards after every
buffer the binding allocates); the two must agree bit for bit.  Run as a module, it is that child:

    QSA_DEBUG=1 python -m tests.debug_cases OUT.pt
"""
from __future__ import annotations

import sys

import torch

from hybrid_sparse_attention_qsa_b200 import inputs as I
from hybrid_sparse_attention_qsa_b200 import qsa as Q


_checked = [0]   # canary guards checked so far (debug library only)


def _ok(name: str):
    """No device-side check or argument fault recorded, and (debug mode) the guard after every live
    buffer the binding allocated is intact, while this case's workspaces are still alive."""
    st = Q.qsa_get_device_status()
    if st != Q.QSA_OK:
        raise RuntimeError(f"{name}: device status {Q.status_string(st)}")
    _checked[0] += Q.qsa_check_canaries()


def run_cases(dev="cuda:0") -> dict:
    """Results of every case on the host.  With the debug library, canaries_checked() then counts
    the guard checks made along the way."""
    res = {}
    # prefill through the whole path: pooling, scores, materialised top-k, row attention
    w = I.WORKLOADS["prefill_32k"].with_(T=3000, k=64, seed=501)
    x = I.make_prefill(w, dev)
    r = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=w.k)
    _ok("prefill")
    res.update(prefill_kp=r["kp"], prefill_idx=r["idx"], prefill_out=r["out"], prefill_lse=r["lse"])
    # query-tile attention (tcgen05) over the same lists
    Q.qsa_set_attn_options(Q.QSA_ATTN_TILES)
    try:
        o, l = Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], r["idx"])
        _ok("tile attention")
    finally:
        Q.qsa_set_attn_options(Q.QSA_ATTN_AUTO)
    res.update(tiles_out=o, tiles_lse=l)
    # the filtered selection (forced) at an offset
    w2 = I.WORKLOADS["prefill_32k"].with_(T=9000, seed=502)
    x2 = I.make_prefill(w2, dev)
    kp2 = Q.qsa_pool_block_keys(x2["ki"])
    Q.qsa_set_select_options(Q.QSA_SELECT_FILTERED, 0)
    try:
        res["filtered_idx"] = Q.qsa_select_topk(w2.k, qi=x2["qi"][:, 4000:].contiguous(), kp=kp2, q_pos0=4000)
        _ok("filtered selection")
    finally:
        Q.qsa_set_select_options(Q.QSA_SELECT_AUTO, 0)
    # the model's attention shape (24 query heads over 2 KV heads at D = 256): the wide kernel
    w3 = I.WORKLOADS["prefill_32k_model"].with_(T=900, k=40, seed=503)
    x3 = I.make_prefill(w3, dev)
    r3 = Q.prefill(x3["q"], x3["k"], x3["v"], x3["qi"], x3["ki"], topk=w3.k)
    _ok("model-shape prefill")
    res.update(model_out=r3["out"], model_lse=r3["lse"])
    # the host-memory prefill (chunked copies overlapping the kernels)
    hx = {n: t.cpu().pin_memory() for n, t in x.items()}
    rh = Q.prefill_host(hx["q"], hx["k"], hx["v"], hx["qi"], hx["ki"], topk=w.k, device=dev, chunks=4)
    torch.cuda.synchronize()
    _ok("host prefill")
    res["host_out"] = rh["out"]
    # decode: the folded pooling + cluster top-k, the cluster merge, the partial merge and the
    # allocation-free entry point
    w4 = I.WORKLOADS["decode_256k"].with_(B=5, T=20000, seed=504)
    x4 = I.make_decode(w4, dev, seqlens=[20000, 19999, 9001, 4096, 7])
    kp4 = Q.qsa_pool_block_keys(x4["ki"])
    idx4 = Q.qsa_decode_select(w4.k, qi=x4["qi"], kp=kp4, ki=x4["ki"], seqlens=x4["seqlens"])
    o4, l4 = Q.qsa_sparse_attn_decode(x4["q"], x4["k"], x4["v"], x4["seqlens"], idx4)
    o5, l5 = Q.qsa_sparse_attn_decode(x4["q"], x4["k"], x4["v"], x4["seqlens"], idx4, num_splits=12)
    o6, _ = Q.qsa_sparse_attn_decode_noalloc(x4["q"], x4["k"], x4["v"], x4["seqlens"], idx4, num_splits=12)
    _ok("decode")
    res.update(decode_idx=idx4, decode_out=o4, decode_lse=l4, decode_out12=o5, decode_lse12=l5, noalloc_out=o6)
    return {n: t.detach().cpu() for n, t in res.items()}


def canaries_checked() -> int:
    return _checked[0]


if __name__ == "__main__":
    if not Q.DEBUG:
        raise SystemExit("set QSA_DEBUG=1: this run is meant for the debug library")
    out = run_cases()
    n = canaries_checked()
    if n == 0:
        raise SystemExit("no canary guard was checked")
    torch.save({"results": out, "canaries_checked": n, "lib": Q.LIB_PATH}, sys.argv[1])
    print(f"debug run ok: {len(out)} results, {n} canary guards intact")

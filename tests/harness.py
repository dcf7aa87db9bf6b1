"""Test harness: run the CUDA path through the C ABI and the CPU oracle on the same seeded inputs,
and compare them with the parity rules of tests/parity.py.  Host logic only; the GPU tests call it.
"""
from __future__ import annotations

import concurrent.futures as cf
import math

import numpy as np
import torch

import oracle as O
from hybrid_sparse_attention_qsa_b200 import inputs as I
from tests import parity as P


def sample_rows(T: int, k: int, n_random: int = 24, seed: int = 0) -> list[int]:
    """Deterministic query rows: edges, the budget boundary, tile boundaries, random, the tail."""
    rows = {0, 1, 2, 3, 4, 5, 7, 63, 64, 127, 128, 255, 256, 257}
    for c in (4 * k - 1, 4 * k, 4 * k + 1, 4 * k + 3, 4 * k + 4, 4 * k + 5):
        rows.add(c)
    rows.update(range(T - 6, T))
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, T, n_random).tolist())
    return sorted(r for r in rows if 0 <= r < T)


def _pool(n):
    return cf.ThreadPoolExecutor(max_workers=max(1, min(16, O.hardware_threads())))


def oracle_prefill_rows(q_rows, qi_rows, k_b, v_b, kp_b, positions, *, topk, rope_theta=0.0, mode=O.RELU_SUM,
                        head_w=None, idx_in=None):
    """Oracle for individual query rows of one batch: q_rows [n,Hq,D], qi_rows [n,Hi,Di] (bits),
    k_b/v_b [Tk,Hkv,D], kp_b [NBk,Di], positions [n].  Rows run in parallel threads."""
    n = len(positions)

    def one(i):
        r = O.prefill_rows(q_rows[i][None, None], k_b[None], v_b[None], qi_rows[i][None, None], kp_b[None], [(0, 0)],
                           topk=topk, q_pos0=int(positions[i]), rope_theta=rope_theta, mode=mode, head_w=head_w,
                           idx_in=None if idx_in is None else idx_in[i][None], nthreads=1)
        return r

    with _pool(n) as ex:
        res = list(ex.map(one, range(n)))
    out = dict(out=np.stack([r["out"][0] for r in res]), lse=np.stack([r["lse"][0] for r in res]))
    if idx_in is None:
        out["idx"] = np.stack([r["idx"][0] for r in res])
        out["kth"] = np.stack([r["kth"][0] for r in res])
    return out


def compare_prefill(gpu_idx, gpu_out, gpu_lse, q_rows, qi_rows, k_b, v_b, kp_b, positions, *, topk,
                    rope_theta=0.0, mode=O.RELU_SUM, head_w=None, lse_atol=2e-2):
    """Selection and output parity for sampled rows of one batch.  gpu_* are host numpy arrays of
    the sampled rows.  Returns a stats dict; raises AssertionError on a parity failure."""
    ora = oracle_prefill_rows(q_rows, qi_rows, k_b, v_b, kp_b, positions, topk=topk, rope_theta=rope_theta, mode=mode,
                              head_w=head_w)
    nb = np.array([min(p // 4, kp_b.shape[0]) for p in positions])
    bad_rows = P.check_index_rows(gpu_idx, nb, topk)
    assert not bad_rows, f"malformed index rows at {[positions[r] for r in bad_rows[:5]]}"

    def score_row(r):
        qr = qi_rows[r]
        if rope_theta > 0:
            qr = O.rope_rows(qr[None], np.array([positions[r]]), rope_theta)[0]
        return O.index_scores(qr, kp_b, int(nb[r]), head_w=head_w, mode=mode)

    sel = P.compare_selection(gpu_idx, ora["idx"], ora["kth"], score_row)
    assert not sel["bad"], "selection parity: " + "; ".join(f"row {positions[r]}: {m}" for r, m in sel["bad"][:5])
    ref_out, ref_lse = ora["out"].copy(), ora["lse"].copy()
    if sel["tie"]:
        rows = sel["tie"]
        re = oracle_prefill_rows(q_rows[rows], qi_rows[rows], k_b, v_b, kp_b, [positions[r] for r in rows], topk=topk,
                                 idx_in=gpu_idx[rows])
        ref_out[rows] = re["out"]
        ref_lse[rows] = re["lse"]
    mx, mean = P.assert_outputs_close(gpu_out, ref_out)
    if gpu_lse is not None:
        dl = np.abs(gpu_lse.astype(np.float64) - ref_lse.astype(np.float64))
        assert np.all(np.isfinite(gpu_lse)) and dl.max() <= lse_atol, f"lse max-abs {dl.max():.3g}"
    return dict(rows=len(positions), exact=len(sel["exact"]), tie=len(sel["tie"]), max_abs=mx, mean_abs=mean)


def oracle_decode_seqs(q, kc, vc, qi, kp, seqlens, seqs, *, topk, rope_theta=0.0, idx_in=None):
    """Oracle decode for listed sequences (host bits; kc/vc/kp may hold only those sequences when
    ``seqs`` indexes into them)."""
    def one(i):
        b = seqs[i]
        return O.decode(q[b:b + 1], kc[b:b + 1], vc[b:b + 1], qi[b:b + 1], kp[b:b + 1], seqlens[b:b + 1], topk=topk,
                        rope_theta=rope_theta, idx_in=None if idx_in is None else idx_in[i][None], nthreads=1)

    with _pool(len(seqs)) as ex:
        res = list(ex.map(one, range(len(seqs))))
    out = dict(out=np.stack([r["out"][0] for r in res]), lse=np.stack([r["lse"][0] for r in res]))
    if idx_in is None:
        out["idx"] = np.stack([r["idx"][0] for r in res])
        out["kth"] = np.stack([r["kth"][0] for r in res])
    return out


def compare_decode(gpu_idx, gpu_out, gpu_lse, q, kc, vc, qi, kp, seqlens, seqs, *, topk, rope_theta=0.0):
    ora = oracle_decode_seqs(q, kc, vc, qi, kp, seqlens, seqs, topk=topk, rope_theta=rope_theta)
    pos = [int(seqlens[b]) - 1 for b in seqs]
    nb = np.array([min(p // 4, kp.shape[1]) for p in pos])
    assert not P.check_index_rows(gpu_idx, nb, topk), "malformed decode index rows"

    def score_row(r):
        b = seqs[r]
        qr = qi[b]
        if rope_theta > 0:
            qr = O.rope_rows(qr[None], np.array([pos[r]]), rope_theta)[0]
        return O.index_scores(qr, kp[b], int(nb[r]))

    sel = P.compare_selection(gpu_idx, ora["idx"], ora["kth"], score_row)
    assert not sel["bad"], "decode selection parity: " + "; ".join(f"seq {seqs[r]}: {m}" for r, m in sel["bad"][:5])
    ref_out, ref_lse = ora["out"].copy(), ora["lse"].copy()
    if sel["tie"]:
        rows = sel["tie"]
        re = oracle_decode_seqs(q, kc, vc, qi, kp, seqlens, [seqs[r] for r in rows], topk=topk, idx_in=gpu_idx[rows])
        ref_out[rows] = re["out"]
        ref_lse[rows] = re["lse"]
    mx, mean = P.assert_outputs_close(gpu_out, ref_out)
    dl = np.abs(gpu_lse.astype(np.float64) - ref_lse.astype(np.float64))
    assert dl.max() <= 2e-2, f"decode lse max-abs {dl.max():.3g}"
    return dict(seqs=len(seqs), exact=len(sel["exact"]), tie=len(sel["tie"]), max_abs=mx, mean_abs=mean)


def bits(t):
    return I.bits(t)

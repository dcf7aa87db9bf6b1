"""Parity rules shared by the GPU tests (host logic only; the CPU tests check it too).

Selection: the block index lists must match exactly, except in rows where the oracle's fp32 score
gap between the k-th and (k+1)-th block is below ``TIE_EPS``.  In such a row every block that the
two sides disagree on must lie within ``TIE_EPS`` of the oracle's k-th score, and the oracle then
re-runs attention on the GPU's list, which the outputs are compared against.

Outputs (bf16): max-abs error <= ``MAX_ABS`` and mean-abs error <= ``MEAN_ABS`` against the oracle
(double arithmetic, rounded once to bf16).
"""
from __future__ import annotations

import numpy as np

TIE_EPS = 1e-4
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_index_rows(idx: np.ndarray, nb: np.ndarray, k: int) -> list[int]:
    """Rows of a [n, k] index list that are malformed: not ascending, duplicated, outside
    [0, nb), wrong count (min(nb, k)) or not -1 padded at the end.  Returns the bad row numbers."""
    bad = []
    for r in range(idx.shape[0]):
        row = idx[r]
        m = int(min(nb[r], k))
        head, tail = row[:m], row[m:]
        if np.any(tail != -1) or np.any(head < 0) or np.any(head >= nb[r]) or np.any(np.diff(head) <= 0):
            bad.append(r)
    return bad


def compare_selection(gpu_idx: np.ndarray, ora_idx: np.ndarray, kth: np.ndarray, score_row) -> dict:
    """gpu_idx, ora_idx [n, k]; kth [n, 2] oracle (s_k, s_k+1); score_row(r) -> oracle fp32 scores
    of row r.  Returns dict(exact=[rows], tie=[rows], bad=[(row, reason)])."""
    exact, tie, bad = [], [], []
    for r in range(gpu_idx.shape[0]):
        a = set(int(x) for x in gpu_idx[r] if x >= 0)
        b = set(int(x) for x in ora_idx[r] if x >= 0)
        if a == b:
            exact.append(r)
            continue
        sk, sk1 = float(kth[r, 0]), float(kth[r, 1])
        if not (sk - sk1 < TIE_EPS):
            bad.append((r, f"sets differ with score gap {sk - sk1:.3g} >= {TIE_EPS}"))
            continue
        if len(a) != len(b):
            bad.append((r, f"selected {len(a)} blocks, oracle {len(b)}"))
            continue
        s = score_row(r)
        diff = sorted(a ^ b)
        off = [d for d in diff if abs(float(s[d]) - sk) > TIE_EPS]
        if off:
            bad.append((r, f"blocks {off[:4]} differ but lie outside the tie band"))
            continue
        tie.append(r)
    return dict(exact=exact, tie=tie, bad=bad)


def output_errors(got_bits: np.ndarray, ref_bits: np.ndarray) -> tuple[float, float]:
    a = bf16_bits_to_f64(got_bits)
    b = bf16_bits_to_f64(ref_bits)
    if not np.all(np.isfinite(a)):
        return float("inf"), float("inf")
    d = np.abs(a - b)
    return float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0


def assert_outputs_close(got_bits, ref_bits, what="out"):
    mx, mean = output_errors(got_bits, ref_bits)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3g} (<= {MAX_ABS}), mean-abs {mean:.3g} (<= {MEAN_ABS})"
    return mx, mean

"""QSA oracle (test infrastructure only).

A plain, slow, host-only C++ restatement of the Qwen Sparse Attention layer (see qsa_oracle.cpp for
the source passages and readings), wrapped with ctypes over numpy arrays.  bf16 tensors travel as
their uint16 bit patterns.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this
package.  It shares no code with the CUDA library and never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libqsa_oracle.so")
_lib = None

RELU_SUM = 0
LINEAR = 1


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/libqsa_oracle.so with the host C++ compiler."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["g++", "-O2", "-std=c++17", "-fno-fast-math", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def build_mutant(mutant: int, path: str) -> str:
    """Compile a deliberately wrong oracle (planted mistake number ``mutant``) to ``path``; used only
    by the test that checks the pins catch planted mistakes."""
    cmd = ["g++", "-O2", "-std=c++17", "-fno-fast-math", "-shared", "-fPIC", "-pthread", f"-DQO_MUTANT={mutant}",
           _SRC, "-o", path]
    subprocess.run(cmd, check=True)
    return path


def use_library(path: str | None) -> None:
    """Switch the wrapper to another build of the oracle (None: the default build)."""
    global _lib, _lib_path_override
    _lib = None
    _lib_path_override = path


_lib_path_override = None


def _load():
    global _lib
    if _lib is None:
        path = _lib_path_override
        if path is None:
            build()
            path = _LIB_PATH
        lib = ctypes.CDLL(path)
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.qo_bf16_round_f64.argtypes = [P, P, I64]
        lib.qo_pool_block_keys.argtypes = [P, P, I64, I64, I64, I64, D, I64]
        lib.qo_rope_rows.argtypes = [P, P, I64, I64, I64, P, D]
        lib.qo_pool_block_keys_yarn.argtypes = [P, P, I64, I64, I64, I64, D, I64, D, D, D, D, D]
        lib.qo_rope_rows_yarn.argtypes = [P, P, I64, I64, I64, P, D, D, D, D, D, D]
        lib.qo_index_scores.argtypes = [P, P, P, I64, I64, I64, I32, P]
        lib.qo_select_topk.argtypes = [P, I64, I64, P, P]
        lib.qo_select_topk.restype = I64
        lib.qo_attend.argtypes = [P, P, P, I64, P, I64, I64, I64, I64, I64, D, P, P]
        lib.qo_attend.restype = I32
        lib.qo_prefill_rows.argtypes = [P] * 6 + [I64] * 12 + [D, I32, D, P, I64, P, P, P, P, P, I32]
        lib.qo_prefill_rows.restype = I32
        lib.qo_decode.argtypes = [P] * 7 + [I64] * 10 + [D, I32, D, P, I64, P, P, P, P, P, I32]
        lib.qo_decode.restype = I32
        lib.qo_hardware_threads.restype = I32
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def hardware_threads() -> int:
    return int(_load().qo_hardware_threads())


# ---------------------------------------------------------------------------- bf16 conversions
def bf16_round(x: np.ndarray) -> np.ndarray:
    """double -> bf16 bit patterns, round to nearest even in one step."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(x.shape, dtype=np.uint16)
    _load().qo_bf16_round_f64(_p(x), _p(y), x.size)
    return y


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------- the four steps
def _yarn_args(yarn):
    """YaRN parameters (factor, orig_ctx, alpha, beta, mscale); None = plain RoPE."""
    if not yarn:
        return (1.0, 0.0, 1.0, 32.0, 0.0)
    return (float(yarn["factor"]), float(yarn["orig_ctx"]), float(yarn.get("alpha", 1.0)),
            float(yarn.get("beta", 32.0)), float(yarn.get("mscale", 0.0)))


def pool_block_keys(ki: np.ndarray, blk: int = 4, rope_theta: float = 0.0, pos0: int = 0, yarn=None) -> np.ndarray:
    """ki [B, L, Di] bf16 bits -> kp [B, L // blk, Di]; `yarn` = dict(factor, orig_ctx[, alpha, beta,
    mscale]) scales the rotary frequencies when RoPE is on."""
    ki = _u16(ki)
    B, L, Di = ki.shape
    kp = np.empty((B, L // blk, Di), dtype=np.uint16)
    if yarn:
        _load().qo_pool_block_keys_yarn(_p(ki), _p(kp), B, L, Di, blk, float(rope_theta), pos0, *_yarn_args(yarn))
    else:
        _load().qo_pool_block_keys(_p(ki), _p(kp), B, L, Di, blk, float(rope_theta), pos0)
    return kp


def rope_rows(x: np.ndarray, pos: np.ndarray, theta: float, yarn=None) -> np.ndarray:
    """x [rows, H, Di] bf16 bits rotated at pos [rows] (YaRN-scaled with `yarn`)."""
    x = _u16(x)
    rows, H, Di = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    y = np.empty_like(x)
    if yarn:
        _load().qo_rope_rows_yarn(_p(x), _p(y), rows, H, Di, _p(pos), float(theta), *_yarn_args(yarn))
    else:
        _load().qo_rope_rows(_p(x), _p(y), rows, H, Di, _p(pos), float(theta))
    return y


def index_scores(qi_row: np.ndarray, kp: np.ndarray, nb: int, head_w=None, mode: int = RELU_SUM) -> np.ndarray:
    """One fp32 score row for a (rotated) query qi_row [Hi, Di] over kp [NB, Di], b < nb."""
    qi_row = _u16(qi_row)
    kp = _u16(kp)
    Hi, Di = qi_row.shape
    s = np.empty(max(nb, 1), dtype=np.float32)
    w = None if head_w is None else np.ascontiguousarray(head_w, dtype=np.float32)
    _load().qo_index_scores(_p(qi_row), _p(kp), _p(w), Hi, Di, nb, mode, _p(s))
    return s[:nb]


def select_topk(s: np.ndarray, k: int):
    """-> (idx [k] int32 ascending, -1 padded; (s_k, s_k+1))."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    idx = np.empty(k, dtype=np.int32)
    kth = np.empty(2, dtype=np.float32)
    _load().qo_select_topk(_p(s), s.size, k, _p(idx), _p(kth))
    return idx, (float(kth[0]), float(kth[1]))


def attend(q_row, kc, vc, pos: int, idx, blk: int = 4, scale: float | None = None):
    """q_row [Hq, D], kc/vc [L, Hkv, D] bf16 bits -> (out [Hq, D] bf16 bits, lse [Hq])."""
    q_row, kc, vc = _u16(q_row), _u16(kc), _u16(vc)
    Hq, D = q_row.shape
    Hkv = kc.shape[1]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.empty((Hq, D), dtype=np.uint16)
    lse = np.empty(Hq, dtype=np.float32)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    rc = _load().qo_attend(_p(q_row), _p(kc), _p(vc), pos, _p(idx), idx.size, Hq, Hkv, D, blk,
                           float(scale), _p(out), _p(lse))
    if rc:
        raise ValueError("index outside the causal range")
    return out, lse


# ---------------------------------------------------------------------------- whole-layer drivers
def prefill_rows(q, k, v, qi, kp, rows, *, topk: int, blk: int = 4, q_pos0: int = 0, rope_theta: float = 0.0,
                 mode: int = RELU_SUM, head_w=None, scale: float | None = None, idx_in=None, nthreads: int = 0):
    """The QSA layer for the listed (b, t) query rows of a prefill.

    q [B,Tq,Hq,D], k/v [B,Tk,Hkv,D], qi [B,Tq,Hi,Di] (unrotated), kp [B,NBk,Di] from pool_block_keys.
    Returns dict(idx [n,k], kth [n,2], out [n,Hq,D] bf16 bits, lse [n,Hq]).  With idx_in the
    selection step is skipped and attention runs over the given index lists.
    """
    q, k, v, qi, kp = map(_u16, (q, k, v, qi, kp))
    B, Tq, Hq, D = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    Hi, Di = qi.shape[2], qi.shape[3]
    NBk = kp.shape[1]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    n = rows.shape[0]
    idx_out = np.empty((n, topk), dtype=np.int32)
    kth = np.empty((n, 2), dtype=np.float32)
    out = np.empty((n, Hq, D), dtype=np.uint16)
    lse = np.empty((n, Hq), dtype=np.float32)
    w = None if head_w is None else np.ascontiguousarray(head_w, dtype=np.float32)
    ii = None if idx_in is None else np.ascontiguousarray(idx_in, dtype=np.int32).reshape(n, topk)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    rc = _load().qo_prefill_rows(_p(q), _p(k), _p(v), _p(qi), _p(kp), _p(w), B, Tq, Tk, NBk, Hq, Hkv, D, Hi, Di,
                                 blk, topk, q_pos0, float(rope_theta), mode, float(scale), _p(rows), n, _p(ii),
                                 _p(idx_out), _p(kth), _p(out), _p(lse), nthreads)
    if rc:
        raise ValueError("index outside the causal range")
    res = dict(out=out, lse=lse)
    if idx_in is None:
        res.update(idx=idx_out, kth=kth)
    return res


def decode(q, kc, vc, qi, kp, seqlens, seqs=None, *, topk: int, blk: int = 4, rope_theta: float = 0.0,
           mode: int = RELU_SUM, head_w=None, scale: float | None = None, idx_in=None, nthreads: int = 0):
    """One decode step for the listed sequences.

    q [B,Hq,D], kc/vc [B,Lmax,Hkv,D], qi [B,Hi,Di] (unrotated), kp [B,NBk,Di], seqlens [B] (new
    token included).  Returns dict(idx, kth, out [n,Hq,D], lse [n,Hq]).
    """
    q, kc, vc, qi, kp = map(_u16, (q, kc, vc, qi, kp))
    B, Hq, D = q.shape
    Lmax, Hkv = kc.shape[1], kc.shape[2]
    Hi, Di = qi.shape[1], qi.shape[2]
    NBk = kp.shape[1]
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    seqs = np.arange(B, dtype=np.int64) if seqs is None else np.ascontiguousarray(seqs, dtype=np.int64)
    n = seqs.size
    idx_out = np.empty((n, topk), dtype=np.int32)
    kth = np.empty((n, 2), dtype=np.float32)
    out = np.empty((n, Hq, D), dtype=np.uint16)
    lse = np.empty((n, Hq), dtype=np.float32)
    w = None if head_w is None else np.ascontiguousarray(head_w, dtype=np.float32)
    ii = None if idx_in is None else np.ascontiguousarray(idx_in, dtype=np.int32).reshape(n, topk)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    rc = _load().qo_decode(_p(q), _p(kc), _p(vc), _p(qi), _p(kp), _p(w), _p(seqlens), B, Lmax, NBk, Hq, Hkv, D, Hi,
                           Di, blk, topk, float(rope_theta), mode, float(scale), _p(seqs), n, _p(ii), _p(idx_out),
                           _p(kth), _p(out), _p(lse), nthreads)
    if rc:
        raise ValueError("index outside the causal range")
    res = dict(out=out, lse=lse)
    if idx_in is None:
        res.update(idx=idx_out, kth=kth)
    return res

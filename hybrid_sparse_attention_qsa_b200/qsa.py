"""ctypes binding of libqsa_b200.so (include/qsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.  PyTorch
supplies device memory (``data_ptr()``) and the current CUDA stream.  There is no fallback: if the
library is missing or the call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
import weakref

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# QSA_DEBUG=1 in the environment (read at import) selects the debug build of the library, whose
# device-side bounds checks record QSA_ERR_DEVICE_CHECK instead of touching memory out of range,
# and puts a canary guard after every buffer this binding allocates (checked by qsa_check_canaries).
DEBUG = os.environ.get("QSA_DEBUG", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libqsa_b200_debug.so" if DEBUG else "libqsa_b200.so")

QSA_OK = 0
QSA_ERR_INVALID_ARGUMENT = 1
QSA_ERR_UNSUPPORTED = 2
QSA_ERR_WORKSPACE_TOO_SMALL = 3
QSA_ERR_CUDA = 4
QSA_ERR_TIMEOUT = 5
QSA_ERR_DEVICE_CHECK = 6

QSA_SCORE_RELU_SUM = 0
QSA_SCORE_LINEAR = 1

QSA_OP_SELECT_TOPK = 1
QSA_OP_SPARSE_ATTN_DECODE = 2
QSA_OP_SPARSE_ATTN_PREFILL = 3

QSA_ATTN_AUTO = 0
QSA_ATTN_ROWS = 1
QSA_ATTN_TILES = 2

# name -> (restype, argtypes), in the order of include/qsa.h
_P, _I, _I64, _F, _SZ, _U64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t,
                               ctypes.c_uint64)
SIGNATURES = {
    "qsa_status_string": (ctypes.c_char_p, [_I]),
    "qsa_abi_version": (_I, []),
    "qsa_pool_block_keys": (_I, [_P, _P, _I, _I, _I, _I, _F, _I64, _I64, _I64, _P]),
    "qsa_pool_block_keys_rope": (_I, [_P, _P, _I, _I, _I, _I, _P, _I64, _I64, _I64, _P]),
    "qsa_rope_index_queries": (_I, [_P, _P, _I, _I, _I, _I, _I64, _P, _F, _P]),
    "qsa_rope_index_queries_rope": (_I, [_P, _P, _I, _I, _I, _I, _I64, _P, _P, _P]),
    "qsa_index_score": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I64, _I, _P, _I64, _P]),
    "qsa_select_topk": (_I, [_P, _I64, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I64, _I, _I, _P, _P, _SZ, _P]),
    "qsa_decode_select": (_I, [_P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P, _P, _SZ, _P]),
    "qsa_sparse_attn_prefill": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I64, _F, _P, _P, _P]),
    "qsa_sparse_attn_prefill_ws": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I64, _F, _P, _P, _P, _SZ,
                                        _P]),
    "qsa_set_attn_options": (_I, [_I]),
    "qsa_attn_prefill_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "qsa_interleave_kv": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I64, _I64, _P]),
    "qsa_sparse_attn_prefill_kv": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I64, _F, _P, _P, _P]),
    "qsa_sparse_attn_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _P]),
    "qsa_sparse_attn_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P]),
    "qsa_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "qsa_decode_default_splits": (_I, [_I, _I]),
    "qsa_decode_split_merge": (_I, [_I, _I, _I, _I, _I]),
    "qsa_get_device_status": (_I, [_P]),
    "qsa_set_select_options": (_I, [_I, _I]),
    "qsa_set_wait_timeout_ns": (None, [_U64]),
    "qsa_wait_timeout_selftest": (_I, [_U64, _P]),
    "qsa_probe_gather": (_I, [_P, _SZ, _I, _I, _I, _I, _I, _I, _I, _U64, _P]),
    "qsa_prefill_host": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I64, _F, _I, _P, _P,
                              _I, _I, _P, _SZ, _P, _P, _P]),
    "qsa_prefill_host_device_bytes": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I64, _I, _I, _I]),
}

_lib = None


class QSAError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call} failed: {status_string(status)} ({status})")


def lib():
    """Load the library once.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m hybrid_sparse_attention_qsa_b200.build`"
                               " (or __graft_entry__.build()); there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().qsa_status_string(status).decode()


def _check(status: int, call: str):
    if status != QSA_OK:
        raise QSAError(status, call)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ------------------------------------------------------------------------------- canary guards
# In debug mode every device buffer this binding allocates (outputs, workspaces, staged inputs) is
# followed by CANARY_BYTES bytes of CANARY_BYTE.  A kernel that writes past the end of its buffer
# changes them; qsa_check_canaries() finds it.
CANARY_BYTES = 256
CANARY_BYTE = 0xA5
_guards: list = []   # (weak reference to the returned tensor, bytes in use, what it holds)


def _empty(*shape, dtype, device, what: str = "buffer") -> torch.Tensor:
    """torch.empty; in debug mode the allocation carries a canary guard after its last byte."""
    if len(shape) == 1 and isinstance(shape[0], (tuple, list, torch.Size)):
        shape = tuple(shape[0])
    if not DEBUG:
        return torch.empty(shape, dtype=dtype, device=device)
    numel = math.prod(shape)
    esz = torch.empty((), dtype=dtype).element_size()
    raw = torch.empty(numel + CANARY_BYTES // esz, dtype=dtype, device=device)
    raw[numel:].view(torch.uint8).fill_(CANARY_BYTE)
    t = raw[:numel].view(shape)   # t._base is raw
    n = numel * esz
    if len(_guards) > 4096:
        _guards[:] = [g for g in _guards if g[0]() is not None]
    _guards.append((weakref.ref(t), n, what))
    return t


def _empty_like(t: torch.Tensor, what: str = "buffer") -> torch.Tensor:
    return _empty(t.shape, dtype=t.dtype, device=t.device, what=what)


def qsa_check_canaries() -> int:
    """Debug mode: synchronise and check the guard after every live buffer the binding allocated.
    Returns how many were checked; raises RuntimeError naming the buffers whose guard changed."""
    if not DEBUG:
        return 0
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    bad, checked = [], 0
    for ref, n, what in _guards:
        t = ref()
        if t is None:     # freed: no longer checked
            continue
        guard = t._base[t.numel():].view(torch.uint8)
        checked += 1
        if bool((guard != CANARY_BYTE).any()):
            bad.append(f"{what} ({n} bytes)")
    if bad:
        raise RuntimeError("canary guard overwritten after: " + ", ".join(bad))
    return checked


# ---------------------------------------------------------------------------------------- ABI calls
def qsa_abi_version() -> int:
    return lib().qsa_abi_version()


def _batch_view_ok(t: torch.Tensor) -> bool:
    """[B, rows, Di] whose rows are packed inside each batch element (batch stride free)."""
    return t.dim() == 3 and t.stride(2) == 1 and t.stride(1) == t.shape[2]


class RopeParams(ctypes.Structure):
    """qsa_rope_params_t: the indexer's rotary base and optional YaRN scaling."""
    _fields_ = [("theta", ctypes.c_double), ("yarn_factor", ctypes.c_double), ("yarn_orig_ctx", ctypes.c_double),
                ("yarn_alpha", ctypes.c_double), ("yarn_beta", ctypes.c_double), ("yarn_mscale", ctypes.c_double)]


def _rope_params(theta: float, yarn: dict | None) -> RopeParams:
    """yarn = dict(factor, orig_ctx[, alpha=1, beta=32, mscale=0 (the paper's default)])."""
    y = yarn or {}
    return RopeParams(float(theta), float(y.get("factor", 1.0)), float(y.get("orig_ctx", 0.0)),
                      float(y.get("alpha", 1.0)), float(y.get("beta", 32.0)), float(y.get("mscale", 0.0)))


def qsa_pool_block_keys(ki: torch.Tensor, kp: torch.Tensor | None = None, *, blk: int = 4, rope_theta: float = 0.0,
                        pos0: int = 0, yarn: dict | None = None) -> torch.Tensor:
    """ki [B, L, Di] bf16 -> kp [B, L // blk, Di] bf16.  ki and kp may be batch-strided views (for
    example the newest block of every sequence of a decode cache: ki[:, 4j:4j+4], kp[:, j:j+1]).
    ``yarn`` (dict(factor, orig_ctx[, alpha, beta, mscale])) scales the rotary frequencies."""
    if not ki.is_cuda or ki.dtype != torch.bfloat16 or not _batch_view_ok(ki):
        raise ValueError("ki must be a CUDA bf16 [B, L, Di] tensor with packed rows")
    B, L, Di = ki.shape
    if kp is None:
        kp = _empty(B, L // blk, Di, dtype=torch.bfloat16, device=ki.device, what="kp")
    if kp.dtype != torch.bfloat16 or not _batch_view_ok(kp) or tuple(kp.shape) != (B, L // blk, Di):
        raise ValueError("kp must be a bf16 [B, L // blk, Di] tensor with packed rows")
    if yarn:
        rp = _rope_params(rope_theta, yarn)
        _check(lib().qsa_pool_block_keys_rope(_ptr(ki), _ptr(kp), B, L, Di, blk, ctypes.byref(rp), pos0, ki.stride(0),
                                              kp.stride(0), _stream(ki.device)), "qsa_pool_block_keys_rope")
        return kp
    _check(lib().qsa_pool_block_keys(_ptr(ki), _ptr(kp), B, L, Di, blk, rope_theta, pos0, ki.stride(0), kp.stride(0),
                                     _stream(ki.device)), "qsa_pool_block_keys")
    return kp


def qsa_rope_index_queries(qi: torch.Tensor, qi_out: torch.Tensor | None = None, *, rope_theta: float, q_pos0: int = 0,
                           seqlens: torch.Tensor | None = None, yarn: dict | None = None) -> torch.Tensor:
    """qi [B, Tq, Hi, Di] (or [B, Hi, Di] with seqlens) rotated at its positions."""
    _need(qi, torch.bfloat16, "qi")
    if seqlens is not None:
        _need(seqlens, torch.int32, "seqlens")
        B, Hi, Di = qi.shape
        Tq = 1
    else:
        B, Tq, Hi, Di = qi.shape
    if qi_out is None:
        qi_out = _empty_like(qi, what="rotated qi")
    if yarn:
        rp = _rope_params(rope_theta, yarn)
        _check(lib().qsa_rope_index_queries_rope(_ptr(qi), _ptr(qi_out), B, Tq, Hi, Di, q_pos0, _ptr(seqlens),
                                                 ctypes.byref(rp), _stream(qi.device)), "qsa_rope_index_queries_rope")
        return qi_out
    _check(lib().qsa_rope_index_queries(_ptr(qi), _ptr(qi_out), B, Tq, Hi, Di, q_pos0, _ptr(seqlens), rope_theta,
                                        _stream(qi.device)), "qsa_rope_index_queries")
    return qi_out


def qsa_index_score(qi: torch.Tensor, kp: torch.Tensor, *, head_w: torch.Tensor | None = None,
                    seqlens: torch.Tensor | None = None, q_pos0: int = 0, mode: int = QSA_SCORE_RELU_SUM,
                    scores: torch.Tensor | None = None, blk: int = 4) -> torch.Tensor:
    """Prefill: qi [B, Tq, Hi, Di]; decode: qi [B, Hi, Di] with seqlens [B].  kp [B, NBk, Di].
    Returns scores [B, Tq, NBk] fp32 (entries beyond each query's candidates are left as they were)."""
    _need(qi, torch.bfloat16, "qi")
    _need(kp, torch.bfloat16, "kp")
    if seqlens is not None:
        _need(seqlens, torch.int32, "seqlens")
        B, Hi, Di = qi.shape
        Tq = 1
    else:
        B, Tq, Hi, Di = qi.shape
    NBk = kp.shape[1]
    if scores is None:
        scores = _empty((B, Tq, max(NBk, 1)), dtype=torch.float32, device=qi.device, what="scores").fill_(float("nan"))
    _need(scores, torch.float32, "scores")
    if head_w is not None:
        _need(head_w, torch.float32, "head_w")
    _check(lib().qsa_index_score(_ptr(qi), _ptr(kp), _ptr(head_w), _ptr(seqlens), B, Tq, NBk, Hi, Di, blk, q_pos0,
                                 mode, _ptr(scores), scores.shape[-1], _stream(qi.device)), "qsa_index_score")
    return scores


def qsa_workspace_size(op: int, B: int, Tq: int, NBk: int, k: int, Hq: int, D: int, num_splits: int = 0) -> int:
    return int(lib().qsa_workspace_size(op, B, Tq, NBk, k, Hq, D, num_splits))


def qsa_select_topk(k: int, *, scores: torch.Tensor | None = None, qi: torch.Tensor | None = None,
                    kp: torch.Tensor | None = None, head_w: torch.Tensor | None = None,
                    seqlens: torch.Tensor | None = None, q_pos0: int = 0, mode: int = QSA_SCORE_RELU_SUM,
                    NBk: int | None = None, idx: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                    blk: int = 4) -> torch.Tensor:
    """Top-k block lists idx [B, Tq, k] int32 (decode: [B, k]).

    From materialised ``scores`` [B, Tq, ld] (then NBk must be given or defaults to ld), or from
    ``qi``/``kp`` with the scores computed chunk-wise in ``workspace`` (allocated if omitted)."""
    ref = scores if scores is not None else qi
    dev = ref.device
    if scores is not None:
        _need(scores, torch.float32, "scores")
        B, Tq, ld = scores.shape
        NBk = ld if NBk is None else NBk
        Hi = Di = 0
    else:
        _need(qi, torch.bfloat16, "qi")
        _need(kp, torch.bfloat16, "kp")
        if seqlens is not None:
            B, Hi, Di = qi.shape
            Tq = 1
        else:
            B, Tq, Hi, Di = qi.shape
        NBk = kp.shape[1]
        ld = 0
        if workspace is None:
            nbytes = qsa_workspace_size(QSA_OP_SELECT_TOPK, B, Tq, NBk, k, 0, 0)
            workspace = _empty(nbytes, dtype=torch.uint8, device=dev, what="select workspace")
    if seqlens is not None:
        _need(seqlens, torch.int32, "seqlens")
    if idx is None:
        idx = _empty((B, k) if seqlens is not None else (B, Tq, k), dtype=torch.int32, device=dev, what="idx")
    _need(idx, torch.int32, "idx")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().qsa_select_topk(_ptr(scores), ld, _ptr(qi), _ptr(kp), _ptr(head_w), _ptr(seqlens), B, Tq, NBk, Hi,
                                 Di, blk, q_pos0, mode, k, _ptr(idx), _ptr(workspace), ws_bytes, _stream(dev)),
           "qsa_select_topk")
    return idx


def qsa_decode_select(k: int, *, qi: torch.Tensor, kp: torch.Tensor, ki: torch.Tensor, seqlens: torch.Tensor,
                      head_w: torch.Tensor | None = None, mode: int = QSA_SCORE_RELU_SUM, rope_theta: float = 0.0,
                      yarn: dict | None = None, idx: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None, blk: int = 4) -> torch.Tensor:
    """One decode step's selection with the pooling of the newest block folded in: for every
    sequence whose new token completes a block, kp[b, seqlens[b] // blk - 1] is pooled from the
    key cache ki [B, Lmax, Di] first (as qsa_pool_block_keys would), then idx [B, k] is selected as
    qsa_select_topk(k, qi=qi, kp=kp, seqlens=seqlens).  kp is updated in place."""
    _need(qi, torch.bfloat16, "qi")
    _need(kp, torch.bfloat16, "kp")
    _need(seqlens, torch.int32, "seqlens")
    if not ki.is_cuda or ki.dtype != torch.bfloat16 or not _batch_view_ok(ki):
        raise ValueError("ki must be a CUDA bf16 [B, Lmax, Di] tensor with packed rows")
    B, Hi, Di = qi.shape
    NBk = kp.shape[1]
    if workspace is None:
        workspace = _empty(qsa_workspace_size(QSA_OP_SELECT_TOPK, B, 1, NBk, k, 0, 0), dtype=torch.uint8,
                           device=qi.device, what="select workspace")
    if idx is None:
        idx = _empty((B, k), dtype=torch.int32, device=qi.device, what="idx")
    _need(idx, torch.int32, "idx")
    # without YaRN the rotary base goes through fp32, as in qsa_pool_block_keys(rope_theta=...)
    rp = _rope_params(rope_theta if yarn else ctypes.c_float(rope_theta).value, yarn)
    _check(lib().qsa_decode_select(_ptr(qi), _ptr(kp), _ptr(ki), ki.stride(0), _ptr(head_w), _ptr(seqlens), B, NBk,
                                   Hi, Di, blk, mode, ctypes.byref(rp), k, _ptr(idx), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(qi.device)),
           "qsa_decode_select")
    return idx


def qsa_sparse_attn_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor, *, q_pos0: int = 0,
                            scale: float | None = None, out: torch.Tensor | None = None,
                            lse: torch.Tensor | None = None, want_lse: bool = True, blk: int = 4,
                            workspace: torch.Tensor | None = None, tiles: bool = True):
    """q [B, Tq, Hq, D], k/v [B, Tk, Hkv, D], idx [B, Tq, kb] -> (out [B, Tq, Hq, D], lse [B, Tq, Hq]).

    With ``tiles`` (default) the call goes through qsa_sparse_attn_prefill_ws with ``workspace``
    (allocated here when omitted, qsa_attn_prefill_workspace_size bytes), which runs the path
    qsa_set_attn_options chose (automatic: row by row over K/V interleaved by block in the
    workspace where the shape allows; QSA_ATTN_ROWS: row by row over k and v; QSA_ATTN_TILES: query
    tiles on tcgen05 where the shape allows).  ``tiles=False`` calls qsa_sparse_attn_prefill (row by
    row, no workspace)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    _need(idx, torch.int32, "idx")
    B, Tq, Hq, D = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    kb = idx.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if out is None:
        out = _empty_like(q, what="out")
    if lse is None and want_lse:
        lse = _empty(B, Tq, Hq, dtype=torch.float32, device=q.device, what="lse")
    if not tiles:
        _check(lib().qsa_sparse_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), B, Tq, Tk, Hq, Hkv, D, kb, blk,
                                             q_pos0, scale, _ptr(out), _ptr(lse), _stream(q.device)),
               "qsa_sparse_attn_prefill")
        return out, lse
    if workspace is None:
        nbytes = qsa_attn_prefill_workspace_size(B, Tq, Tk, Hq, Hkv, D, kb)
        workspace = _empty(max(nbytes, 16), dtype=torch.uint8, device=q.device, what="attention workspace")
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().qsa_sparse_attn_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), B, Tq, Tk, Hq, Hkv, D, kb, blk,
                                            q_pos0, scale, _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
                                            _stream(q.device)), "qsa_sparse_attn_prefill_ws")
    return out, lse


def qsa_attn_prefill_workspace_size(B: int, Tq: int, Tk: int, Hq: int, Hkv: int, D: int, k_blocks: int) -> int:
    return int(lib().qsa_attn_prefill_workspace_size(B, Tq, Tk, Hq, Hkv, D, k_blocks))


def qsa_interleave_kv(k: torch.Tensor, v: torch.Tensor, kv: torch.Tensor | None = None, *, pos_lo: int = 0,
                      pos_hi: int | None = None, blk: int = 4) -> torch.Tensor:
    """k, v [B, Tk, Hkv, D] -> kv [B, ceil(Tk / blk), 2, blk, Hkv, D]: K and V interleaved by block
    (positions >= Tk zero); writes the blocks holding positions [pos_lo, pos_hi)."""
    _need(k, torch.bfloat16, "k")
    _need(v, torch.bfloat16, "v")
    B, Tk, Hkv, D = k.shape
    if kv is None:
        kv = _empty(B, (Tk + blk - 1) // blk, 2, blk, Hkv, D, dtype=torch.bfloat16, device=k.device,
                    what="interleaved kv")
    _need(kv, torch.bfloat16, "kv")
    pos_hi = Tk if pos_hi is None else pos_hi
    _check(lib().qsa_interleave_kv(_ptr(k), _ptr(v), _ptr(kv), B, Tk, Hkv, D, blk, pos_lo, pos_hi,
                                   _stream(k.device)), "qsa_interleave_kv")
    return kv


def qsa_sparse_attn_prefill_kv(q: torch.Tensor, kv: torch.Tensor, idx: torch.Tensor, *, Tk: int, q_pos0: int = 0,
                               scale: float | None = None, out: torch.Tensor | None = None,
                               lse: torch.Tensor | None = None, blk: int = 4):
    """qsa_sparse_attn_prefill over kv from qsa_interleave_kv (Tk: the positions of k and v)."""
    _need(q, torch.bfloat16, "q")
    _need(kv, torch.bfloat16, "kv")
    _need(idx, torch.int32, "idx")
    B, Tq, Hq, D = q.shape
    Hkv = kv.shape[4]
    kb = idx.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if out is None:
        out = _empty_like(q, what="out")
    if lse is None:
        lse = _empty(B, Tq, Hq, dtype=torch.float32, device=q.device, what="lse")
    _check(lib().qsa_sparse_attn_prefill_kv(_ptr(q), _ptr(kv), _ptr(idx), B, Tq, Tk, Hq, Hkv, D, kb, blk, q_pos0,
                                            scale, _ptr(out), _ptr(lse), _stream(q.device)),
           "qsa_sparse_attn_prefill_kv")
    return out, lse


def qsa_set_attn_options(path: int = QSA_ATTN_AUTO) -> None:
    """Prefill attention of qsa_sparse_attn_prefill_ws for later calls: QSA_ATTN_AUTO (row by row),
    QSA_ATTN_ROWS or QSA_ATTN_TILES."""
    _check(lib().qsa_set_attn_options(path), "qsa_set_attn_options")


def qsa_sparse_attn_decode(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, seqlens: torch.Tensor,
                           idx: torch.Tensor, *, scale: float | None = None, num_splits: int = 0,
                           out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None, want_lse: bool = True, blk: int = 4):
    """q [B, Hq, D], caches [B, Lmax, Hkv, D], seqlens [B], idx [B, kb] -> (out [B, Hq, D], lse [B, Hq])."""
    for t, n in ((q, "q"), (kcache, "kcache"), (vcache, "vcache")):
        _need(t, torch.bfloat16, n)
    _need(seqlens, torch.int32, "seqlens")
    _need(idx, torch.int32, "idx")
    B, Hq, D = q.shape
    Lmax, Hkv = kcache.shape[1], kcache.shape[2]
    kb = idx.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if out is None:
        out = _empty_like(q, what="out")
    if lse is None and want_lse:
        lse = _empty(B, Hq, dtype=torch.float32, device=q.device, what="lse")
    if workspace is None:
        nbytes = qsa_workspace_size(QSA_OP_SPARSE_ATTN_DECODE, B, 1, 0, kb, Hq, D, num_splits)
        workspace = _empty(max(nbytes, 16), dtype=torch.uint8, device=q.device, what="attention workspace")
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().qsa_sparse_attn_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(idx), B, Lmax, Hq, Hkv,
                                        D, kb, blk, scale, num_splits, _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
                                        _stream(q.device)), "qsa_sparse_attn_decode")
    return out, lse


def qsa_sparse_attn_decode_noalloc(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor,
                                   seqlens: torch.Tensor, idx: torch.Tensor, *, scale: float | None = None,
                                   num_splits: int = 0, out: torch.Tensor | None = None,
                                   lse: torch.Tensor | None = None, blk: int = 4):
    """qsa_sparse_attn_decode without a workspace: the split partials live in the library's own
    per-GPU scratch array (for callers that cannot allocate).  Pass ``out``/``lse`` to allocate
    nothing at all here either."""
    for t, n in ((q, "q"), (kcache, "kcache"), (vcache, "vcache")):
        _need(t, torch.bfloat16, n)
    _need(seqlens, torch.int32, "seqlens")
    _need(idx, torch.int32, "idx")
    B, Hq, D = q.shape
    Lmax, Hkv = kcache.shape[1], kcache.shape[2]
    kb = idx.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if out is None:
        out = _empty_like(q, what="out")
    _check(lib().qsa_sparse_attn_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(idx), B,
                                                Lmax, Hq, Hkv, D, kb, blk, scale, num_splits, _ptr(out), _ptr(lse),
                                                _stream(q.device)), "qsa_sparse_attn_decode_noalloc")
    return out, lse


def qsa_decode_default_splits(B: int, k_blocks: int) -> int:
    """Split count qsa_sparse_attn_decode picks for num_splits == 0 on the current device."""
    return lib().qsa_decode_default_splits(B, k_blocks)


def qsa_decode_split_merge(B: int, Hq: int, Hkv: int, D: int, num_splits: int) -> int:
    """0: one split; 1: splits merged inside thread-block clusters; 2: through workspace partials and
    the merge kernel; -1: invalid sizes or no usable device."""
    return lib().qsa_decode_split_merge(B, Hq, Hkv, D, num_splits)


def qsa_get_device_status(device=None) -> int:
    """Synchronise the current stream and read + clear the device status word."""
    return int(lib().qsa_get_device_status(_stream(device)))


QSA_SELECT_AUTO, QSA_SELECT_MATERIALISED, QSA_SELECT_FILTERED = 0, 1, 2


def qsa_set_select_options(path: int = QSA_SELECT_AUTO, sample_rank: int = 0) -> None:
    """How qsa_select_topk computes a prefill selection without given scores (process-wide)."""
    _check(lib().qsa_set_select_options(path, sample_rank), "qsa_set_select_options")


def qsa_set_wait_timeout_ns(ns: int) -> None:
    lib().qsa_set_wait_timeout_ns(ns)


def qsa_wait_timeout_selftest(timeout_ns: int, device=None) -> None:
    _check(lib().qsa_wait_timeout_selftest(timeout_ns, _stream(device)), "qsa_wait_timeout_selftest")


# ---------------------------------------------------------------------------------------- whole path
def qsa_probe_gather(src: torch.Tensor, *, chunk_bytes: int = 2048, method: int = 0, issuer_warps: int = 4,
                     stages: int = 3, slots_per_warp: int = 8, iterations: int = 1000, ctas: int = 0,
                     seed: int = 1) -> int:
    """Gather-rate probe over the bytes of ``src`` (a contiguous CUDA tensor); returns the bytes the
    launch delivers to shared memory.  Time it with CUDA events on the current stream."""
    if not src.is_cuda or not src.is_contiguous():
        raise ValueError("src must be a contiguous CUDA tensor")
    nbytes = src.numel() * src.element_size()
    _check(lib().qsa_probe_gather(_ptr(src), nbytes, chunk_bytes, method, issuer_warps, stages, slots_per_warp,
                                  iterations, ctas, seed, _stream(src.device)), "qsa_probe_gather")
    n_ctas = ctas or torch.cuda.get_device_properties(src.device).multi_processor_count
    return n_ctas * issuer_warps * iterations * slots_per_warp * chunk_bytes


def prefill(q, k, v, qi, ki, *, topk: int, q_pos0: int = 0, rope_theta: float = 0.0, head_w=None,
            mode: int = QSA_SCORE_RELU_SUM, scale: float | None = None, workspace=None, kp=None, yarn=None):
    """The QSA layer for a prefill: pool (+RoPE) -> [RoPE queries] -> score + top-k -> sparse attention.
    Returns dict(out, lse, idx, kp)."""
    if kp is None:
        kp = qsa_pool_block_keys(ki, rope_theta=rope_theta, yarn=yarn)
    qr = qsa_rope_index_queries(qi, rope_theta=rope_theta, q_pos0=q_pos0, yarn=yarn) if rope_theta > 0 else qi
    idx = qsa_select_topk(topk, qi=qr, kp=kp, head_w=head_w, q_pos0=q_pos0, mode=mode, workspace=workspace)
    out, lse = qsa_sparse_attn_prefill(q, k, v, idx, q_pos0=q_pos0, scale=scale)
    return dict(out=out, lse=lse, idx=idx, kp=kp)


def decode(q, kcache, vcache, qi, kp, seqlens, *, topk: int, rope_theta: float = 0.0, head_w=None,
           mode: int = QSA_SCORE_RELU_SUM, scale: float | None = None, num_splits: int = 0, workspace=None,
           yarn=None):
    """One decode step on a pooled indexer-key cache kp [B, NBk, Di]: [RoPE query] -> score + top-k
    -> split-KV sparse attention.  Returns dict(out, lse, idx)."""
    qr = qsa_rope_index_queries(qi, rope_theta=rope_theta, seqlens=seqlens, yarn=yarn) if rope_theta > 0 else qi
    idx = qsa_select_topk(topk, qi=qr, kp=kp, head_w=head_w, seqlens=seqlens, mode=mode, workspace=workspace)
    out, lse = qsa_sparse_attn_decode(q, kcache, vcache, seqlens, idx, scale=scale, num_splits=num_splits)
    return dict(out=out, lse=lse, idx=idx)



def qsa_prefill_host_device_bytes(B: int, Tq: int, Tk: int, Hq: int, Hkv: int, D: int, Hi: int, Di: int, k: int, *,
                                  q_pos0: int = 0, rope: bool = False, chunks: int = 0, sel_chunks: int = 2,
                                  blk: int = 4) -> int:
    return int(lib().qsa_prefill_host_device_bytes(B, Tq, Tk, Hq, Hkv, D, Hi, Di, k, blk, q_pos0, 1 if rope else 0,
                                                   chunks, sel_chunks))


def prefill_host(q, k, v, qi, ki, *, topk: int, device="cuda", out=None, q_pos0: int = 0, rope_theta: float = 0.0,
                 head_w=None, mode: int = QSA_SCORE_RELU_SUM, scale: float | None = None,
                 device_buffers: dict | None = None, chunks: int = 0, sel_chunks: int = 2, yarn=None):
    """The QSA layer for a prefill whose inputs live in (pinned) host memory, through
    qsa_prefill_host: the library copies the inputs in causal row chunks on its own copy streams,
    starts each chunk's pooling + selection and attention as soon as its data has arrived, and sends
    each chunk's output rows back while the next is computed (``chunks`` equal attention chunks, or
    0: quarters, then halving chunks).  ``device_buffers`` (a dict) keeps the
    device scratch ("scratch"), the index lists ("idx") and the log-sum-exps ("lse") for reuse.
    Returns dict(out=host tensor, lse=device tensor, idx=device tensor); the output is complete once
    the current stream of ``device`` has reached this call."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (qi, "qi"), (ki, "ki")):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous bf16 host tensor")
    dev = torch.device(device)
    B, Tq, Hq, D = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    Hi, Di = qi.shape[2], qi.shape[3]
    rope = _rope_params(rope_theta, yarn) if rope_theta > 0 else None
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    nbytes = qsa_prefill_host_device_bytes(B, Tq, Tk, Hq, Hkv, D, Hi, Di, topk, q_pos0=q_pos0, rope=rope is not None,
                                           chunks=chunks, sel_chunks=sel_chunks)
    if nbytes == 0:
        raise ValueError("invalid sizes for qsa_prefill_host")
    bufs = device_buffers if device_buffers is not None else {}
    if "scratch" not in bufs or bufs["scratch"].numel() < nbytes:
        bufs["scratch"] = _empty(nbytes, dtype=torch.uint8, device=dev, what="host pipeline scratch")
    if "idx" not in bufs:
        bufs["idx"] = _empty(B, Tq, topk, dtype=torch.int32, device=dev, what="idx")
    if "lse" not in bufs:
        bufs["lse"] = _empty(B, Tq, Hq, dtype=torch.float32, device=dev, what="lse")
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if head_w is not None:
        _need(head_w, torch.float32, "head_w")
    scratch, idx, lse = bufs["scratch"], bufs["idx"], bufs["lse"]
    with torch.cuda.device(dev):
        _check(lib().qsa_prefill_host(_ptr(q), _ptr(k), _ptr(v), _ptr(qi), _ptr(ki), _ptr(out), B, Tq, Tk, Hq, Hkv, D,
                                      Hi, Di, topk, 4, q_pos0, scale, mode, _ptr(head_w),
                                      ctypes.byref(rope) if rope is not None else None, chunks, sel_chunks,
                                      _ptr(scratch), scratch.numel(), _ptr(idx), _ptr(lse), _stream(dev)),
               "qsa_prefill_host")
    return dict(out=out, lse=lse, idx=idx)

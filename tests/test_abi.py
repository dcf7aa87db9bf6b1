"""The C-ABI library: it loads without a GPU, exports every symbol include/qsa.h declares, and
rejects bad arguments on the host before any launch (no GPU needed for those paths)."""
import ctypes
import os
import re

import pytest

from hybrid_sparse_attention_qsa_b200 import build as B
from hybrid_sparse_attention_qsa_b200 import qsa as Q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return Q.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "qsa.h")).read()
    return sorted(set(re.findall(r"QSA_API\s+[\w\s\*]+?\b(qsa_\w+)\s*\(", src)))


def test_header_declares_the_four_hot_path_calls():
    names = declared_symbols()
    for n in ("qsa_index_score", "qsa_select_topk", "qsa_sparse_attn_prefill", "qsa_sparse_attn_decode",
              "qsa_pool_block_keys"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(Q.SIGNATURES), "binding and header disagree"


def test_debug_library_exports_the_same_symbols():
    # the debug build (-DQSA_DEBUG): same ABI, device-side bounds checks compiled in
    path = B.build(debug=True)
    assert path == B.LIB_DEBUG
    dl = ctypes.CDLL(path)
    for n in declared_symbols():
        assert hasattr(dl, n), n
    dl.qsa_status_string.restype = ctypes.c_char_p
    assert dl.qsa_status_string(Q.QSA_ERR_DEVICE_CHECK) == b"QSA_ERR_DEVICE_CHECK"


def test_abi_version_and_status_strings(lib):
    assert Q.qsa_abi_version() == 1
    assert Q.status_string(Q.QSA_ERR_WORKSPACE_TOO_SMALL) == "QSA_ERR_WORKSPACE_TOO_SMALL"
    assert Q.status_string(99) == "QSA_ERR_UNKNOWN"


P = ctypes.c_void_p
FAKE = P(1 << 20)          # never dereferenced: every call below fails its host-side checks


def test_pool_argument_checks(lib):
    assert lib.qsa_pool_block_keys(None, None, 1, 8, 64, 4, 0.0, 0, 0, 0, None) == Q.QSA_ERR_INVALID_ARGUMENT
    assert lib.qsa_pool_block_keys(FAKE, FAKE, 1, 8, 63, 4, 0.0, 0, 0, 0, None) == Q.QSA_ERR_INVALID_ARGUMENT
    assert lib.qsa_pool_block_keys(FAKE, FAKE, 1, 8, 64, 3, 0.0, 0, 0, 0, None) == Q.QSA_ERR_UNSUPPORTED
    assert lib.qsa_pool_block_keys(P(17), FAKE, 1, 8, 64, 4, 0.0, 0, 0, 0, None) == Q.QSA_ERR_INVALID_ARGUMENT
    assert lib.qsa_pool_block_keys(None, None, 0, 8, 64, 4, 0.0, 0, 0, 0, None) == Q.QSA_OK      # empty: nothing to do
    assert lib.qsa_pool_block_keys(None, None, 1, 3, 64, 4, 0.0, 0, 0, 0, None) == Q.QSA_OK      # no complete block


def test_score_argument_checks(lib):
    args = lambda **kw: dict(dict(qi=FAKE, kp=FAKE, w=None, sl=None, B=1, Tq=8, NBk=2, Hi=4, Di=64, blk=4, q0=0, mode=0,
                                  s=FAKE, ld=2), **kw)

    def call(**kw):
        a = args(**kw)
        return lib.qsa_index_score(a["qi"], a["kp"], a["w"], a["sl"], a["B"], a["Tq"], a["NBk"], a["Hi"], a["Di"],
                                   a["blk"], a["q0"], a["mode"], a["s"], a["ld"], None)

    assert call(Di=128) == Q.QSA_ERR_UNSUPPORTED
    assert call(Hi=3) == Q.QSA_ERR_UNSUPPORTED
    assert call(mode=2) == Q.QSA_ERR_INVALID_ARGUMENT
    # row 11 has 2 candidates and kp holds NBk = 2 rows: valid; row 12 would need 3
    assert call(Tq=13, NBk=2) == Q.QSA_ERR_INVALID_ARGUMENT   # ... row 12 needs 3 > NBk = 2
    assert call(q0=5, Tq=8) == Q.QSA_ERR_INVALID_ARGUMENT      # row at position 12 again
    assert call(ld=1) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(sl=FAKE, Tq=2) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(qi=P(8)) == Q.QSA_ERR_INVALID_ARGUMENT


def test_select_and_attention_argument_checks(lib):
    # k < 1
    assert lib.qsa_select_topk(FAKE, 8, None, None, None, None, 1, 4, 8, 4, 64, 4, 0, 0, 0, FAKE, None, 0,
                               None) == Q.QSA_ERR_INVALID_ARGUMENT
    # scores == NULL needs a workspace
    assert lib.qsa_select_topk(None, 0, FAKE, FAKE, None, None, 1, 40, 10, 4, 64, 4, 0, 0, 8, FAKE, None, 0,
                               None) == Q.QSA_ERR_WORKSPACE_TOO_SMALL
    # decode with too small a workspace
    assert lib.qsa_select_topk(None, 0, FAKE, FAKE, None, FAKE, 2, 1, 10, 4, 64, 4, 0, 0, 8, FAKE, FAKE, 40,
                               None) == Q.QSA_ERR_WORKSPACE_TOO_SMALL
    pre = lambda D=128, Hq=16, Hkv=2, blk=4, Tq=8, Tk=8, q0=0: lib.qsa_sparse_attn_prefill(
        FAKE, FAKE, FAKE, FAKE, 1, Tq, Tk, Hq, Hkv, D, 8, blk, q0, ctypes.c_float(0.1), FAKE, None, None)
    assert pre(D=64) == Q.QSA_ERR_UNSUPPORTED
    assert pre(Hkv=4, Hq=16) == Q.QSA_ERR_UNSUPPORTED
    assert pre(Hq=34, Hkv=2) == Q.QSA_ERR_UNSUPPORTED        # groups of more than 16 query heads
    assert pre(D=512) == Q.QSA_ERR_UNSUPPORTED
    # the model shape (24 query heads over 2 KV heads at head dimension 256) passes the shape checks
    assert pre(Hq=24, Hkv=2, D=256) not in (Q.QSA_ERR_UNSUPPORTED, Q.QSA_ERR_INVALID_ARGUMENT)
    assert pre(Hq=15, Hkv=2) == Q.QSA_ERR_INVALID_ARGUMENT
    assert pre(blk=8) == Q.QSA_ERR_UNSUPPORTED
    assert pre(q0=4) == Q.QSA_ERR_INVALID_ARGUMENT           # q0 + Tq > Tk
    dec = lambda ws, nbytes, splits: lib.qsa_sparse_attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 100, 16, 2, 128, 64, 4,
                                                                ctypes.c_float(0.1), splits, FAKE, None, ws, nbytes,
                                                                None)
    assert dec(None, 0, -1) == Q.QSA_ERR_INVALID_ARGUMENT


def filtered_bytes(rows, nbk, k):
    # the filtered selection's workspace as include/qsa.h states it: per row the sampled scores
    # (every 16th block, padded to 4), threshold, count and failure slot, and the candidate list
    # of 32 * max(64, ceil(2k/16)) (key, block) pairs; plus 128 scratch rows and alignment
    rank = max(64, (2 * k + 15) // 16)
    ns = (nbk - 9) // 16 + 1 if nbk > 8 else 0
    per_row = ((max(ns, 1) + 3) // 4 * 4) * 4 + 12 + 32 * rank * 8
    return 12 * 256 + 4 + 128 * max(nbk, 1) * 4 + rows * per_row


def test_workspace_sizes(lib):
    # 128K prefill: every row fits the filtered path in one chunk (under 4 GiB)
    n = Q.qsa_workspace_size(Q.QSA_OP_SELECT_TOPK, 1, 131072, 32768, 512, 16, 128)
    assert n == filtered_bytes(131072, 32768, 512) and n <= 4 << 30
    # 1M prefill: chunks of rows within 4 GiB, never less than a 512 MiB chunk of score rows
    n = Q.qsa_workspace_size(Q.QSA_OP_SELECT_TOPK, 1, 1048576, 262144, 512, 16, 128)
    assert (512 << 20) <= n <= 4 << 30
    # short prefill: the materialised chunk of all rows can be the larger of the two
    n = Q.qsa_workspace_size(Q.QSA_OP_SELECT_TOPK, 1, 2048, 512, 64, 1, 128)
    assert n == max(2048 * 512 * 4, filtered_bytes(2048, 512, 64))
    assert Q.qsa_workspace_size(Q.QSA_OP_SELECT_TOPK, 32, 1, 65536, 512, 16, 128) == 32 * 65536 * 4
    assert Q.qsa_workspace_size(Q.QSA_OP_SPARSE_ATTN_DECODE, 32, 1, 0, 512, 16, 128, 5) == 32 * 5 * 16 * 130 * 4
    assert Q.qsa_workspace_size(99, 1, 1, 1, 1, 1, 1) == 0


def test_select_options_checks(lib):
    assert lib.qsa_set_select_options(3, 0) == Q.QSA_ERR_INVALID_ARGUMENT
    assert lib.qsa_set_select_options(-1, 0) == Q.QSA_ERR_INVALID_ARGUMENT
    assert lib.qsa_set_select_options(0, -5) == Q.QSA_ERR_INVALID_ARGUMENT
    assert lib.qsa_set_select_options(2, 7) == Q.QSA_OK
    assert lib.qsa_set_select_options(0, 0) == Q.QSA_OK


def test_rope_params_checks(lib):
    rp = Q.RopeParams(10000.0, 4.0, 0.0, 1.0, 32.0, 0.0)      # YaRN without an original context
    assert lib.qsa_pool_block_keys_rope(1, 1, 1, 8, 64, 4, ctypes.byref(rp), 0, 0, 0, None) == Q.QSA_ERR_INVALID_ARGUMENT
    rp = Q.RopeParams(10000.0, 4.0, 4096.0, 32.0, 1.0, 0.0)   # ramp bounds reversed
    assert lib.qsa_pool_block_keys_rope(1, 1, 1, 8, 64, 4, ctypes.byref(rp), 0, 0, 0, None) == Q.QSA_ERR_INVALID_ARGUMENT
    rp = Q.RopeParams(0.0, 1.0, 0.0, 1.0, 32.0, 0.0)          # the query rotation needs a base
    assert lib.qsa_rope_index_queries_rope(1, 1, 1, 4, 4, 64, 0, None, ctypes.byref(rp), None) == Q.QSA_ERR_INVALID_ARGUMENT
    assert lib.qsa_rope_index_queries_rope(1, 1, 1, 4, 4, 64, 0, None, None, None) == Q.QSA_ERR_INVALID_ARGUMENT


def test_decode_split_merge_host_rules(lib):
    # one split never merges; invalid sizes are refused before any device query
    assert lib.qsa_decode_split_merge(32, 16, 2, 128, 1) == 0
    assert lib.qsa_decode_split_merge(0, 16, 2, 128, 4) == -1
    assert lib.qsa_decode_split_merge(4, 16, 3, 128, 4) == -1   # Hq not a multiple of Hkv
    assert lib.qsa_decode_split_merge(4, 16, 2, 128, 0) == -1


def test_decode_select_argument_checks(lib):
    """Host-side checks run before any device work (no GPU needed)."""
    def call(qi=FAKE, kp=FAKE, ki=FAKE, kis=0, sl=FAKE, B=2, NBk=64, Hi=4, Di=64, blk=4, mode=0, rope=None, k=8,
             idx=FAKE, ws=FAKE, wsb=1 << 20):
        return lib.qsa_decode_select(qi, kp, ki, kis, None, sl, B, NBk, Hi, Di, blk, mode, rope, k, idx, ws, wsb, None)
    assert call(k=0) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(blk=8) == Q.QSA_ERR_UNSUPPORTED
    assert call(B=0) == Q.QSA_OK                                  # nothing to do
    assert call(sl=None) == Q.QSA_ERR_INVALID_ARGUMENT            # decode needs the lengths
    assert call(idx=None) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(ki=None) == Q.QSA_ERR_INVALID_ARGUMENT            # the key cache to pool from
    assert call(ki=P(8)) == Q.QSA_ERR_INVALID_ARGUMENT            # misaligned
    assert call(kis=100) == Q.QSA_ERR_INVALID_ARGUMENT            # a row shorter than NBk * blk keys
    assert call(Di=32) == Q.QSA_ERR_UNSUPPORTED
    assert call(mode=2) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(wsb=16) == Q.QSA_ERR_WORKSPACE_TOO_SMALL          # less than the B score rows
    rp = Q.RopeParams(10000.0, 4.0, 0.0, 1.0, 32.0, 0.0)         # YaRN without an original context
    assert call(rope=ctypes.byref(rp)) == Q.QSA_ERR_INVALID_ARGUMENT


def test_declared_attention_shape_limits(lib):
    """The supported-shape line of include/qsa.h and the host checks of the attention calls agree."""
    src = open(os.path.join(ROOT, "include", "qsa.h")).read()
    m = re.search(r"attention D in \{([0-9, ]+)\}, Hkv in \{([0-9, ]+)\}, Hq/Hkv <= (\d+)", src)
    assert m, "the header states the attention shapes"
    dims = [int(x) for x in m.group(1).split(",")]
    hkvs = [int(x) for x in m.group(2).split(",")]
    gmax = int(m.group(3))
    assert dims == [128, 256] and hkvs == [1, 2] and gmax == 16

    def pre(D, Hq, Hkv):
        return lib.qsa_sparse_attn_prefill(FAKE, FAKE, FAKE, FAKE, 1, 8, 8, Hq, Hkv, D, 8, 4, 0, ctypes.c_float(0.1),
                                           FAKE, None, P(0), )

    def dec(D, Hq, Hkv):
        return lib.qsa_sparse_attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 100, Hq, Hkv, D, 64, 4, ctypes.c_float(0.1),
                                          -1, FAKE, None, None, 0, None)

    for D in (64, 96, 192, 512):
        assert pre(D, 16, 2) == Q.QSA_ERR_UNSUPPORTED
    for Hkv in hkvs:
        for D in dims:
            # the largest declared group passes the shape checks (it then fails only on num_splits = -1)
            assert dec(D, gmax * Hkv, Hkv) == Q.QSA_ERR_INVALID_ARGUMENT
            assert dec(D, (gmax + 1) * Hkv, Hkv) == Q.QSA_ERR_UNSUPPORTED
            assert pre(D, (gmax + 1) * Hkv, Hkv) == Q.QSA_ERR_UNSUPPORTED
    assert pre(128, 12, 3) == Q.QSA_ERR_UNSUPPORTED


def test_prefill_host_sizes_and_argument_checks(lib):
    # host arithmetic only: the device bytes grow with the inputs, shrink with more row chunks
    # (smaller per-chunk workspaces), and are 0 for invalid sizes
    full = Q.qsa_prefill_host_device_bytes(1, 131072, 131072, 16, 2, 128, 4, 64, 512, chunks=1, sel_chunks=1)
    chunked = Q.qsa_prefill_host_device_bytes(1, 131072, 131072, 16, 2, 128, 4, 64, 512, chunks=32)
    inputs = 131072 * (2 * 16 * 128 * 2 + 2 * 2 * 128 * 2 + 4 * 64 * 2 + 64 * 2)   # q, out, k, v, qi, ki
    assert full > chunked > inputs
    assert Q.qsa_prefill_host_device_bytes(1, 131072, 131072, 16, 2, 128, 4, 64, 512, chunks=32, rope=True) > chunked
    assert Q.qsa_prefill_host_device_bytes(1, 131072, 131072, 16, 2, 128, 4, 64, 512, chunks=0) > 0
    assert Q.qsa_prefill_host_device_bytes(1, 100, 50, 16, 2, 128, 4, 64, 512) == 0        # Tk < q_pos0 + Tq
    assert Q.qsa_prefill_host_device_bytes(1, 100, 100, 16, 2, 128, 4, 64, 512, chunks=-1) == 0
    args = [FAKE] * 6 + [1, 64, 64, 16, 2, 128, 4, 64, 8, 4, 0, 0.1, 0, None, None, 1, 1, FAKE, 1 << 30, None, None,
                         None]

    def call(**kw):
        a = list(args)
        names = {"q": 0, "dev": 23, "dev_bytes": 24, "Tk": 8, "blk": 15, "scale": 17, "chunks": 21}
        for n, val in kw.items():
            a[names[n]] = val
        return lib.qsa_prefill_host(*a)

    assert call(q=None) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(dev=None) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(dev=P((1 << 20) + 16)) == Q.QSA_ERR_INVALID_ARGUMENT      # not 256-byte aligned
    assert call(Tk=60) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(blk=8) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(scale=0.0) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(chunks=-1) == Q.QSA_ERR_INVALID_ARGUMENT
    assert call(dev_bytes=100) == Q.QSA_ERR_WORKSPACE_TOO_SMALL

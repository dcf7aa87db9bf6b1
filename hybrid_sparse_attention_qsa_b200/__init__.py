"""B200-native Qwen Sparse Attention (QSA) hot path.

``qsa`` is the ctypes binding of the C-ABI library ``libqsa_b200.so`` (declared in include/qsa.h);
``inputs`` draws the seeded synthetic workloads.  The library is loaded on first use and there is
no CPU fallback.
"""
from . import qsa  # noqa: F401
from .qsa import (QSA_SELECT_AUTO, QSA_SELECT_FILTERED, QSA_SELECT_MATERIALISED, QSAError,  # noqa: F401
                  decode, prefill, prefill_host, qsa_abi_version, qsa_decode_select, qsa_get_device_status,
                  qsa_index_score,
                  qsa_pool_block_keys, qsa_rope_index_queries, qsa_select_topk, qsa_set_select_options,
                  qsa_set_wait_timeout_ns, qsa_sparse_attn_decode, qsa_sparse_attn_prefill,
                  qsa_sparse_attn_decode_noalloc, qsa_wait_timeout_selftest, qsa_workspace_size,
                  qsa_set_attn_options, QSA_ATTN_AUTO, QSA_ATTN_ROWS, QSA_ATTN_TILES, qsa_check_canaries)

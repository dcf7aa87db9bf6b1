"""B200-native Qwen Sparse Attention (QSA) hot path: the C-ABI library and its Python binding."""

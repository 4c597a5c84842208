"""SegPagedAttention for NVIDIA B200 (sm_100a): C-ABI library libsegpaged.so and its Python binding."""

"""fp64 CPU oracle for SegPagedAttention -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline legs may import this package.
The product (head_sparse_paged_b200) never imports it and it never imports the product.
"""

"""B200-native query-dependent top-k block-sparse causal attention (NSA / MoBA forward).

The compute path is the C-ABI library ``libnsa_b200.so`` (hand-written CUDA for
sm_100a); ``dynamic_block_sparse_scoring_b200.abi`` is its thin ctypes binding.
``workloads`` holds the named problem shapes and their seeded synthetic inputs.
"""
__all__ = ["abi", "workloads"]

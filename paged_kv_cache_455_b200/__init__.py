"""B200 paged KV-cache decode attention.

The CUDA library (``libpa.so``, built from ``csrc/``) is reached through
``paged_kv_cache_455_b200.pa``; ``workloads`` holds the seeded input
generators.  Importing the package itself loads nothing.
"""

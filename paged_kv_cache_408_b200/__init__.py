"""paged_kv_cache_408_b200 -- paged-KV attention for continuous batching on B200 (sm_100a).

The compute path is the C-ABI library ``libpa.so`` (hand-written CUDA for
sm_100a, declared in ``include/pa.h``); ``ops`` is its thin Python binding and
``runtime`` the host-side block allocator and iteration-level scheduler that
drive it.  Importing the package loads nothing; the first call into ``ops``
loads the library and fails loudly if it is missing.
"""

__all__ = ["ops", "runtime", "inputs"]

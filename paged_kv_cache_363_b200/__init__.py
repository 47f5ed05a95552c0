"""B200-native paged KV-cache decode path (PagedAttention).

The compute lives in libpa.so (hand-written sm_100a CUDA behind a C ABI,
declared in include/pa.h).  `paged_kv_cache_363_b200.pa` is the thin ctypes
binding; `paged_kv_cache_363_b200.workloads` draws seeded synthetic inputs.
"""

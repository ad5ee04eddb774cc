"""B200 (sm_100a) PagedAttention: attention over a KV cache kept in fixed 16-token blocks of one
pooled buffer, addressed through per-request block tables.

The compute lives in libpkv.so (C ABI in include/pkv.h). Import
`paged_kv_cache_446_b200.pkv` for its Python binding (it raises if the library is not built) and
`paged_kv_cache_446_b200.workloads` for the seeded synthetic inputs of the five measured
configurations.
"""

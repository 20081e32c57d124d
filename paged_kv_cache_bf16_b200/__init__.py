"""B200-native paged KV-cache attention (bf16).

The compute lives in libnpv.so (hand-written sm_100a CUDA behind a C ABI, see
include/npv.h).  `paged_kv_cache_bf16_b200.ops` is the thin Python binding;
`paged_kv_cache_bf16_b200.workloads` draws seeded synthetic inputs;
`paged_kv_cache_bf16_b200.tp` runs decode attention head-sharded over ranks
with the output projection's all-reduce.
Importing the package does not load the CUDA library; the first op call does,
and raises if it is missing.
"""

__all__ = ["ops", "workloads", "tp"]

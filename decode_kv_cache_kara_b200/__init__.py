"""B200-native Kara window compression and LaCache ladder compaction over a paged KV cache.

The compute path is the C-ABI CUDA library ``libkara.so`` (sm_100a) declared in
``include/kara.h``; ``decode_kv_cache_kara_b200.kara`` is its thin Python binding (argument
marshalling only) and ``decode_kv_cache_kara_b200.synth`` draws seeded synthetic workloads.
Submodules are imported explicitly so that importing the package never loads CUDA.
"""

__all__ = ["kara", "synth", "build"]

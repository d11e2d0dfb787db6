"""Seeded synthetic inputs for the paged KV-cache decode path.

This package is shared by the oracle-side tests and by the GPU-side tests and
bench. It holds no arithmetic of the method itself: it draws random numbers,
rounds them to the storage type of the cache, and describes the five decode
workloads (sequence counts, head counts, context-length mixes, pool sizes and
the seeded physical placement of blocks). Block tables, slot mappings,
copy-on-write pairs and attention outputs are never produced here.
"""

from .gen import (  # noqa: F401
    f32_to_bits,
    normal_bits,
    seq_kv_bits,
    query_bits,
    own_token_kv_bits,
    bits_dtype_name,
)
from .configs import (  # noqa: F401
    DecodeWorkload,
    SharedPrefixWorkload,
    WORKLOADS,
    workload,
)

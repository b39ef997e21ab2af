"""B200 (sm_100a) hot path of Memory Sparse Attention: document-wise RoPE + chunk-mean pooling,
cosine router scoring on tcgen05 tensor cores, top-k document selection, host-bank KV fetch,
sparse GQA attention and the Memory Interleave round — behind the C ABI of include/msa.h.

Importing this package loads libmsa.so and raises if it is missing: there is no fallback path.
"""
from .api import *  # noqa: F401,F403
from .api import InterleaveGraph, InterleaveRound, MSAError, device_status, rope_table, chunk_doc_map, version  # noqa: F401

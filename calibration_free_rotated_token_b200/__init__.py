"""Rotated-token KV-cache quantization (TurboQuant form) for B200 / sm_100a.

The compute lives in ``libkvq.so`` (CUDA kernels behind the C ABI of
``include/kvq.h``); this package only builds it (``build``), binds it
(``_abi``: functions named like the C entry points) and draws seeded
synthetic inputs (``workloads``).  Importing the package does not load the
library; the first call does, and fails loudly if it is missing.
"""
from ._abi import (  # noqa: F401
    EXPORTED, KVQ_BETA_CODEBOOK, KVQ_BF16, KVQ_F16, KVQ_F32, KVQ_LAYOUT_BLOCK32, KVQ_LAYOUT_TOKEN, KVQ_QJL, Handle,
    KvqCache, KvqDecodeDesc, KvqError, KvqQuantJob, alloc_packed, kvq_codebook, kvq_decode_attend, kvq_decode_attend_ex, kvq_decode_attend_noalloc,
    kvq_decode_workspace, kvq_destroy, kvq_get_constants, kvq_init, kvq_last_error, kvq_nsn_decode_attend,
    kvq_nsn_quantize, kvq_probe_wait_timeout, kvq_quantize, kvq_quantize_batch, kvq_status, load, make_cache, packed_shapes,
)

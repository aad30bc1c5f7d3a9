"""B200 (sm_100a) WSVD low-rank KV-cache decode: C-ABI library + thin binding."""
from ._lib import (  # noqa: F401
    LIB_PATH,
    WsvdError,
    dense_cache_bytes,
    dense_decode_attention,
    dense_decode_workspace_size,
    load,
    shared_cache_bytes,
    shared_decode_workspace_size,
    shared_latent_svd_decode,
    workspace,
    wsvd_append_and_decode,
    wsvd_append_workspace_size,
    wsvd_cache_bytes,
    wsvd_decode_attention,
    wsvd_decode_workspace_size,
    wsvd_latent_append,
)

"""Causal grouped-query attention on B200 (sm_100a): prefill, split-KV decode and KV append,
over a contiguous or a paged KV cache, with an optional sliding window, the prefill's backward
pass, and MLA decode over a latent cache.

The computation lives in the CUDA library ``libgqa_b200.so`` behind the C ABI of
``include/gqa.h``; this package is a thin ctypes binding over it (``_lib``) plus the build script
(``build``). Importing the package fails if the library has not been built: there is no CPU path.
"""

from ._lib import (  # noqa: F401
    GQAError,
    LIB_PATH,
    debug_expire_waits,
    decode,
    decode_noalloc,
    decode_paged,
    decode_workspace_size,
    get_device_error,
    kv_append,
    kv_append_paged,
    mla_decode,
    prefill,
    prefill_backward,
    status_string,
    version,
    workspace,
)
